"""The Python binding without a GPU: every tensor's shape and dtype are checked
against the sizes handed to the library before anything reaches the device
(a buffer smaller than those sizes would be read or written out of bounds),
then that the tensors are contiguous CUDA tensors on one device.  CPU tensors
are used throughout, so each bad argument must be caught by the shape/dtype
checks, and a well-formed CPU call must stop at the device check."""
import pytest
import torch

bf, f32, e4 = torch.bfloat16, torch.float32, torch.float8_e4m3fn


@pytest.fixture(scope="module")
def h():
    from head_attention_qk_b200 import build

    build.build()
    import head_attention_qk_b200 as pkg

    return pkg


def t(*shape, dtype=bf):
    return torch.zeros(shape, dtype=dtype)


def fwd_args(**kw):
    a = dict(q=t(1, 4, 64, 128), k=t(1, 2, 96, 128), v=t(1, 2, 96, 128))
    a.update(kw)
    return a


@pytest.mark.parametrize("kw,exc", [
    (dict(v=t(1, 2, 95, 128)), ValueError),              # V shorter than K
    (dict(k=t(2, 2, 96, 128), v=t(2, 2, 96, 128)), ValueError),   # batch mismatch
    (dict(k=t(1, 2, 96, 64), v=t(1, 2, 96, 64)), ValueError),     # head dim mismatch
    (dict(q=t(4, 64, 128)), ValueError),                 # not 4-d
    (dict(v=t(1, 2, 96, 128, dtype=f32)), TypeError),    # V of another type
    (dict(q=t(1, 4, 64, 128, dtype=f32)), TypeError),    # fp32 inputs are refused
    (dict(out=t(1, 4, 63, 128)), ValueError),            # output too small
    (dict(out=t(1, 4, 64, 128, dtype=f32)), TypeError),
    (dict(lse=t(1, 4, 64, dtype=bf)), TypeError),
    (dict(lse=t(1, 4, 32, dtype=f32)), ValueError),
])
def test_fwd_argument_checks(h, kw, exc):
    with pytest.raises(exc):
        h.attn_fwd(**fwd_args(**kw))


def test_fwd_e4m3_descale_checks(h):
    q, k, v = t(1, 4, 64, 128, dtype=e4), t(1, 2, 96, 128, dtype=e4), t(1, 2, 96, 128, dtype=e4)
    good = dict(q_descale=t(1, 4, dtype=f32), k_descale=t(1, 2, dtype=f32), v_descale=t(1, 2, dtype=f32))
    # which descales must be given is the library's check (HATTN_EINVAL, see test_abi.py)
    with pytest.raises(ValueError):                      # one value per tensor is not enough
        h.attn_fwd(q, k, v, **dict(good, k_descale=t(1, dtype=f32)))
    with pytest.raises(TypeError):
        h.attn_fwd(q, k, v, **dict(good, v_descale=t(1, 2, dtype=bf)))
    with pytest.raises(ValueError, match="CUDA"):        # well-formed: stops at the device check
        h.attn_fwd(q, k, v, **good)


def test_fwd_well_formed_cpu_call_stops_at_device_check(h):
    with pytest.raises(ValueError, match="CUDA"):
        h.attn_fwd(**fwd_args())
    with pytest.raises(ValueError, match="contiguous|CUDA"):
        h.attn_fwd(**fwd_args(q=t(1, 4, 128, 64).transpose(2, 3)))


def test_quantize_argument_checks(h):
    x = t(1, 3, 70, 128)
    with pytest.raises(TypeError):
        h.quantize_e4m3(x.float())
    with pytest.raises(ValueError):
        h.quantize_e4m3(x, codes=t(1, 3, 69, 128, dtype=e4))
    with pytest.raises(TypeError):
        h.quantize_e4m3(x, codes=t(1, 3, 70, 128, dtype=torch.uint8))
    with pytest.raises(ValueError):
        h.quantize_e4m3(x, descale=t(1, 2, dtype=f32))
    with pytest.raises(ValueError, match="CUDA"):
        h.quantize_e4m3(x, codes=t(1, 3, 70, 128, dtype=e4), descale=t(3, dtype=f32))


def test_kvblocks_argument_checks(h):
    q = t(1, 4, 64, 128)
    ks = [t(1, 2, 100, 128), t(1, 2, 37, 128)]
    vs = [t(1, 2, 100, 128), t(1, 2, 37, 128)]
    with pytest.raises(ValueError):
        h.attn_fwd_kvblocks(q, ks, vs[:1])
    with pytest.raises(ValueError):                      # V block shorter than its K block
        h.attn_fwd_kvblocks(q, ks, [vs[0], t(1, 2, 36, 128)])
    with pytest.raises(ValueError):                      # KV heads differ between blocks
        h.attn_fwd_kvblocks(q, [ks[0], t(1, 1, 37, 128)], [vs[0], t(1, 1, 37, 128)])
    with pytest.raises(TypeError):
        h.attn_fwd_kvblocks(q, ks, [vs[0], t(1, 2, 37, 128, dtype=f32)])
    with pytest.raises(ValueError):
        h.attn_fwd_kvblocks(q, ks, vs, lse=t(1, 4, 65, dtype=f32))
    with pytest.raises(ValueError, match="CUDA"):
        h.attn_fwd_kvblocks(q, ks, vs)


def bwd_args(**kw):
    a = dict(q=t(2, 4, 64, 128), k=t(2, 2, 80, 128), v=t(2, 2, 80, 128), out=t(2, 4, 64, 128),
             lse=t(2, 4, 64, dtype=f32), dout=t(2, 4, 64, 128))
    a.update(kw)
    return a


@pytest.mark.parametrize("kw,exc", [
    (dict(v=t(2, 2, 79, 128)), ValueError),
    (dict(out=t(2, 4, 63, 128)), ValueError),
    (dict(dout=t(2, 4, 64, 128, dtype=f32)), TypeError),
    (dict(lse=t(2, 4, 64, dtype=bf)), TypeError),
    (dict(lse=t(2, 4, 63, dtype=f32)), ValueError),
    (dict(dq=t(2, 4, 32, 128)), ValueError),
    (dict(dk=t(2, 4, 80, 128)), ValueError),             # dK has the KV heads
    (dict(dv=t(2, 2, 80, 128, dtype=f32)), TypeError),
    (dict(q=t(2, 4, 64, 128, dtype=e4), k=t(2, 2, 80, 128, dtype=e4), v=t(2, 2, 80, 128, dtype=e4)),
     TypeError),                                         # no fp8 backward
])
@pytest.mark.parametrize("fn", ["attn_bwd", "attn_bwd_noalloc"])
def test_bwd_argument_checks(h, fn, kw, exc):
    with pytest.raises(exc):
        getattr(h, fn)(**bwd_args(**kw))


@pytest.mark.parametrize("fn", ["attn_bwd", "attn_bwd_noalloc"])
def test_bwd_well_formed_cpu_call_stops_at_device_check(h, fn):
    with pytest.raises(ValueError, match="CUDA"):
        getattr(h, fn)(**bwd_args())
