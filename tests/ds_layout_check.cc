// CPU check of the stored dS^T tile layout (head_attention_qk_b200/csrc/ds_layout.h):
// compiled and run by tests/test_ds_layout.py with g++.
#include <cstdio>
#include <vector>

#include "../head_attention_qk_b200/csrc/ds_layout.h"

#define CHECK(c)                                                              \
  do {                                                                        \
    if (!(c)) {                                                               \
      std::fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #c);    \
      return 1;                                                               \
    }                                                                         \
  } while (0)

int main() {
  using hattn::ds_tile_offset;
  // a bijection of the 128 x 128 tile onto 0 .. 16383
  std::vector<int> seen(16384, 0);
  for (int k = 0; k < 128; ++k)
    for (int q = 0; q < 128; ++q) {
      const int o = ds_tile_offset(k, q);
      CHECK(o >= 0 && o < 16384);
      ++seen[o];
    }
  for (int o = 0; o < 16384; ++o) CHECK(seen[o] == 1);
  // a compute warp (key quarter kq: rows 32 kq + lane) storing 8 queries a
  // lane (16 bytes) of its 32-query group writes 512 contiguous bytes
  for (int kq = 0; kq < 4; ++kq)
    for (int q0 = 0; q0 < 128; q0 += 8) {
      const int base = ds_tile_offset(32 * kq, q0);
      for (int lane = 0; lane < 32; ++lane)
        for (int e = 0; e < 8; ++e) CHECK(ds_tile_offset(32 * kq + lane, q0 + e) == base + 8 * lane + e);
    }
  // the dQ product's A operand: for the 16 keys of MMA k, core blocks (8 keys
  // x 8 queries, 128 contiguous bytes, keys 16 bytes apart) start at byte
  // 8192 (k / 2) + 256 (k % 2), step 128 bytes along keys and 512 along queries
  for (int k = 0; k < 8; ++k) {
    const int start = ds_tile_offset(16 * k, 0);
    CHECK(2 * start == 8192 * (k / 2) + 256 * (k % 2));
    for (int kb = 0; kb < 2; ++kb)
      for (int qb = 0; qb < 16; ++qb)
        for (int kr = 0; kr < 8; ++kr)
          for (int qe = 0; qe < 8; ++qe)
            CHECK(2 * ds_tile_offset(16 * k + 8 * kb + kr, 8 * qb + qe) ==
                  2 * start + 128 * kb + 512 * qb + 16 * kr + 2 * qe);
  }
  std::printf("ds_layout ok\n");
  return 0;
}
