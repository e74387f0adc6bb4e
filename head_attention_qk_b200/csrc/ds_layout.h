// ds_layout.h -- layout of a stored 128 x 128 dS^T tile (attn_bwd_dsbuf).
//
// Written by the dK/dV kernel's compute warps, read back by the dQ product
// kernel as a no-swizzle MN-major operand.  Plain C++ (no CUDA types), so the
// map's properties can be checked on the host (tests/ds_layout_check.cc).
#pragma once

#if defined(__CUDACC__)
#define HATTN_HD __host__ __device__
#else
#define HATTN_HD
#endif

namespace hattn {

// Element offset of dS^T[key][query] within a stored tile: 8-key x 8-query
// core blocks of 128 bytes (keys 16 bytes apart), ordered key-group (8 keys)
// fastest within a 32-key quarter, then 8-query groups, then 32-query groups,
// then key quarters:
//     key = 32 kq + 8 kb + kr, query = 32 qg + 8 q8 + qe
//     offset = 4096 kq + 1024 qg + 256 q8 + 64 kb + 8 kr + qe.
// A compute warp (one key quarter, 32 queries) then stores 512 contiguous
// bytes per instruction, and the tile is the no-swizzle MN-major operand
// layout of the dQ product (core blocks 512 bytes apart along queries, 128
// along keys).
HATTN_HD constexpr int ds_tile_offset(int key, int query) {
  return 4096 * (key >> 5) + 1024 * (query >> 5) + 256 * ((query >> 3) & 3) + 64 * ((key >> 3) & 3) +
         8 * (key & 7) + (query & 7);
}

}  // namespace hattn
