// phi.cuh - the linear-attention feature map phi(x) = elu(x) + 1 applied in
// place to a 128-byte-swizzled bf16 tile in shared memory.
#pragma once

#include "sm100.cuh"

namespace vdn {

__device__ __forceinline__ float phi_f(float x) { return x > 0.f ? x + 1.f : __expf(x); }

// Tile: 128 rows x (nbox * 64) bf16 columns as loaded by TMA with 128-byte
// swizzle (box b at byte offset b * 16384, row r at r * 128 inside a box, the
// 16-byte chunk index XOR-ed with r % 8).  Rows >= n_valid and columns >=
// d_real become 0; every other element x becomes bf16(phi(x)).  Called by
// nthreads threads with tid in [0, nthreads).
__device__ __forceinline__ void phi_tile_inplace(uint8_t* tile, int nbox, int n_valid, int d_real, int tid,
                                                 int nthreads) {
  const int nchunks = nbox * 1024;
#pragma unroll 4
  for (int q = tid; q < nchunks; q += nthreads) {
    const int bx = q >> 10, w = q & 1023;
    const int row = w >> 3, c16 = w & 7;
    const int a0 = bx * 64 + ((c16 ^ (row & 7)) << 3);
    uint4* ptr = reinterpret_cast<uint4*>(tile + bx * 16384 + row * 128 + c16 * 16);
    uint4 v = *ptr;
    uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int a = a0 + 2 * e;
      const float lo = (row < n_valid && a < d_real) ? phi_f(bf16_lo(u[e])) : 0.f;
      const float hi = (row < n_valid && a + 1 < d_real) ? phi_f(bf16_hi(u[e])) : 0.f;
      u[e] = pack_bf16x2(lo, hi);
    }
    *ptr = make_uint4(u[0], u[1], u[2], u[3]);
  }
}

}  // namespace vdn
