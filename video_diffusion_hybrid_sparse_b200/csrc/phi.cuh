// phi.cuh - the linear-attention feature map phi(x) = elu(x) + 1 applied in
// place to a 128-byte-swizzled bf16 tile in shared memory.
#pragma once

#include "sm100.cuh"

namespace vdn {

// phi(x) = max(x, 0) + exp(min(x, 0)): x + 1 for x > 0 (exp(0) = 1), exp(x)
// otherwise.  Written without a branch so the exponentials of a chunk issue
// back to back.
__device__ __forceinline__ float phi_f(float x) {
  return fmaxf(x, 0.f) + ex2_approx(fminf(x, 0.f) * 1.4426950408889634f);
}

// phi of the two bf16 halves of w, packed back to bf16: the arithmetic of
// phi_f on each half (fp32 min, multiply, ex2, add, one rounding to bf16)
// with max(x, 0) formed as x - min(x, 0), which is exact, so that the
// multiply and the two adds run as packed f32x2 instructions.
__device__ __forceinline__ uint32_t phi_bf16x2(uint32_t w) {
  const float x0 = bf16_lo(w), x1 = bf16_hi(w);
  const uint64_t x = f32x2_pack(x0, x1);
  const uint64_t t = f32x2_pack(fminf(x0, 0.f), fminf(x1, 0.f));
  float a0, a1;
  f32x2_unpack(f32x2_mul(t, f32x2_pack(1.4426950408889634f, 1.4426950408889634f)), a0, a1);
  float r0, r1;
  f32x2_unpack(f32x2_add(f32x2_sub(x, t), f32x2_pack(ex2_approx(a0), ex2_approx(a1))), r0, r1);
  return pack_bf16x2(r0, r1);
}

// Tile: 128 rows x (nbox * 64) bf16 columns as loaded by TMA with 128-byte
// swizzle (box b at byte offset b * 16384, row r at r * 128 inside a box, the
// 16-byte chunk index XOR-ed with r % 8).  Rows >= n_valid and columns >=
// d_real become 0; every other element x becomes bf16(phi(x)).  Called by
// nthreads threads with tid in [0, nthreads).  kB chunks per thread and
// batch: all loads first, then compute and store, so the shared-memory round
// trips of a thread overlap; with kB = nbox * 1024 / nthreads every thread
// takes exactly its chunks in one batch (a larger kB computes phi of chunks
// that are then not stored).
template <int kB = 8>
__device__ __forceinline__ void phi_tile_inplace(uint8_t* tile, int nbox, int n_valid, int d_real, int tid,
                                                 int nthreads) {
  const int nchunks = nbox * 1024;
  if (n_valid >= 128 && d_real >= nbox * 64) {
    // nothing to zero: chunk q is the 16 bytes at 16 q (the swizzle only
    // decides which columns they hold)
    uint4* base = reinterpret_cast<uint4*>(tile);
    for (int q0 = tid; q0 < nchunks; q0 += kB * nthreads) {
      uint4 v[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const int q = q0 + u * nthreads;
        v[u] = base[q < nchunks ? q : q0];  // out-of-range slots re-read a valid chunk and are not stored
      }
#pragma unroll
      for (int u = 0; u < kB; ++u)
        v[u] = make_uint4(phi_bf16x2(v[u].x), phi_bf16x2(v[u].y), phi_bf16x2(v[u].z), phi_bf16x2(v[u].w));
#pragma unroll
      for (int u = 0; u < kB; ++u)
        if (q0 + u * nthreads < nchunks) base[q0 + u * nthreads] = v[u];
    }
    return;
  }
  for (int q0 = tid; q0 < nchunks; q0 += kB * nthreads) {
    uint4 v[kB];
    uint4* ptr[kB];
    int a0[kB], row[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const int q = q0 + u * nthreads;
      const int qq = q < nchunks ? q : q0;  // out-of-range slots re-read a valid chunk and are not stored
      const int bx = qq >> 10, w = qq & 1023;
      row[u] = w >> 3;
      const int c16 = w & 7;
      a0[u] = bx * 64 + ((c16 ^ (row[u] & 7)) << 3);
      ptr[u] = reinterpret_cast<uint4*>(tile + bx * 16384 + row[u] * 128 + c16 * 16);
      v[u] = *ptr[u];
    }
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      uint32_t w4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int a = a0[u] + 2 * e;
        const bool rv = row[u] < n_valid;
        const float lo = (rv && a < d_real) ? 1.f : 0.f;
        const float hi = (rv && a + 1 < d_real) ? 1.f : 0.f;
        w4[e] = pack_bf16x2(lo * phi_f(bf16_lo(w4[e])), hi * phi_f(bf16_hi(w4[e])));
      }
      v[u] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
#pragma unroll
    for (int u = 0; u < kB; ++u)
      if (q0 + u * nthreads < nchunks) *ptr[u] = v[u];
  }
}

}  // namespace vdn
