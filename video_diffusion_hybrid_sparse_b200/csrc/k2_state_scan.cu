// k2_state_scan.cu - forward/backward states of the VDN-H3 linear branch
// (article section 双分支混合注意力机制: a forward state sums the context before
// the local window, a backward state the context after it, both without the
// window and the anchor frames; the text is written at half weight into each).
//
// Per element group of [S | z] (batch, head, row n in [0, Dp], 4 consecutive
// columns a) one thread:
//   1. sums the slice partials of every non-anchor frame into its chunk,
//      cs[c] = sum_{f in chunk c, f not an anchor} [S|z]_f  (fp32; partials
//      are read in batches of kScanBatch for memory-level parallelism; parts
//      are ordered by frame, so one register sum per chunk is kept and
//      written out when the chunk changes), and the text partials into t;
//   2. turns cs into running prefix sums P[c] = sum_{c' <= c} cs[c'] and forms
//      F_c = t/2 + P[c-2],  B_c = t/2 + (P[Nc-1] - P[c+1]),  M_c = F_c + B_c
//      (B_c is exactly t/2 for the last two chunks);
//   3. writes M_c as a bf16 hi/lo pair (hi = bf16(M), lo = bf16(M - hi)) into
//      the readout's B-operand image: rows n (value column; row Dp = z, rows
//      Dp+1..Dp+15 zero, written by the threads of rows 0..14, one row
//      each), K = a, K-major with the 128-byte swizzle, so the readout copies
//      it to shared memory with one bulk copy;
//   4. optionally exports F_c and B_c in fp32.
// The chunk sums live in shared memory, thread-fastest ([Nc][4][threads]).
#include "kernels.h"
#include "sm100.cuh"

namespace vdn {

namespace {

#ifndef VDN_K2_BATCH
#define VDN_K2_BATCH 10
#endif
constexpr int kScanBatch = VDN_K2_BATCH;  // partial loads in flight per thread
constexpr int kScanThreads = 128;

__device__ __forceinline__ uint32_t mt_offset(int n, int a, int rows) {
  // byte offset of element (row n, column a) in one K-major SW128 B-tile image
  const int ac = a >> 6;
  const int chunk = ((a & 63) >> 3) ^ (n & 7);
  return (uint32_t)(ac * rows * 128 + n * 128 + chunk * 16 + (a & 7) * 2);
}

}  // namespace

__global__ void __launch_bounds__(kScanThreads) k2_state_scan(const __grid_constant__ K2Params p, int n_threads_total) {
  extern __shared__ float scan_smem[];
  const Geom& g = p.g;
  const int Dp = g.Dp;
  const int Nc = g.Nc;
  const int T_ = blockDim.x;
  float* cs = scan_smem + threadIdx.x;  // cs[(c * 4 + e) * T_]
  const int gid = blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= n_threads_total) return;

  const int a4s = Dp / 4;
  int rem = gid;
  const int a4 = rem % a4s; rem /= a4s;
  const int n = rem % (Dp + 1); rem /= (Dp + 1);
  const int h = rem % g.H;
  const int b = rem / g.H;
  const size_t part_stride = (size_t)g.B * g.H * (Dp + 1) * Dp;
  const float* src0 = p.parts + (((size_t)b * g.H + h) * (Dp + 1) + n) * Dp + a4 * 4;

  for (int c = 0; c < Nc; ++c)
#pragma unroll
    for (int e = 0; e < 4; ++e) cs[(c * 4 + e) * T_] = 0.f;
  float t[4] = {0.f, 0.f, 0.f, 0.f};
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  int cur = -1;  // chunk held in acc

  for (int p0 = 0; p0 < g.n_parts; p0 += kScanBatch) {
    float4 x[kScanBatch];
#pragma unroll
    for (int u = 0; u < kScanBatch; ++u)
      if (p0 + u < g.n_parts) x[u] = __ldg(reinterpret_cast<const float4*>(src0 + (size_t)(p0 + u) * part_stride));
#pragma unroll
    for (int u = 0; u < kScanBatch; ++u) {
      const int pp = p0 + u;
      if (pp >= g.n_parts) break;
      if (pp < g.n_video_parts) {
        const int ch = part_frame(pp, g) / g.C;
        if (ch != cur) {
          if (cur >= 0)
#pragma unroll
            for (int e = 0; e < 4; ++e) cs[(cur * 4 + e) * T_] = acc[e];
          cur = ch;
          acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
        }
        acc[0] += x[u].x; acc[1] += x[u].y; acc[2] += x[u].z; acc[3] += x[u].w;
      } else {
        t[0] += x[u].x; t[1] += x[u].y; t[2] += x[u].z; t[3] += x[u].w;
      }
    }
  }
  if (cur >= 0)
#pragma unroll
    for (int e = 0; e < 4; ++e) cs[(cur * 4 + e) * T_] = acc[e];

  // running prefix sums in place
  for (int c = 1; c < Nc; ++c)
#pragma unroll
    for (int e = 0; e < 4; ++e) cs[(c * 4 + e) * T_] += cs[((c - 1) * 4 + e) * T_];

  const int rows = Dp + 16;
  const size_t tile_bytes = (size_t)rows * Dp * 2;
  const int d = g.d;
  const bool exp_row = (n < d) || (n == Dp);
  const int exp_n = (n == Dp) ? d : n;
  const uint32_t off = mt_offset(n, a4 * 4, rows);
  const bool zero_row = n < 15;
  const uint32_t off_z = mt_offset(Dp + 1 + (zero_row ? n : 0), a4 * 4, rows);
  for (int c = 0; c < Nc; ++c) {
    const int fl = fwd_last_chunk(c), bf = bwd_first_chunk(c);
    float Fv[4], Bv[4], M[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float pre = fl >= 0 ? cs[(fl * 4 + e) * T_] : 0.f;
      const float suf = bf <= Nc - 1 ? cs[((Nc - 1) * 4 + e) * T_] - cs[((bf - 1) * 4 + e) * T_] : 0.f;
      Fv[e] = 0.5f * t[e] + pre;
      Bv[e] = 0.5f * t[e] + suf;
      M[e] = Fv[e] + Bv[e];
    }
    uint8_t* tile = p.mt + (((size_t)b * Nc + c) * g.H + h) * 2 * tile_bytes;
    uint32_t hi[2], lo[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const __nv_bfloat16 h0 = __float2bfloat16_rn(M[2 * e]), h1 = __float2bfloat16_rn(M[2 * e + 1]);
      const float r0 = M[2 * e] - __bfloat162float(h0), r1 = M[2 * e + 1] - __bfloat162float(h1);
      hi[e] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
      lo[e] = pack_bf16x2(r0, r1);
    }
    *reinterpret_cast<uint2*>(tile + off) = make_uint2(hi[0], hi[1]);
    *reinterpret_cast<uint2*>(tile + tile_bytes + off) = make_uint2(lo[0], lo[1]);
    if (zero_row) {
      *reinterpret_cast<uint2*>(tile + off_z) = make_uint2(0, 0);
      *reinterpret_cast<uint2*>(tile + tile_bytes + off_z) = make_uint2(0, 0);
    }
    if (p.export_fwd && exp_row) {
      const size_t base = ((((size_t)b * Nc + c) * g.H + h) * (d + 1) + exp_n) * d;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int a = a4 * 4 + e;
        if (a < d) {
          p.export_fwd[base + a] = Fv[e];
          p.export_bwd[base + a] = Bv[e];
        }
      }
    }
  }
}

int k2_threads_per_block(int Nc) {
  // chunk sums in shared memory: Nc * 16 bytes per thread, at most ~96 KB per block
  int tpb = (96 * 1024) / (Nc * 16);
  tpb = (tpb / 32) * 32;
  if (tpb > kScanThreads) tpb = kScanThreads;
  return tpb;
}

cudaError_t launch_state_scan(const K2Params& p, cudaStream_t st) {
  const Geom& g = p.g;
  const int total = g.B * g.H * (g.Dp + 1) * (g.Dp / 4);
  const int tpb = k2_threads_per_block(g.Nc);
  if (tpb < 32) return cudaErrorInvalidValue;
  const int smem = tpb * g.Nc * 16;
  cudaError_t e = cudaFuncSetAttribute(k2_state_scan, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  k2_state_scan<<<(total + tpb - 1) / tpb, tpb, smem, st>>>(p, total);
  return cudaGetLastError();
}

}  // namespace vdn
