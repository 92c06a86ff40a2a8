// k2_state_scan.cu - forward/backward states of the VDN-H3 linear branch
// (article section 双分支混合注意力机制: a forward state sums the context before
// the local window, a backward state the context after it, both without the
// window and the anchor frames; the text is written at half weight into each).
//
// Per element e of [S | z] (batch, head, row n in [0, Dp], 8 consecutive
// columns a) one thread:
//   1. sums the slice partials of every non-anchor frame into its chunk:
//      cs[c] = sum_{f in chunk c, f not an anchor} [S|z]_f      (fp32)
//      and the text partials into t;
//   2. forms, exactly by running sums in both directions,
//      F_c = t/2 + sum_{c' <= c-2} cs[c'],   B_c = t/2 + sum_{c' >= c+2} cs[c'],
//      M_c = F_c + B_c;
//   3. writes M_c as a bf16 hi/lo pair (hi = bf16(M), lo = bf16(M - hi)) into
//      the readout's B-operand image: rows n (value column; row Dp = z, rows
//      Dp+1..Dp+15 zero), K = a, K-major with the 128-byte swizzle, so the
//      readout copies it to shared memory with one bulk copy;
//   4. optionally exports F_c and B_c in fp32.
// The chunk sums and backward sums of a thread live in shared memory
// (2 x n_chunks x 8 floats each).
#include "kernels.h"
#include "sm100.cuh"

namespace vdn {

namespace {

__device__ __forceinline__ uint32_t mt_offset(int n, int a, int Dp, int rows) {
  // byte offset of element (row n, column a) in one K-major SW128 B-tile image
  const int ac = a >> 6;
  const int chunk = ((a & 63) >> 3) ^ (n & 7);
  return (uint32_t)(ac * rows * 128 + n * 128 + chunk * 16 + (a & 7) * 2);
}

}  // namespace

__global__ void k2_state_scan(const __grid_constant__ K2Params p, int n_threads_total) {
  extern __shared__ float scan_smem[];  // [2][Nc][8][blockDim.x]: thread-fastest, no bank conflicts
  const Geom& g = p.g;
  const int Dp = g.Dp;
  const int Nc = g.Nc;
  const int gid = blockIdx.x * blockDim.x + threadIdx.x;
  const int T_ = blockDim.x;
  float* cs = scan_smem + threadIdx.x;  // cs[(c * 8 + e) * T_]
  if (gid >= n_threads_total) return;

  const int a8s = Dp / 8;
  int rem = gid;
  const int a8 = rem % a8s; rem /= a8s;
  const int n = rem % (Dp + 1); rem /= (Dp + 1);
  const int h = rem % g.H;
  const int b = rem / g.H;
  const size_t part_stride = (size_t)g.B * g.H * (Dp + 1) * Dp;
  const size_t elem = (((size_t)b * g.H + h) * (Dp + 1) + n) * Dp + a8 * 8;

  for (int c = 0; c < Nc; ++c)
#pragma unroll
    for (int e = 0; e < 8; ++e) cs[(c * 8 + e) * T_] = 0.f;
  float t[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) t[e] = 0.f;

  for (int pp = 0; pp < g.n_parts; ++pp) {
    const float4* src = reinterpret_cast<const float4*>(p.parts + pp * part_stride + elem);
    const float4 x0 = src[0], x1 = src[1];
    const float x[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    if (pp < g.n_video_parts) {
      float* dst = cs + (part_frame(pp, g) / g.C) * 8 * T_;
#pragma unroll
      for (int e = 0; e < 8; ++e) dst[e * T_] += x[e];
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) t[e] += x[e];
    }
  }

  // bw[c] = sum of cs[c'] for c' >= bwd_first_chunk(c), by a backward running sum
  float* bw = cs + (size_t)T_ * Nc * 8;  // second array, same layout
  {
    float run[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) run[e] = 0.f;
    int next = Nc - 1;  // highest chunk not yet added to run
    for (int c = Nc - 1; c >= 0; --c) {
      for (; next >= 0 && next >= bwd_first_chunk(c); --next)
#pragma unroll
        for (int e = 0; e < 8; ++e) run[e] += cs[(next * 8 + e) * T_];
#pragma unroll
      for (int e = 0; e < 8; ++e) bw[(c * 8 + e) * T_] = run[e];
    }
  }

  const int rows = Dp + 16;
  const size_t tile_bytes = (size_t)rows * Dp * 2;
  const int d = g.d;
  const bool exp_row = (n < d) || (n == Dp);
  const int exp_n = (n == Dp) ? d : n;
  float fw[8];  // sum of cs[c'] for c' <= fwd_last_chunk(c), forward running sum
#pragma unroll
  for (int e = 0; e < 8; ++e) fw[e] = 0.f;
  int next_f = 0;  // lowest chunk not yet added to fw
  for (int c = 0; c < Nc; ++c) {
    for (; next_f < Nc && next_f <= fwd_last_chunk(c); ++next_f)
#pragma unroll
      for (int e = 0; e < 8; ++e) fw[e] += cs[(next_f * 8 + e) * T_];
    float Fv[8], Bv[8], M[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      Fv[e] = 0.5f * t[e] + fw[e];
      Bv[e] = 0.5f * t[e] + bw[(c * 8 + e) * T_];
      M[e] = Fv[e] + Bv[e];
    }
    uint8_t* tile = p.mt + (((size_t)b * Nc + c) * g.H + h) * 2 * tile_bytes;
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat16 h0 = __float2bfloat16_rn(M[2 * e]), h1 = __float2bfloat16_rn(M[2 * e + 1]);
      const float r0 = M[2 * e] - __bfloat162float(h0), r1 = M[2 * e + 1] - __bfloat162float(h1);
      hi[e] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
      lo[e] = pack_bf16x2(r0, r1);
    }
    const uint32_t off = mt_offset(n, a8 * 8, Dp, rows);
    *reinterpret_cast<uint4*>(tile + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(tile + tile_bytes + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    if (n == Dp) {
      for (int z = Dp + 1; z < rows; ++z) {  // zero padding rows
        const uint32_t oz = mt_offset(z, a8 * 8, Dp, rows);
        *reinterpret_cast<uint4*>(tile + oz) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(tile + tile_bytes + oz) = make_uint4(0, 0, 0, 0);
      }
    }
    if (p.export_fwd && exp_row) {
      const size_t base = ((((size_t)b * Nc + c) * g.H + h) * (d + 1) + exp_n) * d;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int a = a8 * 8 + e;
        if (a < d) {
          p.export_fwd[base + a] = Fv[e];
          p.export_bwd[base + a] = Bv[e];
        }
      }
    }
  }
}

int k2_threads_per_block(int Nc) {
  // chunk sums + backward sums in shared memory: Nc * 64 bytes per thread, at most ~200 KB per block
  int tpb = (200 * 1024) / (Nc * 64);
  tpb = (tpb / 32) * 32;
  if (tpb > 128) tpb = 128;
  return tpb;
}

cudaError_t launch_state_scan(const K2Params& p, cudaStream_t st) {
  const Geom& g = p.g;
  const int total = g.B * g.H * (g.Dp + 1) * (g.Dp / 8);
  const int tpb = k2_threads_per_block(g.Nc);
  if (tpb < 32) return cudaErrorInvalidValue;
  const int smem = tpb * g.Nc * 64;
  cudaError_t e = cudaFuncSetAttribute(k2_state_scan, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  k2_state_scan<<<(total + tpb - 1) / tpb, tpb, smem, st>>>(p, total);
  return cudaGetLastError();
}

}  // namespace vdn
