// k0_misc.cu - input staging (fp32 -> bf16, head_dim 32 -> 64 zero padding)
// and the device-side membership table.
#include "kernels.h"
#include "sm100.cuh"

namespace vdn {

// dst[row, head, 0:Dp] = bf16(src[row, head, 0:d]) with zeros in [d, Dp).
template <bool FP32_IN>
__global__ void k0_stage(const void* __restrict__ src, __nv_bfloat16* __restrict__ dst, long long n_vec, int d,
                         int Dp) {
  const int per_row = Dp / 8;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n_vec; i += (long long)gridDim.x * blockDim.x) {
    const long long rh = i / per_row;
    const int a0 = (int)(i - rh * per_row) * 8;
    float x[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int a = a0 + e;
      if (a < d) {
        if constexpr (FP32_IN) x[e] = static_cast<const float*>(src)[rh * d + a];
        else x[e] = __bfloat162float(static_cast<const __nv_bfloat16*>(src)[rh * d + a]);
      } else {
        x[e] = 0.f;
      }
    }
    *reinterpret_cast<uint4*>(dst + rh * Dp + a0) =
        make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
  }
}

cudaError_t launch_stage(const void* src, int fp32_in, __nv_bfloat16* dst, long long rows, int H, int d, int Dp,
                         cudaStream_t st) {
  const long long n_vec = rows * H * (Dp / 8);
  if (n_vec == 0) return cudaSuccess;
  const int tpb = 256;
  long long blocks = (n_vec + tpb - 1) / tpb;
  if (blocks > 148 * 64) blocks = 148 * 64;
  if (fp32_in) k0_stage<true><<<(int)blocks, tpb, 0, st>>>(src, dst, n_vec, d, Dp);
  else k0_stage<false><<<(int)blocks, tpb, 0, st>>>(src, dst, n_vec, d, Dp);
  return cudaGetLastError();
}

// table[f * F + x]: 1 if the softmax kernel's KV ranges of f's query segment
// cover key frame x, 2 if the scan puts x in f's forward state, 3 if in the
// backward state (none for a GLOBAL anchor query, whose readout is zeroed);
// 255 if not exactly one of them.
__global__ void k_membership(const __grid_constant__ Geom g, uint8_t* table) {
  const int total = g.F * g.F;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const int f = i / g.F, x = i % g.F;
    const int c = f / g.C;
    const int glob = no_linear_read(f, g);
    KvRanges r;
    seg_ranges(glob ? kAllFrames : c, g, r);
    const long long s0 = (long long)x * g.P, e0 = s0 + g.P;
    int soft = 0;
    for (int k = 0; k < r.n; ++k)
      if (r.start[k] <= s0 && e0 <= r.start[k] + r.len[k]) soft = 1;
    const int has_state = !glob && x >= 1 && x <= g.F - 2;  // frames that own state parts
    const int cx = x / g.C;
    const int fwd = has_state && cx <= fwd_last_chunk(c);
    const int bwd = has_state && cx >= bwd_first_chunk(c);
    uint8_t code = 255;
    if (soft + fwd + bwd == 1) code = soft ? 1 : (fwd ? 2 : 3);
    table[i] = code;
  }
}

cudaError_t launch_membership(const Geom& g, uint8_t* table, cudaStream_t st) {
  const int total = g.F * g.F;
  k_membership<<<(total + 255) / 256, 256, 0, st>>>(g, table);
  return cudaGetLastError();
}

}  // namespace vdn
