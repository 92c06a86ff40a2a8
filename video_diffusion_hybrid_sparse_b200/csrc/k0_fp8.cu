// k0_fp8.cu - e4m3 operands of the fp8 softmax branch.
//
// The pages run their VDN-H3 headline at FP8 (section 性能实测表现); they do
// not describe the scheme, so this is the plain one: one scale per (batch,
// head) for q, one for k and text_k together, one for v and text_v together,
// scale = amax / 448 (448 = largest finite e4m3), values x / scale rounded to
// nearest-even and saturated to the finite range.
//   * k_fp8_amax: |x| maxima of q, k, v, text_k, text_v per (batch, head);
//   * k_fp8_rows: q, k, text_k as e4m3 in their [rows, H * D] layout;
//   * k_fp8_vt:   v, text_v as e4m3 transposed per (batch, head) to
//                 [(b * H + h) * D + dd, token] (row pitch a multiple of 16
//                 bytes), the K-major operand of P.V.
#include "kernels.h"
#include "sm100.cuh"

namespace vdn {

namespace {

__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {  // a in the low byte
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}

// 448 / amax of tensor t (0 q, 1 k, 2 v, 3 text_k, 4 text_v) for (batch, head)
// bh; k and text_k share the larger of their maxima, v and text_v too.
__device__ __forceinline__ float inv_scale(const float* amax, int t, int BH, int bh) {
  float a = amax[t * BH + bh];
  if (t > 0) {
    const int u = t <= 2 ? t : t - 2;  // k / v
    a = fmaxf(amax[u * BH + bh], amax[(u + 2) * BH + bh]);
  }
  return a > 0.f ? 448.0f / a : 1.0f;
}

}  // namespace

// amax[t * BH + b * H + h] = max |x| of tensor t in (batch b, head h).  The
// 16 vectors of one (row, head) sit in 16 consecutive lanes, which reduce
// with shuffles before one lane folds into shared memory; blocks then fold
// into the global maxima (float bits of non-negative values order like
// unsigned integers, so the result does not depend on the order of updates).
// Four vectors per thread and step are loaded before any is reduced.
__global__ void k_fp8_amax(Fp8Src src, int B, long long N, int T, int H, float* amax) {
  extern __shared__ uint32_t s_max[];  // [5 * B * H]
  const int BH = B * H;
  for (int i = threadIdx.x; i < 5 * BH; i += blockDim.x) s_max[i] = 0u;
  __syncthreads();
  const int c8 = 128 / 8;  // 16-byte vectors per (row, head), head_dim 128
  const long long stride = (long long)gridDim.x * blockDim.x;  // a multiple of 32
  for (int t = 0; t < 5; ++t) {
    const __nv_bfloat16* x = src.p[t];
    const long long per_b = t < 3 ? N : (long long)T;
    const long long vecs = per_b * B * H * c8;
    for (long long i0 = blockIdx.x * (long long)blockDim.x + threadIdx.x; i0 - threadIdx.x % 32 < vecs;
         i0 += 4 * stride) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const long long i = i0 + u * stride;
        v[u] = i < vecs ? __ldg(reinterpret_cast<const uint4*>(x) + i) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const long long i = i0 + u * stride;
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        float m = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) m = fmax3(m, fabsf(bf16_lo(w[e])), fabsf(bf16_hi(w[e])));
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if ((threadIdx.x & 15) == 0 && i < vecs) {
          const long long row = i / (H * c8);
          const int h = (int)((i / c8) % H);
          const int b = (int)(row / per_b);
          atomicMax(&s_max[t * BH + b * H + h], __float_as_uint(m));
        }
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 5 * BH; i += blockDim.x)
    if (s_max[i]) atomicMax(reinterpret_cast<unsigned int*>(amax) + i, s_max[i]);
}

// q, k, text_k: e4m3 in place of bf16, same [rows, H * D] layout (one byte
// each).  Four vectors per thread and step are loaded before any is converted.
__global__ void k_fp8_rows(Fp8Src src, Fp8Dst dst, int B, long long N, int T, int H, const float* amax) {
  const int BH = B * H;
  const int c8 = 128 / 8;
  const int which[3] = {0, 1, 3};  // q, k, text_k
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (int u = 0; u < 3; ++u) {
    const int t = which[u];
    const __nv_bfloat16* x = src.p[t];
    uint8_t* y = u == 0 ? dst.q : (u == 1 ? dst.k : dst.tk);
    const long long per_b = (t < 3 ? N : (long long)T);
    const long long vecs = per_b * B * H * c8;
    for (long long i0 = blockIdx.x * (long long)blockDim.x + threadIdx.x; i0 < vecs; i0 += 4 * stride) {
      uint4 v[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const long long i = i0 + r * stride;
        if (i < vecs) v[r] = __ldg(reinterpret_cast<const uint4*>(x) + i);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const long long i = i0 + r * stride;
        if (i >= vecs) break;
        const long long row = i / (H * c8);
        const int h = (int)((i / c8) % H);
        const int b = (int)(row / per_b);
        const float s = inv_scale(amax, t, BH, b * H + h);
        uint2 o;
        o.x = e4m3x2(bf16_lo(v[r].x) * s, bf16_hi(v[r].x) * s) |
              (e4m3x2(bf16_lo(v[r].y) * s, bf16_hi(v[r].y) * s) << 16);
        o.y = e4m3x2(bf16_lo(v[r].z) * s, bf16_hi(v[r].z) * s) |
              (e4m3x2(bf16_lo(v[r].w) * s, bf16_hi(v[r].w) * s) << 16);
        reinterpret_cast<uint2*>(y)[i] = o;
      }
    }
  }
}

// v (t = 2) or text_v (t = 4) transposed: block (token tile of 64, b * H + h),
// 256 threads, reads 64 tokens x 128 head_dim values and writes 128 rows x 64
// bytes.  Thread (g, c) loads the 8 values of vector c for the four tokens
// 4g..4g+3 and stores, per head_dim slot, their four bytes as one word.
__global__ void __launch_bounds__(256) k_fp8_vt(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ y, int t,
                                               int B, long long rows_b, long long pitch, int H, const float* amax) {
  __shared__ uint32_t tile32[128][16 + 1];  // [head_dim][token / 4], padded rows
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const long long tok0 = (long long)blockIdx.x * 64;
  const float s = inv_scale(amax, t, B * H, bh);
  {
    const int c = threadIdx.x & 15, g = threadIdx.x >> 4;  // vector, token group
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const long long tok = tok0 + 4 * g + u;
      v[u] = tok < rows_b ? __ldg(reinterpret_cast<const uint4*>(x + ((b * rows_b + tok) * H + h) * 128) + c)
                          : make_uint4(0, 0, 0, 0);
    }
    uint32_t pr[4][4];  // [token][value pair]
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) pr[u][e] = e4m3x2(bf16_lo(w[e]) * s, bf16_hi(w[e]) * s);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      // head_dim slots 8c + 2e (low bytes) and 8c + 2e + 1 (high bytes)
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        lo |= (pr[u][e] & 0xFFu) << (8 * u);
        hi |= (pr[u][e] >> 8) << (8 * u);
      }
      tile32[c * 8 + 2 * e][g] = lo;
      tile32[c * 8 + 2 * e + 1][g] = hi;
    }
  }
  __syncthreads();
  const uint8_t(*tile)[4 * (16 + 1)] = reinterpret_cast<const uint8_t(*)[4 * (16 + 1)]>(tile32);
  // store: 128 rows x 64 bytes (4 x 16 bytes), tokens past the end skipped
  for (int i = threadIdx.x; i < 128 * 4; i += blockDim.x) {
    const int dd = i >> 2, c = i & 3;
    const long long tok = tok0 + c * 16;
    if (tok >= rows_b) continue;
    uint8_t* dstp = y + ((long long)bh * 128 + dd) * pitch + tok;
    if (tok + 16 <= rows_b) {
      const uint32_t* src = &tile32[dd][c * 4];
      *reinterpret_cast<uint4*>(dstp) = make_uint4(src[0], src[1], src[2], src[3]);
    } else {
      for (int e = 0; tok + e < rows_b; ++e) dstp[e] = tile[dd][c * 16 + e];
    }
  }
}

cudaError_t launch_fp8_quant(const Fp8Src& src, const Fp8Dst& dst, int B, long long N, int T, int H, float* amax,
                             cudaStream_t st) {
  const int BH = B * H;
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float) * 5 * BH, st);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const size_t smem = sizeof(uint32_t) * 5 * BH;
  if (smem > 48 * 1024) return cudaErrorInvalidValue;
  k_fp8_amax<<<sms * 4, 256, smem, st>>>(src, B, N, T, H, amax);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  k_fp8_rows<<<sms * 4, 256, 0, st>>>(src, dst, B, N, T, H, amax);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  k_fp8_vt<<<dim3((unsigned)((N + 63) / 64), BH), 256, 0, st>>>(src.p[2], dst.vt, 2, B, N, dst.pitch_v, H, amax);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (T > 0) {
    k_fp8_vt<<<dim3((unsigned)((T + 63) / 64), BH), 256, 0, st>>>(src.p[4], dst.tvt, 4, B, T, dst.pitch_t, H, amax);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace vdn
