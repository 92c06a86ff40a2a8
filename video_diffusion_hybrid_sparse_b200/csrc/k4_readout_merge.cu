// k4_readout_merge.cu - linear-branch readout and gated fusion of the VDN-H3
// hybrid attention (article sections 双分支混合注意力机制 and
// 自适应门控融合双分支输出).
//
// One CTA (256 threads) handles 128 query rows of one (batch, chunk, head):
//   1. TMA loads the q tile (128-byte swizzle) and one bulk copy brings the
//      chunk's readout operand M_c = F_c + B_c as a bf16 hi/lo pair
//      (rows: value column b, row Dp = z; K = head_dim slot a);
//   2. phi is applied to the q tile in place;
//   3. one thread issues D = phi(Q) M_hi^T + phi(Q) M_lo^T on the tensor cores
//      (M = 128, N = Dp + 16, fp32 in TMEM): columns [0, Dp) are the
//      numerators phi(q)^T M, column Dp is the denominator phi(q) . z;
//   4. two warps share each TMEM row (one per half of the columns):
//      o_l = num / den (0 when the states of the chunk hold no token), the
//      row's sum of squares is combined through shared memory, and
//      r = o_l / sqrt(mean(o_l^2) + eps) is staged in shared memory (fp32,
//      16-byte chunks XOR-swizzled by row, over the no longer needed operand
//      buffers);
//   5. a coalesced pass, 16 bytes per thread per item, reads o_s and both
//      gates, applies gamma, and writes out = sigmoid(g_s) o_s + sigmoid(g_l) r.
#include "kernels.h"
#include "phi.cuh"
#include "sm100.cuh"

namespace vdn {

namespace {

template <int D>
struct K4Layout {
  static constexpr int kRows = D + 16;
  static constexpr int kA = 0;
  static constexpr int kATile = 128 * D * 2;
  static constexpr int kBTile = kRows * D * 2;
  static constexpr int kB = kA + kATile;
  static constexpr int kR = 0;                 // r staging [128][D] fp32, reuses A and B
  static constexpr int kRBytes = 128 * D * 4;
  static constexpr int kOperandEnd = kB + 2 * kBTile;
  static_assert(kRBytes <= kOperandEnd, "r staging must fit in the operand buffers");
  static constexpr int kSs = kOperandEnd;      // [2][128] partial sums of squares
  static constexpr int kBar = kSs + 2 * 128 * 4;
  static constexpr int kBytes = kBar + 64 + 1024;
};

__device__ __forceinline__ float sigmoid_f(float x) { return 1.0f / (1.0f + __expf(-x)); }

template <bool FP32>
__device__ __forceinline__ void load8(const void* base, size_t idx, float (&x)[8]) {
  if constexpr (FP32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  } else {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + idx));
    x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x); x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
    x[4] = bf16_lo(u.z); x[5] = bf16_hi(u.z); x[6] = bf16_lo(u.w); x[7] = bf16_hi(u.w);
  }
}

template <bool FP32>
__device__ __forceinline__ void store8(void* base, size_t idx, const float (&x)[8]) {
  if constexpr (FP32) {
    float4* p = reinterpret_cast<float4*>(static_cast<float*>(base) + idx);
    p[0] = make_float4(x[0], x[1], x[2], x[3]);
    p[1] = make_float4(x[4], x[5], x[6], x[7]);
  } else {
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + idx) =
        make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
  }
}

// r staging: row-major fp32 [128][D]; the 16-byte chunk j of row r is stored
// at chunk j ^ (r % (D/4)) so that 32 rows written column-wise, or 2 rows read
// row-wise, spread over all banks.
template <int D>
__device__ __forceinline__ float4* r_chunk(uint8_t* base, int row, int j) {
  constexpr int kChunks = D / 4;
  return reinterpret_cast<float4*>(base + (size_t)row * D * 4 + ((j ^ (row & (kChunks - 1))) << 4));
}

}  // namespace

template <int D, bool FP32>
__global__ void __launch_bounds__(256)
    k4_readout_merge(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ K4Params p) {
  using L = K4Layout<D>;
  constexpr int kCols = D + 16;
  constexpr int kAlloc = kCols <= 128 ? 128 : 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);  // [0] loads, [1] mma
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + 16);
  int* abort_flag = reinterpret_cast<int*>(smem + L::kBar + 20);
  float* ss_part = reinterpret_cast<float*>(smem + L::kSs);

  const Geom& g = p.g;
  const int r0 = blockIdx.x * 128;  // first row of the tile within the chunk
  const int c = blockIdx.y;
  const int b = blockIdx.z / g.H, h = blockIdx.z % g.H;
  const int nrows = min(128, g.rows_per_chunk - r0);
  const int tid = threadIdx.x;
  const uint32_t warp = warp_id(), lane = lane_id();

  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kAlloc);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const CtaAbort ab{abort_flag, p.status};

  if (tid == 0) {
    mbar_expect_tx(&bars[0], (uint32_t)(L::kATile + 2 * L::kBTile));
    for (int bx = 0; bx < D / 64; ++bx)
      tma_load_2d(smem + L::kA + bx * 16384, &tm_q, &bars[0], h * D + bx * 64,
                  b * (int)g.N + c * g.rows_per_chunk + r0);
    const uint8_t* src = p.mt + (((size_t)b * g.Nc + c) * g.H + h) * 2 * (size_t)L::kBTile;
    bulk_load(smem + L::kB, src, (uint32_t)(2 * L::kBTile), &bars[0]);
  }
  bool issued = false;
  bool ok = mbar_wait(&bars[0], 0, ab);
  if (__syncthreads_or(!ok)) {
    if (tid == 0) mbar_drain(&bars[0], 0);
  } else {
    phi_tile_inplace(smem + L::kA, D / 64, 128, g.d, tid, 256);
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16_f32(128, kCols, 0, 0);
      const uint32_t a_addr = smem_u32(smem + L::kA);
      const uint32_t b_addr = smem_u32(smem + L::kB);
#pragma unroll
      for (int hl = 0; hl < 2; ++hl)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = smem_desc(a_addr + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kLayoutSw128);
          const uint64_t bd = smem_desc(b_addr + hl * L::kBTile + (kk >> 2) * (L::kRows * 128) + (kk & 3) * 32, 16,
                                        1024, kLayoutSw128);
          mma_ss(tmem, a, bd, idesc, (hl | kk) ? 1u : 0u);
        }
      mma_commit(&bars[1]);
      issued = true;
    }
    ok = mbar_wait(&bars[1], 0, ab);
    if (!__syncthreads_or(!ok)) {
      tc_fence_after();
      // ---------------------------------------------------------- TMEM -> r (two warps per row)
      const uint32_t quarter = warp & 3, half = warp >> 2;
      const int row = quarter * 32 + lane;
      const int col0 = half * (D / 2);
      const int d = g.d;
      float num[D / 2];
#pragma unroll
      for (int i = 0; i < D / 64; ++i) {
        uint32_t r[32];
        tmem_ld32(tmem_addr(tmem, quarter * 32, col0 + 32 * i), r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) num[32 * i + e] = __uint_as_float(r[e]);
      }
      uint32_t dr;
      tmem_ld1(tmem_addr(tmem, quarter * 32, D), dr);
      tmem_wait_ld();
      const bool empty = state_tokens(c, g) == 0;
      const float inv_den = empty ? 0.f : 1.0f / __uint_as_float(dr);
      float ss = 0.f;
#pragma unroll
      for (int a = 0; a < D / 2; ++a) {
        num[a] *= inv_den;
        if (col0 + a < d) ss = fmaf(num[a], num[a], ss);
      }
      ss_part[half * 128 + row] = ss;
      __syncthreads();
      const float inv_rms = (p.flags & 4) ? 1.0f : rsqrtf((ss_part[row] + ss_part[128 + row]) / (float)d + g.eps);
#pragma unroll
      for (int j = 0; j < D / 8; ++j) {
        const float4 v = make_float4(num[4 * j] * inv_rms, num[4 * j + 1] * inv_rms, num[4 * j + 2] * inv_rms,
                                     num[4 * j + 3] * inv_rms);
        *r_chunk<D>(smem + L::kR, row, col0 / 4 + j) = v;
      }
      __syncthreads();
      // ---------------------------------------------------------- coalesced merge
      const int c8s = d / 8;
      const int items = 128 * c8s;
      const size_t tok0 = (size_t)b * g.N + (size_t)(c * g.rows_per_chunk + r0);
#pragma unroll 4
      for (int it = tid; it < items; it += 256) {
        const int rr = it / c8s, c8 = it - rr * c8s;
        if (rr >= nrows) continue;
        const size_t tok = tok0 + rr;
        float os[8], gs[8], gl[8], o[8];
        load8<false>(p.o_s, (tok * g.H + h) * D + c8 * 8, os);
        load8<FP32>(p.gate_s, (tok * g.H + h) * d + c8 * 8, gs);
        load8<FP32>(p.gate_l, (tok * g.H + h) * d + c8 * 8, gl);
        const float4 ra = *r_chunk<D>(smem + L::kR, rr, 2 * c8);
        const float4 rb = *r_chunk<D>(smem + L::kR, rr, 2 * c8 + 1);
        float r[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
        if (p.gamma && !(p.flags & 4)) {
          const float4 ga = __ldg(reinterpret_cast<const float4*>(p.gamma + h * d + c8 * 8));
          const float4 gb = __ldg(reinterpret_cast<const float4*>(p.gamma + h * d + c8 * 8) + 1);
          r[0] *= ga.x; r[1] *= ga.y; r[2] *= ga.z; r[3] *= ga.w;
          r[4] *= gb.x; r[5] *= gb.y; r[6] *= gb.z; r[7] *= gb.w;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float v;
          if (p.flags & 1) v = os[e];        // softmax branch only
          else if (p.flags & 6) v = r[e];    // linear read: normalised (2) or raw (4)
          else v = sigmoid_f(gs[e]) * os[e] + sigmoid_f(gl[e]) * r[e];
          o[e] = v;
        }
        store8<FP32>(p.out, (tok * g.H + h) * d + c8 * 8, o);
      }
    }
  }
  if (issued) mbar_drain(&bars[1], 0);  // the MMA finished before TMEM is released
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kAlloc);
  }
}

template <int D, bool FP32>
static cudaError_t launch_k4(const Maps& m, const K4Params& p, cudaStream_t st) {
  const int smem = K4Layout<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(k4_readout_merge<D, FP32>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.g.rows_per_chunk + 127) / 128, p.g.Nc, p.g.B * p.g.H);
  k4_readout_merge<D, FP32><<<grid, 256, smem, st>>>(m.q, p);
  return cudaGetLastError();
}

cudaError_t launch_readout_merge(const Maps& m, const K4Params& p, cudaStream_t st) {
  if (p.g.Dp == 128) return p.g.fp32_io ? launch_k4<128, true>(m, p, st) : launch_k4<128, false>(m, p, st);
  return p.g.fp32_io ? launch_k4<64, true>(m, p, st) : launch_k4<64, false>(m, p, st);
}

}  // namespace vdn
