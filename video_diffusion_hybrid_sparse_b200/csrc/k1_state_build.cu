// k1_state_build.cu - per-slice linear-attention states of the VDN-H3 linear
// branch (article section 双分支混合注意力机制: the frame-wise linear memory).
//
// For one slice of up to 2048 key tokens of one non-anchor frame (or of the
// text), one batch and one head, it computes on the tensor cores
//
//     [S | z] = phi(K)^T [V | 1],   S: d x d,  z: d,   phi = elu + 1,
//
// with bf16 operands and fp32 accumulation in TMEM.  Anchor frames get no
// state (no state ever reads them).  The output partial is stored transposed,
// part[b_col][a] with row Dp holding z, which is the K-major order the
// readout consumes.
//
// Per 128-token tile: TMA brings the K tile and the V tile (128-byte swizzle);
// sixteen warps apply phi in place on the K tile (zeroing rows past the slice and
// padded head_dim columns) and fence it to the async proxy; one thread issues
//   D[:, 0:Dp]    += phi(K)^T V      (A and B both MN-major, M = 128 = head_dim slots)
//   D[:, Dp:Dp+16] += phi(K)^T 1     (B = a block of ones)
// Three pipeline stages keep the HBM stream busy.
#include "kernels.h"
#include "phi.cuh"
#include "sm100.cuh"

namespace vdn {

namespace {

template <int D>
struct K1Layout {
  static constexpr int kStages = 3;
  static constexpr int kATile = 128 * 128 * 2;  // K tile as A operand: always 128 head_dim slots (zero-padded)
  static constexpr int kBTile = 128 * D * 2;    // V tile
  static constexpr int kStage = kATile + kBTile;
  static constexpr int kOnes = kStages * kStage;
  static constexpr int kOnesBytes = 4096;
  static constexpr int kBar = kOnes + kOnesBytes;
  static constexpr int kBytes = kBar + 256 + 1024;
};

enum { kFull = 0, kPhi = 3, kEmpty = 6, kAcc = 9, kNumBars1 = 10 };
constexpr int kPhiThreads = 512;  // warps 2..17
constexpr int kK1Threads = 64 + kPhiThreads;

}  // namespace

template <int D>
__global__ void __launch_bounds__(kK1Threads, 1)
    k1_state_build(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_tk, const __grid_constant__ CUtensorMap tm_tv,
                   const __grid_constant__ K1Params p) {
  using L = K1Layout<D>;
  constexpr int kCols = D + 16;
  constexpr int kAlloc = kCols <= 128 ? 128 : 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + kNumBars1 * 8);
  int* abort_flag = reinterpret_cast<int*>(smem + L::kBar + kNumBars1 * 8 + 4);

  const Geom& g = p.g;
  // (batch, head) is the fastest grid index: CTAs that run together read
  // whole [H, d] token rows of k and v rather than scattered 256-byte pieces
  const int bh = blockIdx.x;
  const int part = blockIdx.y;
  const int b = bh / g.H, h = bh % g.H;
  const uint32_t warp = warp_id(), lane = lane_id();

  // token range of this part
  const bool text = part >= g.n_video_parts;
  int row0, ntok;
  if (!text) {
    const int f = part_frame(part, g);
    const int s = part % g.n_slices;
    row0 = b * (int)g.N + f * g.P + s * kSliceTokens;
    ntok = min(kSliceTokens, g.P - s * kSliceTokens);
  } else {
    const int tp = part - g.n_video_parts;
    row0 = b * g.T + tp * kSliceTokens;
    ntok = min(kSliceTokens, g.T - tp * kSliceTokens);
  }
  const int ntiles = (ntok + 127) / 128;
  const CUtensorMap* mk = text ? &tm_tk : &tm_k;
  const CUtensorMap* mv = text ? &tm_tv : &tm_v;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&bars[kFull + s], 1);
      mbar_init(&bars[kPhi + s], kPhiThreads);
      mbar_init(&bars[kEmpty + s], 1);
    }
    mbar_init(&bars[kAcc], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // ones block for z; zero the unused upper head_dim half of each A tile (D = 64)
  for (int i = threadIdx.x; i < L::kOnesBytes / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(smem + L::kOnes)[i] = 0x3F803F80u;  // two bf16 1.0
  if (D < 128) {
    for (int s = 0; s < L::kStages; ++s)
      for (int i = threadIdx.x; i < 16384 / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(smem + s * L::kStage + 16384)[i] = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(tmem_slot, kAlloc);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const CtaAbort ab{abort_flag, p.status, p.record, 1};

  if (warp == 0) {
    if (lane == 0) {
      int i = 0;
      bool ok = true;
      for (; i < ntiles; ++i) {
        const int st = i % L::kStages;
        const uint32_t ph = (i / L::kStages) & 1;
        if (!mbar_wait(&bars[kEmpty + st], ph ^ 1, ab)) { ok = false; break; }
        mbar_expect_tx(&bars[kFull + st], (D / 64) * 16384 * 2);
        uint8_t* sa = smem + st * L::kStage;
        uint8_t* sb = sa + L::kATile;
        for (int bx = 0; bx < D / 64; ++bx) {
          tma_load_2d(sa + bx * 16384, mk, &bars[kFull + st], h * D + bx * 64, row0 + i * 128);
          tma_load_2d(sb + bx * 16384, mv, &bars[kFull + st], h * D + bx * 64, row0 + i * 128);
        }
      }
      if (!ok)
        for (int k = (i > L::kStages ? i - L::kStages : 0); k < i; ++k)
          mbar_drain(&bars[kFull + k % L::kStages], (k / L::kStages) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_v = idesc_bf16_f32(128, D, 1, 1);
      constexpr uint32_t idesc_1 = idesc_bf16_f32(128, 16, 1, 1);
      const uint32_t ones = smem_u32(smem + L::kOnes);
      // failure-path test: wait (with a short limit) for the accumulator
      // phase, which only this thread's final commit completes; the wait runs
      // out, the CTA gives up and the status word records the timeout
      const bool injected = p.inject_timeout && blockIdx.x == 0 && blockIdx.y == 0 &&
                            !mbar_wait(&bars[kAcc], 0, ab, 10000000ll);
      for (int i = 0; i < ntiles && !injected; ++i) {
        const int st = i % L::kStages;
        if (!mbar_wait(&bars[kPhi + st], (i / L::kStages) & 1, ab)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + st * L::kStage);
        const uint32_t sb = sa + L::kATile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = smem_desc(sa + kk * 2048, 16384, 1024, kLayoutSw128);
          const uint64_t bv = smem_desc(sb + kk * 2048, 16384, 1024, kLayoutSw128);
          const uint64_t b1 = smem_desc(ones, 256, 256, kLayoutNone);
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          mma_ss(tmem, a, bv, idesc_v, acc);
          mma_ss(tmem + D, a, b1, idesc_1, acc);
        }
        mma_commit(&bars[kEmpty + st]);
      }
      mma_commit(&bars[kAcc]);
    }
  } else {
    // warps 2..17: phi workers; warps 2..5 then read the accumulator out
    const int tid = threadIdx.x - 64;
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      const int st = i % L::kStages;
      const bool got = mbar_wait(&bars[kFull + st], (i / L::kStages) & 1, ab);
      if (__any_sync(0xffffffffu, !got)) { ok = false; break; }
      phi_tile_inplace(smem + st * L::kStage, D / 64, ntok - i * 128, g.d, tid, kPhiThreads);
      fence_proxy_async_smem();
      mbar_arrive(&bars[kPhi + st]);
    }
    if (ok && warp < 6) {
      const bool got = mbar_wait(&bars[kAcc], 0, ab);
      if (!__any_sync(0xffffffffu, !got)) {
        tc_fence_after();
        const uint32_t quarter = warp & 3;
        const int a = quarter * 32 + lane;  // TMEM lane = head_dim slot of phi(k)
        float* dst = p.parts + (((size_t)part * g.B + b) * g.H + h) * (size_t)(D + 1) * D;
#pragma unroll
        for (int i = 0; i < kCols / 16; ++i) {
          uint32_t r[16];
          tmem_ld16(tmem_addr(tmem, quarter * 32, 16 * i), r);
          tmem_wait_ld();
          if (a < D) {
            if (16 * i < D) {
#pragma unroll
              for (int e = 0; e < 16; ++e) dst[(size_t)(16 * i + e) * D + a] = __uint_as_float(r[e]);
            } else {
              dst[(size_t)D * D + a] = __uint_as_float(r[0]);  // z
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    // every MMA of this CTA completed (kAcc) before the columns are released
    mbar_drain(&bars[kAcc], 0);
    tmem_dealloc(tmem, kAlloc);
  }
}

cudaError_t launch_state_build(const Maps& m, const K1Params& p, cudaStream_t st) {
  dim3 grid(p.g.B * p.g.H, p.g.n_parts);
  if (p.g.n_parts == 0) return cudaSuccess;
  if (p.g.Dp == 128) {
    const int smem = K1Layout<128>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(k1_state_build<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k1_state_build<128><<<grid, kK1Threads, smem, st>>>(m.k, m.v, m.tk, m.tv, p);
  } else {
    const int smem = K1Layout<64>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(k1_state_build<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k1_state_build<64><<<grid, kK1Threads, smem, st>>>(m.k, m.v, m.tk, m.tv, p);
  }
  return cudaGetLastError();
}

}  // namespace vdn
