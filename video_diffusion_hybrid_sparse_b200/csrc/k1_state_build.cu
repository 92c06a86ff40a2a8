// k1_state_build.cu - linear-attention states of the VDN-H3 linear branch
// (article section 双分支混合注意力机制: the frame-wise linear memory).
//
// For every (batch, head) and state segment -- the non-anchor frames of one
// chunk, or the text -- the states are
//
//     [S | z] = phi(K)^T [V | 1],   S: d x d,  z: d,   phi = elu + 1,
//
// computed on the tensor cores with bf16 operands and fp32 accumulation in
// TMEM.  Anchor frames get no state (no state ever reads them).
//
// Work split (stream-K): the 128-token tiles of every (batch, head, segment)
// form one list, (batch, head)-major; the grid is one wave of CTAs and CTA k
// takes the k-th of `grid` equal contiguous ranges of that list, so every SM
// streams the same number of tiles.  A CTA accumulates over the run of its
// tiles that lies in one segment (a "piece") and writes that run's sum as one
// partial to the segment's slot for this CTA; the scan adds a segment's
// partials.  Partials are stored transposed, part[n][a] with row n = value
// column (row Dp holds z) and a = phi(k) slot, which is the K-major order the
// readout consumes.
//
// Roles (22 warps):
//   * warp 0 (one thread): TMA loads of the K and V tiles (128-byte swizzle),
//     three stages;
//   * warps 2-17: phi in place on the K tile (rows past the segment and padded
//     head_dim columns zeroed), fenced to the async proxy;
//   * warp 1 (one thread): D[:, 0:Dp] += phi(K)^T V and D[:, Dp:Dp+16] +=
//     phi(K)^T 1 (both operands MN-major, M = 128 head_dim slots; B = a block
//     of bf16 ones gives z) into one of two TMEM accumulators, one per piece
//     in turn, so a piece's read-out overlaps the next piece's products;
//   * warps 18-21: read a finished accumulator (TMEM lane = phi slot) and
//     store the partial.
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
  static constexpr int kCols = D + 16;                     // accumulator columns: values, z (+ padding)
  static constexpr int kAccCols = kCols <= 128 ? 128 : 256;  // one accumulator slot
};

enum { kFull = 0, kPhi = 3, kEmpty = 6, kAccFull = 9, kAccEmpty = 11, kDone = 13, kNumBars1 = 14 };
constexpr int kPhiWarps = 16;        // warps 2..17
constexpr int kPhiThreads = 32 * kPhiWarps;
constexpr int kEpiWarp0 = 2 + kPhiWarps;  // warps 18..21
constexpr int kK1Threads = 32 * (kEpiWarp0 + 4);

// Walk over the tiles of this CTA's range: (batch, head), tile within the
// (batch, head) and its segment, advanced one tile at a time (one division
// at the start of the range, none per tile).
struct SbCursor {
  int bh, lt, seg;

  __device__ __forceinline__ SbCursor(long long t, const StatePlan& sp) {
    bh = (int)(t / sp.tiles_per_bh);
    lt = (int)(t - (long long)bh * sp.tiles_per_bh);
    seg = sb_seg_of(lt, sp);
  }
  // The tile is the last of its segment (the next one starts another piece).
  __device__ __forceinline__ bool seg_ends(const StatePlan& sp) const { return lt + 1 == sp.seg_tile0[seg + 1]; }
  __device__ __forceinline__ void next(const StatePlan& sp) {
    if (++lt == sp.tiles_per_bh) {
      lt = 0;
      seg = 0;
      ++bh;
    } else if (lt == sp.seg_tile0[seg + 1]) {
      ++seg;
    }
  }
  __device__ __forceinline__ bool text(const StatePlan& sp) const { return seg >= sp.n_vsegs; }
  // first token row of the tile in the [B * N] video or [B * T] text rows
  __device__ __forceinline__ int row(const Geom& g, const StatePlan& sp) const {
    const int b = bh / g.H;
    return (text(sp) ? b * g.T : b * (int)g.N) + sp.seg_row0[seg] + (lt - sp.seg_tile0[seg]) * 128;
  }
  __device__ __forceinline__ int n_valid(const StatePlan& sp) const {
    return min(128, sp.seg_rows[seg] - (lt - sp.seg_tile0[seg]) * 128);
  }
};

}  // namespace

template <int D>
__global__ void __launch_bounds__(kK1Threads, 1)
    k1_state_build(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_tk, const __grid_constant__ CUtensorMap tm_tv,
                   const __grid_constant__ K1Params p) {
  using L = K1Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + kNumBars1 * 8);
  int* abort_flag = reinterpret_cast<int*>(smem + L::kBar + kNumBars1 * 8 + 4);

  const Geom& g = p.g;
  const StatePlan& sp = p.sp;
  const long long t_begin = sp.grid > 0 ? sb_range_start(blockIdx.x, sp) : 0;
  const long long t_end = sp.grid > 0 ? sb_range_start(blockIdx.x + 1, sp) : 0;
  const int ntiles = (int)(t_end - t_begin);
  const uint32_t warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0 && blockIdx.x == 0 && p.scan_counter) *p.scan_counter = 0ull;
  if (blockIdx.x == 0 && p.scan_done)
    for (int i = threadIdx.x; i < p.g.B * p.g.H; i += blockDim.x) p.scan_done[i] = 0u;
  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&bars[kFull + s], 1);
      mbar_init(&bars[kPhi + s], kPhiThreads);
      mbar_init(&bars[kEmpty + s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bars[kAccFull + a], 1);
      mbar_init(&bars[kAccEmpty + a], 128);
    }
    mbar_init(&bars[kDone], 1);
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
    tmem_alloc(tmem_slot, 2 * L::kAccCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const CtaAbort ab{abort_flag, p.status, p.record, 1};

  if (warp == 0) {
    // ------------------------------------------------------------ loads
    if (lane == 0) {
      int i = 0;
      bool ok = true;
      SbCursor cur(t_begin, sp);
      for (; i < ntiles; ++i, cur.next(sp)) {
        const int st = i % L::kStages;
        const uint32_t ph = (i / L::kStages) & 1;
        if (!mbar_wait(&bars[kEmpty + st], ph ^ 1, ab)) { ok = false; break; }
        const int h = cur.bh % g.H, row = cur.row(g, sp);
        const CUtensorMap* mk = cur.text(sp) ? &tm_tk : &tm_k;
        const CUtensorMap* mv = cur.text(sp) ? &tm_tv : &tm_v;
        mbar_expect_tx(&bars[kFull + st], (D / 64) * 16384 * 2);
        uint8_t* sa = smem + st * L::kStage;
        uint8_t* sb = sa + L::kATile;
        for (int bx = 0; bx < D / 64; ++bx) {
          tma_load_2d(sa + bx * 16384, mk, &bars[kFull + st], h * D + bx * 64, row);
          tma_load_2d(sb + bx * 16384, mv, &bars[kFull + st], h * D + bx * 64, row);
        }
      }
      if (!ok)
        for (int k = (i > L::kStages ? i - L::kStages : 0); k < i; ++k)
          mbar_drain(&bars[kFull + k % L::kStages], (k / L::kStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t idesc_v = idesc_bf16_f32(128, D, 1, 1);
      constexpr uint32_t idesc_1 = idesc_bf16_f32(128, 16, 1, 1);
      const uint32_t ones = smem_u32(smem + L::kOnes);
      // failure-path test: wait (with a short limit) for the first
      // accumulator phase, which only this thread's own commit completes; the
      // wait runs out, the CTA gives up and the status word records the timeout
      const bool injected = p.inject_timeout && blockIdx.x == 0 && !mbar_wait(&bars[kAccFull], 0, ab, 10000000ll);
      int piece = 0;
      bool first = true;  // first tile of the current piece
      SbCursor cur(t_begin, sp);
      for (int i = 0; i < ntiles && !injected; ++i, cur.next(sp)) {
        const int st = i % L::kStages;
        const int a = piece & 1;
        if (first && !mbar_wait(&bars[kAccEmpty + a], ((piece >> 1) & 1) ^ 1, ab)) break;
        if (!mbar_wait(&bars[kPhi + st], (i / L::kStages) & 1, ab)) break;
        tc_fence_after();
        const uint32_t acc = tmem + a * L::kAccCols;
        const uint32_t sa = smem_u32(smem + st * L::kStage);
        const uint32_t sb = sa + L::kATile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t da = smem_desc(sa + kk * 2048, 16384, 1024, kLayoutSw128);
          const uint64_t bv = smem_desc(sb + kk * 2048, 16384, 1024, kLayoutSw128);
          const uint64_t b1 = smem_desc(ones, 256, 256, kLayoutNone);
          const uint32_t accum = (!first || kk > 0) ? 1u : 0u;
          mma_ss(acc, da, bv, idesc_v, accum);
          mma_ss(acc + D, da, b1, idesc_1, accum);
        }
        mma_commit(&bars[kEmpty + st]);
        first = i + 1 == ntiles || cur.seg_ends(sp);  // this tile ends its piece
        if (first) {
          mma_commit(&bars[kAccFull + a]);
          ++piece;
        }
      }
      // every MMA of this thread completes before TMEM is released
      mma_commit(&bars[kDone]);
    }
  } else if (warp < kEpiWarp0) {
    // ------------------------------------------------------------ phi workers
    const int tid = threadIdx.x - 64;
    SbCursor cur(t_begin, sp);
    for (int i = 0; i < ntiles; ++i, cur.next(sp)) {
      const int st = i % L::kStages;
      const bool got = mbar_wait(&bars[kFull + st], (i / L::kStages) & 1, ab);
      if (__any_sync(0xffffffffu, !got)) break;
      phi_tile_inplace<D / 64 * 1024 / kPhiThreads>(smem + st * L::kStage, D / 64, cur.n_valid(sp), g.d, tid,
                                                     kPhiThreads);
      fence_proxy_async_smem();
      mbar_arrive(&bars[kPhi + st]);
    }
  } else {
    // ------------------------------------------------------------ read-out of finished pieces
    const uint32_t quarter = warp & 3;
    const int a = quarter * 32 + lane;  // TMEM lane = head_dim slot of phi(k)
    int piece = 0;
    SbCursor cur(t_begin, sp);
    for (int i = 0; i < ntiles; ++i, cur.next(sp)) {
      if (!(i + 1 == ntiles || cur.seg_ends(sp))) continue;  // not the last tile of a piece
      const int buf = piece & 1;
      const bool got = mbar_wait(&bars[kAccFull + buf], (piece >> 1) & 1, ab);
      if (__any_sync(0xffffffffu, !got)) break;
      tc_fence_after();
      // this CTA's contributor index within the segment
      const long long seg_first = (long long)cur.bh * sp.tiles_per_bh + sp.seg_tile0[cur.seg];
      const int u = (int)blockIdx.x - sb_cta_of(seg_first, sp);
      float* dst = p.parts + sb_slot(cur.bh, cur.seg, u, sp) * (long long)(D + 1) * D;
      const uint32_t acc = tmem + buf * L::kAccCols;
#pragma unroll
      for (int c = 0; c < L::kCols / 16; ++c) {
        uint32_t r[16];
        tmem_ld16(tmem_addr(acc, quarter * 32, 16 * c), r);
        tmem_wait_ld();
        if (a < D) {
          if (16 * c < D) {
#pragma unroll
            for (int e = 0; e < 16; ++e) dst[(size_t)(16 * c + e) * D + a] = __uint_as_float(r[e]);
          } else {
            dst[(size_t)D * D + a] = __uint_as_float(r[0]);  // z
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars[kAccEmpty + buf]);
      ++piece;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    // every MMA of this CTA completed (kDone) before the columns are released
    mbar_drain(&bars[kDone], 0);
    tmem_dealloc(tmem, 2 * L::kAccCols);
  }
}

cudaError_t launch_state_build(const Maps& m, const K1Params& p, cudaStream_t st) {
  // one CTA even without tiles: it zeroes the scan counter
  const int grid = p.sp.grid > 0 ? p.sp.grid : 1;
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
