// k4_readout_merge.cu - linear-branch readout and gated fusion of the VDN-H3
// hybrid attention (article sections 双分支混合注意力机制 and
// 自适应门控融合双分支输出).
//
// Work item: 128 query rows (a tile) of one (batch, chunk, head).  Persistent
// CTAs: with S = max(1, SMs / H) streams, CTA k keeps head k % H and walks the
// tile positions (batch, chunk, tile) s, s + S, s + 2S, ... of stream
// s = k / H.  At any moment the CTAs therefore cover every head of a few
// neighbouring tiles, so together they read whole [H, d] token rows from HBM
// rather than scattered 256-byte pieces, and consecutive items of a CTA mostly
// share the chunk's readout operand M_c.  Warp roles:
//   * warp 0 (one thread): bulk-copies M_c = F_c + B_c as a bf16 hi/lo pair
//     (rows: value column b, row Dp = z; K = head_dim slot a; already in the
//     K-major 128-byte-swizzled operand image) whenever (batch, chunk, head)
//     changes, and TMA-loads each q tile into one of two buffers;
//   * warp 1 (one thread): D = phi(Q) M_hi^T + phi(Q) M_lo^T on the tensor
//     cores (M = 128, N = Dp + 16, fp32) into one of two TMEM accumulators:
//     columns [0, Dp) are the numerators phi(q)^T M, column Dp the
//     denominator phi(q) . z;
//   * warps 2-9 (256 threads): apply phi to q tile i in place, then finish
//     tile i-1 while the MMA of tile i runs: two warps per TMEM row compute
//     o_l = num / den (0 when the chunk's states hold no token) and the
//     row's RMS, stage r = o_l / sqrt(mean(o_l^2) + eps) in shared memory, and
//     a coalesced pass reads o_s and both gates (prefetched into L2 one tile
//     ahead), applies gamma and writes out = sigmoid(g_s) o_s + sigmoid(g_l) r
//     (SPLIT: the two terms to out and out_linear).  Rows of a GLOBAL anchor
//     query read nothing through the states (o_l = 0).
// Every wait is bounded; the worker warps agree on giving up through a
// barrier with an OR reduction, so none is left waiting for another.
#include "k4_common.cuh"
#include "kernels.h"
#include "phi.cuh"
#include "sm100.cuh"

namespace vdn {

namespace {

using namespace k4;

template <int D>
struct K4Layout {
  static constexpr int kRows = D + 16;
  static constexpr int kATile = 128 * D * 2;
  static constexpr int kBTile = kRows * D * 2;
  static constexpr int kA = 0;                       // two q tiles
  static constexpr int kB = kA + 2 * kATile;         // M_c hi, lo
  static constexpr int kR = kB + 2 * kBTile;         // r staging [128][D] fp32
  static constexpr int kSs = kR + 128 * D * 4;       // [2][128] partial sums of squares
  static constexpr int kBar = kSs + 2 * 128 * 4;
  static constexpr int kBytes = kBar + 128 + 1024;
  static constexpr int kAccCols = D + 16 <= 128 ? 128 : 256;  // one accumulator
};

enum { kAFull = 0, kAReady = 2, kAEmpty = 4, kAccFull = 6, kAccEmpty = 8, kBFull = 10, kBEmpty = 11, kDone4 = 12,
       kNumBars4 = 13 };
constexpr int kWorkers = 256;
constexpr int kK4Threads = 64 + kWorkers;

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
__global__ void __launch_bounds__(kK4Threads, 1)
    k4_readout_merge(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ K4Params p, int n_streams) {
  using L = K4Layout<D>;
  constexpr int kCols = D + 16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + kNumBars4 * 8);
  int* abort_flag = reinterpret_cast<int*>(smem + L::kBar + kNumBars4 * 8 + 4);
  float* ss_part = reinterpret_cast<float*>(smem + L::kSs);

  const Geom& g = p.g;
  const int tiles = (g.rows_per_chunk + 127) / 128;
  const int head = blockIdx.x % g.H, stream = blockIdx.x / g.H;
  const int positions = g.B * g.Nc * tiles;
  const int n_mine = stream < positions ? (positions - stream + n_streams - 1) / n_streams : 0;
  const int first = 0, last = n_mine;  // item index i in [first, last)
  const uint32_t warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[kAFull + s], 1);
      mbar_init(&bars[kAReady + s], kWorkers);
      mbar_init(&bars[kAEmpty + s], 1);
      mbar_init(&bars[kAccFull + s], 1);
      mbar_init(&bars[kAccEmpty + s], kWorkers);
    }
    mbar_init(&bars[kBFull], 1);
    mbar_init(&bars[kBEmpty], 1);
    mbar_init(&bars[kDone4], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * L::kAccCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const CtaAbort ab{abort_flag, p.status, p.record, 41};

  if (warp == 0) {
    // ------------------------------------------------------------ loads
    if (lane == 0) {
      int prev_key = -1, b_loads = 0, a_issued = 0;
      bool ok = true;
      for (int item = first; item < last && ok; ++item) {
        const Item4 it = decode4(item, head, stream, n_streams, g, tiles);
        const int i = item - first, s = i & 1;
        if (it.key != prev_key) {
          if (b_loads > 0 && !mbar_wait(&bars[kBEmpty], (b_loads - 1) & 1, ab)) { ok = false; break; }
          mbar_expect_tx(&bars[kBFull], (uint32_t)(2 * L::kBTile));
          bulk_load(smem + L::kB, p.mt + (((size_t)it.b * g.Nc + it.c) * g.H + it.h) * 2 * (size_t)L::kBTile,
                    (uint32_t)(2 * L::kBTile), &bars[kBFull]);
          ++b_loads;
          prev_key = it.key;
        }
        if (!mbar_wait(&bars[kAEmpty + s], ((i >> 1) & 1) ^ 1, ab)) { ok = false; break; }
        mbar_expect_tx(&bars[kAFull + s], (uint32_t)L::kATile);
        for (int bx = 0; bx < D / 64; ++bx)
          tma_load_2d(smem + L::kA + s * L::kATile + bx * 16384, &tm_q, &bars[kAFull + s], it.h * D + bx * 64,
                      it.b * (int)g.N + it.c * g.rows_per_chunk + it.tile * 128);
        ++a_issued;
      }
      if (!ok) {
        for (int k = (a_issued > 2 ? a_issued - 2 : 0); k < a_issued; ++k)
          mbar_drain(&bars[kAFull + (k & 1)], (k >> 1) & 1);
        if (b_loads > 0) mbar_drain(&bars[kBFull], (b_loads - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, kCols, 0, 0);
      int prev_key = -1, b_loads = 0;
      for (int item = first; item < last; ++item) {
        const Item4 it = decode4(item, head, stream, n_streams, g, tiles);
        const int i = item - first, s = i & 1;
        const uint32_t ph = (i >> 1) & 1;
        if (it.key != prev_key) {
          if (p.stall_ns > 0 && i > 0) sleep_ns(p.stall_ns);  // debug: let the other warps run ahead
          ++b_loads;
          prev_key = it.key;
          if (!mbar_wait(&bars[kBFull], (b_loads - 1) & 1, ab)) break;
        }
        if (!mbar_wait(&bars[kAReady + s], ph, ab)) break;
        if (!mbar_wait(&bars[kAccEmpty + s], ph ^ 1, ab)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + L::kA + s * L::kATile);
        const uint32_t b_addr = smem_u32(smem + L::kB);
#pragma unroll
        for (int hl = 0; hl < 2; ++hl)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = smem_desc(a_addr + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, kLayoutSw128);
            const uint64_t bd = smem_desc(b_addr + hl * L::kBTile + (kk >> 2) * (L::kRows * 128) + (kk & 3) * 32,
                                          16, 1024, kLayoutSw128);
            mma_ss(tmem + s * L::kAccCols, a, bd, idesc, (hl | kk) ? 1u : 0u);
          }
        mma_commit(&bars[kAccFull + s]);
        mma_commit(&bars[kAEmpty + s]);
        const bool key_ends = item + 1 >= last || decode4(item + 1, head, stream, n_streams, g, tiles).key != it.key;
        if (key_ends) mma_commit(&bars[kBEmpty]);
      }
      mma_commit(&bars[kDone4]);
      mbar_drain(&bars[kDone4], 0);
    }
  } else {
    // ------------------------------------------------------------ workers
    const int tid = threadIdx.x - 64;
    const uint32_t quarter = warp & 3, half = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;
    const int col0 = half * (D / 2);
    const int d = g.d;
    const int c8s = d / 8;
    // output: 0 merged, 1 softmax branch only, 2 linear read (normalised or raw)
    const int mode = (p.flags & 1) ? 1 : ((p.flags & 6) ? 2 : 0);
    const bool use_gamma = p.gamma != nullptr && !(p.flags & 4);
    const bool split = p.out_linear != nullptr;  // out gets sigmoid(g_s) o_s, out_linear sigmoid(g_l) r

    // Finish tile `item` (slot s): TMEM -> r -> coalesced merge.  Returns false on a timeout.
    auto finish = [&](int item, int s) -> bool {
      const Item4 it = decode4(item, head, stream, n_streams, g, tiles);
      const int i = item - first;
      const bool got = mbar_wait(&bars[kAccFull + s], (i >> 1) & 1, ab);
      if (workers_any(!got)) return false;
      tc_fence_after();
      float num[D / 2];
#pragma unroll
      for (int k = 0; k < D / 64; ++k) {
        uint32_t r[32];
        tmem_ld32(tmem_addr(tmem + s * L::kAccCols, quarter * 32, col0 + 32 * k), r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) num[32 * k + e] = __uint_as_float(r[e]);
      }
      uint32_t dr;
      tmem_ld1(tmem_addr(tmem + s * L::kAccCols, quarter * 32, D), dr);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars[kAccEmpty + s]);  // the accumulator may be overwritten now
      // zero read: the chunk's states hold no token, or the row is a GLOBAL anchor query
      const int qrow = it.c * g.rows_per_chunk + it.tile * 128 + row;
      const bool empty = state_tokens(it.c, g) == 0 || no_linear_read(qrow / g.P, g);
      const float inv_den = empty ? 0.f : 1.0f / __uint_as_float(dr);
      float ss = 0.f;
#pragma unroll
      for (int a = 0; a < D / 2; ++a) {
        num[a] *= inv_den;
        if (col0 + a < d) ss = fmaf(num[a], num[a], ss);
      }
      ss_part[half * 128 + row] = ss;
      workers_any(false);
      const float inv_rms = (p.flags & 4) ? 1.0f : rsqrtf((ss_part[row] + ss_part[128 + row]) / (float)d + g.eps);
#pragma unroll
      for (int j = 0; j < D / 8; ++j) {
        const float4 v = make_float4(num[4 * j] * inv_rms, num[4 * j + 1] * inv_rms, num[4 * j + 2] * inv_rms,
                                     num[4 * j + 3] * inv_rms);
        *r_chunk<D>(smem + L::kR, row, col0 / 4 + j) = v;
      }
      workers_any(false);
      // coalesced merge: each thread issues the raw 16-byte loads of a whole
      // batch of items (eight for bf16 gates, two for fp32) before using any
      constexpr int kBatch = FP32 ? 2 : 4;
      constexpr int kGv = FP32 ? 2 : 1;  // 16-byte vectors per 8 gate values
      const int nrows = min(128, g.rows_per_chunk - it.tile * 128);
      const int items = 128 * c8s;
      const size_t tok0 = (size_t)it.b * g.N + (size_t)(it.c * g.rows_per_chunk + it.tile * 128);
      for (int e0 = tid; e0 < items; e0 += kBatch * kWorkers) {
        uint4 vos[kBatch], vgs[kBatch][kGv], vgl[kBatch][kGv];
        size_t tok[kBatch];
        int rrs[kBatch], c8v[kBatch];
        bool valid[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int e = e0 + u * kWorkers;
          const int rr = e / c8s, c8 = e - rr * c8s;
          valid[u] = e < items && rr < nrows;
          rrs[u] = valid[u] ? rr : 0;
          c8v[u] = valid[u] ? c8 : 0;
          tok[u] = tok0 + rrs[u];
          const size_t row_h = tok[u] * g.H + it.h;
          vos[u] = __ldg(reinterpret_cast<const uint4*>(p.o_s + row_h * D + c8v[u] * 8));
          const uint4* gsp = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.gate_s) +
                                                            (row_h * d + c8v[u] * 8) * (FP32 ? 4 : 2));
          const uint4* glp = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.gate_l) +
                                                            (row_h * d + c8v[u] * 8) * (FP32 ? 4 : 2));
#pragma unroll
          for (int k = 0; k < kGv; ++k) {
            vgs[u][k] = __ldg(gsp + k);
            vgl[u][k] = __ldg(glp + k);
          }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const float4 ra = *r_chunk<D>(smem + L::kR, rrs[u], 2 * c8v[u]);
          const float4 rb = *r_chunk<D>(smem + L::kR, rrs[u], 2 * c8v[u] + 1);
          float r[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
          if (use_gamma) {
            const float4 ga = __ldg(reinterpret_cast<const float4*>(p.gamma + it.h * d + c8v[u] * 8));
            const float4 gb = __ldg(reinterpret_cast<const float4*>(p.gamma + it.h * d + c8v[u] * 8) + 1);
            r[0] *= ga.x; r[1] *= ga.y; r[2] *= ga.z; r[3] *= ga.w;
            r[4] *= gb.x; r[5] *= gb.y; r[6] *= gb.z; r[7] *= gb.w;
          }
          const uint32_t ow[4] = {vos[u].x, vos[u].y, vos[u].z, vos[u].w};
          float os[8], gs[8], gl[8];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            os[2 * k] = bf16_lo(ow[k]);
            os[2 * k + 1] = bf16_hi(ow[k]);
          }
          if constexpr (FP32) {
            const float* fs = reinterpret_cast<const float*>(&vgs[u][0]);
            const float* fl = reinterpret_cast<const float*>(&vgl[u][0]);
#pragma unroll
            for (int k = 0; k < 8; ++k) { gs[k] = fs[k]; gl[k] = fl[k]; }
          } else {
            const uint32_t sw[4] = {vgs[u][0].x, vgs[u][0].y, vgs[u][0].z, vgs[u][0].w};
            const uint32_t lw[4] = {vgl[u][0].x, vgl[u][0].y, vgl[u][0].z, vgl[u][0].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              gs[2 * k] = bf16_lo(sw[k]); gs[2 * k + 1] = bf16_hi(sw[k]);
              gl[2 * k] = bf16_lo(lw[k]); gl[2 * k + 1] = bf16_hi(lw[k]);
            }
          }
          float o[8];
          const size_t oidx = (tok[u] * g.H + it.h) * d + c8v[u] * 8;
          if (split) {
            float ol[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              o[k] = sigmoid_f(gs[k]) * os[k];
              ol[k] = sigmoid_f(gl[k]) * r[k];
            }
            if (valid[u]) store8<FP32>(p.out_linear, oidx, ol);
          } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float merged = sigmoid_f(gs[k]) * os[k] + sigmoid_f(gl[k]) * r[k];
              o[k] = mode == 0 ? merged : (mode == 1 ? os[k] : r[k]);
            }
          }
          if (valid[u]) store8<FP32>(p.out, oidx, o);
        }
      }
      workers_any(false);  // r staging is rewritten by the next tile
      return true;
    };

    bool ok = true;
    for (int item = first; item < last && ok; ++item) {
      const Item4 it = decode4(item, head, stream, n_streams, g, tiles);
      const int i = item - first, s = i & 1;
      // bring this tile's o_s and gate rows into L2 for its merge (one tile later):
      // thread t covers row t % 128 of o_s (t < 128) or of both gates (t >= 128)
      {
        const int rr = tid & 127;
        if (rr < min(128, g.rows_per_chunk - it.tile * 128)) {
          const size_t row_h = ((size_t)it.b * g.N + (size_t)(it.c * g.rows_per_chunk + it.tile * 128 + rr)) * g.H + it.h;
          if (tid < 128) {
            const uint8_t* o = reinterpret_cast<const uint8_t*>(p.o_s + row_h * D);
#pragma unroll
            for (int l = 0; l < D * 2 / 128; ++l) prefetch_l2(o + l * 128);
          } else {
            const size_t rb = row_h * (size_t)d * (FP32 ? 4 : 2);
            for (int l = 0; l < d * (FP32 ? 4 : 2); l += 128) {
              prefetch_l2(static_cast<const uint8_t*>(p.gate_s) + rb + l);
              prefetch_l2(static_cast<const uint8_t*>(p.gate_l) + rb + l);
            }
          }
        }
      }
      const bool got = mbar_wait(&bars[kAFull + s], (i >> 1) & 1, ab);
      if (workers_any(!got)) { ok = false; break; }
      phi_tile_inplace<D / 64 * 1024 / kWorkers>(smem + L::kA + s * L::kATile, D / 64, 128, d, tid, kWorkers);
      fence_proxy_async_smem();
      mbar_arrive(&bars[kAReady + s]);
      if (item > first) ok = finish(item - 1, (i - 1) & 1);
    }
    if (ok && last > first) finish(last - 1, (last - 1 - first) & 1);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * L::kAccCols);
  }
}

template <int D, bool FP32>
static cudaError_t launch_k4(const Maps& m, const K4Params& p, cudaStream_t st) {
  const int smem = K4Layout<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(k4_readout_merge<D, FP32>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int tiles = (p.g.rows_per_chunk + 127) / 128;
  const int positions = tiles * p.g.Nc * p.g.B;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int n_streams = sms / p.g.H;
  if (n_streams < 1) n_streams = 1;
  if (n_streams > positions) n_streams = positions;
  k4_readout_merge<D, FP32><<<n_streams * p.g.H, kK4Threads, smem, st>>>(m.q, p, n_streams);
  return cudaGetLastError();
}

cudaError_t launch_readout_merge(const Maps& m, const K4Params& p, cudaStream_t st) {
  if (p.g.Dp == 128) return p.g.fp32_io ? launch_k4<128, true>(m, p, st) : launch_k4<128, false>(m, p, st);
  return p.g.fp32_io ? launch_k4<64, true>(m, p, st) : launch_k4<64, false>(m, p, st);
}

}  // namespace vdn
