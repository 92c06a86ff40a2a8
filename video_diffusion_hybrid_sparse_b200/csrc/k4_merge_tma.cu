// k4_merge_tma.cu - linear-branch readout and gated fusion of the VDN-H3
// hybrid attention (article sections 双分支混合注意力机制 and
// 自适应门控融合双分支输出) for bf16 tensors whose head_dim needs no padding
// (64 or 128): every input tile arrives by TMA and, on the merge path, the
// output tile leaves by TMA.
//
// The work is the list of (head, batch, chunk, 128-row tile) positions, head
// outermost; CTA k of G takes the contiguous range [k P / G, (k + 1) P / G)
// of the P positions, so the readout operand M_c (one per head, batch and
// chunk) changes only at a chunk boundary inside the range, and the grid is
// one CTA per SM whatever the head count.  Per tile:
//   * warp 0 (one thread) TMA-loads the q tile, and, one tile later, the
//     tile's o_s and gate_l tiles (128 rows x head_dim each), and gate_s only
//     when the softmax kernel left o_s ungated (o_s holds sigmoid(g_s) * o_s
//     when it was given the gate, and the gate_s slot then holds a second q
//     tile, so two q tiles are in flight); it bulk-copies M_c (bf16 hi/lo readout
//     operand) when the chunk changes, prefetches the next tiles into L2 and,
//     once the workers have merged a full tile into the o_s buffer, TMA-stores
//     it to out before that buffer is reloaded;
//   * warp 1 (one thread): D = phi(Q) M_hi^T + phi(Q) M_lo^T (M = 128,
//     N = head_dim + 16, fp32) into one of two TMEM accumulators: numerators
//     in the first head_dim columns, the denominator phi(q) . z after them;
//     phi(Q) itself is the A operand, read from TMEM (columns of the same
//     accumulator slot that the accumulator leaves free);
//   * warps 2-17 (512 threads): warp w holds TMEM lanes 32 (w % 4) .. + 31
//     (the tile's rows) and a quarter of the columns, (w - 2) / 4.  Each
//     thread applies phi to its quarter row of the q tile and stores it to
//     TMEM as bf16 (its q slot is free for a later tile's load right
//     after), then finishes the previous tile: o_l = num / den (0 for an empty
//     state or a GLOBAL anchor query row), the row's sum of squares from the
//     four quarter rows, and the merge out = sigmoid(g_s) o_s +
//     sigmoid(g_l) r, r = o_l / sqrt(mean(o_l^2) + eps) * gamma, over its own
//     8-column pieces of the 128-byte-swizzled shared tiles.  A full tile's
//     output overwrites its o_s pieces in place and goes out in one TMA store;
//     a ragged tile (the end of a chunk whose rows are not a multiple of 128),
//     the SPLIT output and the debug outputs are stored 16 bytes at a time.
// Every wait is bounded; worker warps agree on giving up through barriers
// with an OR reduction, so none is left waiting for another.
#include <type_traits>

#include "k4_common.cuh"
#include "kernels.h"
#include "phi.cuh"
#include "sm100.cuh"

namespace vdn {

namespace {

using namespace k4;

template <int D>
struct K4TLayout {
  static constexpr int kRows = D + 16;
  static constexpr int kTile = 128 * D * 2;   // one bf16 128-row tile (q, o_s, g_s or g_l)
  static constexpr int kBTile = kRows * D * 2;
  static constexpr int kA = 0;                // q tile
  static constexpr int kB = kA + kTile;       // M_c hi, lo
  static constexpr int kG = kB + 2 * kBTile;  // o_s (then out), g_s, g_l tiles of the tile being merged
  static constexpr int kSs = kG + 3 * kTile;  // [2 tiles][4 quarters][128] sums of squares
  static constexpr int kBar = kSs + 2 * 4 * 128 * 4;
  static constexpr int kBytes = kBar + 128 + 1024;
  static constexpr int kAccCols = D + 16 <= 128 ? 128 : 256;  // one accumulator slot
  static constexpr int kPhiCol = kAccCols - D / 2;             // phi(Q) (bf16 pairs) at the slot's end
  static_assert(kPhiCol >= D + 16, "phi(Q) must not overlap the accumulator");
  static_assert(kBytes <= 227 * 1024, "shared memory");
};

enum {
  kTAFull = 0, kTAReady = 2, kTAEmpty = 4, kTAccFull = 6, kTAccEmpty = 8, kTBFull = 10, kTBEmpty = 11,
  kTGFull = 12, kTGEmpty = 13, kTDone = 14, kTNumBars = 15
};
// kTAFull + q / kTAEmpty + q: q tile slot q (the slot of tile i is i % nq;
// nq = 2 when the softmax kernel applied the gate, whose g_s slot in the G
// region then holds the second q tile, else 1).
// kTAReady + s: phi(Q) of a tile of accumulator slot s is in TMEM (workers);
// kTAEmpty: the workers have read the q tile out of shared memory (the
// producer may load the next one); kTGEmpty: the workers are done with the
// o_s / gate tiles (and, on the TMA-store path, have written the output tile
// over o_s).  kTAReady is one barrier per slot because the workers' next
// arrival depends only on the producer (q of the next tile), not on the MMA
// thread having seen the previous phase: with one barrier, a MMA thread held
// up on a readout-operand load could find two phases completed and wait on
// the parity of a third that never comes.  Per slot, the next arrival (tile
// i + 2) follows finish(i), which waits for the MMA of tile i, so the MMA
// thread is never a whole phase behind.
constexpr int kTWorkers = 512;
constexpr int kTThreads = 64 + kTWorkers;

// Byte offset of the 16-byte piece (8 bf16) of row `row`, columns
// [col, col + 8), in a 128-row tile loaded by TMA as 64-column boxes with
// the 128-byte swizzle.
__device__ __forceinline__ int piece_off(int row, int col) {
  const int box = col >> 6, chunk = (col & 63) >> 3;
  return box * 16384 + row * 128 + ((chunk ^ (row & 7)) << 4);
}

// 2-D tiled TMA store of the box at (x, y) from shared memory (bulk group).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the committed stores have read their shared-memory source.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until the committed stores are complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Barrier of all workers that also ORs a predicate.
__device__ __forceinline__ bool all_workers_any(bool pred) { return bar_any(1, kTWorkers, pred); }
// Barrier of the four worker warps that hold the same TMEM lanes (named
// barrier 2 + lane quarter), also ORing a predicate.
__device__ __forceinline__ bool quad_any(uint32_t quarter, bool pred) { return bar_any(2 + quarter, 128, pred); }

// Position `pos` of the (head, batch, chunk, tile) list.
__device__ __forceinline__ Item4 decode_pos(int pos, const Geom& g, int tiles) {
  Item4 it;
  it.tile = pos % tiles;
  const int rem = pos / tiles;  // (head, batch, chunk): identifies the readout operand
  it.key = rem;
  it.c = rem % g.Nc;
  it.b = (rem / g.Nc) % g.B;
  it.h = rem / (g.Nc * g.B);
  return it;
}

// Item4 of consecutive positions, advanced without divisions.
__device__ __forceinline__ void next_pos(Item4& it, const Geom& g, int tiles) {
  if (++it.tile < tiles) return;
  it.tile = 0;
  ++it.key;
  if (++it.c < g.Nc) return;
  it.c = 0;
  if (++it.b < g.B) return;
  it.b = 0;
  ++it.h;
}

}  // namespace

// kGeneral: the debug outputs or the SPLIT output (flags & 7 or out_linear set)
template <int D, bool kGeneral>
__global__ void __launch_bounds__(kTThreads, 1)
    k4_merge_tma(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_os,
                 const __grid_constant__ CUtensorMap tm_gs, const __grid_constant__ CUtensorMap tm_gl,
                 const __grid_constant__ CUtensorMap tm_out, const __grid_constant__ K4Params p) {
  using L = K4TLayout<D>;
  constexpr int kCols = D + 16;
  constexpr int kQC = D / 4;  // columns of a worker thread (a quarter row)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + kTNumBars * 8);
  int* abort_flag = reinterpret_cast<int*>(smem + L::kBar + kTNumBars * 8 + 4);
  float* ss_part = reinterpret_cast<float*>(smem + L::kSs);

  const Geom& g = p.g;
  const int tiles = (g.rows_per_chunk + 127) / 128;
  const long long positions = (long long)g.H * g.B * g.Nc * tiles;
  const int first = (int)(blockIdx.x * positions / gridDim.x);
  const int n = (int)((blockIdx.x + 1) * positions / gridDim.x) - first;  // tiles of this CTA
  const uint32_t warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    for (int q = 0; q < 2; ++q) {
      mbar_init(&bars[kTAFull + q], 1);
      mbar_init(&bars[kTAEmpty + q], kTWorkers);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[kTAReady + s], kTWorkers);
      mbar_init(&bars[kTAccFull + s], 1);
      mbar_init(&bars[kTAccEmpty + s], kTWorkers);
    }
    mbar_init(&bars[kTBFull], 1);
    mbar_init(&bars[kTBEmpty], 1);
    mbar_init(&bars[kTGFull], 1);
    mbar_init(&bars[kTGEmpty], kTWorkers);
    mbar_init(&bars[kTDone], 1);
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
  const CtaAbort ab{abort_flag, p.status, p.record, 4};
  auto row0_of = [&](const Item4& it) { return it.b * (int)g.N + it.c * g.rows_per_chunk + it.tile * 128; };
  auto item = [&](int i) { return decode_pos(first + i, g, tiles); };
  // o_s already holds sigmoid(g_s) * o_s (the softmax kernel was given the
  // gate): g_s is then neither loaded nor applied
  const bool gated = p.os_gated != nullptr && __ldg(p.os_gated) != 0;
  // q tiles in flight: the g_s slot is free for a second one when o_s comes gated
  const int nq = gated ? 2 : 1;
  auto q_slot = [&](int i) { return i % nq == 0 ? smem + L::kA : smem + L::kG + L::kTile; };
  // a full tile of the plain merge leaves by one TMA store from the o_s buffer
  // (the debug outputs and the SPLIT output take 16-byte stores)
  auto tma_out = [&](const Item4& it) { return !kGeneral && g.rows_per_chunk - it.tile * 128 >= 128; };

  if (warp == 0) {
    // ------------------------------------------------------------ loads, output stores
    if (lane == 0) {
      int prev_key = -1, b_loads = 0, a_issued = 0, g_issued = 0;
      bool ok = true;
      // the output tile of tile j (merged in the o_s buffer) goes out before
      // that buffer is reloaded
      auto store_out = [&](const Item4& it) {
        if (!tma_out(it)) return;
        for (int bx = 0; bx < D / 64; ++bx) tma_store_2d(&tm_out, smem + L::kG + bx * 16384, it.h * D + bx * 64, row0_of(it));
        bulk_commit();
        bulk_wait_read();
      };
      // step i: q of tile i, then o_s and the gates of tile i - 1 (they are
      // needed one tile later, once the merge of tile i - 2 has freed the buffer)
      // items i + 1, i, i - 1 and i - 2 of the step
      Item4 nx = item(0), cur = nx, prev1 = nx, prev2 = nx;
      for (int i = 0; i <= n && ok; ++i) {
        prev2 = prev1;
        prev1 = cur;
        cur = nx;
        next_pos(nx, g, tiles);
        if (i < n) {
          const Item4& it = cur;
          if (it.key != prev_key) {
            if (b_loads > 0 && !mbar_wait(&bars[kTBEmpty], (b_loads - 1) & 1, ab)) { ok = false; break; }
            mbar_expect_tx(&bars[kTBFull], (uint32_t)(2 * L::kBTile));
            bulk_load(smem + L::kB, p.mt + (((size_t)it.b * g.Nc + it.c) * g.H + it.h) * 2 * (size_t)L::kBTile,
                      (uint32_t)(2 * L::kBTile), &bars[kTBFull]);
            ++b_loads;
            prev_key = it.key;
          }
          const int qs = i % nq;
          if (!mbar_wait(&bars[kTAEmpty + qs], ((i / nq) & 1) ^ 1, ab)) { ok = false; break; }
          mbar_expect_tx(&bars[kTAFull + qs], (uint32_t)L::kTile);
          for (int bx = 0; bx < D / 64; ++bx)
            tma_load_2d(q_slot(i) + bx * 16384, &tm_q, &bars[kTAFull + qs], it.h * D + bx * 64, row0_of(it));
          ++a_issued;
          // warm L2 for what the next steps load
          if (i + 1 < n)
            for (int bx = 0; bx < D / 64; ++bx) tma_prefetch_2d(&tm_q, nx.h * D + bx * 64, row0_of(nx));
          for (int bx = 0; bx < D / 64; ++bx) {
            tma_prefetch_2d(&tm_os, it.h * D + bx * 64, row0_of(it));
            if (!gated) tma_prefetch_2d(&tm_gs, it.h * D + bx * 64, row0_of(it));
            tma_prefetch_2d(&tm_gl, it.h * D + bx * 64, row0_of(it));
          }
        }
        if (i >= 1) {
          const Item4& it = prev1;
          if (!mbar_wait(&bars[kTGEmpty], ((i - 1) & 1) ^ 1, ab)) { ok = false; break; }
          if (i >= 2) store_out(prev2);
          mbar_expect_tx(&bars[kTGFull], (uint32_t)((gated ? 2 : 3) * L::kTile));
          for (int bx = 0; bx < D / 64; ++bx) {
            tma_load_2d(smem + L::kG + bx * 16384, &tm_os, &bars[kTGFull], it.h * D + bx * 64, row0_of(it));
            if (!gated)
              tma_load_2d(smem + L::kG + L::kTile + bx * 16384, &tm_gs, &bars[kTGFull], it.h * D + bx * 64,
                          row0_of(it));
            tma_load_2d(smem + L::kG + 2 * L::kTile + bx * 16384, &tm_gl, &bars[kTGFull], it.h * D + bx * 64,
                        row0_of(it));
          }
          ++g_issued;
        }
      }
      // the last tile's output
      // (the loop ended after step n: prev1 is item n - 1)
      if (ok && n > 0 && mbar_wait(&bars[kTGEmpty], (n - 1) & 1, ab)) store_out(prev1);
      if (!ok) {  // let loads in flight land before the CTA exits
        for (int i = (a_issued > nq ? a_issued - nq : 0); i < a_issued; ++i)
          mbar_drain(&bars[kTAFull + i % nq], (i / nq) & 1);
        if (g_issued > 0) mbar_drain(&bars[kTGFull], (g_issued - 1) & 1);
        if (b_loads > 0) mbar_drain(&bars[kTBFull], (b_loads - 1) & 1);
      }
      bulk_wait_all();  // every output store complete before the CTA exits
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, kCols, 0, 0);
      const uint64_t b_desc0 = smem_desc(smem_u32(smem + L::kB), 16, 1024, kLayoutSw128);
      int prev_key = -1, b_loads = 0;
      Item4 it = item(0), nx = it;
      next_pos(nx, g, tiles);
      for (int i = 0; i < n; ++i, it = nx, next_pos(nx, g, tiles)) {
        const int s = i & 1;
        if (it.key != prev_key) {
          if (p.stall_ns > 0 && i > 0) sleep_ns(p.stall_ns);  // debug: let the other warps run ahead
          ++b_loads;
          prev_key = it.key;
          if (!mbar_wait(&bars[kTBFull], (b_loads - 1) & 1, ab)) break;
        }
        if (!mbar_wait(&bars[kTAReady + s], (i >> 1) & 1, ab)) break;
        if (!mbar_wait(&bars[kTAccEmpty + s], ((i >> 1) & 1) ^ 1, ab)) break;
        tc_fence_after();
#pragma unroll
        for (int hl = 0; hl < 2; ++hl)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t b =
                b_desc0 + (uint64_t)((hl * L::kBTile + (kk >> 2) * (L::kRows * 128) + (kk & 3) * 32) >> 4);
            mma_ts(tmem + s * L::kAccCols, tmem + s * L::kAccCols + L::kPhiCol + kk * 8, b, idesc,
                   (hl | kk) ? 1u : 0u);
          }
        mma_commit(&bars[kTAccFull + s]);
        const bool key_ends = i + 1 >= n || nx.key != it.key;
        if (key_ends) mma_commit(&bars[kTBEmpty]);
      }
      mma_commit(&bars[kTDone]);
      mbar_drain(&bars[kTDone], 0);
    }
  } else {
    // ------------------------------------------------------------ workers
    const uint32_t quarter = warp & 3, part = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;  // TMEM lane = tile row
    const int col0 = part * kQC;          // this thread's columns [col0, col0 + kQC)
    const int d = g.d;
    const int mode = (p.flags & 1) ? 1 : ((p.flags & 6) ? 2 : 0);  // 0 merged, 1 o_s, 2 linear read
    const bool use_gamma = p.gamma != nullptr && !(p.flags & 4);
    const bool split = p.out_linear != nullptr;

    // Finish tile j: TMEM -> o_l, RMS, merge from the shared tiles.  V = 0:
    // gated o_s, plain merge; 1: ungated o_s, plain merge; 2: the general
    // merge (debug outputs, SPLIT).  Returns false on a timeout (the four
    // warps of a row quarter agree).
    Item4 wit = item(0);  // the item of the next finish (tiles are finished in order)
    auto finish = [&](int j, auto variant) -> bool {
      constexpr int V = decltype(variant)::value;
      const Item4 it = wit;
      const int s = j & 1;
      const bool got = mbar_wait(&bars[kTAccFull + s], (j >> 1) & 1, ab);
      if (quad_any(quarter, !got)) return false;
      tc_fence_after();
      const int qrow = it.c * g.rows_per_chunk + it.tile * 128 + row;
      const bool empty = state_tokens(it.c, g) == 0 || no_linear_read(qrow / g.P, g);
      uint32_t dr, v[kQC];
      tmem_ld1(tmem_addr(tmem + s * L::kAccCols, quarter * 32, D), dr);
      if constexpr (kQC == 32) {
        tmem_ld32(tmem_addr(tmem + s * L::kAccCols, quarter * 32, col0), v);
      } else {
        tmem_ld16(tmem_addr(tmem + s * L::kAccCols, quarter * 32, col0), v);
      }
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars[kTAccEmpty + s]);  // the accumulator may be overwritten now
      // o_l = num * inv_den; its sum of squares is inv_den^2 * sum(num^2)
      const float inv_den = empty ? 0.f : 1.0f / __uint_as_float(dr);
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < kQC; ++e) ss = fmaf(__uint_as_float(v[e]), __uint_as_float(v[e]), ss);
      ss *= inv_den * inv_den;
      float* ssb = ss_part + s * 512;
      ssb[part * 128 + row] = ss;
      quad_any(quarter, false);
      const float tot = (ssb[row] + ssb[128 + row]) + (ssb[256 + row] + ssb[384 + row]);
      const float inv_rms = (p.flags & 4) ? 1.0f : rsqrtf(tot / (float)d + g.eps);
      const float scale = inv_den * inv_rms;  // r = num * scale
      const bool gok = mbar_wait(&bars[kTGFull], j & 1, ab);
      if (quad_any(quarter, !gok)) return false;
      const int nrows = min(128, g.rows_per_chunk - it.tile * 128);
      const bool via_tma = V != 2 && nrows == 128;  // the producer's tma_out(it)
      const size_t row_h = ((size_t)it.b * g.N + (size_t)qrow) * g.H + it.h;
      uint8_t* t_os = smem + L::kG;
      const uint8_t* t_gs = smem + L::kG + L::kTile;
      const uint8_t* t_gl = smem + L::kG + 2 * L::kTile;
      if constexpr (V != 2) {
        // plain merge, two columns per packed f32x2 operation
        const uint64_t scale2 = f32x2_pack(scale, scale);
#pragma unroll
        for (int c8 = 0; c8 < kQC / 8; ++c8) {
          const int col = col0 + 8 * c8;
          const int off = piece_off(row, col);
          const uint4 vo = *reinterpret_cast<const uint4*>(t_os + off);
          const uint4 vl = *reinterpret_cast<const uint4*>(t_gl + off);
          const uint32_t ow[4] = {vo.x, vo.y, vo.z, vo.w};
          const uint32_t lw[4] = {vl.x, vl.y, vl.z, vl.w};
          uint32_t sw[4] = {0u, 0u, 0u, 0u};
          if constexpr (V == 1) {
            const uint4 vs = *reinterpret_cast<const uint4*>(t_gs + off);
            sw[0] = vs.x; sw[1] = vs.y; sw[2] = vs.z; sw[3] = vs.w;
          }
          const float2* gam = reinterpret_cast<const float2*>(p.gamma + it.h * d + col);
          float o[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            // the softmax branch's gated term sigmoid(g_s) * o_s
            uint64_t st2 = f32x2_pack(bf16_lo(ow[e]), bf16_hi(ow[e]));
            if constexpr (V == 1) st2 = f32x2_mul(sigmoid2_tanh(f32x2_pack(bf16_lo(sw[e]), bf16_hi(sw[e]))), st2);
            uint64_t rr2 = f32x2_mul(f32x2_pack(__uint_as_float(v[8 * c8 + 2 * e]), __uint_as_float(v[8 * c8 + 2 * e + 1])),
                                     scale2);
            if (use_gamma) {
              const float2 g2 = __ldg(gam + e);
              rr2 = f32x2_mul(rr2, f32x2_pack(g2.x, g2.y));
            }
            const uint64_t o2 = f32x2_fma(sigmoid2_tanh(f32x2_pack(bf16_lo(lw[e]), bf16_hi(lw[e]))), rr2, st2);
            f32x2_unpack(o2, o[2 * e], o[2 * e + 1]);
          }
          if (via_tma) {
            // in place of this thread's own o_s piece, for the TMA store
            *reinterpret_cast<uint4*>(t_os + off) = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                                                               pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
          } else if (row < nrows) {
            store8<false>(p.out, row_h * d + col, o);
          }
        }
      } else {
        // general merge: debug outputs, SPLIT (16-byte stores)
#pragma unroll
        for (int c8 = 0; c8 < kQC / 8; ++c8) {
          const int col = col0 + 8 * c8;
          const int off = piece_off(row, col);
          const uint4 vo = *reinterpret_cast<const uint4*>(t_os + off);
          const uint4 vl = *reinterpret_cast<const uint4*>(t_gl + off);
          const uint32_t ow[4] = {vo.x, vo.y, vo.z, vo.w};
          const uint32_t lw[4] = {vl.x, vl.y, vl.z, vl.w};
          float os[8], gl[8], rr[8], sterm[8];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            os[2 * k] = bf16_lo(ow[k]); os[2 * k + 1] = bf16_hi(ow[k]);
            gl[2 * k] = bf16_lo(lw[k]); gl[2 * k + 1] = bf16_hi(lw[k]);
          }
          // the softmax branch's gated term sigmoid(g_s) * o_s
          if (gated) {
#pragma unroll
            for (int k = 0; k < 8; ++k) sterm[k] = os[k];
          } else {
            const uint4 vs = *reinterpret_cast<const uint4*>(t_gs + off);
            const uint32_t sw[4] = {vs.x, vs.y, vs.z, vs.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              sterm[2 * k] = sigmoid_f(bf16_lo(sw[k])) * os[2 * k];
              sterm[2 * k + 1] = sigmoid_f(bf16_hi(sw[k])) * os[2 * k + 1];
            }
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) rr[k] = __uint_as_float(v[8 * c8 + k]) * scale;
          if (use_gamma) {
            const float4 ga = __ldg(reinterpret_cast<const float4*>(p.gamma + it.h * d + col));
            const float4 gb = __ldg(reinterpret_cast<const float4*>(p.gamma + it.h * d + col) + 1);
            rr[0] *= ga.x; rr[1] *= ga.y; rr[2] *= ga.z; rr[3] *= ga.w;
            rr[4] *= gb.x; rr[5] *= gb.y; rr[6] *= gb.z; rr[7] *= gb.w;
          }
          float o[8];
          if (split) {
            float ol[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              o[k] = sterm[k];
              ol[k] = sigmoid_f(gl[k]) * rr[k];
            }
            if (row < nrows) store8<false>(p.out_linear, row_h * d + col, ol);
          } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float merged = sterm[k] + sigmoid_f(gl[k]) * rr[k];
              o[k] = mode == 0 ? merged : (mode == 1 ? os[k] : rr[k]);
            }
          }
          if (row < nrows) store8<false>(p.out, row_h * d + col, o);
        }
      }
      if (via_tma) fence_proxy_async_smem();  // the output tile is read by the async proxy
      mbar_arrive(&bars[kTGEmpty]);           // the shared tiles may be reloaded (after the store)
      next_pos(wit, g, tiles);
      return true;
    };
    auto fin = [&](int j) -> bool {
      if constexpr (kGeneral) {
        return finish(j, std::integral_constant<int, 2>());
      } else {
        return gated ? finish(j, std::integral_constant<int, 0>()) : finish(j, std::integral_constant<int, 1>());
      }
    };

    bool ok = true;
    for (int i = 0; i < n && ok; ++i) {
      const bool got = mbar_wait(&bars[kTAFull + i % nq], (i / nq) & 1, ab);
      if (all_workers_any(!got)) { ok = false; break; }
      // phi of this thread's quarter row, bf16 pairs into the free columns of
      // accumulator slot i % 2 (the MMA of tile i - 2, which read that slot's
      // phi(Q), completed before finish(i - 2) returned)
      {
        uint32_t pk[kQC / 2];
#pragma unroll
        for (int c8 = 0; c8 < kQC / 8; ++c8) {
          const uint4 v = *reinterpret_cast<const uint4*>(q_slot(i) + piece_off(row, col0 + 8 * c8));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) pk[4 * c8 + e] = phi_bf16x2(w[e]);
        }
        mbar_arrive(&bars[kTAEmpty + i % nq]);  // q tile read: its slot may be reloaded
        const uint32_t base = tmem_addr(tmem + (i & 1) * L::kAccCols, quarter * 32, L::kPhiCol + col0 / 2);
        if constexpr (kQC == 32) {
          tmem_st16(base, pk);
        } else {
          tmem_st8(base, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[kTAReady + (i & 1)]);
      }
      if (i > 0) ok = !all_workers_any(!fin(i - 1));
    }
    if (ok && n > 0) fin(n - 1);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * L::kAccCols);
  }
}

size_t k4_merge_tma_smem(int Dp) {
  return Dp == 128 ? (size_t)K4TLayout<128>::kBytes : (size_t)K4TLayout<64>::kBytes;
}

template <int D, bool kGeneral>
static cudaError_t launch_k4t(const MergeMaps& m, const K4Params& p, cudaStream_t st) {
  const int smem = K4TLayout<D>::kBytes;
  cudaError_t e =
      cudaFuncSetAttribute(k4_merge_tma<D, kGeneral>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long positions = (long long)((p.g.rows_per_chunk + 127) / 128) * p.g.Nc * p.g.B * p.g.H;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = (int)(positions < sms ? (positions > 0 ? positions : 1) : sms);
  k4_merge_tma<D, kGeneral><<<grid, kTThreads, smem, st>>>(m.q, m.os, m.gs, m.gl, m.out, p);
  return cudaGetLastError();
}

cudaError_t launch_readout_merge_tma(const MergeMaps& m, const K4Params& p, cudaStream_t st) {
  const bool general = (p.flags & 7) != 0 || p.out_linear != nullptr;
  if (p.g.Dp == 128) return general ? launch_k4t<128, true>(m, p, st) : launch_k4t<128, false>(m, p, st);
  return general ? launch_k4t<64, true>(m, p, st) : launch_k4t<64, false>(m, p, st);
}

}  // namespace vdn
