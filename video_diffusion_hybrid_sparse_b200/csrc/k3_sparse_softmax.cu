// k3_sparse_softmax.cu - softmax branch of the VDN-H3 hybrid attention
// (article section 双分支混合注意力机制): exact attention of every video query
// over the keys of its chunk window (chunk c-1..c+1, clipped), the two anchor
// frames and all text tokens.
//
// Design (sm_100a):
//  * persistent CTAs, one per SM; a work item is two 128-row query tiles of
//    one (batch, head, query segment), a segment being the rows of one chunk
//    (under the GLOBAL anchor reading the rows of frames 0 and F-1 are
//    segments of their own whose key set is every frame); items are handed
//    out statically in blocks ordered (batch, head, segment, pair), so the
//    CTAs running at once share one head's keys and values in L2
//    (plan_items in api.cu chooses the blocks);
//  * only the KV tiles of the item's key set are enumerated: at most three
//    merged video token ranges plus the text range, 128 keys per tile; the
//    last tile of a range is masked past the range end;
//  * warp 0 issues TMA loads (Q once per item, K and V per tile, two stages);
//    warp 1 issues tcgen05 MMAs from one thread: S_t = Q_t K^T (both operands
//    K-major in shared memory, fp32 accumulator in TMEM) and O_t += P_t V
//    (P_t read from TMEM, V MN-major in shared memory);
//  * warps 4-7 and 8-11 are the softmax warpgroups of query tile 0 and 1
//    (warp w reads TMEM lanes 32*(w%4)..+31); each thread owns one query row
//    (TMEM lane), so row max and row sum are in-thread; P is written back as
//    bf16 over the first half of S's columns;
//  * TMEM: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D);
//  * when asked to, warps 2-3 (idle in the attention itself) and, after their
//    last item, the softmax warps run the forward/backward scan of the linear
//    branch (scan.cuh), taking units from a counter in the workspace (zeroed
//    by the state build), so CTAs that finish their items early do most of
//    the scan's tail.
//
// Online softmax.  The running max m moves only when a tile's max exceeds it
// by more than 8 (log2 units; O is then rescaled in TMEM and the final 1/l
// is applied in the epilogue), so P <= 2^8.  Of every eight key pairs, the
// pairs in kEmuPairs get 2^x from a cubic on the FMA pipe (exp2x2_fma) and
// the others from the special-function unit: at head_dim 128 a 128-key tile
// costs the SFU as many cycles as the tensor core, so moving part of the
// exponentials to the FMA pipe leaves the SFU slack to absorb the hand-offs
// between the roles.  Masked keys (past the end of a key range) get s = -inf:
// a weight of 0 from the SFU, below 2^-126 from the FMA-pipe form.
//
// The MMA issue order per KV tile j is PV_0(j), S_0(j+1), PV_1(j), S_1(j+1), so
// the tensor core works on one tile while the other tile's softmax runs.  P is
// handed over in two halves (keys 0-63, then 64-127): the P.V of the first
// half runs while the second half is exponentiated, which takes its time off
// the tile's critical chain (S -> softmax -> P.V -> next S).  A commit after
// S_t(j+1) also covers PV_t(j), so when the softmax of tile t sees S_t(j+1)
// its O_t is quiescent and may be rescaled (before the first half is handed
// over).
//
// Fused readout (kFused, bf16 and head_dim 128): the linear branch's read and
// the gated merge run in this kernel's item epilogue instead of a readout
// kernel of their own (the frame-7 paragraph of 双分支混合注意力机制 combines
// the linear read with the local branch at the query's position), so o_s is
// never written and q is read once.  The forward/backward scan runs in warps
// 2-3 as on the other path and counts its completed units per (batch, head);
// an item's readout waits (bounded) until its (batch, head) is complete, which
// it is long before the first item ends.  Per item:
//  * the producer sends M_c of the item's (batch, chunk, head) through the
//    K/V ring as one more stage, the hi image in the K slot and the lo image
//    in the V slot (rows 0..127 of each: the numerator columns);
//  * after handing over the last P of the item, softmax warpgroup t applies
//    phi to its query row in place in Q_t (its S MMAs are complete) and forms
//    the denominator phi(q) . z on the CUDA cores (z = row 128 of the images);
//  * the MMA thread issues num_t = phi(Q_t) M_hi + phi(Q_t) M_lo into S_t's
//    TMEM columns (behind the item's last P.V, which reads P_t from them),
//    then releases the stage and Q;
//  * the epilogue reads num_t and O_t: o_l = num / den (0 for an empty state
//    or a GLOBAL anchor segment), r = o_l / sqrt(mean(o_l^2) + eps) * gamma,
//    out = sigmoid(g_s) O / l + sigmoid(g_l) r; then S_t's columns are free
//    for the next item's first S_t (kRDone).
#include <type_traits>

#include "k3_common.cuh"
#include "kernels.h"
#include "phi.cuh"
#include "scan.cuh"
#include "sm100.cuh"

namespace vdn {

namespace {

using namespace k3;

template <int D>
struct K3Layout {
  static constexpr int kTile = kBlockM * D * 2;  // bytes of one 128-row bf16 tile
  static constexpr int kStages = 2;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + 2 * kTile;
  static constexpr int kV = kK + kStages * kTile;
  static constexpr int kBar = kV + kStages * kTile;
  static constexpr int kBytes = kBar + 256 + 1024;  // + barriers + alignment slack
};

// Barriers of the fused readout, after the common ones.  kPhiFull + t:
// phi(Q_t) is in shared memory (128 arrivals); kRFull + t: num_t is in TMEM;
// kRDone + t: the epilogue has read num_t (128 arrivals).
enum { kPhiFull = kNumBars, kRFull = kNumBars + 2, kRDone = kNumBars + 4, kNumBarsAll = kNumBars + 6 };

// Readout operand image of one (batch, chunk, head) at head_dim 128 (scan.cuh):
// hi then lo, each two K halves of 144 rows x 128 bytes; rows 0..127 hold the
// numerator columns, row 128 holds z.
constexpr int kMtHalf = 144 * 128;
constexpr int kMtImage = 2 * kMtHalf;

constexpr int kThreads = 384;  // warp 0 loads, warp 1 MMA, warps 2-3 scan, warps 4-11 softmax
constexpr uint32_t kLaunchRegs = 168;  // per thread at launch (65536 / 384, in steps of 8)
constexpr uint32_t kLowRegs = 120;     // warpgroup 0
constexpr uint32_t kHighRegs = 184;    // softmax warpgroups

// Key pairs (bit e of each group of eight) exponentiated on the FMA pipe.
constexpr uint32_t kEmuPairs = 0x0u;

// Exponentials of one 16-key group: P (bf16 pairs) and the row sum (two
// packed partial sums).
__device__ __forceinline__ void exp_group(const uint32_t* s, uint64_t sl2x2, uint64_t negm, uint32_t (&pk)[8],
                                          uint64_t& l0, uint64_t& l1) {
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const uint64_t x = f32x2_fma(f32x2_pack(__uint_as_float(s[2 * e]), __uint_as_float(s[2 * e + 1])), sl2x2, negm);
    uint64_t pp;
    if ((kEmuPairs >> e) & 1u) {
      pp = exp2x2_fma(x);
    } else {
      float x0, x1;
      f32x2_unpack(x, x0, x1);
      pp = f32x2_pack(ex2_approx(x0), ex2_approx(x1));
    }
    if (e & 1) l1 = f32x2_add(l1, pp);
    else l0 = f32x2_add(l0, pp);
    float p0, p1;
    f32x2_unpack(pp, p0, p1);
    pk[e] = pack_bf16x2(p0, p1);
  }
}

// Scan units taken 32 at a time (one per lane) from the workspace counter
// until none is left.
__device__ __forceinline__ void scan_dynamic(const K3Params& p, uint32_t lane) {
  const long long units = scan_units(p.g);
  while (true) {
    long long base = 0;
    if (lane == 0) base = (long long)atomicAdd(p.scan_counter, 32ull);
    base = __shfl_sync(0xffffffffu, base, 0);
    if (base >= units) break;
    if (base + lane < units) {
      scan_unit(p.scan, base + lane);
      if (p.scan_done) {
        // release: this unit's M_c writes before the count that says so
        __threadfence();
        atomicAdd(p.scan_done + (base + lane) / scan_units_per_bh(p.g), 1u);
      }
    }
  }
}

// The fused readout and merge of query tile t of an item (kFused), run by the
// tile's softmax warpgroup after it handed over the item's last P: phi(Q_t)
// in place and den, the wait for O_t and num_t, the RMSNorm and the merge.
// Returns false when a wait ran out.
template <int D>
__device__ __forceinline__ bool fused_readout_tile(const K3Params& p, int item, int t, int row, uint32_t lane_base,
                                                uint32_t tmem, uint8_t* sQ, uint64_t* bars, uint32_t o_cnt,
                                                float l_run, CtaAbort ab) {
  using L = K3Layout<D>;
  const Geom& g = p.g;
  const Item it = decode_item(item, p);
  const bool no_read = it.c == kAllFrames || state_tokens(it.c, g) == 0;
  const uint8_t* img =
      p.mt + (((size_t)it.b * g.Nc + (it.c == kAllFrames ? 0 : it.c)) * g.H + it.h) * (size_t)kMtImage * 2;
  const int nrows = min(kBlockM, it.nrows - t * kBlockM);  // valid rows of this tile
  const size_t row_el = (((size_t)it.b * g.N + (size_t)(it.row0 + t * kBlockM + row)) * g.H + it.h) * D;
  const uint4* gsp = reinterpret_cast<const uint4*>(p.gate_s + row_el);
  const uint4* glp = reinterpret_cast<const uint4*>(p.gate_l + row_el);
  // z of M_c (read below) comes from this kernel's own scan under do_scan
  const bool z_ready = !p.do_scan || counter_wait(p.scan_done + it.b * g.H + it.h, (unsigned)scan_units_per_bh(g), ab);
  if (__any_sync(0xffffffffu, !z_ready)) return false;
  // phi(q) in place over this thread's row of Q_t (K-major, 128-byte
  // swizzle: 16-byte chunk c of row r sits at chunk c ^ (r % 8)) and
  // den = phi(q) . (z_hi + z_lo), with the bf16 phi(q) the MMA reads
  uint8_t* qrow = sQ + t * L::kTile + row * 128;
  uint64_t den2 = f32x2_pack(0.f, 0.f);
#pragma unroll 1
  for (int bx = 0; bx < 2; ++bx) {
    const uint4* zh = reinterpret_cast<const uint4*>(img + bx * kMtHalf + 128 * 128);
    const uint4* zl = reinterpret_cast<const uint4*>(img + kMtImage + bx * kMtHalf + 128 * 128);
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      uint4* pq = reinterpret_cast<uint4*>(qrow + bx * 16384 + ((ch ^ (row & 7)) << 4));
      const uint4 w = *pq;
      const uint4 f = make_uint4(phi_bf16x2(w.x), phi_bf16x2(w.y), phi_bf16x2(w.z), phi_bf16x2(w.w));
      *pq = f;
      const uint4 a = __ldcg(zh + ch), b = __ldcg(zl + ch);  // written in this kernel under do_scan: not __ldg
      const uint32_t fw[4] = {f.x, f.y, f.z, f.w}, aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        den2 = f32x2_fma(f32x2_pack(bf16_lo(fw[e]), bf16_hi(fw[e])),
                         f32x2_add(f32x2_pack(bf16_lo(aw[e]), bf16_hi(aw[e])),
                                   f32x2_pack(bf16_lo(bw[e]), bf16_hi(bw[e]))),
                         den2);
    }
  }
  fence_proxy_async_smem();
  mbar_arrive(&bars[kPhiFull + t]);
  bool got = mbar_wait(&bars[kOFull + t], o_cnt & 1, ab);
  got = got && mbar_wait(&bars[kRFull + t], o_cnt & 1, ab);  // one num_t per O_t
  if (__any_sync(0xffffffffu, !got)) return false;
  tc_fence_after();
  float d0, d1;
  f32x2_unpack(den2, d0, d1);
  const float inv_den = no_read ? 0.f : 1.0f / (d0 + d1);
  const uint32_t n_addr = tmem_addr(tmem, lane_base, t * 128);
  const uint32_t o_addr = tmem_addr(tmem, lane_base, 256 + t * D);
  // the row's sum of squares of num (o_l = num / den)
  uint64_t ss2 = f32x2_pack(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < D / 32; ++i) {
    uint32_t v[32];
    tmem_ld32(n_addr + 32 * i, v);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint64_t x = f32x2_pack(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
      ss2 = f32x2_fma(x, x, ss2);
    }
  }
  float s0, s1;
  f32x2_unpack(ss2, s0, s1);
  const float scale = inv_den * rsqrtf((s0 + s1) * inv_den * inv_den / (float)g.d + g.eps);  // r = num * scale
  const uint64_t scale2 = f32x2_pack(scale, scale);
  const float inv_l = 1.0f / l_run;
  const uint64_t inv_l2 = f32x2_pack(inv_l, inv_l);
  const float* gam = p.gamma ? p.gamma + (size_t)it.h * D : nullptr;
#pragma unroll 1
  for (int i = 0; i < D / 32; ++i) {
    uint32_t nm[32], o[32];
    tmem_ld32(n_addr + 32 * i, nm);
    tmem_ld32(o_addr + 32 * i, o);
    tmem_wait_ld();
    if (i + 1 == D / 32) {
      tc_fence_before();
      mbar_arrive(&bars[kRDone + t]);  // S_t's columns may take the next item's S_t
    }
    if (row < nrows) {
      // the gates of these 32 columns (in L2 since the item's start): loaded
      // only once num and O are in registers, so that no gate registers are
      // held across the TMEM reads (holding them, or the next group's,
      // spilled registers of the KV loop and cost more than the load waits)
      uint4 cs[4], cl[4];
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4) {
        cs[v4] = __ldg(gsp + 4 * i + v4);
        cl[v4] = __ldg(glp + 4 * i + v4);
      }
      uint4* d4 = reinterpret_cast<uint4*>(p.out + row_el + 32 * i);
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4) {
        const uint32_t sw[4] = {cs[v4].x, cs[v4].y, cs[v4].z, cs[v4].w};
        const uint32_t lw[4] = {cl[v4].x, cl[v4].y, cl[v4].z, cl[v4].w};
        uint32_t ow[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int k = 8 * v4 + 2 * e;
          // sigmoid(g_s) o_s + sigmoid(g_l) r
          const uint64_t st2 = f32x2_mul(sigmoid2_tanh(f32x2_pack(bf16_lo(sw[e]), bf16_hi(sw[e]))),
                                         f32x2_mul(f32x2_pack(__uint_as_float(o[k]), __uint_as_float(o[k + 1])),
                                                   inv_l2));
          uint64_t rr2 = f32x2_mul(f32x2_pack(__uint_as_float(nm[k]), __uint_as_float(nm[k + 1])), scale2);
          if (gam) {
            const float2 g2 = __ldg(reinterpret_cast<const float2*>(gam + 32 * i + k));
            rr2 = f32x2_mul(rr2, f32x2_pack(g2.x, g2.y));
          }
          float y0, y1;
          f32x2_unpack(f32x2_fma(sigmoid2_tanh(f32x2_pack(bf16_lo(lw[e]), bf16_hi(lw[e]))), rr2, st2), y0, y1);
          ow[e] = pack_bf16x2(y0, y1);
        }
        d4[v4] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
      }
    }
  }
  return true;
}

}  // namespace

template <int D, bool kFused>
__global__ void __launch_bounds__(kThreads, 1)
    k3_sparse_softmax(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_tk,
                      const __grid_constant__ CUtensorMap tm_tv, const __grid_constant__ K3Params p) {
  using L = K3Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + kNumBarsAll * 8);
  int* abort_flag = reinterpret_cast<int*>(smem + L::kBar + kNumBarsAll * 8 + 4);
  static_assert(kNumBarsAll * 8 + 8 <= 256, "barrier region");
  static_assert(!kFused || D == 128, "the fused readout is built for head_dim 128");

  const Geom& g = p.g;
  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();

  if (threadIdx.x == 0) {
    mbar_init(&bars[kQFull], 1);
    mbar_init(&bars[kQEmpty], 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&bars[kKFull + s], 1);
      mbar_init(&bars[kKEmpty + s], 1);
      mbar_init(&bars[kVFull + s], 1);
      mbar_init(&bars[kVEmpty + s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars[kSFull + t], 1);
      mbar_init(&bars[kPFull + t], kBlockM);
      mbar_init(&bars[kPFull2 + t], kBlockM);
      mbar_init(&bars[kOFull + t], 1);
    }
    mbar_init(&bars[kDone], 1);
    if (kFused) {
      for (int t = 0; t < 2; ++t) {
        mbar_init(&bars[kPhiFull + t], kBlockM);
        mbar_init(&bars[kRFull + t], 1);
        mbar_init(&bars[kRDone + t], kBlockM);
      }
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const CtaAbort ab{abort_flag, p.status, p.record, 3};
  // Register re-split between the warpgroups: the launch gives every thread
  // kLaunchRegs; warpgroup 0 (loads, MMA issue, scan) hands registers to the
  // two softmax warpgroups.  The re-split never asks for more than the launch
  // holds (128 * kLowRegs + 256 * kHighRegs <= 384 * kLaunchRegs), or the
  // increase would wait for registers that never come.
  static_assert(128 * kLowRegs + 256 * kHighRegs <= kThreads * kLaunchRegs, "register re-split exceeds the launch");

  uint8_t* sQ = smem + L::kQ;
  uint8_t* sK = smem + L::kK;
  uint8_t* sV = smem + L::kV;

  if (warp < 4) {
  regs_dec<kLowRegs>();
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && blockIdx.x == 0 && p.os_gated) *p.os_gated = p.gate_s != nullptr;  // for the readout
    if (lane == 0) {
      uint32_t kv_cnt = 0, item_cnt = 0, q_loads = 0;  // q_loads: Q loads issued (the last is drained on an abort)
      bool ok = true;
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++item_cnt) {
        const Item it = decode_item(item, p);
        if (item_cnt > 0 && !mbar_wait(&bars[kQEmpty], (item_cnt - 1) & 1, ab)) { ok = false; break; }
        ++q_loads;
        mbar_expect_tx(&bars[kQFull], it.ntiles * L::kTile);
        for (int t = 0; t < it.ntiles; ++t)
          for (int bx = 0; bx < D / 64; ++bx)
            tma_load_2d(sQ + t * L::kTile + bx * 16384, &tm_q, &bars[kQFull], it.h * D + bx * 64,
                        it.b * (int)g.N + it.row0 + t * kBlockM);
        KvRanges kr;
        seg_ranges(it.c, g, kr);
        for (int ri = 0; ri <= kr.n && ok; ++ri) {
          const bool text = (ri == kr.n);
          const int len = text ? g.T : (int)kr.len[ri];
          const int base = text ? it.b * g.T : it.b * (int)g.N + (int)kr.start[ri];
          const CUtensorMap* mk = text ? &tm_tk : &tm_k;
          const CUtensorMap* mv = text ? &tm_tv : &tm_v;
          for (int off = 0; off < len; off += kBlockN, ++kv_cnt) {
            const int st = kv_cnt % L::kStages;
            const uint32_t ph = (kv_cnt / L::kStages) & 1;
            if (!mbar_wait(&bars[kKEmpty + st], ph ^ 1, ab)) { ok = false; break; }
            mbar_expect_tx(&bars[kKFull + st], L::kTile);
            for (int bx = 0; bx < D / 64; ++bx)
              tma_load_2d(sK + st * L::kTile + bx * 16384, mk, &bars[kKFull + st], it.h * D + bx * 64, base + off);
            if (!mbar_wait(&bars[kVEmpty + st], ph ^ 1, ab)) { ok = false; ++kv_cnt; break; }
            mbar_expect_tx(&bars[kVFull + st], L::kTile);
            for (int bx = 0; bx < D / 64; ++bx)
              tma_load_2d(sV + st * L::kTile + bx * 16384, mv, &bars[kVFull + st], it.h * D + bx * 64, base + off);
          }
        }
        if (kFused && ok) {
          // the item's readout operand as one more stage: M_hi rows 0..127 in
          // the K slot, M_lo rows 0..127 in the V slot (a GLOBAL anchor
          // segment reads nothing through the states; it takes chunk 0's
          // operand and the epilogue zeroes its read)
          const int st = kv_cnt % L::kStages;
          const uint32_t ph = (kv_cnt / L::kStages) & 1;
          const int mc = it.c == kAllFrames ? 0 : it.c;
          const uint8_t* img = p.mt + (((size_t)it.b * g.Nc + mc) * g.H + it.h) * (size_t)kMtImage * 2;
          ++kv_cnt;
          if (p.do_scan) {
            // M_c of this (batch, head) comes from the kernel's own scan (a
            // test of the failure path asks CTA 0 for one unit more, 10 ms)
            const bool inject = p.inject_scan_wait && blockIdx.x == 0;
            if (!counter_wait(p.scan_done + it.b * g.H + it.h, (unsigned)scan_units_per_bh(g) + (inject ? 1u : 0u),
                              ab, inject ? 10000000ll : kWaitNs)) {
              ok = false;
              break;
            }
            fence_proxy_async_global();
          }
          if (!mbar_wait(&bars[kKEmpty + st], ph ^ 1, ab)) { ok = false; break; }
          mbar_expect_tx(&bars[kKFull + st], L::kTile);
          for (int bx = 0; bx < 2; ++bx)
            bulk_load(sK + st * L::kTile + bx * 16384, img + bx * kMtHalf, 16384, &bars[kKFull + st]);
          if (!mbar_wait(&bars[kVEmpty + st], ph ^ 1, ab)) { ok = false; break; }
          mbar_expect_tx(&bars[kVFull + st], L::kTile);
          for (int bx = 0; bx < 2; ++bx)
            bulk_load(sV + st * L::kTile + bx * 16384, img + kMtImage + bx * kMtHalf, 16384, &bars[kVFull + st]);
        }
      }
      if (!ok) {
        // Let loads already in flight land before the CTA's shared memory goes away.
        for (uint32_t i = (kv_cnt > (uint32_t)L::kStages ? kv_cnt - L::kStages : 0); i < kv_cnt; ++i) {
          mbar_drain(&bars[kKFull + i % L::kStages], (i / L::kStages) & 1);
          mbar_drain(&bars[kVFull + i % L::kStages], (i / L::kStages) & 1);
        }
        if (q_loads > 0) mbar_drain(&bars[kQFull], (q_loads - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kBlockN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      // descriptors of tile 0 / stage 0; tiles, stages and K steps add byte offsets >> 4
      const uint64_t q_desc0 = smem_desc(smem_u32(sQ), 16, 1024, kLayoutSw128);
      const uint64_t k_desc0 = smem_desc(smem_u32(sK), 16, 1024, kLayoutSw128);
      const uint64_t v_desc0 = smem_desc(smem_u32(sV), 16384, 1024, kLayoutSw128);
      const uint64_t m_lo_desc0 = smem_desc(smem_u32(sV), 16, 1024, kLayoutSw128);  // fused readout: M_lo, K-major
      uint32_t kv_cnt = 0, item_cnt = 0, p_cnt[2] = {0, 0};
      // fused readout: phi(Q_t) hand-overs seen, kRDone phases waited, and
      // whether S_t's columns still hold a num_t the epilogue may be reading
      uint32_t phi_cnt[2] = {0, 0}, rd_cnt[2] = {0, 0};
      bool rd_pend[2] = {false, false};
      bool ok = true;

      auto issue_qk = [&](int t, int st) {
        const uint32_t d_tmem = tmem + t * 128;
        const uint64_t qd = q_desc0 + (uint64_t)((t * L::kTile) >> 4);
        const uint64_t kd = k_desc0 + (uint64_t)((st * L::kTile) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
          mma_ss(d_tmem, qd + off, kd + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      // O_t += P_t·V over keys 64*part .. 64*part + 63 of the tile
      auto issue_pv = [&](int t, int st, int part, bool acc) {
        const uint32_t d_tmem = tmem + 256 + t * D;
        const uint64_t vd = v_desc0 + (uint64_t)((st * L::kTile) >> 4);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int kk = 4 * part + k;
          mma_ts(d_tmem, tmem + t * 128 + kk * 8, vd + (uint64_t)((kk * 2048) >> 4), idesc_pv,
                 (acc || kk > 0) ? 1u : 0u);
        }
      };

      // num_t = phi(Q_t) (M_hi + M_lo) over the numerator columns, into S_t's columns
      auto issue_readout = [&](int t, int st) {
        const uint32_t d_tmem = tmem + t * 128;
        const uint64_t qd = q_desc0 + (uint64_t)((t * L::kTile) >> 4);
        const uint64_t hd = k_desc0 + (uint64_t)((st * L::kTile) >> 4);
        const uint64_t ld = m_lo_desc0 + (uint64_t)((st * L::kTile) >> 4);
#pragma unroll
        for (int hl = 0; hl < 2; ++hl)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            mma_ss(d_tmem, qd + off, (hl ? ld : hd) + off, idesc_qk, (hl | kk) ? 1u : 0u);
          }
      };

      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++item_cnt) {
        const Item it = decode_item(item, p);
        const int nkv = seg_kv_tiles(it.c, g);
        if (!mbar_wait(&bars[kQFull], item_cnt & 1, ab)) { ok = false; break; }
        {
          const int st = kv_cnt % L::kStages;
          if (!mbar_wait(&bars[kKFull + st], (kv_cnt / L::kStages) & 1, ab)) { ok = false; break; }
          tc_fence_after();
          for (int t = 0; t < it.ntiles; ++t) {
            if (kFused && rd_pend[t]) {
              // S_t's columns hold the previous item's num_t until its epilogue has read it
              if (!mbar_wait(&bars[kRDone + t], rd_cnt[t] & 1, ab)) { ok = false; break; }
              ++rd_cnt[t];
              rd_pend[t] = false;
              tc_fence_after();
            }
            issue_qk(t, st);
            mma_commit(&bars[kSFull + t]);
          }
          if (!ok) break;
          mma_commit(&bars[kKEmpty + st]);
        }
        for (int j = 0; j < nkv; ++j, ++kv_cnt) {
          const int st = kv_cnt % L::kStages;
          const int nst = (kv_cnt + 1) % L::kStages;
          const bool has_next = j + 1 < nkv;
          if (!mbar_wait(&bars[kVFull + st], (kv_cnt / L::kStages) & 1, ab)) { ok = false; break; }
          for (int t = 0; t < it.ntiles; ++t) {
            if (!mbar_wait(&bars[kPFull + t], p_cnt[t] & 1, ab)) { ok = false; break; }
            tc_fence_after();
            issue_pv(t, st, 0, j > 0);
            if (!mbar_wait(&bars[kPFull2 + t], p_cnt[t] & 1, ab)) { ok = false; break; }
            tc_fence_after();
            issue_pv(t, st, 1, true);
            ++p_cnt[t];
            if (!has_next) mma_commit(&bars[kOFull + t]);
            if (has_next) {
              if (t == 0 && !mbar_wait(&bars[kKFull + nst], ((kv_cnt + 1) / L::kStages) & 1, ab)) {
                ok = false;
                break;
              }
              tc_fence_after();
              issue_qk(t, nst);
              mma_commit(&bars[kSFull + t]);
            }
          }
          if (!ok) break;
          mma_commit(&bars[kVEmpty + st]);
          if (has_next) mma_commit(&bars[kKEmpty + nst]);
        }
        if (!ok) break;
        if (kFused) {
          // the readout stage: M_hi in the K slot, M_lo in the V slot
          const int st = kv_cnt % L::kStages;
          const uint32_t ph = (kv_cnt / L::kStages) & 1;
          ++kv_cnt;
          if (!mbar_wait(&bars[kKFull + st], ph, ab) || !mbar_wait(&bars[kVFull + st], ph, ab)) {
            ok = false;
            break;
          }
          for (int t = 0; t < it.ntiles; ++t) {
            if (!mbar_wait(&bars[kPhiFull + t], phi_cnt[t] & 1, ab)) { ok = false; break; }
            ++phi_cnt[t];
            tc_fence_after();
            issue_readout(t, st);
            mma_commit(&bars[kRFull + t]);
            rd_pend[t] = true;
          }
          if (!ok) break;
          mma_commit(&bars[kKEmpty + st]);
          mma_commit(&bars[kVEmpty + st]);
        }
        mma_commit(&bars[kQEmpty]);
      }
      // All MMAs issued by this thread complete before TMEM is released.
      mma_commit(&bars[kDone]);
      mbar_drain(&bars[kDone], 0);
    }
  } else {
    // ------------------------------------------------------------ forward/backward scan
    if (p.do_scan) scan_dynamic(p, lane);
  }
  } else {
    regs_inc<kHighRegs>();
    // ------------------------------------------------------------ softmax warpgroups
    const int t = (warp - 4) >> 2;
    const uint32_t quarter = warp & 3;
    const int row = quarter * 32 + lane;  // query row of the tile == TMEM lane
    const uint32_t lane_base = quarter * 32;
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f32x2_pack(sl2, sl2);
    uint32_t s_cnt = 0, o_cnt = 0;
    bool ok = true;

    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      // only the key set and the tile count live across the KV loop; the
      // epilogue decodes the item again (fewer registers held in the loop)
      int seg_c, ntiles;
      {
        const Item it = decode_item(item, p);
        seg_c = it.c;
        ntiles = it.ntiles;
        // the row's gate logits are read in the epilogue: bring them into L2 now
        if (p.gate_s && t < ntiles && row < it.nrows - t * kBlockM) {
          const __nv_bfloat16* gr =
              p.gate_s + (((size_t)it.b * g.N + (size_t)(it.row0 + t * kBlockM + row)) * g.H + it.h) * D;
#pragma unroll
          for (int i = 0; i < D / 64; ++i) prefetch_l2(gr + 64 * i);
          if (kFused) {
            const __nv_bfloat16* gl = p.gate_l + (gr - p.gate_s);
#pragma unroll
            for (int i = 0; i < D / 64; ++i) prefetch_l2(gl + 64 * i);
          }
        }
      }
      if (t >= ntiles) continue;
      float m_run = 0.f, l_run = 0.f;
      // keys left in the current key range (video ranges, then text); only
      // these scalars live across the loop, the ranges are re-derived at
      // range ends
      const int nkv = seg_kv_tiles(seg_c, g);
      int range = 0, left = seg_range_len(seg_c, g, 0);
      for (int j = 0; j < nkv; ++j) {
        while (left == 0) left = seg_range_len(seg_c, g, ++range);
        const int n_valid = min(kBlockN, left);
        left -= n_valid;
        const bool got = mbar_wait(&bars[kSFull + t], s_cnt & 1, ab);
        if (__any_sync(0xffffffffu, !got)) { ok = false; break; }
        ++s_cnt;
        tc_fence_after();
        const uint32_t s_addr = tmem_addr(tmem, lane_base, t * 128);  // S_t, then P_t over its first half
        float alpha = 1.0f;
        bool rescale = false;
        uint64_t l0 = f32x2_pack(0.f, 0.f), l1 = l0;
        // One KV tile: the row max over all 128 scores, then the exponentials.
        // kMasked: the last tile of a key range, whose keys past n_valid get
        // s = -inf (a weight of 0 from the SFU, below 2^-126 from the FMA-pipe
        // form); the full tiles run a copy of the code without the masking.
        auto tile = [&](auto masked_tag) {
          constexpr bool kMasked = decltype(masked_tag)::value;
          uint32_t s[128];
#pragma unroll
          for (int i = 0; i < 4; ++i) tmem_ld32(s_addr + 32 * i, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * i]));
          tmem_wait_ld();
          if (kMasked) {
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (i >= n_valid) s[i] = __float_as_uint(-INFINITY);
          }
          // row max: eight independent fmax3 chains of eight (the max's
          // latency, not its instruction count, is on the critical path)
          float mc[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) mc[c] = fmaxf(__uint_as_float(s[2 * c]), __uint_as_float(s[2 * c + 1]));
#pragma unroll
          for (int i = 16; i < 128; i += 16)
#pragma unroll
            for (int c = 0; c < 8; ++c) mc[c] = fmax3(mc[c], __uint_as_float(s[i + 2 * c]), __uint_as_float(s[i + 2 * c + 1]));
          const float mxs =
              fmaxf(fmaxf(fmax3(mc[0], mc[1], mc[2]), fmax3(mc[3], mc[4], mc[5])), fmaxf(mc[6], mc[7])) * sl2;
          // lazy rescale: move the running max only when this tile's max is
          // more than 2^8 above it (O is rescaled below, once P is stored)
          if (j == 0) {
            m_run = mxs;
          } else {
            const bool need = mxs > m_run + 8.0f;
            rescale = __any_sync(0xffffffffu, need);
            if (need) {
              alpha = ex2_approx(m_run - mxs);
              m_run = mxs;
            }
          }
          // p = 2^(s * scale * log2(e) - m); P goes to TMEM 16 columns (32
          // keys) at a time
          const uint64_t negm = f32x2_pack(-m_run, -m_run);
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            uint32_t pk[16];
            exp_group(&s[16 * i], sl2x2, negm, *reinterpret_cast<uint32_t(*)[8]>(&pk[0]), l0, l1);
            exp_group(&s[16 * i + 16], sl2x2, negm, *reinterpret_cast<uint32_t(*)[8]>(&pk[8]), l0, l1);
            tmem_st16(s_addr + 8 * i, pk);
            if (i == 2) {
              if (rescale) {
#pragma unroll 1
                for (int c = 0; c < D / 16; ++c) {
                  uint32_t o[16];
                  const uint32_t ta = tmem_addr(tmem, lane_base, 256 + t * D + 16 * c);
                  tmem_ld16(ta, o);
                  tmem_wait_ld();
#pragma unroll
                  for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                  tmem_st16(ta, o);
                }
              }
              tmem_wait_st();
              tc_fence_before();
              mbar_arrive(&bars[kPFull + t]);  // keys 0-63: the P.V of the first half may start
            }
          }
        };
        if (n_valid < kBlockN) tile(std::true_type());
        else tile(std::false_type());
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[kPFull2 + t]);
        float c0, c1, c2, c3;
        f32x2_unpack(l0, c0, c1);
        f32x2_unpack(l1, c2, c3);
        l_run = l_run * alpha + ((c0 + c1) + (c2 + c3));
      }
      if (!ok) break;
      if constexpr (kFused) {
        // ---------------------------------------------------------- fused readout and merge
        const bool good = fused_readout_tile<D>(p, item, t, row, lane_base, tmem, sQ, bars, o_cnt, l_run, ab);
        ++o_cnt;
        if (!good) { ok = false; break; }
        continue;
      }
      // ---------------------------------------------------------- epilogue: o_s = O / l
      // (times sigmoid(g_s) when the gate is given: the softmax branch's term
      // of the gated merge; the gate logits were brought into L2 at the start
      // of the item).
      const bool got = mbar_wait(&bars[kOFull + t], o_cnt & 1, ab);
      if (__any_sync(0xffffffffu, !got)) { ok = false; break; }
      ++o_cnt;
      tc_fence_after();
      const Item it = decode_item(item, p);
      const int nrows = min(kBlockM, it.nrows - t * kBlockM);  // valid rows of this tile
      const size_t row_el = (((size_t)it.b * g.N + (size_t)(it.row0 + t * kBlockM + row)) * g.H + it.h) * D;
      const bool gated = p.gate_s != nullptr;
      const float inv_l = 1.0f / l_run;
      __nv_bfloat16* dst = p.o_s + row_el;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        uint32_t o[32];
        uint4 gv[4];
        if (gated && row < nrows) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) gv[v4] = __ldg(reinterpret_cast<const uint4*>(p.gate_s + row_el) + 4 * i + v4);
        }
        tmem_ld32(tmem_addr(tmem, lane_base, 256 + t * D + 32 * i), o);
        tmem_wait_ld();
        if (row < nrows) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * i);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(o[8 * v4 + e]) * inv_l;
            if (gated) {
              const uint4 gq = gv[v4];
              const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                x[2 * e] *= sigmoid_tanh(bf16_lo(gw[e]));
                x[2 * e + 1] *= sigmoid_tanh(bf16_hi(gw[e]));
              }
            }
            d4[v4] = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                                pack_bf16x2(x[6], x[7]));
          }
        }
      }
    }
    // the scan's tail: warps that finish their items early take the remaining units
    if (ok && p.do_scan) scan_dynamic(p, lane);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

size_t k3_smem_bytes(int Dp) {
  // At least ~116 KB so that a second CTA never shares the SM (each claims all 512 TMEM columns).
  const size_t need = Dp == 128 ? (size_t)K3Layout<128>::kBytes : (size_t)K3Layout<64>::kBytes;
  return need < 118 * 1024 ? 118 * 1024 : need;
}

template <int D, bool kFused>
static cudaError_t launch_k3(const Maps& m, const K3Params& p, int grid, cudaStream_t st) {
  const size_t smem = k3_smem_bytes(D);
  cudaError_t e =
      cudaFuncSetAttribute(k3_sparse_softmax<D, kFused>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k3_sparse_softmax<D, kFused><<<grid, kThreads, smem, st>>>(m.q, m.k, m.v, m.tk, m.tv, p);
  return cudaGetLastError();
}

cudaError_t launch_sparse_softmax(const Maps& m, const K3Params& p, int grid, cudaStream_t st) {
  if (p.out) {
    // fused readout: bf16, head_dim 128, gates and out given; its own scan
    // needs the per-(batch, head) counters
    if (p.g.Dp != 128 || p.g.d != 128 || !p.gate_s || !p.gate_l || !p.mt || (p.do_scan && !p.scan_done))
      return cudaErrorInvalidValue;
    return launch_k3<128, true>(m, p, grid, st);
  }
  return p.g.Dp == 128 ? launch_k3<128, false>(m, p, grid, st) : launch_k3<64, false>(m, p, grid, st);
}

}  // namespace vdn
