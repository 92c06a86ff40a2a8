// k3_fp8.cu - softmax branch of the VDN-H3 hybrid attention with e4m3
// operands (section 双分支混合注意力机制 for the computation; section
// 性能实测表现 runs the model at FP8): the same block-sparse walk, pipeline
// and online softmax as k3_sparse_softmax, head_dim 128, with
//  * Q, K (video and text) and V^T (video and text) in e4m3, one scale per
//    (batch, head) and tensor (K and text K share one, V and text V share
//    one), written by the quantisation pass; the scales are folded into the
//    exponent (q.k scale) and into the epilogue (v scale);
//  * S_t = Q_t K^T and O_t += P_t V with tcgen05 kind::f8f6f4 (fp32
//    accumulators in TMEM), P_t written to TMEM as e4m3, four per column;
//  * P = 2^(s - m + 4): the running max moves when a tile's max exceeds it by
//    more than 4 (in log2 units), so P <= 256 fits e4m3 (max 448) and weights
//    down to 2^-13 of the row maximum keep at least one significant bit; the
//    row sum is taken over the same (unrounded) P, so the common factor
//    cancels in o_s = v_scale * O / l.
// V enters transposed (rows = head_dim, keys contiguous), so both operands of
// P.V are K-major.
#include "k3_common.cuh"
#include "kernels.h"
#include "scan.cuh"
#include "sm100.cuh"

namespace vdn {

namespace {

using namespace k3;

template <int D>
struct K3Layout {
  static constexpr int kTile = kBlockM * D;  // bytes of one 128 x 128 e4m3 tile (Q, K or V^T)
  static constexpr int kStages = 2;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + 2 * kTile;
  static constexpr int kV = kK + kStages * kTile;
  static constexpr int kBar = kV + kStages * kTile;
  static constexpr int kBytes = kBar + 256 + 1024;  // + barriers + alignment slack
};

// With kPolyEvery = n > 0, one column pair in n is exponentiated on the FMA
// pipe instead of the special-function unit.  With e4m3 operands the tensor
// work per KV tile halves and the exponential unit is the tighter limit, so
// one pair in eight goes to the FMA pipe (measured 1.7 % faster at 768p than
// none, and than one in four).
constexpr int kPolyEvery = 8;

// two fp32 to e4m3 (round to nearest even, saturate), a in the low byte
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}

__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t (&r)[4]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
               "r"(r[2]), "r"(r[3])
               : "memory");
}
__host__ __device__ constexpr bool poly_pair(int e) { return e % kPolyEvery == kPolyEvery - 1; }

}  // namespace

template <int D>
__global__ void __launch_bounds__(384, 1)
    k3_fp8(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_tk,
           const __grid_constant__ CUtensorMap tm_tv, const __grid_constant__ K3Params p) {
  static_assert(D == 128, "the fp8 branch is built for head_dim 128");
  using L = K3Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + kNumBars * 8);
  int* abort_flag = reinterpret_cast<int*>(smem + L::kBar + kNumBars * 8 + 4);

  const Geom& g = p.g;
  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();

  if (threadIdx.x == 0 && blockIdx.x == 0 && p.os_gated) *p.os_gated = 0;  // o_s is left ungated
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
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const CtaAbort ab{abort_flag, p.status, p.record, 31};

  uint8_t* sQ = smem + L::kQ;
  uint8_t* sK = smem + L::kK;
  uint8_t* sV = smem + L::kV;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t kv_cnt = 0, item_cnt = 0, q_loads = 0;  // q_loads: Q loads issued (the last is drained on an abort)
      bool ok = true;
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x, ++item_cnt) {
        const Item it = decode_item(item, p);
        if (item_cnt > 0 && !mbar_wait(&bars[kQEmpty], (item_cnt - 1) & 1, ab)) { ok = false; break; }
        ++q_loads;
        mbar_expect_tx(&bars[kQFull], it.ntiles * L::kTile);
        for (int t = 0; t < it.ntiles; ++t)
          tma_load_2d(sQ + t * L::kTile, &tm_q, &bars[kQFull], it.h * D, it.b * (int)g.N + it.row0 + t * kBlockM);
        KvRanges kr;
        seg_ranges(it.c, g, kr);
        for (int ri = 0; ri <= kr.n && ok; ++ri) {
          const bool text = (ri == kr.n);
          const int len = text ? g.T : (int)kr.len[ri];
          const int base = text ? it.b * g.T : it.b * (int)g.N + (int)kr.start[ri];  // K rows
          const int vx = text ? 0 : (int)kr.start[ri];  // V^T columns: token within the batch
          const int vy = (it.b * g.H + it.h) * D;       // V^T rows of this (batch, head)
          const CUtensorMap* mk = text ? &tm_tk : &tm_k;
          const CUtensorMap* mv = text ? &tm_tv : &tm_v;
          for (int off = 0; off < len; off += kBlockN, ++kv_cnt) {
            const int st = kv_cnt % L::kStages;
            const uint32_t ph = (kv_cnt / L::kStages) & 1;
            if (!mbar_wait(&bars[kKEmpty + st], ph ^ 1, ab)) { ok = false; break; }
            mbar_expect_tx(&bars[kKFull + st], L::kTile);
            tma_load_2d(sK + st * L::kTile, mk, &bars[kKFull + st], it.h * D, base + off);
            if (!mbar_wait(&bars[kVEmpty + st], ph ^ 1, ab)) { ok = false; ++kv_cnt; break; }
            mbar_expect_tx(&bars[kVFull + st], L::kTile);
            tma_load_2d(sV + st * L::kTile, mv, &bars[kVFull + st], vx + off, vy);
          }
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
      constexpr uint32_t idesc_qk = idesc_e4m3_f32(128, kBlockN);
      constexpr uint32_t idesc_pv = idesc_e4m3_f32(128, D);
      // descriptors of tile 0 / stage 0 (K-major, 128-byte rows, 128-byte
      // swizzle); tiles, stages and K steps (32 e4m3 = 32 bytes) add byte offsets >> 4
      const uint64_t q_desc0 = smem_desc(smem_u32(sQ), 16, 1024, kLayoutSw128);
      const uint64_t k_desc0 = smem_desc(smem_u32(sK), 16, 1024, kLayoutSw128);
      const uint64_t v_desc0 = smem_desc(smem_u32(sV), 16, 1024, kLayoutSw128);
      uint32_t kv_cnt = 0, item_cnt = 0, p_cnt[2] = {0, 0};
      bool ok = true;

      auto issue_qk = [&](int t, int st) {
        const uint32_t d_tmem = tmem + t * 128;
        const uint64_t qd = q_desc0 + (uint64_t)((t * L::kTile) >> 4);
        const uint64_t kd = k_desc0 + (uint64_t)((st * L::kTile) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) mma_ss_f8(d_tmem, qd + 2 * kk, kd + 2 * kk, idesc_qk, kk > 0 ? 1u : 0u);
      };
      // O_t += P_t·V over keys 64*part .. 64*part + 63 of the tile
      auto issue_pv = [&](int t, int st, int part, bool acc) {
        const uint32_t d_tmem = tmem + 256 + t * D;
        const uint64_t vd = v_desc0 + (uint64_t)((st * L::kTile) >> 4);
#pragma unroll
        for (int k = 0; k < 2; ++k) {  // 32 keys: 8 TMEM columns of P, 32 bytes of a V^T row
          const int kk = 2 * part + k;
          mma_ts_f8(d_tmem, tmem + t * 128 + kk * 8, vd + 2 * kk, idesc_pv, (acc || kk > 0) ? 1u : 0u);
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
            issue_qk(t, st);
            mma_commit(&bars[kSFull + t]);
          }
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
        mma_commit(&bars[kQEmpty]);
      }
      // All MMAs issued by this thread complete before TMEM is released.
      mma_commit(&bars[kDone]);
      mbar_drain(&bars[kDone], 0);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ linear-branch scan (no barriers)
    if (p.do_scan)
      scan_range(p.scan, (long long)blockIdx.x * 64 + (threadIdx.x - 64), (long long)gridDim.x * 64);
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int t = (warp - 4) >> 2;
    const uint32_t quarter = warp & 3;
    const int row = quarter * 32 + lane;  // query row of the tile == TMEM lane
    const uint32_t lane_base = quarter * 32;
    uint32_t s_cnt = 0, o_cnt = 0;

    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
      // only the key set and the tile count live across the KV loop; the
      // epilogue decodes the item again (fewer registers held in the loop)
      int seg_c, ntiles;
      float sl2;  // scale * log2(e) * q scale * k scale of this (batch, head)
      {
        const Item it = decode_item(item, p);
        seg_c = it.c;
        ntiles = it.ntiles;
        const int bh = it.b * g.H + it.h, BH = g.B * g.H;
        sl2 = p.scale_log2 * (p.fp8_amax[bh] / 448.f) * (fmaxf(p.fp8_amax[BH + bh], p.fp8_amax[3 * BH + bh]) / 448.f);
      }
      if (t >= ntiles) continue;
      float m_run = 0.f, l_run = 0.f;
      bool ok = true;
      // keys left in the current key range (video ranges, then text); only
      // these scalars live across the loop, the ranges are re-derived at
      // range ends
      const int nkv = seg_kv_tiles(seg_c, g);
      int range = 0, left = seg_range_len(seg_c, g, 0);
      {
        for (int j = 0; j < nkv; ++j) {
          while (left == 0) left = seg_range_len(seg_c, g, ++range);
          const int n_valid = min(kBlockN, left);
          left -= n_valid;
          const bool got = mbar_wait(&bars[kSFull + t], s_cnt & 1, ab);
          if (__any_sync(0xffffffffu, !got)) { ok = false; break; }
          ++s_cnt;
          tc_fence_after();
          uint32_t s[128];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t (&chunk)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32 * i]);
            tmem_ld32(tmem_addr(tmem, lane_base, t * 128 + 32 * i), chunk);
          }
          tmem_wait_ld();
          if (n_valid < kBlockN) {
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (i >= n_valid) s[i] = __float_as_uint(-INFINITY);
          }
          // row max: four independent fmax3 chains
          float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
          for (int i = 0; i < 128; i += 8) {
            a0 = fmax3(a0, __uint_as_float(s[i]), __uint_as_float(s[i + 1]));
            a1 = fmax3(a1, __uint_as_float(s[i + 2]), __uint_as_float(s[i + 3]));
            a2 = fmax3(a2, __uint_as_float(s[i + 4]), __uint_as_float(s[i + 5]));
            a3 = fmax3(a3, __uint_as_float(s[i + 6]), __uint_as_float(s[i + 7]));
          }
          const float mx = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
          const float mxs = mx * sl2;
          // lazy rescale: move the running max only when this tile's max is
          // more than 2^4 above it (O is rescaled below, once P is stored)
          float alpha = 1.0f;
          bool rescale = false;
          if (j == 0) {
            m_run = mxs;
          } else {
            const bool need = mxs > m_run + 4.0f;
            rescale = __any_sync(0xffffffffu, need);
            if (need) {
              alpha = ex2_approx(m_run - mxs);
              m_run = mxs;
            }
          }
          l_run *= alpha;
          // p = 2^(s * scale * log2(e) - m): the exponent argument and the
          // row sum in packed f32x2; P goes to TMEM 8 columns (16 keys) at a
          // time, which keeps the live registers under the 168 of a 384-thread
          // CTA (no spills).
          const uint64_t sl2x2 = f32x2_pack(sl2, sl2);
          const uint64_t negm = f32x2_pack(4.0f - m_run, 4.0f - m_run);  // P = 2^(s - m + 4)
          uint64_t lsum0 = f32x2_pack(0.f, 0.f), lsum1 = lsum0;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            uint32_t pk[4];  // 16 keys as e4m3, four per TMEM column
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const uint64_t sx = f32x2_pack(__uint_as_float(s[16 * i + 2 * e]), __uint_as_float(s[16 * i + 2 * e + 1]));
              float x0, x1;
              f32x2_unpack(f32x2_fma(sx, sl2x2, negm), x0, x1);
              float p0, p1;
              if (poly_pair(e)) {
                p0 = exp2_fma(x0);
                p1 = exp2_fma(x1);
              } else {
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
              }
              if (e & 1) lsum1 = f32x2_add(lsum1, f32x2_pack(p0, p1));
              else lsum0 = f32x2_add(lsum0, f32x2_pack(p0, p1));
              const uint32_t pr = e4m3x2(p0, p1);
              if (e & 1) pk[e >> 1] |= pr << 16;
              else pk[e >> 1] = pr;
            }
            tmem_st4(tmem_addr(tmem, lane_base, t * 128 + 4 * i), pk);
            if (i == 3) {
              if (rescale) {
                // O_t is quiescent here: S_t(j) completing implies PV_t(j-1)
                // completed, and PV_t(j) starts only after P_t(j) is handed over.
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
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&bars[kPFull2 + t]);
          {
            float l0, l1, l2, l3;
            f32x2_unpack(lsum0, l0, l1);
            f32x2_unpack(lsum1, l2, l3);
            l_run += (l0 + l1) + (l2 + l3);
          }
        }
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue: o_s = O / l
      const bool got = mbar_wait(&bars[kOFull + t], o_cnt & 1, ab);
      if (__any_sync(0xffffffffu, !got)) break;
      ++o_cnt;
      tc_fence_after();
      const Item it = decode_item(item, p);
      const int bh = it.b * g.H + it.h, BH = g.B * g.H;
      const float inv_l = (fmaxf(p.fp8_amax[2 * BH + bh], p.fp8_amax[4 * BH + bh]) / 448.f) / l_run;
      const int nrows = min(kBlockM, it.nrows - t * kBlockM);  // valid rows of this tile
      __nv_bfloat16* dst = p.o_s + (((size_t)it.b * g.N + (size_t)(it.row0 + t * kBlockM + row)) * g.H + it.h) * D;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        uint32_t o[32];
        tmem_ld32(tmem_addr(tmem, lane_base, 256 + t * D + 32 * i), o);
        tmem_wait_ld();
        if (row < nrows) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * i);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * v4 + 0]) * inv_l, __uint_as_float(o[8 * v4 + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(o[8 * v4 + 2]) * inv_l, __uint_as_float(o[8 * v4 + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(o[8 * v4 + 4]) * inv_l, __uint_as_float(o[8 * v4 + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(o[8 * v4 + 6]) * inv_l, __uint_as_float(o[8 * v4 + 7]) * inv_l);
            d4[v4] = w;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
}

cudaError_t launch_sparse_softmax_fp8(const Maps& m, const K3Params& p, int grid, cudaStream_t st) {
  const size_t need = (size_t)K3Layout<128>::kBytes;
  const size_t smem = need < 118 * 1024 ? 118 * 1024 : need;  // one CTA per SM (all TMEM columns)
  cudaError_t e = cudaFuncSetAttribute(k3_fp8<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k3_fp8<128><<<grid, 384, smem, st>>>(m.q, m.k, m.v, m.tk, m.tv, p);
  return cudaGetLastError();
}

}  // namespace vdn
