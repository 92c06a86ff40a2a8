// scan.cuh - forward/backward states of the VDN-H3 linear branch (article
// section 双分支混合注意力机制: a forward state sums the context before the
// local window, a backward state the context after it, both without the window
// and the anchor frames; the text is written at half weight into each), from
// the state-build partials.
//
// One unit = (batch, head, row n in [0, Dp], 4 consecutive columns a) of
// [S | z] (row Dp = z).  Per unit:
//   1. segment sums: each state segment's partials (one per state-build CTA
//      that met the segment) are added in slot order and stored as the
//      segment state; the video segments (in chunk order) are also added into
//      the running total, the text segment gives t;
//   2. a walk over the chunks keeps Pref(c-2) and the chunk sums CS(c-1),
//      CS(c), CS(c+1) and forms
//          F_c = t/2 + Pref(c-2),   B_c = t/2 + (Total - Pref(c+1)),
//      with B_c exactly t/2 when no chunk lies at or past c+2 (Pref is
//      accumulated in the same order as Total, so Total - Pref is exact where
//      nothing is left);
//   3. M_c = F_c + B_c is written as a bf16 hi/lo pair (hi = bf16(M), lo =
//      bf16(M - hi)) into the readout's B-operand image: rows n (value
//      column; row Dp = z; rows Dp+1..Dp+15 zero, written by the units of
//      rows 0..14, one row each), K = a, K-major with the 128-byte swizzle,
//      so the readout copies it to shared memory with one bulk copy;
//   4. optionally F_c and B_c are exported in fp32.
// Four segments' (and four chunks') loads are issued before any is added, for
// memory-level parallelism.  Deterministic: a fixed order of additions.
#pragma once

#include "kernels.h"
#include "sm100.cuh"

namespace vdn {

__device__ __forceinline__ uint32_t mt_offset(int n, int a, int rows) {
  // byte offset of element (row n, column a) in one K-major SW128 B-tile image
  const int ac = a >> 6;
  const int chunk = ((a & 63) >> 3) ^ (n & 7);
  return (uint32_t)(ac * rows * 128 + n * 128 + chunk * 16 + (a & 7) * 2);
}

__device__ __forceinline__ float4 f4add(float4 x, float4 y) {
  return make_float4(x.x + y.x, x.y + y.y, x.z + y.z, x.w + y.w);
}

// Units of the scan: B * H * (Dp + 1) * (Dp / 4).
__host__ __device__ __forceinline__ long long scan_units(const Geom& g) {
  return (long long)g.B * g.H * (g.Dp + 1) * (g.Dp / 4);
}

// Units of one (batch, head): unit u belongs to (batch, head) u / this.
__host__ __device__ __forceinline__ int scan_units_per_bh(const Geom& g) { return (g.Dp + 1) * (g.Dp / 4); }

__device__ __forceinline__ void scan_unit(const ScanArgs& sa, long long unit) {
  const Geom& g = sa.g;
  const StatePlan& sp = sa.sp;
  const int Dp = g.Dp;
  const int a4s = Dp / 4;
  const int a4 = (int)(unit % a4s);
  long long rem = unit / a4s;
  const int n = (int)(rem % (Dp + 1));
  const int bh = (int)(rem / (Dp + 1));
  const size_t st_elems = (size_t)(Dp + 1) * Dp;
  const size_t off = (size_t)n * Dp + a4 * 4;
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);

  // ---- 1. segment sums, total and text
  float4 total = zero, t = zero;
  for (int s0 = 0; s0 < sp.n_segs; s0 += 4) {
    float4 x[4][2];
    int nc[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int s = s0 + q;
      nc[q] = s < sp.n_segs ? sb_contributors(bh, s, sp) : 0;
      x[q][0] = x[q][1] = zero;
      if (nc[q] > 0) x[q][0] = __ldg(reinterpret_cast<const float4*>(sa.parts + sb_slot(bh, s, 0, sp) * st_elems + off));
      if (nc[q] > 1) x[q][1] = __ldg(reinterpret_cast<const float4*>(sa.parts + sb_slot(bh, s, 1, sp) * st_elems + off));
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int s = s0 + q;
      if (s >= sp.n_segs) break;
      float4 cs = x[q][0];
      if (nc[q] > 1) cs = f4add(cs, x[q][1]);
      for (int u = 2; u < nc[q]; ++u)
        cs = f4add(cs, __ldg(reinterpret_cast<const float4*>(sa.parts + sb_slot(bh, s, u, sp) * st_elems + off)));
      *reinterpret_cast<float4*>(sa.segst + ((size_t)bh * sp.n_segs + s) * st_elems + off) = cs;
      if (s < sp.n_vsegs) total = f4add(total, cs);
      else t = cs;
    }
  }

  // ---- 2./3./4. chunk walk
  const int Nc = g.Nc;
  const int c_first = sp.n_vsegs > 0 ? sp.seg_chunk[0] : Nc;  // video segments are chunks c_first, c_first+1, ...
  auto load_cs = [&](int c) -> float4 {
    const int s = c - c_first;
    if (c >= Nc || s < 0 || s >= sp.n_vsegs) return zero;
    return *reinterpret_cast<const float4*>(sa.segst + ((size_t)bh * sp.n_segs + s) * st_elems + off);
  };
  const int rows = Dp + 16;
  const size_t tile_bytes = (size_t)rows * Dp * 2;
  const int d = g.d;
  const bool exp_row = (n < d) || (n == Dp);
  const int exp_n = (n == Dp) ? d : n;
  const uint32_t mo = mt_offset(n, a4 * 4, rows);
  const bool zero_row = n < 15;
  const uint32_t mo_z = mt_offset(Dp + 1 + (zero_row ? n : 0), a4 * 4, rows);
  const int b = bh / g.H, h = bh % g.H;
  const float4 half_t = make_float4(0.5f * t.x, 0.5f * t.y, 0.5f * t.z, 0.5f * t.w);
  float4 pm2 = zero, cs_m1 = zero, cs_0 = load_cs(0);
  for (int c0 = 0; c0 < Nc; c0 += 4) {
    float4 nx[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) nx[q] = load_cs(c0 + q + 1);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = c0 + q;
      if (c >= Nc) break;
      const float4 cs_p1 = nx[q];
      // Pref(c+1) in the same order as Total
      const float4 pref1 = f4add(f4add(f4add(pm2, cs_m1), cs_0), cs_p1);
      const bool has_suffix = c + 2 <= Nc - 1;
      float Fv[4], Bv[4], M[4];
      const float pre[4] = {pm2.x, pm2.y, pm2.z, pm2.w};
      const float tot[4] = {total.x, total.y, total.z, total.w};
      const float p1[4] = {pref1.x, pref1.y, pref1.z, pref1.w};
      const float ht[4] = {half_t.x, half_t.y, half_t.z, half_t.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        Fv[e] = ht[e] + pre[e];
        Bv[e] = ht[e] + (has_suffix ? tot[e] - p1[e] : 0.f);
        M[e] = Fv[e] + Bv[e];
      }
      uint8_t* tile = sa.mt + (((size_t)b * Nc + c) * g.H + h) * 2 * tile_bytes;
      uint32_t hi[2], lo[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const __nv_bfloat16 h0 = __float2bfloat16_rn(M[2 * e]), h1 = __float2bfloat16_rn(M[2 * e + 1]);
        const float r0 = M[2 * e] - __bfloat162float(h0), r1 = M[2 * e + 1] - __bfloat162float(h1);
        hi[e] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
        lo[e] = pack_bf16x2(r0, r1);
      }
      *reinterpret_cast<uint2*>(tile + mo) = make_uint2(hi[0], hi[1]);
      *reinterpret_cast<uint2*>(tile + tile_bytes + mo) = make_uint2(lo[0], lo[1]);
      if (zero_row) {
        *reinterpret_cast<uint2*>(tile + mo_z) = make_uint2(0, 0);
        *reinterpret_cast<uint2*>(tile + tile_bytes + mo_z) = make_uint2(0, 0);
      }
      if (sa.export_fwd && exp_row) {
        const size_t base = ((((size_t)b * Nc + c) * g.H + h) * (d + 1) + exp_n) * d;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int a = a4 * 4 + e;
          if (a < d) {
            sa.export_fwd[base + a] = Fv[e];
            sa.export_bwd[base + a] = Bv[e];
          }
        }
      }
      // advance: Pref(c-1) = Pref(c-2) + CS(c-1)
      pm2 = f4add(pm2, cs_m1);
      cs_m1 = cs_0;
      cs_0 = cs_p1;
    }
  }
}

// Units unit0, unit0 + stride, ... of the scan.
__device__ __forceinline__ void scan_range(const ScanArgs& sa, long long unit0, long long stride) {
  const long long n = scan_units(sa.g);
  for (long long u = unit0; u < n; u += stride) scan_unit(sa, u);
}

}  // namespace vdn
