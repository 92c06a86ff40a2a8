// plan.h - problem geometry, workspace layout and the index rules of the
// hybrid attention, shared by the host (validation, membership table, launch
// set-up) and the kernels (KV tile enumeration, state membership).
//
// Index rules (VDN-H3 article, section 双分支混合注意力机制):
//   * latent frames are grouped into chunks of C consecutive frames;
//   * the softmax branch of chunk c reads the window chunks
//     max(0, c-1) .. min(Nc-1, c+1) plus the anchor frames 0 and F-1 plus the
//     text; an anchor already inside the window is read once;
//   * the forward state of chunk c holds chunks 0 .. c-2, the backward state
//     chunks c+2 .. Nc-1, both without the anchor frames;
//   * each state also holds half of the text state;
//   * anchor frames as queries follow the same rule (LOCAL), or, under the
//     GLOBAL reading of "the first and last frames interact with all frames",
//     attend by softmax to every frame and read nothing through the states.
#pragma once

#include <cstddef>
#include <cstdint>

#ifdef __CUDACC__
#define VDN_HD __host__ __device__ __forceinline__
#else
#define VDN_HD inline
#endif

namespace vdn {

constexpr int kMaxChunks = 256;     // chunk-order table carried in kernel parameters
constexpr int kStateBuildCtas = 148;  // state-build ranges: one per SM of a B200
constexpr int kBlockM = 128;        // query rows per tile
constexpr int kBlockN = 128;        // keys per tile
constexpr int kMaxSegs = kMaxChunks + 2;  // query segments (chunks, plus the anchor frames under GLOBAL)

struct Geom {
  int B, F, P, H, d, T, C;  // batch, frames, tokens/frame, heads, head_dim, text tokens, chunk frames
  int Dp;                   // head_dim as stored for the tensor cores (64 or 128)
  int Nc;                   // chunks
  long long N;              // F * P video tokens per batch
  int staged;               // inputs are converted/padded into the workspace first
  int fp32_io;              // q/k/v/text/gates/out are fp32
  int n_state_segs;         // state segments per (batch, head): chunks with a non-anchor frame, + text
  long long n_part_slots;   // state-build partial slots: B * H * n_state_segs * cmax
  int rows_per_chunk;       // C * P query rows
  int n_pairs;              // work items of two 128-row query tiles per chunk
  int mt_rows;              // rows of one readout B-tile: Dp + 16 (values, z, zero padding)
  int anchor_global;        // 1: anchor query frames attend to every frame, no linear read
  float scale;              // softmax scale
  float eps;                // RMSNorm epsilon
  // workspace layout (byte offsets; each 1024-aligned)
  size_t off_status, off_os, off_q, off_k, off_v, off_tk, off_tv, off_parts, off_segst, off_mt, off_done, total;
  int fp8;                  // softmax branch with e4m3 operands
  long long pitch_v8, pitch_t8;  // row pitches (bytes) of the transposed e4m3 v and text_v
  size_t off_q8, off_k8, off_vt8, off_tk8, off_tvt8, off_amax;
};

VDN_HD int is_anchor(int f, int F) { return f == 0 || f == F - 1; }
VDN_HD int n_anchor(int F) { return F == 1 ? 1 : 2; }

// Number of non-anchor frames in chunks [c0, c1] (empty if c1 < c0).
VDN_HD int nonanchor_frames_in_chunks(int c0, int c1, int C, int F) {
  if (c1 < c0) return 0;
  int f0 = c0 * C, f1 = (c1 + 1) * C - 1;  // inclusive frame range
  int n = f1 - f0 + 1;
  if (f0 <= 0 && 0 <= f1) n--;
  if (F - 1 != 0 && f0 <= F - 1 && F - 1 <= f1) n--;
  return n;
}

// Tokens held by the two states of chunk c (text counted once); 0 means an empty read.
VDN_HD long long state_tokens(int c, const Geom& g) {
  int nf = nonanchor_frames_in_chunks(0, c - 2, g.C, g.F) + nonanchor_frames_in_chunks(c + 2, g.Nc - 1, g.C, g.F);
  return (long long)g.T + (long long)g.P * nf;
}

// Video key token ranges [start, start+len) read by the softmax branch of
// chunk c: window plus anchors, adjacent ranges merged, at most three.
struct KvRanges {
  long long start[3];
  long long len[3];
  int n;
};

VDN_HD void kv_ranges(int c, const Geom& g, KvRanges& r) {
  const int wlo = (c - 1 > 0 ? c - 1 : 0) * g.C;                        // first window frame
  const int whi = ((c + 1 < g.Nc - 1 ? c + 1 : g.Nc - 1) + 1) * g.C;    // one past last window frame
  long long s[3], e[3];
  int n = 0;
  if (wlo > 0) { s[n] = 0; e[n] = g.P; n++; }                            // anchor 0 before the window
  s[n] = (long long)wlo * g.P; e[n] = (long long)whi * g.P; n++;          // window
  if (whi < g.F) { s[n] = (long long)(g.F - 1) * g.P; e[n] = (long long)g.F * g.P; n++; }  // last anchor after it
  // merge touching ranges
  r.n = 0;
  for (int i = 0; i < n; ++i) {
    if (r.n > 0 && r.start[r.n - 1] + r.len[r.n - 1] == s[i]) {
      r.len[r.n - 1] += e[i] - s[i];
    } else {
      r.start[r.n] = s[i];
      r.len[r.n] = e[i] - s[i];
      r.n++;
    }
  }
}

VDN_HD int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

// KV tiles of 128 keys enumerated by the softmax kernel for chunk c.
VDN_HD int kv_tiles(int c, const Geom& g) {
  KvRanges r;
  kv_ranges(c, g, r);
  int n = 0;
  for (int i = 0; i < r.n; ++i) n += ceil_div(r.len[i], kBlockN);
  return n + ceil_div(g.T, kBlockN);
}

// A query segment: rows [row0, row0 + nrows) of one batch that read the same
// key set through the softmax branch: the window of chunk c (c >= 0) or every
// video frame (c = kAllFrames).
constexpr int kAllFrames = -1;
struct QSeg {
  int row0, nrows, c;
};

// Video key ranges of a segment's key set.
VDN_HD void seg_ranges(int c, const Geom& g, KvRanges& r) {
  if (c == kAllFrames) {
    r.n = 1;
    r.start[0] = 0;
    r.len[0] = g.N;
    return;
  }
  kv_ranges(c, g, r);
}

// Keys in range r of a segment's key set (video ranges in order, then the
// text as the last range); 0 past the end.
VDN_HD int seg_range_len(int c, const Geom& g, int r) {
  KvRanges kr;
  seg_ranges(c, g, kr);
  for (int i = 0; i < 3; ++i)
    if (i < kr.n && i == r) return (int)kr.len[i];
  return r == kr.n ? g.T : 0;
}

VDN_HD int seg_kv_tiles(int c, const Geom& g) {
  KvRanges r;
  seg_ranges(c, g, r);
  int n = 0;
  for (int i = 0; i < r.n; ++i) n += ceil_div(r.len[i], kBlockN);
  return n + ceil_div(g.T, kBlockN);
}

// Query frame f reads nothing through the states (GLOBAL anchor).
VDN_HD int no_linear_read(int f, const Geom& g) { return g.anchor_global && is_anchor(f, g.F); }

// The query segments in row order; returns their number (<= Nc + 2).
inline int query_segments(const Geom& g, QSeg* out) {
  int n = 0;
  for (int c = 0; c < g.Nc; ++c) {
    int lo = c * g.C, hi = (c + 1) * g.C;  // frames [lo, hi)
    if (!g.anchor_global) {
      out[n++] = QSeg{lo * g.P, (hi - lo) * g.P, c};
      continue;
    }
    if (lo == 0) { out[n++] = QSeg{0, g.P, kAllFrames}; lo = 1; }
    const bool last_here = hi == g.F && g.F - 1 >= lo;
    if (last_here) hi = g.F - 1;
    if (hi > lo) out[n++] = QSeg{lo * g.P, (hi - lo) * g.P, c};
    if (last_here) out[n++] = QSeg{(g.F - 1) * g.P, g.P, kAllFrames};
  }
  return n;
}

// Last chunk summed by the forward state of chunk c, first chunk summed by
// its backward state (the window is c-1 .. c+1).
VDN_HD int fwd_last_chunk(int c) { return c - 2; }
VDN_HD int bwd_first_chunk(int c) { return c + 2; }

// ---------------------------------------------------------------- state build plan
//
// The state build walks, for every (batch, head), the state segments in
// order: one video segment per chunk that holds a non-anchor frame (its
// non-anchor frames are consecutive token rows) and, when T > 0, the text.
// A segment is cut into 128-token tiles; the tiles of all (batch, head)
// pairs, (batch, head)-major, form one list that is split into `grid` equal
// contiguous ranges, one per CTA (every CTA gets the same number of tiles,
// +-1).  A CTA accumulates phi(K)^T [V | 1] over the run of its tiles that
// falls in one segment and writes it as one partial; a segment gets one
// partial from each CTA whose range meets it, in slots
// seg_slot0(gseg) + 0, 1, ... (at most `cmax` per segment).

constexpr int kMaxStateSegs = kMaxChunks + 1;  // video segments (one per chunk) + text

struct StatePlan {
  int n_segs;                         // segments per (batch, head)
  int n_vsegs;                        // of which video (chunk) segments; the text segment is last
  int seg_chunk[kMaxStateSegs];       // chunk of a video segment
  int seg_row0[kMaxStateSegs];        // first token row within the batch (video rows, or text rows)
  int seg_rows[kMaxStateSegs];        // token rows of the segment
  int seg_tile0[kMaxStateSegs + 1];   // first tile of the segment within one (batch, head)
  int tiles_per_bh;
  int grid;                           // state-build CTAs (ranges)
  int cmax;                           // partial slots per segment
  long long total_tiles;              // B * H * tiles_per_bh
};

// CTA whose range holds global tile t: ranges start at floor(k * TT / G).
VDN_HD int sb_cta_of(long long t, const StatePlan& sp) {
  return (int)(((t + 1) * sp.grid - 1) / sp.total_tiles);
}
VDN_HD long long sb_range_start(int k, const StatePlan& sp) { return (long long)k * sp.total_tiles / sp.grid; }

// Partial slot of contributor u (0, 1, ...) of segment s of (batch, head) bh.
VDN_HD long long sb_slot(int bh, int s, int u, const StatePlan& sp) {
  return ((long long)bh * sp.n_segs + s) * sp.cmax + u;
}

// Number of CTAs whose range meets segment s of bh (partials written for it).
VDN_HD int sb_contributors(int bh, int s, const StatePlan& sp) {
  const long long t0 = (long long)bh * sp.tiles_per_bh + sp.seg_tile0[s];
  const long long t1 = (long long)bh * sp.tiles_per_bh + sp.seg_tile0[s + 1] - 1;
  return sb_cta_of(t1, sp) - sb_cta_of(t0, sp) + 1;
}

// Host: the state-build plan of a problem (segments, tile ranges, slots).
// Needs g.B, g.H, g.P, g.T, g.C, g.F, g.Nc.
inline void build_state_plan(const Geom& g, StatePlan& sp) {
  sp.n_segs = 0;
  int tiles = 0;
  for (int c = 0; c < g.Nc; ++c) {
    // the chunk's frames [c*C, (c+1)*C) without the anchors 0 and F-1 are consecutive
    const int f0 = c * g.C > 1 ? c * g.C : 1;
    const int f1 = (c + 1) * g.C < g.F - 1 ? (c + 1) * g.C : g.F - 1;
    if (f1 <= f0) continue;
    const int n = sp.n_segs++;
    sp.seg_chunk[n] = c;
    sp.seg_row0[n] = f0 * g.P;
    sp.seg_rows[n] = (f1 - f0) * g.P;
    sp.seg_tile0[n] = tiles;
    tiles += ceil_div(sp.seg_rows[n], 128);
  }
  sp.n_vsegs = sp.n_segs;
  if (g.T > 0) {
    const int n = sp.n_segs++;
    sp.seg_chunk[n] = -1;
    sp.seg_row0[n] = 0;
    sp.seg_rows[n] = g.T;
    sp.seg_tile0[n] = tiles;
    tiles += ceil_div(g.T, 128);
  }
  sp.seg_tile0[sp.n_segs] = tiles;
  sp.tiles_per_bh = tiles;
  sp.total_tiles = (long long)g.B * g.H * tiles;
  sp.grid = (int)(sp.total_tiles < kStateBuildCtas ? sp.total_tiles : kStateBuildCtas);
  sp.cmax = 0;
  if (sp.grid == 0) return;
  for (int bh = 0; bh < g.B * g.H; ++bh)
    for (int s = 0; s < sp.n_segs; ++s) {
      const int n = sb_contributors(bh, s, sp);
      if (n > sp.cmax) sp.cmax = n;
    }
}

// Segment of local tile lt of a (batch, head) (binary search over seg_tile0).
VDN_HD int sb_seg_of(int lt, const StatePlan& sp) {
  int lo = 0, hi = sp.n_segs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sp.seg_tile0[mid] <= lt) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

}  // namespace vdn
