// api.cu - host side of libvdnattn: argument checks, geometry and workspace
// layout, the host membership table, TMA descriptors and the launch sequence
// of the hybrid attention (declared in include/vdnattn.h).
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <numeric>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "kernels.h"
#include "vdnattn.h"

namespace vdn {
namespace {

// NVTX range around the host-side launch of one step (the ranges a profiler
// shows next to the kernels; without a profiler attached they cost a few
// nanoseconds).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr int kMaxScanChunks = kMaxChunks;  // state segments carried in kernel parameters

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The softmax kernel's fused readout epilogue: bf16 tensors of head_dim 128,
// bf16 softmax operands, the merged output without debug outputs.
bool fused_readout_supported(const vdn_cfg* cfg) {
  return cfg->dtype == VDN_BF16 && cfg->head_dim == 128 && cfg->softmax_precision == VDN_PREC_BF16 &&
         cfg->output_mode == VDN_OUTPUT_MERGED &&
         !(cfg->debug_flags & (VDN_OUT_SOFTMAX_ONLY | VDN_OUT_LINEAR_ONLY | VDN_OUT_LINEAR_RAW));
}

vdn_status make_geom(const vdn_cfg* cfg, Geom& g) {
  if (!cfg) return VDN_ERR_INVALID_ARG;
  if (cfg->batch < 1 || cfg->frames < 1 || cfg->tokens_per_frame < 1 || cfg->heads < 1 || cfg->text_tokens < 0 ||
      cfg->chunk_frames < 1)
    return VDN_ERR_INVALID_ARG;
  if (cfg->softmax_precision != VDN_PREC_BF16 && cfg->softmax_precision != VDN_PREC_FP8) return VDN_ERR_INVALID_ARG;
  if (cfg->softmax_precision == VDN_PREC_FP8 &&
      (cfg->head_dim != 128 || cfg->dtype != VDN_BF16 || cfg->tokens_per_frame % 16 != 0 ||
       (long long)cfg->batch * cfg->heads * 5 * 4 > 48 * 1024))
    return VDN_ERR_UNSUPPORTED;
  if (cfg->anchor_query_mode != VDN_ANCHOR_LOCAL && cfg->anchor_query_mode != VDN_ANCHOR_GLOBAL)
    return VDN_ERR_INVALID_ARG;
  if (cfg->output_mode != VDN_OUTPUT_MERGED && cfg->output_mode != VDN_OUTPUT_SPLIT) return VDN_ERR_INVALID_ARG;
  if (cfg->output_mode == VDN_OUTPUT_SPLIT &&
      (cfg->debug_flags & (VDN_OUT_SOFTMAX_ONLY | VDN_OUT_LINEAR_ONLY | VDN_OUT_LINEAR_RAW)))
    return VDN_ERR_INVALID_ARG;
  if (cfg->readout_mode != VDN_READOUT_SEPARATE && cfg->readout_mode != VDN_READOUT_FUSED) return VDN_ERR_INVALID_ARG;
  if (cfg->readout_mode == VDN_READOUT_FUSED && !fused_readout_supported(cfg)) return VDN_ERR_UNSUPPORTED;
  if (cfg->frames % cfg->chunk_frames != 0) return VDN_ERR_INVALID_ARG;
  if (cfg->head_dim != 32 && cfg->head_dim != 64 && cfg->head_dim != 128) return VDN_ERR_UNSUPPORTED;
  if (cfg->dtype != VDN_BF16 && cfg->dtype != VDN_FP32) return VDN_ERR_UNSUPPORTED;
  if (cfg->debug_flags &
      ~(VDN_OUT_SOFTMAX_ONLY | VDN_OUT_LINEAR_ONLY | VDN_OUT_LINEAR_RAW | VDN_EXPORT_STATES | VDN_INJECT_TIMEOUT |
        VDN_INJECT_TIMEOUT_SCAN |
        VDN_STALL_READOUT_MMA | VDN_POISON_WS))
    return VDN_ERR_INVALID_ARG;
  const int Nc = cfg->frames / cfg->chunk_frames;
  if (Nc > kMaxScanChunks) return VDN_ERR_UNSUPPORTED;
  const long long N = (long long)cfg->frames * cfg->tokens_per_frame;
  // TMA row coordinates and tile arithmetic are 32-bit
  if ((long long)cfg->batch * N >= (1ll << 30) || (long long)cfg->batch * cfg->text_tokens >= (1ll << 30) ||
      (long long)cfg->chunk_frames * cfg->tokens_per_frame >= (1ll << 28) || cfg->heads > 4096)
    return VDN_ERR_UNSUPPORTED;

  std::memset(&g, 0, sizeof(g));
  g.B = cfg->batch;
  g.F = cfg->frames;
  g.P = cfg->tokens_per_frame;
  g.H = cfg->heads;
  g.d = cfg->head_dim;
  g.T = cfg->text_tokens;
  g.C = cfg->chunk_frames;
  g.Dp = g.d == 128 ? 128 : 64;
  g.Nc = Nc;
  g.N = N;
  g.fp32_io = cfg->dtype == VDN_FP32;
  g.staged = g.fp32_io || g.d != g.Dp;
  {
    StatePlan sp;
    build_state_plan(g, sp);
    g.n_state_segs = sp.n_segs;
    g.n_part_slots = (long long)g.B * g.H * sp.n_segs * sp.cmax;
  }
  g.rows_per_chunk = g.C * g.P;
  g.n_pairs = (g.rows_per_chunk + 2 * kBlockM - 1) / (2 * kBlockM);
  g.mt_rows = g.Dp + 16;
  g.anchor_global = cfg->anchor_query_mode == VDN_ANCHOR_GLOBAL;
  g.scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.0f / std::sqrt((float)g.d);
  g.eps = cfg->rms_eps < 0.f ? 1e-6f : cfg->rms_eps;

  const size_t vid = (size_t)g.B * g.N * g.H * g.Dp * 2;
  const size_t txt = (size_t)g.B * g.T * g.H * g.Dp * 2;
  size_t off = 0;
  g.off_status = off; off = align_up(off + 256, 1024);
  g.off_os = off; off = align_up(off + vid, 1024);
  if (g.staged) {
    g.off_q = off; off = align_up(off + vid, 1024);
    g.off_k = off; off = align_up(off + vid, 1024);
    g.off_v = off; off = align_up(off + vid, 1024);
    g.off_tk = off; off = align_up(off + txt, 1024);
    g.off_tv = off; off = align_up(off + txt, 1024);
  }
  const size_t state_bytes = (size_t)(g.Dp + 1) * g.Dp * 4;
  g.off_parts = off; off = align_up(off + (size_t)g.n_part_slots * state_bytes, 1024);
  g.off_segst = off; off = align_up(off + (size_t)g.B * g.H * g.n_state_segs * state_bytes, 1024);
  g.off_mt = off; off = align_up(off + (size_t)g.B * g.Nc * g.H * 2 * g.mt_rows * g.Dp * 2, 1024);
  g.off_done = off; off = align_up(off + (size_t)g.B * g.H * 4, 1024);  // scan units done per (batch, head)
  g.fp8 = cfg->softmax_precision == VDN_PREC_FP8;
  if (g.fp8) {
    g.pitch_v8 = (long long)align_up((size_t)g.N, 16);
    g.pitch_t8 = (long long)align_up((size_t)g.T, 16);
    const size_t vid8 = (size_t)g.B * g.N * g.H * 128, txt8 = (size_t)g.B * g.T * g.H * 128;
    g.off_q8 = off; off = align_up(off + vid8, 1024);
    g.off_k8 = off; off = align_up(off + vid8, 1024);
    g.off_vt8 = off; off = align_up(off + (size_t)g.B * g.H * 128 * g.pitch_v8, 1024);
    g.off_tk8 = off; off = align_up(off + txt8, 1024);
    g.off_tvt8 = off; off = align_up(off + (size_t)g.B * g.H * 128 * g.pitch_t8, 1024);
    g.off_amax = off; off = align_up(off + sizeof(float) * 5 * g.B * g.H, 1024);
  }
  g.total = off;
  return VDN_OK;
}

vdn_status check_ws(const vdn_cfg* cfg, const Geom& g) {
  if (!cfg->workspace || cfg->workspace_bytes < g.total) return VDN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(cfg->workspace) & 255u) != 0) return VDN_ERR_ALIGNMENT;
  if (cfg->status_word && (reinterpret_cast<uintptr_t>(cfg->status_word) & 3u) != 0) return VDN_ERR_ALIGNMENT;
  if (cfg->rms_weight && (reinterpret_cast<uintptr_t>(cfg->rms_weight) & 15u) != 0) return VDN_ERR_ALIGNMENT;
  return VDN_OK;
}

vdn_status check_ptrs(std::initializer_list<const void*> required) {
  for (const void* p : required) {
    if (!p) return VDN_ERR_INVALID_ARG;
    if (!aligned16(p)) return VDN_ERR_ALIGNMENT;
  }
  return VDN_OK;
}

uint8_t* ws(const vdn_cfg* cfg, size_t off) { return static_cast<uint8_t*>(cfg->workspace) + off; }

int* status_ptr(const vdn_cfg* cfg, const Geom& g) {
  return cfg->status_word ? cfg->status_word : reinterpret_cast<int*>(ws(cfg, g.off_status));
}

// VDN_POISON_WS: 0xFF over the workspace past the 256-byte status slot.
cudaError_t poison_ws(const vdn_cfg* cfg, const Geom& g, cudaStream_t st) {
  if (!(cfg->debug_flags & VDN_POISON_WS) || g.total <= 256) return cudaSuccess;
  return cudaMemsetAsync(ws(cfg, 256), 0xFF, g.total - 256, st);
}

// Timeout record of the kernels' bounded waits: 16 int words at byte 64 of
// the workspace's status slot (the workspace status word, when used, is at
// byte 0).  Written only when a wait runs out; cleared by the caller.
int* record_ptr(const vdn_cfg* cfg, const Geom& g) {
  return reinterpret_cast<int*>(ws(cfg, g.off_status) + 64);
}

// ---------------------------------------------------------------- TMA descriptors

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 view [rows, H*Dp] (row pitch H*Dp*2 bytes), box box_rows rows x
// 64 columns, 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, long long rows, int H, int Dp, int box_rows = 128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  if (rows < 1) rows = 1;
  const cuuint64_t dims[2] = {(cuuint64_t)H * Dp, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)H * Dp * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D e4m3 (byte) view [rows, cols] with the given row pitch (bytes), box 128 x
// 128, 128-byte swizzle.
bool make_map8(CUtensorMap* m, const void* base, long long rows, long long cols, long long pitch) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  if (rows < 1) rows = 1;
  if (cols < 1) cols = 1;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(pitch < 16 ? 16 : pitch)};
  const cuuint32_t box[2] = {128, 128};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Srcs {
  const void *q, *k, *v, *tk, *tv;
};

// Tensors the kernels read: the caller's (bf16, head_dim 64/128) or the staged copies.
Srcs kernel_srcs(const vdn_cfg* cfg, const Geom& g, const void* q, const void* k, const void* v, const void* tk,
                 const void* tv) {
  if (!g.staged) return Srcs{q, k, v, tk, tv};
  return Srcs{ws(cfg, g.off_q), ws(cfg, g.off_k), ws(cfg, g.off_v), ws(cfg, g.off_tk), ws(cfg, g.off_tv)};
}

bool make_maps(Maps& m, const Geom& g, const Srcs& s, int box_rows = 128) {
  const long long vrows = (long long)g.B * g.N;
  const long long trows = (long long)g.B * g.T;
  bool ok = make_map(&m.q, s.q, vrows, g.H, g.Dp, box_rows) && make_map(&m.k, s.k, vrows, g.H, g.Dp, box_rows) &&
            make_map(&m.v, s.v, vrows, g.H, g.Dp, box_rows);
  if (g.T > 0) {
    ok = ok && make_map(&m.tk, s.tk, trows, g.H, g.Dp, box_rows) && make_map(&m.tv, s.tv, trows, g.H, g.Dp, box_rows);
  } else {  // never read; any valid descriptor
    m.tk = m.q;
    m.tv = m.q;
  }
  return ok;
}

vdn_status cuda_status(cudaError_t e) { return e == cudaSuccess ? VDN_OK : VDN_ERR_CUDA; }

// ---------------------------------------------------------------- steps

vdn_status step_stage(const vdn_cfg* cfg, const Geom& g, const void* q, const void* k, const void* v, const void* tk,
                      const void* tv, cudaStream_t st) {
  NvtxRange nvtx("vdn:stage");
  if (!g.staged) return VDN_OK;
  const long long vrows = (long long)g.B * g.N, trows = (long long)g.B * g.T;
  cudaError_t e = launch_stage(q, g.fp32_io, reinterpret_cast<__nv_bfloat16*>(ws(cfg, g.off_q)), vrows, g.H, g.d, g.Dp, st);
  if (e == cudaSuccess) e = launch_stage(k, g.fp32_io, reinterpret_cast<__nv_bfloat16*>(ws(cfg, g.off_k)), vrows, g.H, g.d, g.Dp, st);
  if (e == cudaSuccess) e = launch_stage(v, g.fp32_io, reinterpret_cast<__nv_bfloat16*>(ws(cfg, g.off_v)), vrows, g.H, g.d, g.Dp, st);
  if (e == cudaSuccess && g.T > 0)
    e = launch_stage(tk, g.fp32_io, reinterpret_cast<__nv_bfloat16*>(ws(cfg, g.off_tk)), trows, g.H, g.d, g.Dp, st);
  if (e == cudaSuccess && g.T > 0)
    e = launch_stage(tv, g.fp32_io, reinterpret_cast<__nv_bfloat16*>(ws(cfg, g.off_tv)), trows, g.H, g.d, g.Dp, st);
  return cuda_status(e);
}

// 8-byte counter of the scan units the softmax kernel has handed out, at byte
// 128 of the workspace's status slot.
unsigned long long* scan_counter_ptr(const vdn_cfg* cfg, const Geom& g) {
  return reinterpret_cast<unsigned long long*>(ws(cfg, g.off_status) + 128);
}

// Scan units completed per (batch, head), counted by the softmax kernel's
// scan and zeroed by the state build (the fused readout waits for its
// (batch, head) to be complete before it reads M_c).
unsigned* scan_done_ptr(const vdn_cfg* cfg, const Geom& g) { return reinterpret_cast<unsigned*>(ws(cfg, g.off_done)); }

// Flag at byte 136 of the status slot, written by the softmax kernel: 1 when
// o_s in the workspace holds sigmoid(g_s) * o_s.
int* os_gated_ptr(const vdn_cfg* cfg, const Geom& g) { return reinterpret_cast<int*>(ws(cfg, g.off_status) + 136); }

// The readout reads everything by TMA (bf16, head_dim without padding); only
// then does the softmax kernel take the gate of its branch.
bool tma_readout(const Geom& g) { return !g.fp32_io && g.d == g.Dp; }

vdn_status step_state_build(const vdn_cfg* cfg, const Geom& g, const Srcs& s, cudaStream_t st) {
  NvtxRange nvtx("vdn:state_build");
  K1Params p;
  p.g = g;
  build_state_plan(g, p.sp);
  Maps m;
  if (!make_maps(m, g, s)) return VDN_ERR_CUDA;
  p.parts = reinterpret_cast<float*>(ws(cfg, g.off_parts));
  p.status = status_ptr(cfg, g);
  p.record = record_ptr(cfg, g);
  p.inject_timeout = (cfg->debug_flags & VDN_INJECT_TIMEOUT) != 0;
  p.scan_counter = scan_counter_ptr(cfg, g);
  p.scan_done = scan_done_ptr(cfg, g);
  return cuda_status(launch_state_build(m, p, st));
}

void make_scan_args(const vdn_cfg* cfg, const Geom& g, ScanArgs& sa) {
  sa.g = g;
  build_state_plan(g, sa.sp);
  sa.parts = reinterpret_cast<const float*>(ws(cfg, g.off_parts));
  sa.segst = reinterpret_cast<float*>(ws(cfg, g.off_segst));
  sa.mt = ws(cfg, g.off_mt);
  const bool exp = (cfg->debug_flags & VDN_EXPORT_STATES) != 0;
  sa.export_fwd = exp ? cfg->export_fwd : nullptr;
  sa.export_bwd = exp ? cfg->export_bwd : nullptr;
}

vdn_status step_state_scan(const vdn_cfg* cfg, const Geom& g, cudaStream_t st) {
  NvtxRange nvtx("vdn:state_scan");
  ScanArgs sa;
  make_scan_args(cfg, g, sa);
  return cuda_status(launch_state_scan(sa, st));
}

// Work items of the softmax kernel.  Block 0: the segments that read every
// frame (GLOBAL anchor rows), the longest items, first.  Block 1: the chunk
// segments in chunk order, so that the items the persistent CTAs run at the
// same time share a head's keys and values (and neighbouring chunks two of
// their three window chunks).  Each block is ordered (batch, head, segment,
// pair).
void plan_items(const Geom& g, K3Params& p) {
  QSeg segs[kMaxSegs];
  const int n = query_segments(g, segs);
  int k = 0, nb = 0;
  p.blk_seg0[0] = 0;
  for (int blk = 0; blk < 2; ++blk) {
    const int k0 = k;
    for (int i = 0; i < n; ++i)
      if ((segs[i].c == kAllFrames) == (blk == 0)) p.segs[k++] = segs[i];
    if (k > k0) p.blk_seg0[++nb] = k;
  }
  p.n_blocks = nb;
  p.seg_pair0[0] = 0;
  for (int i = 0; i < k; ++i)
    p.seg_pair0[i + 1] = p.seg_pair0[i] + (p.segs[i].nrows + 2 * kBlockM - 1) / (2 * kBlockM);
  p.blk_item0[0] = 0;
  for (int b = 0; b < nb; ++b)
    p.blk_item0[b + 1] = p.blk_item0[b] + g.B * g.H * (p.seg_pair0[p.blk_seg0[b + 1]] - p.seg_pair0[p.blk_seg0[b]]);
  p.n_items = p.blk_item0[nb];
}

// The softmax branch; with do_scan, the kernel also runs the forward/backward
// scan of the state partials in the workspace; with gate_s (bf16 tensors whose
// head_dim needs no padding, not under VDN_OUT_SOFTMAX_ONLY), o_s is written
// as sigmoid(gate_s) * o_s.  With out (the fused readout): the kernel writes
// the merged output itself, from gate_s, gate_l and the readout operands.
vdn_status step_sparse_softmax(const vdn_cfg* cfg, const Geom& g, const Srcs& s, cudaStream_t st, bool do_scan,
                               const void* gate_s, const void* gate_l = nullptr, void* out = nullptr) {
  NvtxRange nvtx("vdn:sparse_softmax");
  Maps m;
  if (!make_maps(m, g, s)) return VDN_ERR_CUDA;
  K3Params p;
  std::memset(&p, 0, sizeof(p));
  p.g = g;
  if (g.fp8) {
    // e4m3 operands, then the same walk with kind::f8f6f4 MMAs
    Fp8Src src{{static_cast<const __nv_bfloat16*>(s.q), static_cast<const __nv_bfloat16*>(s.k),
                static_cast<const __nv_bfloat16*>(s.v), static_cast<const __nv_bfloat16*>(s.tk),
                static_cast<const __nv_bfloat16*>(s.tv)}};
    Fp8Dst dst{ws(cfg, g.off_q8), ws(cfg, g.off_k8), ws(cfg, g.off_vt8), ws(cfg, g.off_tk8), ws(cfg, g.off_tvt8),
               g.pitch_v8, g.pitch_t8};
    float* amax = reinterpret_cast<float*>(ws(cfg, g.off_amax));
    cudaError_t e = launch_fp8_quant(src, dst, g.B, g.N, g.T, g.H, amax, st);
    if (e != cudaSuccess) return VDN_ERR_CUDA;
    const long long vrows = (long long)g.B * g.N, trows = (long long)g.B * g.T, vtrows = (long long)g.B * g.H * 128;
    if (!make_map8(&m.q, dst.q, vrows, (long long)g.H * 128, (long long)g.H * 128) ||
        !make_map8(&m.k, dst.k, vrows, (long long)g.H * 128, (long long)g.H * 128) ||
        !make_map8(&m.v, dst.vt, vtrows, g.N, g.pitch_v8))
      return VDN_ERR_CUDA;
    if (g.T > 0) {
      if (!make_map8(&m.tk, dst.tk, trows, (long long)g.H * 128, (long long)g.H * 128) ||
          !make_map8(&m.tv, dst.tvt, vtrows, g.T, g.pitch_t8))
        return VDN_ERR_CUDA;
    } else {
      m.tk = m.q;
      m.tv = m.q;
    }
    p.fp8_amax = amax;
  }
  p.scale_log2 = g.scale * 1.4426950408889634f;
  p.o_s = reinterpret_cast<__nv_bfloat16*>(ws(cfg, g.off_os));
  p.status = status_ptr(cfg, g);
  p.record = record_ptr(cfg, g);
  plan_items(g, p);
  p.do_scan = do_scan ? 1 : 0;
  p.scan_counter = scan_counter_ptr(cfg, g);
  p.os_gated = os_gated_ptr(cfg, g);
  p.gate_s = (gate_s && tma_readout(g) && !g.fp8 && !(cfg->debug_flags & VDN_OUT_SOFTMAX_ONLY))
                 ? static_cast<const __nv_bfloat16*>(gate_s)
                 : nullptr;
  if (out) {
    // fused readout: the kernel writes out itself from the scan's M_c
    p.out = static_cast<__nv_bfloat16*>(out);
    p.gate_s = static_cast<const __nv_bfloat16*>(gate_s);
    p.gate_l = static_cast<const __nv_bfloat16*>(gate_l);
    p.mt = ws(cfg, g.off_mt);
    p.gamma = cfg->rms_weight;
    p.scan_done = do_scan ? scan_done_ptr(cfg, g) : nullptr;
    p.inject_scan_wait = do_scan && (cfg->debug_flags & VDN_INJECT_TIMEOUT_SCAN) ? 1 : 0;
  }
  if (do_scan) make_scan_args(cfg, g, p.scan);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::min(p.n_items, sms);
  return cuda_status(g.fp8 ? launch_sparse_softmax_fp8(m, p, grid, st) : launch_sparse_softmax(m, p, grid, st));
}

vdn_status step_readout_merge(const vdn_cfg* cfg, const Geom& g, const Srcs& s, const void* gs, const void* gl,
                              void* out, cudaStream_t st) {
  NvtxRange nvtx("vdn:readout_merge");
  Maps m;
  if (!make_maps(m, g, s)) return VDN_ERR_CUDA;
  K4Params p;
  p.g = g;
  p.o_s = reinterpret_cast<const __nv_bfloat16*>(ws(cfg, g.off_os));
  p.mt = ws(cfg, g.off_mt);
  p.gamma = cfg->rms_weight;
  p.gate_s = gs;
  p.gate_l = gl;
  p.out = out;
  p.out_linear = cfg->output_mode == VDN_OUTPUT_SPLIT ? cfg->out_linear : nullptr;
  p.flags = cfg->debug_flags & (VDN_OUT_SOFTMAX_ONLY | VDN_OUT_LINEAR_ONLY | VDN_OUT_LINEAR_RAW);
  p.stall_ns = (cfg->debug_flags & VDN_STALL_READOUT_MMA) ? 50000 : 0;
  p.os_gated = os_gated_ptr(cfg, g);
  p.status = status_ptr(cfg, g);
  p.record = record_ptr(cfg, g);
  if (tma_readout(g)) {
    // bf16 tensors without head_dim padding: every input tile by TMA
    MergeMaps mm;
    mm.q = m.q;
    const long long vrows = (long long)g.B * g.N;
    if (!make_map(&mm.os, ws(cfg, g.off_os), vrows, g.H, g.Dp) || !make_map(&mm.gs, gs, vrows, g.H, g.Dp) ||
        !make_map(&mm.gl, gl, vrows, g.H, g.Dp) || !make_map(&mm.out, out, vrows, g.H, g.Dp))
      return VDN_ERR_CUDA;
    return cuda_status(launch_readout_merge_tma(mm, p, st));
  }
  return cuda_status(launch_readout_merge(m, p, st));
}

vdn_status check_inputs(const vdn_cfg* cfg, const Geom& g, std::initializer_list<const void*> video,
                        std::initializer_list<const void*> text) {
  vdn_status s = check_ws(cfg, g);
  if (s != VDN_OK) return s;
  s = check_ptrs(video);
  if (s != VDN_OK) return s;
  if (g.T > 0) s = check_ptrs(text);
  return s;
}

// ---------------------------------------------------------------- calls on host tensors

// Device staging of vdn_hybrid_attn_fwd_host: the caller's tensors in their
// own dtype and layout, 256-byte aligned slots.
struct HostStaging {
  size_t q, k, v, tk, tv, gs, gl, out, out_lin, total;
};

HostStaging host_staging(const vdn_cfg* cfg, const Geom& g) {
  const size_t e = g.fp32_io ? 4 : 2;
  const size_t vid = (size_t)g.B * g.N * g.H * g.d * e, txt = (size_t)g.B * g.T * g.H * g.d * e;
  HostStaging h;
  size_t off = 0;
  auto take = [&](size_t n) {
    const size_t o = off;
    off = align_up(off + n, 256);
    return o;
  };
  h.q = take(vid);
  h.k = take(vid);
  h.v = take(vid);
  h.tk = take(txt);
  h.tv = take(txt);
  h.gs = take(vid);
  h.gl = take(vid);
  h.out = take(vid);
  h.out_lin = cfg->output_mode == VDN_OUTPUT_SPLIT ? take(vid) : h.out;
  h.total = off;
  return h;
}

// One non-blocking copy stream per device, created on first use.
cudaStream_t copy_stream() {
  static std::mutex mu;
  static cudaStream_t streams[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!streams[dev] && cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking) != cudaSuccess)
    streams[dev] = nullptr;
  return streams[dev];
}

}  // namespace
}  // namespace vdn

using namespace vdn;

extern "C" {

int32_t vdn_version(void) { return (1 << 16) | 0; }

const char* vdn_status_string(vdn_status s) {
  switch (s) {
    case VDN_OK: return "ok";
    case VDN_ERR_INVALID_ARG: return "invalid argument";
    case VDN_ERR_UNSUPPORTED: return "unsupported configuration";
    case VDN_ERR_ALIGNMENT: return "pointer not aligned";
    case VDN_ERR_WORKSPACE: return "workspace missing or too small";
    case VDN_ERR_CUDA: return "CUDA error";
    case VDN_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

vdn_status vdn_validate(const vdn_cfg* cfg) {
  Geom g;
  return make_geom(cfg, g);
}

size_t vdn_workspace_bytes(const vdn_cfg* cfg) {
  Geom g;
  return make_geom(cfg, g) == VDN_OK ? g.total : 0;
}

vdn_status vdn_plan_membership(const vdn_cfg* cfg, uint8_t* table) {
  Geom g;
  vdn_status s = make_geom(cfg, g);
  if (s != VDN_OK) return s;
  if (!table) return VDN_ERR_INVALID_ARG;
  for (int f = 0; f < g.F; ++f) {
    const int c = f / g.C;
    const int wlo = std::max(0, c - 1), whi = std::min(g.Nc - 1, c + 1);
    for (int x = 0; x < g.F; ++x) {
      const int cx = x / g.C;
      uint8_t code;
      if ((cx >= wlo && cx <= whi) || is_anchor(x, g.F) || no_linear_read(f, g)) code = 1;
      else if (cx <= fwd_last_chunk(c)) code = 2;
      else code = 3;
      table[f * g.F + x] = code;
    }
  }
  return VDN_OK;
}

vdn_status vdn_membership_device(const vdn_cfg* cfg, uint8_t* table_dev, void* stream) {
  Geom g;
  vdn_status s = make_geom(cfg, g);
  if (s != VDN_OK) return s;
  if (!table_dev) return VDN_ERR_INVALID_ARG;
  return cuda_status(launch_membership(g, table_dev, static_cast<cudaStream_t>(stream)));
}

vdn_status vdn_stage_inputs(const void* q, const void* k, const void* v, const void* text_k, const void* text_v,
                            const vdn_cfg* cfg, void* stream) {
  Geom g;
  vdn_status s = make_geom(cfg, g);
  if (s != VDN_OK) return s;
  s = check_inputs(cfg, g, {q, k, v}, {text_k, text_v});
  if (s != VDN_OK) return s;
  return step_stage(cfg, g, q, k, v, text_k, text_v, static_cast<cudaStream_t>(stream));
}

vdn_status vdn_state_build(const void* k, const void* v, const void* text_k, const void* text_v, const vdn_cfg* cfg,
                           void* stream) {
  Geom g;
  vdn_status s = make_geom(cfg, g);
  if (s != VDN_OK) return s;
  s = check_inputs(cfg, g, {k, v}, {text_k, text_v});
  if (s != VDN_OK) return s;
  return step_state_build(cfg, g, kernel_srcs(cfg, g, k, k, v, text_k, text_v), static_cast<cudaStream_t>(stream));
}

vdn_status vdn_state_scan(const vdn_cfg* cfg, void* stream) {
  Geom g;
  vdn_status s = make_geom(cfg, g);
  if (s != VDN_OK) return s;
  s = check_ws(cfg, g);
  if (s != VDN_OK) return s;
  if ((cfg->debug_flags & VDN_EXPORT_STATES) && (!cfg->export_fwd || !cfg->export_bwd)) return VDN_ERR_INVALID_ARG;
  return step_state_scan(cfg, g, static_cast<cudaStream_t>(stream));
}

vdn_status vdn_export_states(const vdn_cfg* cfg, float* fwd, float* bwd, void* stream) {
  if (!cfg || !fwd || !bwd) return VDN_ERR_INVALID_ARG;
  if (((reinterpret_cast<uintptr_t>(fwd) | reinterpret_cast<uintptr_t>(bwd)) & 15u) != 0) return VDN_ERR_ALIGNMENT;
  vdn_cfg c = *cfg;
  c.debug_flags |= VDN_EXPORT_STATES;
  c.export_fwd = fwd;
  c.export_bwd = bwd;
  return vdn_state_scan(&c, stream);
}

vdn_status vdn_sparse_softmax(const void* q, const void* k, const void* v, const void* text_k, const void* text_v,
                              const vdn_cfg* cfg, void* stream) {
  Geom g;
  vdn_status s = make_geom(cfg, g);
  if (s != VDN_OK) return s;
  s = check_inputs(cfg, g, {q, k, v}, {text_k, text_v});
  if (s != VDN_OK) return s;
  return step_sparse_softmax(cfg, g, kernel_srcs(cfg, g, q, k, v, text_k, text_v), static_cast<cudaStream_t>(stream),
                             false, nullptr);
}

vdn_status vdn_softmax_and_scan(const void* q, const void* k, const void* v, const void* text_k, const void* text_v,
                                const void* gate_s, const vdn_cfg* cfg, void* stream) {
  Geom g;
  vdn_status s = make_geom(cfg, g);
  if (s != VDN_OK) return s;
  s = check_inputs(cfg, g, {q, k, v}, {text_k, text_v});
  if (s != VDN_OK) return s;
  if ((cfg->debug_flags & VDN_EXPORT_STATES) && (!cfg->export_fwd || !cfg->export_bwd)) return VDN_ERR_INVALID_ARG;
  if (gate_s && (s = check_ptrs({gate_s})) != VDN_OK) return s;
  return step_sparse_softmax(cfg, g, kernel_srcs(cfg, g, q, k, v, text_k, text_v), static_cast<cudaStream_t>(stream),
                             true, gate_s);
}

vdn_status vdn_readout_merge(const void* q, const void* gate_s, const void* gate_l, void* out, const vdn_cfg* cfg,
                             void* stream) {
  Geom g;
  vdn_status s = make_geom(cfg, g);
  if (s != VDN_OK) return s;
  s = check_inputs(cfg, g, {q, gate_s, gate_l, out}, {});
  if (s != VDN_OK) return s;
  if (cfg->output_mode == VDN_OUTPUT_SPLIT && (s = check_ptrs({cfg->out_linear})) != VDN_OK) return s;
  return step_readout_merge(cfg, g, kernel_srcs(cfg, g, q, q, q, q, q), gate_s, gate_l, out,
                            static_cast<cudaStream_t>(stream));
}

vdn_status vdn_sparse_softmax_merge(const void* q, const void* k, const void* v, const void* text_k,
                                    const void* text_v, const void* gate_s, const void* gate_l, void* out,
                                    const vdn_cfg* cfg, void* stream) {
  Geom g;
  vdn_status s = make_geom(cfg, g);
  if (s != VDN_OK) return s;
  if (!fused_readout_supported(cfg)) return VDN_ERR_UNSUPPORTED;
  s = check_inputs(cfg, g, {q, k, v, gate_s, gate_l, out}, {text_k, text_v});
  if (s != VDN_OK) return s;
  if ((cfg->debug_flags & VDN_EXPORT_STATES) && (!cfg->export_fwd || !cfg->export_bwd)) return VDN_ERR_INVALID_ARG;
  return step_sparse_softmax(cfg, g, kernel_srcs(cfg, g, q, k, v, text_k, text_v), static_cast<cudaStream_t>(stream),
                             true, gate_s, gate_l, out);
}

vdn_status vdn_hybrid_attn_fwd(const void* q, const void* k, const void* v, const void* text_k, const void* text_v,
                               const void* gate_s, const void* gate_l, void* out, const vdn_cfg* cfg, void* stream) {
  Geom g;
  vdn_status s = make_geom(cfg, g);
  if (s != VDN_OK) return s;
  s = check_inputs(cfg, g, {q, k, v, gate_s, gate_l, out}, {text_k, text_v});
  if (s != VDN_OK) return s;
  if (cfg->output_mode == VDN_OUTPUT_SPLIT && (s = check_ptrs({cfg->out_linear})) != VDN_OK) return s;
  if ((cfg->debug_flags & VDN_EXPORT_STATES) && (!cfg->export_fwd || !cfg->export_bwd)) return VDN_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Srcs src = kernel_srcs(cfg, g, q, k, v, text_k, text_v);
  if (poison_ws(cfg, g, st) != cudaSuccess) return VDN_ERR_CUDA;
  if ((s = step_stage(cfg, g, q, k, v, text_k, text_v, st)) != VDN_OK) return s;
  if ((s = step_state_build(cfg, g, src, st)) != VDN_OK) return s;
  if (cfg->readout_mode == VDN_READOUT_FUSED)  // the scan runs inside as well
    return step_sparse_softmax(cfg, g, src, st, true, gate_s, gate_l, out);
  if ((s = step_sparse_softmax(cfg, g, src, st, true, gate_s)) != VDN_OK) return s;  // the scan runs inside
  return step_readout_merge(cfg, g, src, gate_s, gate_l, out, st);
}

size_t vdn_host_staging_bytes(const vdn_cfg* cfg) {
  Geom g;
  return make_geom(cfg, g) == VDN_OK ? host_staging(cfg, g).total : 0;
}

vdn_status vdn_hybrid_attn_fwd_host(const void* q, const void* k, const void* v, const void* text_k,
                                    const void* text_v, const void* gate_s, const void* gate_l, void* out,
                                    void* staging, size_t staging_bytes, const vdn_cfg* cfg, void* stream) {
  Geom g;
  vdn_status s = make_geom(cfg, g);
  if (s != VDN_OK) return s;
  for (const void* p : {q, k, v, gate_s, gate_l, static_cast<const void*>(out)})
    if (!p) return VDN_ERR_INVALID_ARG;
  if (g.T > 0 && (!text_k || !text_v)) return VDN_ERR_INVALID_ARG;
  if (cfg->output_mode == VDN_OUTPUT_SPLIT && !cfg->out_linear) return VDN_ERR_INVALID_ARG;
  if ((cfg->debug_flags & VDN_EXPORT_STATES) && (!cfg->export_fwd || !cfg->export_bwd)) return VDN_ERR_INVALID_ARG;
  if ((s = check_ws(cfg, g)) != VDN_OK) return s;
  const HostStaging h = host_staging(cfg, g);
  if (!staging || staging_bytes < h.total) return VDN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(staging) & 255u) != 0) return VDN_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaStream_t cs = copy_stream();
  if (!cs) return VDN_ERR_CUDA;
  uint8_t* dv = static_cast<uint8_t*>(staging);
  const size_t e = g.fp32_io ? 4 : 2;
  const size_t vid = (size_t)g.B * g.N * g.H * g.d * e, txt = (size_t)g.B * g.T * g.H * g.d * e;
  cudaEvent_t ev[4] = {};  // start, k/v/text landed, q landed, gates landed
  for (auto& x : ev)
    if (cudaEventCreateWithFlags(&x, cudaEventDisableTiming) != cudaSuccess) x = nullptr;
  auto finish = [&](vdn_status r) {
    for (auto& x : ev)
      if (x) cudaEventDestroy(x);  // released once the GPU has passed them
    return r;
  };
  if (!ev[0] || !ev[1] || !ev[2] || !ev[3]) return finish(VDN_ERR_CUDA);
  auto h2d = [&](size_t off, const void* src, size_t n) {
    return n == 0 ? cudaSuccess : cudaMemcpyAsync(dv + off, src, n, cudaMemcpyHostToDevice, cs);
  };
  // Copies on the copy stream, in the order the kernels need them, so the
  // state build runs while q lands and the softmax branch while the gates land.
  if (poison_ws(cfg, g, st) != cudaSuccess) return finish(VDN_ERR_CUDA);
  cudaError_t ce = cudaEventRecord(ev[0], st);  // earlier work on st may still read the staging
  if (ce == cudaSuccess) ce = cudaStreamWaitEvent(cs, ev[0], 0);
  if (ce == cudaSuccess && g.T > 0) ce = h2d(h.tk, text_k, txt);
  if (ce == cudaSuccess && g.T > 0) ce = h2d(h.tv, text_v, txt);
  if (ce == cudaSuccess) ce = h2d(h.k, k, vid);
  if (ce == cudaSuccess) ce = h2d(h.v, v, vid);
  if (ce == cudaSuccess) ce = cudaEventRecord(ev[1], cs);
  if (ce == cudaSuccess) ce = h2d(h.q, q, vid);
  if (ce == cudaSuccess) ce = cudaEventRecord(ev[2], cs);
  if (ce == cudaSuccess) ce = h2d(h.gs, gate_s, vid);
  if (ce == cudaSuccess) ce = h2d(h.gl, gate_l, vid);
  if (ce == cudaSuccess) ce = cudaEventRecord(ev[3], cs);
  if (ce != cudaSuccess) return finish(VDN_ERR_CUDA);

  vdn_cfg c = *cfg;
  if (c.output_mode == VDN_OUTPUT_SPLIT) c.out_linear = dv + h.out_lin;
  const void* dq = dv + h.q;
  const void* dk = dv + h.k;
  const void* dvv = dv + h.v;
  const void* dtk = g.T > 0 ? dv + h.tk : nullptr;
  const void* dtv = g.T > 0 ? dv + h.tv : nullptr;
  const Srcs src = kernel_srcs(&c, g, dq, dk, dvv, dtk, dtv);
  if (cudaStreamWaitEvent(st, ev[1], 0) != cudaSuccess) return finish(VDN_ERR_CUDA);
  if (g.staged) {  // staging converts q as well
    if (cudaStreamWaitEvent(st, ev[2], 0) != cudaSuccess) return finish(VDN_ERR_CUDA);
    if ((s = step_stage(&c, g, dq, dk, dvv, dtk, dtv, st)) != VDN_OK) return finish(s);
  }
  if ((s = step_state_build(&c, g, src, st)) != VDN_OK) return finish(s);
  if (c.readout_mode == VDN_READOUT_FUSED) {
    // the fused softmax kernel (which runs the scan as well) reads q and both gates
    if (cudaStreamWaitEvent(st, ev[3], 0) != cudaSuccess) return finish(VDN_ERR_CUDA);
    if ((s = step_sparse_softmax(&c, g, src, st, true, dv + h.gs, dv + h.gl, dv + h.out)) != VDN_OK)
      return finish(s);
  } else {
    // the softmax branch runs while the gates are still in flight, so here it
    // leaves o_s ungated and the readout applies both gates
    if (cudaStreamWaitEvent(st, ev[2], 0) != cudaSuccess) return finish(VDN_ERR_CUDA);
    if ((s = step_sparse_softmax(&c, g, src, st, true, nullptr)) != VDN_OK) return finish(s);  // the scan runs inside
    if (cudaStreamWaitEvent(st, ev[3], 0) != cudaSuccess) return finish(VDN_ERR_CUDA);
    if ((s = step_readout_merge(&c, g, src, dv + h.gs, dv + h.gl, dv + h.out, st)) != VDN_OK) return finish(s);
  }
  ce = cudaMemcpyAsync(out, dv + h.out, vid, cudaMemcpyDeviceToHost, st);
  if (ce == cudaSuccess && c.output_mode == VDN_OUTPUT_SPLIT)
    ce = cudaMemcpyAsync(cfg->out_linear, dv + h.out_lin, vid, cudaMemcpyDeviceToHost, st);
  return finish(ce == cudaSuccess ? VDN_OK : VDN_ERR_CUDA);
}

}  // extern "C"
