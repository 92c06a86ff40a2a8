/*
 * vdnattn.h - C ABI of libvdnattn, the sm_100a (B200) implementation of the
 * VDN-H3 dual-branch hybrid attention.
 *
 * Source of the operation: the VDN-H3 article (tahou.com, article
 * 216474224916730885), section "技术核心设计 / 双分支混合注意力机制" (the
 * softmax branch over a chunk window plus boundary anchors plus text; the
 * bidirectional frame-wise linear memory with half-weight text; the frame-7
 * example) and section "自适应门控融合双分支输出" (RMSNorm on the linear
 * branch, one sigmoid gate per branch, sum of the two).
 *
 * The call computes, for every video query token i (batch b, head h):
 *
 *   o_s[i] = softmax over keys J(i) of (scale * q_i . k_j), applied to v_j,
 *            J(i) = tokens of the frames in the window of i's chunk (the chunk
 *            and its two neighbours, clipped at the ends) and of the first and
 *            last frame, each frame once, plus all text tokens;
 *   o_l[i] = phi(q_i)^T (S_F + S_B) / (phi(q_i) . (z_F + z_B)), phi = elu + 1,
 *            S_F/z_F summing phi(k) v^T / phi(k) over the chunks before the
 *            window, S_B/z_B over the chunks after it, both without the two
 *            anchor frames, each holding half of the text state; o_l = 0 when
 *            the states hold no token;
 *   r[i]   = o_l[i] / sqrt(mean_d(o_l[i]^2) + eps) * gamma[h];
 *   out[i] = sigmoid(gate_s[i]) * o_s[i] + sigmoid(gate_l[i]) * r[i].
 *
 * Two readings the article leaves open are selectable (vdn_cfg):
 *   anchor_query_mode = VDN_ANCHOR_LOCAL (default): the rule above for every
 *     query frame, the anchors included (the frame-7 example's rule);
 *     VDN_ANCHOR_GLOBAL: a query in frame 0 or F-1 attends by softmax to
 *     every video frame (plus text) and reads nothing through the states
 *     (o_l = 0 there, so out = sigmoid(gate_s) * o_s); other rows unchanged.
 *   output_mode = VDN_OUTPUT_MERGED (default): out as above;
 *     VDN_OUTPUT_SPLIT: out = sigmoid(gate_s) * o_s and
 *     cfg->out_linear = sigmoid(gate_l) * r, the two gated branch terms
 *     (section 自适应门控融合双分支输出: one output per branch), for callers
 *     that project each branch before summing.
 *
 * Where the linear read and the merge run is selectable too (same result up
 * to rounding):
 *   readout_mode = VDN_READOUT_SEPARATE (default): the softmax kernel stores
 *     sigmoid(gate_s) * o_s (bf16) and a readout kernel of its own reads it
 *     back with q, M_c and gate_l and writes out;
 *     VDN_READOUT_FUSED: the readout, the RMSNorm and the merge run in the
 *     softmax kernel's epilogue (the frame-7 paragraph combines the linear read
 *     with the local branch at the query's position): o_s stays in TMEM in
 *     fp32 and q is read once.  Needs bf16 tensors, head_dim 128,
 *     the BF16 softmax precision and VDN_OUTPUT_MERGED without the VDN_OUT_*
 *     debug outputs (VDN_ERR_UNSUPPORTED otherwise).
 *
 * Layouts (row-major, no padding between rows):
 *   q, k, v, gate_s, gate_l, out : [batch, frames*tokens_per_frame, heads, head_dim]
 *   text_k, text_v               : [batch, text_tokens, heads, head_dim]
 *   token n of a video tensor lies in latent frame n / tokens_per_frame.
 * All of these are DEVICE pointers in the dtype given by vdn_cfg.dtype, each
 * 16-byte aligned; the caller owns them.  Accumulation is always fp32; tensor
 * core operands are bf16 (fp32 inputs are rounded to bf16 before the
 * contractions, and the intermediate softmax output o_s is kept in bf16).
 *
 * Ownership and threading: the library allocates no device memory.  Scratch
 * space is the caller-owned workspace (vdn_workspace_bytes).  Every device
 * function enqueues its work on the given stream and returns without host
 * synchronisation; the caller keeps inputs, outputs and the workspace alive
 * until that work completes.  Two calls that share a workspace must be
 * ordered on the GPU.  Functions are thread-safe.
 *
 * Errors: every argument check happens before anything is enqueued; on an
 * error return nothing was launched.  VDN_ERR_CUDA reports a launch error
 * (cudaGetLastError).  A kernel whose bounded wait runs out (1 s of global
 * time) writes VDN_ERR_TIMEOUT into *status_word (when given) and returns
 * early; that is read by the caller after synchronising.  The first such wait
 * also describes itself in a timeout record, 16 int32 words at byte 64 of the
 * workspace (count of waits that ran out, kernel id, block, warp, barrier as
 * its byte distance to the CTA's abort flag, phase parity, nanoseconds waited
 * as two words, SM); the library never clears it, the caller may.
 */
#ifndef VDNATTN_H
#define VDNATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define VDN_API __attribute__((visibility("default")))
#else
#define VDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VDN_OK = 0,
  VDN_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, frames % chunk != 0 */
  VDN_ERR_UNSUPPORTED = 2, /* head_dim not 32/64/128, unknown dtype, too many chunks */
  VDN_ERR_ALIGNMENT = 3,   /* a pointer is not 16-byte aligned */
  VDN_ERR_WORKSPACE = 4,   /* workspace NULL or smaller than vdn_workspace_bytes */
  VDN_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed */
  VDN_ERR_TIMEOUT = 6      /* written to status_word by a kernel whose wait ran out */
} vdn_status;

typedef enum { VDN_BF16 = 0, VDN_FP32 = 1 } vdn_dtype;

typedef enum { VDN_ANCHOR_LOCAL = 0, VDN_ANCHOR_GLOBAL = 1 } vdn_anchor_query_mode;
typedef enum { VDN_OUTPUT_MERGED = 0, VDN_OUTPUT_SPLIT = 1 } vdn_output_mode;
typedef enum { VDN_READOUT_SEPARATE = 0, VDN_READOUT_FUSED = 1 } vdn_readout_mode;

/* Operand precision of the softmax branch's two contractions.  BF16 (default):
 * bf16 operands, fp32 accumulation.  FP8: q, k, v, text_k, text_v quantised
 * to e4m3 with one scale per (batch, head) for q, one for k and text_k, one for
 * v and text_v (scale = max |x| / 448); P in e4m3; fp32 accumulation; o_s and
 * everything after it as in BF16.  FP8 needs head_dim 128, bf16 tensors and
 * tokens_per_frame % 16 == 0 (VDN_ERR_UNSUPPORTED otherwise), and a larger
 * workspace (vdn_workspace_bytes accounts for it). */
typedef enum { VDN_PREC_BF16 = 0, VDN_PREC_FP8 = 1 } vdn_softmax_precision;

/* debug_flags: what vdn_readout_merge writes into out instead of the merge. */
enum {
  VDN_OUT_SOFTMAX_ONLY = 1, /* out = o_s (no gate) */
  VDN_OUT_LINEAR_ONLY = 2,  /* out = r, the RMS-normalised linear read (no gate) */
  VDN_OUT_LINEAR_RAW = 4,   /* out = o_l, the linear read before RMSNorm */
  VDN_EXPORT_STATES = 8,    /* the scan (vdn_state_scan, or the one inside vdn_softmax_and_scan and
                               the whole calls) also writes S_F/z_F and S_B/z_B (fp32) */
  VDN_INJECT_TIMEOUT = 16,  /* test of the failure path only: in the state build, the MMA thread of
                               CTA 0 first waits, with a 10-ms limit, for a barrier phase
                               that nothing completes; it gives up, the CTA's other warps follow, the
                               kernel writes VDN_ERR_TIMEOUT to status_word and returns.  The call's
                               outputs are then undefined; the context stays usable. */
  VDN_STALL_READOUT_MMA = 32, /* test of the readout's barrier protocol only: the readout's MMA thread
                               sleeps 50 microseconds whenever it moves to another readout operand
                               (batch, chunk, head), letting the other warps run as far ahead as the
                               protocol allows.  Outputs are unchanged. */
  VDN_POISON_WS = 64,         /* vdn_hybrid_attn_fwd, _host and _static first fill the workspace past its
                               256-byte status slot with 0xFF bytes (NaN in bf16 and fp32), so that a
                               read of scratch the call has not written would show in the output.
                               Outputs are unchanged. */
  VDN_INJECT_TIMEOUT_SCAN = 128 /* test of the failure path only: under VDN_READOUT_FUSED, the producer of
                               CTA 0 of the softmax kernel waits, with a 10-ms limit, for one scan unit
                               more than its (batch, head) has; it gives up, the CTA's other warps
                               follow, the kernel writes VDN_ERR_TIMEOUT to status_word and returns.
                               The call's outputs are then undefined; the context stays usable. */
};

typedef struct {
  int32_t batch;            /* B  >= 1 */
  int32_t frames;           /* F  >= 1, latent frames; anchors are frames 0 and F-1 */
  int32_t tokens_per_frame; /* P  >= 1 */
  int32_t heads;            /* H  >= 1 */
  int32_t head_dim;         /* d in {32, 64, 128} */
  int32_t text_tokens;      /* T  >= 0 */
  int32_t chunk_frames;     /* C  >= 1, F % C == 0 (5 in the article's chunking, 1 in its frame-7 example) */
  int32_t dtype;            /* vdn_dtype of q, k, v, text, gates and out */
  float softmax_scale;      /* <= 0 selects 1/sqrt(head_dim) */
  float rms_eps;            /* < 0 selects 1e-6 */
  const float* rms_weight;  /* device [heads, head_dim] fp32 gamma (16-byte aligned), or NULL for ones */
  int32_t debug_flags;      /* VDN_OUT_* / VDN_EXPORT_STATES, 0 in production */
  int32_t anchor_query_mode; /* vdn_anchor_query_mode; 0 = LOCAL */
  void* workspace;          /* device, 256-byte aligned, >= vdn_workspace_bytes(cfg) bytes */
  size_t workspace_bytes;
  int32_t* status_word;     /* optional device int32; set to VDN_ERR_TIMEOUT by a kernel that gave up */
  float* export_fwd;        /* VDN_EXPORT_STATES: device [B, F/C, H, d+1, d] fp32; row d holds z */
  float* export_bwd;        /* same layout, backward states */
  int32_t output_mode;      /* vdn_output_mode; 0 = MERGED.  SPLIT excludes the VDN_OUT_* debug flags */
  int32_t softmax_precision; /* vdn_softmax_precision; 0 = BF16 */
  void* out_linear;         /* SPLIT only: device [B, N, H, d] in dtype, 16-byte aligned; else ignored */
  int32_t readout_mode;     /* vdn_readout_mode; 0 = SEPARATE */
} vdn_cfg;

/* Library version, (major << 16) | minor. */
VDN_API int32_t vdn_version(void);

/* Human-readable name of a status code (static string). */
VDN_API const char* vdn_status_string(vdn_status s);

/* Host-only argument check of cfg (sizes, dtype, head_dim, chunking).  No CUDA call. */
VDN_API vdn_status vdn_validate(const vdn_cfg* cfg);

/* Bytes of workspace a call with this cfg needs; 0 if cfg is invalid.  No CUDA call. */
VDN_API size_t vdn_workspace_bytes(const vdn_cfg* cfg);

/* Host-only membership table of the frame-7 rule: table[f*F + g] = 1 when query
 * frame f reads key frame g through the softmax branch, 2 through the forward
 * state, 3 through the backward state (under VDN_ANCHOR_GLOBAL the rows of
 * frames 0 and F-1 are all 1).  table is HOST memory of F*F bytes. */
VDN_API vdn_status vdn_plan_membership(const vdn_cfg* cfg, uint8_t* table);

/* The same table produced on the GPU by the index logic the kernels use
 * (KV ranges of the softmax kernel, chunk membership of the scan).
 * table_dev is DEVICE memory of F*F bytes.  stream is a cudaStream_t. */
VDN_API vdn_status vdn_membership_device(const vdn_cfg* cfg, uint8_t* table_dev, void* stream);

/* Whole call: staging (fp32 or head_dim 32 only), state build, sparse
 * softmax with the forward/backward scan (and, for bf16 with head_dim 64 or
 * 128, the softmax branch's gate) in the same kernel, readout + merge, all on
 * stream; under VDN_READOUT_FUSED: state build, then the softmax kernel with
 * the scan inside and the readout and merge in its epilogue.  out: [B, N, H, d] in dtype (and cfg->out_linear under
 * VDN_OUTPUT_SPLIT). */
VDN_API vdn_status vdn_hybrid_attn_fwd(const void* q, const void* k, const void* v,
                               const void* text_k, const void* text_v,
                               const void* gate_s, const void* gate_l, void* out,
                               const vdn_cfg* cfg, void* stream);

/* The steps of vdn_hybrid_attn_fwd, for callers that schedule them
 * separately.  vdn_stage_inputs (required first when dtype is fp32 or
 * head_dim is 32; otherwise a no-op), then either
 *   vdn_state_build -> vdn_softmax_and_scan -> vdn_readout_merge
 * (the sequence of the whole call: the scan runs in otherwise idle warps of
 * the softmax kernel), or, with the linear steps independent of the softmax
 * branch (e.g. on a second stream),
 *   vdn_state_build -> vdn_state_scan, and vdn_sparse_softmax, in either
 *   order, then vdn_readout_merge.
 * Each reads what the earlier steps left in the workspace. */
VDN_API vdn_status vdn_stage_inputs(const void* q, const void* k, const void* v,
                            const void* text_k, const void* text_v,
                            const vdn_cfg* cfg, void* stream);
/* Partial states [S | z] = phi(K)^T [V | 1] (tensor cores): for every state
 * segment (the non-anchor frames of one chunk, or the text) of every (batch,
 * head), one partial per state-build CTA whose equal share of the tiles meets
 * the segment. */
VDN_API vdn_status vdn_state_build(const void* k, const void* v, const void* text_k,
                           const void* text_v, const vdn_cfg* cfg, void* stream);
/* Forward/backward chunk states and their sum M_c, fp32 scan. */
VDN_API vdn_status vdn_state_scan(const vdn_cfg* cfg, void* stream);
/* The forward and backward states S_F / z_F and S_B / z_B of every (batch,
 * chunk, head), as fp32 [B, F/C, H, d+1, d] (row n < d: value column n of S;
 * row d: z; column a: key feature a), recomputed by the scan on `stream`
 * from the state partials that the last vdn_hybrid_attn_fwd or
 * vdn_state_build on cfg->workspace left there; the readout operands are
 * rewritten with the values they had.  fwd, bwd: device, 16-byte aligned,
 * B*(F/C)*H*(d+1)*d floats each, caller-owned.  Same as calling
 * vdn_state_scan with VDN_EXPORT_STATES and cfg->export_fwd/export_bwd set. */
VDN_API vdn_status vdn_export_states(const vdn_cfg* cfg, float* fwd, float* bwd, void* stream);
/* Block-sparse softmax branch o_s (window + anchors + text) into the workspace. */
VDN_API vdn_status vdn_sparse_softmax(const void* q, const void* k, const void* v,
                              const void* text_k, const void* text_v,
                              const vdn_cfg* cfg, void* stream);
/* vdn_sparse_softmax and, in the same kernel, vdn_state_scan: must follow
 * vdn_state_build on the same workspace (stream order).  gate_s (the
 * softmax branch's gate logits, [B, N, H, d], or NULL): for bf16 tensors whose
 * head_dim is 64 or 128, and without VDN_OUT_SOFTMAX_ONLY, the kernel stores
 * sigmoid(gate_s) * o_s in place of o_s (the softmax branch's term of the
 * gated merge; one rounding to bf16 either way) and notes so in the
 * workspace, and vdn_readout_merge then takes that term as it is; otherwise
 * o_s is stored and the readout applies the gate.  Errors as
 * vdn_sparse_softmax, plus VDN_ERR_INVALID_ARG for VDN_EXPORT_STATES without
 * export buffers and VDN_ERR_ALIGNMENT for a misaligned gate_s. */
VDN_API vdn_status vdn_softmax_and_scan(const void* q, const void* k, const void* v,
                                        const void* text_k, const void* text_v, const void* gate_s,
                                        const vdn_cfg* cfg, void* stream);
/* phi(Q) M_c readout, RMSNorm, gates and merge into out. */
VDN_API vdn_status vdn_readout_merge(const void* q, const void* gate_s, const void* gate_l,
                             void* out, const vdn_cfg* cfg, void* stream);
/* The steps of a VDN_READOUT_FUSED call: vdn_state_build ->
 * vdn_sparse_softmax_merge, which runs the softmax branch, the
 * forward/backward scan (in otherwise idle warps, as vdn_softmax_and_scan) and,
 * in the kernel's item epilogue, the readout, RMSNorm, gates and merge into
 * out; it must follow vdn_state_build on the same workspace (stream order).
 * Requirements of VDN_READOUT_FUSED apply whatever cfg->readout_mode says
 * (VDN_ERR_UNSUPPORTED otherwise); VDN_ERR_ALIGNMENT for a misaligned
 * pointer; VDN_ERR_INVALID_ARG for VDN_EXPORT_STATES without export buffers. */
VDN_API vdn_status vdn_sparse_softmax_merge(const void* q, const void* k, const void* v,
                                            const void* text_k, const void* text_v,
                                            const void* gate_s, const void* gate_l, void* out,
                                            const vdn_cfg* cfg, void* stream);

/* For callers that cannot allocate device memory (code running inside another
 * runtime's plugin/operator interface that hands over tensors but no
 * allocator, or latency-critical loops where cudaMalloc is not acceptable).
 * There is no counterpart on the article's pages: this is an interface
 * addition, not part of the method.
 *
 * Same operation, arguments and layouts as vdn_hybrid_attn_fwd, but
 * cfg->workspace / workspace_bytes are ignored: the scratch is a static device
 * array of vdn_static_scratch_bytes() (32 MiB) inside the library, which every
 * GPU that loads the library holds until the process exits.  The first call on
 * a device (with that device current) looks up the array's device address
 * with cudaGetSymbolAddress; make that first call before any stream capture.
 * The address is cached with the id of the CUDA context it was looked up in
 * and is valid only there: after cudaDeviceReset (or any replacement of the
 * context) the next call looks it up again, and that call too should precede
 * any capture.  Nothing is allocated.  Returns VDN_ERR_WORKSPACE when
 * vdn_workspace_bytes(cfg) exceeds the static size (it fits, e.g., 15 frames
 * x 256 tokens x 8 heads x head_dim 64); every argument error (sizes,
 * missing or misaligned pointers, including cfg->status_word and
 * cfg->rms_weight) is returned before any CUDA call, with nothing queued.
 * All calls on a device share the one array: calls whose GPU work overlaps
 * race and must be ordered by the caller.  The status slot of the array is
 * cleared on every call. */
VDN_API vdn_status vdn_hybrid_attn_fwd_static(const void* q, const void* k, const void* v,
                                              const void* text_k, const void* text_v,
                                              const void* gate_s, const void* gate_l, void* out,
                                              const vdn_cfg* cfg, void* stream);
/* Size in bytes of the static scratch used by vdn_hybrid_attn_fwd_static. */
VDN_API size_t vdn_static_scratch_bytes(void);

/* The whole call on HOST tensors (same layouts and dtype as vdn_hybrid_attn_fwd;
 * out, and cfg->out_linear under VDN_OUTPUT_SPLIT, are HOST pointers too).
 * Not part of the method: an interface for callers whose tensors live in host
 * memory.  The inputs are copied into `staging`, a caller-owned DEVICE buffer
 * of at least vdn_host_staging_bytes(cfg) bytes (256-byte aligned), on a
 * library-owned copy stream in the order the kernels need them (text, k, v,
 * then q, then the gates), so the state build runs while q is in flight and
 * the softmax branch while the gates are; the output is copied back on
 * `stream`.  cfg->workspace is used as in vdn_hybrid_attn_fwd; the export
 * buffers, if any, are device memory.  Host buffers should be page-locked
 * (cudaHostAlloc / cudaHostRegister): from pageable memory the copies do
 * not overlap.  The call returns once everything is enqueued; the caller
 * synchronises `stream` before reading out and must keep the host and device
 * buffers alive until then.  Errors: as vdn_hybrid_attn_fwd, plus
 * VDN_ERR_WORKSPACE for a missing or small staging buffer and
 * VDN_ERR_ALIGNMENT for a misaligned one. */
VDN_API size_t vdn_host_staging_bytes(const vdn_cfg* cfg);
VDN_API vdn_status vdn_hybrid_attn_fwd_host(const void* q, const void* k, const void* v,
                                            const void* text_k, const void* text_v,
                                            const void* gate_s, const void* gate_l, void* out,
                                            void* staging, size_t staging_bytes,
                                            const vdn_cfg* cfg, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* VDNATTN_H */
