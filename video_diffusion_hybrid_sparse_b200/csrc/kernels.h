// kernels.h - parameter blocks and host launchers of the CUDA kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "plan.h"

namespace vdn {

// The forward/backward scan (scan.cuh): partials in, segment states, the
// readout operands M_c and (optionally) the exported F_c / B_c out.
struct ScanArgs {
  Geom g;
  StatePlan sp;
  const float* parts;      // state-build partial slots [n_part_slots, Dp+1, Dp] fp32 (row Dp holds z)
  float* segst;            // segment states [B * H * n_segs, Dp+1, Dp] fp32
  uint8_t* mt;             // readout B-tiles (hi, lo) per (b, chunk, head)
  float* export_fwd;       // optional [B, Nc, H, d+1, d]
  float* export_bwd;
};

struct K3Params {
  Geom g;
  float scale_log2;        // softmax scale * log2(e)
  __nv_bfloat16* o_s;      // [B, N, H, Dp] bf16
  const float* fp8_amax;   // fp8 branch: [5][B][H] maxima of q, k, v, text_k, text_v
  int* status;
  int* record;             // timeout record (workspace), may be null
  int n_items;             // all work items
  // Work items come in blocks of query segments; block k holds segments
  // [blk_seg0[k], blk_seg0[k + 1]) and items [blk_item0[k], blk_item0[k + 1]),
  // ordered (batch, head, segment, pair of 128-row query tiles).  seg_pair0
  // is the running count of pairs over all segments (pairs of segment i are
  // seg_pair0[i] .. seg_pair0[i + 1]).
  int n_blocks;
  int blk_seg0[kMaxSegs + 1];
  int blk_item0[kMaxSegs + 1];
  QSeg segs[kMaxSegs];
  int seg_pair0[kMaxSegs + 1];
  const __nv_bfloat16* gate_s;  // [B, N, H, Dp] or null: o_s is written as sigmoid(gate_s) * o_s
  int* os_gated;           // workspace flag: 1 when o_s holds the gated term (read by the readout)
  int do_scan;             // the kernel also runs the forward/backward scan (scan below)
  unsigned long long* scan_counter;  // next scan unit to take (workspace; zeroed by the state build)
  ScanArgs scan;
  // Fused readout (out != null; bf16, head_dim 128): the kernel writes the
  // merged output itself from M_c.  With do_scan, M_c comes from this
  // kernel's own scan: the scan counts the units it completed per (batch,
  // head) in scan_done, and an item reads M_c of its (batch, head) once all
  // of them are in; without, the scan ran before the kernel.
  __nv_bfloat16* out;      // [B, N, H, 128] bf16
  const __nv_bfloat16* gate_l;  // [B, N, H, 128]
  const uint8_t* mt;       // readout operand images per (b, chunk, head) (scan.cuh)
  const float* gamma;      // [H, 128] fp32 or null (ones)
  unsigned* scan_done;     // [B * H] (workspace; zeroed by the state build)
  int inject_scan_wait;    // test only: CTA 0's producer waits for one unit more (short limit)
};

struct K1Params {
  Geom g;
  StatePlan sp;
  float* parts;            // partial slots [n_part_slots, Dp+1, Dp] fp32; row Dp holds z
  int* status;
  int* record;             // timeout record (workspace), may be null
  int inject_timeout;      // test only: CTA 0 waits for a phase nothing completes (short limit)
  unsigned long long* scan_counter;  // zeroed by CTA 0 for the scan of the softmax kernel that follows
  unsigned* scan_done;     // [B * H] zeroed by CTA 0 likewise
};

struct K4Params {
  Geom g;
  const __nv_bfloat16* o_s;
  const uint8_t* mt;
  const float* gamma;      // [H, d] or null
  const void* gate_s;
  const void* gate_l;
  void* out;
  void* out_linear;        // SPLIT output: sigmoid(g_l) * r goes here, out gets sigmoid(g_s) * o_s
  int flags;
  int stall_ns;            // > 0: the MMA thread sleeps this long at each readout-operand change
  const int* os_gated;     // workspace flag written by the softmax kernel: o_s already holds sigmoid(g_s) * o_s
  int* status;
  int* record;             // timeout record (workspace), may be null
};

// Tensor maps: 2-D bf16 views [rows, H*Dp] with a 128-row x 64-column box and
// 128-byte swizzle.
struct Maps {
  CUtensorMap q, k, v, tk, tv;
};

cudaError_t launch_stage(const void* src, int fp32_in, __nv_bfloat16* dst, long long rows, int H, int d, int Dp,
                         cudaStream_t st);
cudaError_t launch_state_build(const Maps& m, const K1Params& p, cudaStream_t st);
cudaError_t launch_state_scan(const ScanArgs& sa, cudaStream_t st);
cudaError_t launch_sparse_softmax(const Maps& m, const K3Params& p, int grid, cudaStream_t st);
// fp8 branch (head_dim 128): Maps of the e4m3 q, k, text_k ([rows, H * 128]
// bytes) and of v, text_v transposed ([B * H * 128, tokens] bytes).
cudaError_t launch_sparse_softmax_fp8(const Maps& m, const K3Params& p, int grid, cudaStream_t st);
cudaError_t launch_readout_merge(const Maps& m, const K4Params& p, cudaStream_t st);

// Maps of the TMA-fed readout/merge (bf16, head_dim == Dp): q, o_s and the
// two gates as 2-D [rows, H*Dp] views like Maps.
struct MergeMaps {
  CUtensorMap q, os, gs, gl, out;  // out: the output tensor, same geometry (TMA stores of full tiles)
};
cudaError_t launch_readout_merge_tma(const MergeMaps& m, const K4Params& p, cudaStream_t st);
cudaError_t launch_membership(const Geom& g, uint8_t* table, cudaStream_t st);

// e4m3 operands of the fp8 softmax branch (head_dim 128): q, k, text_k in their
// [rows, H * 128] layout, v and text_v transposed to [(b * H + h) * 128 + dd,
// token] with row pitches pitch_v / pitch_t (multiples of 16 bytes); amax is
// [5][B][H] (q, k, v, text_k, text_v), the scale of a tensor is amax / 448.
struct Fp8Src {
  const __nv_bfloat16* p[5];
};
struct Fp8Dst {
  uint8_t *q, *k, *vt, *tk, *tvt;
  long long pitch_v, pitch_t;
};
cudaError_t launch_fp8_quant(const Fp8Src& src, const Fp8Dst& dst, int B, long long N, int T, int H, float* amax,
                             cudaStream_t st);

size_t k3_smem_bytes(int Dp);

}  // namespace vdn
