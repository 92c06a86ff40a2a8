// k4_common.cuh - pieces shared by the two readout/merge kernels (the
// general one and the TMA-fed one for bf16 tensors whose head_dim needs no
// padding): work-item decoding of the persistent grid, the worker barriers,
// the sigmoid and the 8-value stores.
#pragma once

#include "kernels.h"
#include "sm100.cuh"

namespace vdn {
namespace k4 {

__device__ __forceinline__ float sigmoid_f(float x) { return sigmoid_tanh(x); }

template <bool FP32>
__device__ __forceinline__ void store8(void* base, size_t idx, const float (&x)[8]) {
  if constexpr (FP32) {
    float4* p = reinterpret_cast<float4*>(static_cast<float*>(base) + idx);
    p[0] = make_float4(x[0], x[1], x[2], x[3]);
    p[1] = make_float4(x[4], x[5], x[6], x[7]);
  } else {
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + idx) =
        make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
  }
}

// Barrier among the 256 worker threads (id 1) that also ORs a predicate:
// every worker leaves with the same answer.
__device__ __forceinline__ bool workers_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}

// Barrier of the two worker warps that hold the halves of the same TMEM rows
// (warps w and w + 4, named barrier 2 + w % 4), also ORing a predicate.
__device__ __forceinline__ bool pair_any(uint32_t quarter, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 64, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(2 + quarter)
      : "memory");
  return r != 0;
}

struct Item4 {
  int b, h, c, tile, key;
};

// The i-th item of the CTA (head h, stream s of n_streams): with S streams,
// CTA k keeps head k % H and walks the (batch, chunk, tile) positions
// s, s + S, s + 2S, ... of stream s = k / H.
__device__ __forceinline__ Item4 decode4(int i, int h, int s, int n_streams, const Geom& g, int tiles) {
  Item4 it;
  const int pos = s + i * n_streams;
  it.tile = pos % tiles;
  const int rem = pos / tiles;
  it.c = rem % g.Nc;
  it.b = rem / g.Nc;
  it.h = h;
  it.key = rem;  // (batch, chunk) of this head identifies the readout operand
  return it;
}

}  // namespace k4
}  // namespace vdn
