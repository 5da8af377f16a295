// Shared definitions of the decode kernels: launch parameters and small
// device helpers (bf16 bit conversions, the gate's softplus and sigmoid, a
// warp sum). The arithmetic they serve is the op of
// "lite_boost.ops.recurrent_gated_delta_rule" (MindSpore Lite API page,
// section 算法流程) and the gate of "com.microsoft.LinearAttentionGate"
// (README, section Description).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdr {

constexpr int kSliceCols = 64;  // D_v must be a multiple of this
constexpr int kMaxT = 8;        // decode only: at most 8 tokens per call

struct DecodeParams {
  const uint16_t* query;        // [B, H_qk, T, D_k] bf16
  const uint16_t* key;          // [B, H_qk, T, D_k] bf16
  const uint16_t* value;        // [B, H_v, T, D_v] bf16
  const uint16_t* beta;         // [B, H_v, T] bf16        (plain path)
  const float* g;               // [B, H_v, T] fp32        (plain path)
  const uint16_t* gate_a;       // [B, T, H_v] bf16        (gated path)
  const uint16_t* gate_b;       // [B, T, H_v] bf16        (gated path)
  const float* dt_bias;         // [H_v] fp32              (gated path)
  const float* decay_scale;     // [H_v] fp32              (gated path)
  const float* gk;              // [B, H_v, T, D_k] fp32
  uint16_t* state_pool;         // [pool, H_v, D_k, D_v] bf16, in place
  uint16_t* out;                // [B, H_v, T, D_v] bf16
  const int32_t* seq_lengths;   // [B]
  const int32_t* state_indices; // [B]
  const int32_t* num_accepted;  // [B] or NULL: tokens whose state update is committed
  float scale;
  int B, T, H_qk, H_v, D_v, pool_size;
  int group;  // H_v / H_qk
};

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t x) {
  return __uint_as_float(static_cast<uint32_t>(x) << 16);
}

// Two bf16 values packed in a 32-bit word: element 0 in the low half.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Round two fp32 values to bf16 (round-to-nearest-even) and pack them, lo first.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float x) {
  __nv_bfloat16 v = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&v);
}

// softplus(x) = ln(1 + e^x) = max(x, 0) + ln(1 + e^-|x|), without overflow.
__device__ __forceinline__ float softplus_f32(float x) {
  return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}

// sigmoid(x) = 1 / (1 + e^-x), without overflow for either sign.
__device__ __forceinline__ float sigmoid_f32(float x) {
  const float z = expf(-fabsf(x));
  return x >= 0.0f ? 1.0f / (1.0f + z) : z / (1.0f + z);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace gdr
