// The LinearAttentionGate op on its own ("com.microsoft.LinearAttentionGate",
// sections Description, Inputs, Outputs and Type constraints): per element,
// in float32,
//   decay = decay_scale[h] * softplus(a + dt_bias[h]),  beta = sigmoid(b),
// narrowed to the tensor type on store. h is the index on the last axis.
//
// Elementwise: each thread moves 16-byte vectors of a (and b)
// in and of decay (and beta) out, over a grid-stride loop; tensors that are
// not 16-byte aligned, and the last partial vector, take the scalar path.
// The per-head vectors are read through the read-only cache.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr_decode.cuh"

namespace gdr {

enum GateType { kGateF32 = 0, kGateF16 = 1, kGateBF16 = 2 };

// The gate's two functions. For a float32 output they are the accurate
// library forms of gdr_decode.cuh. For a 16-bit output (one unit in the last
// place is 2^-8 of the value for bf16, 2^-11 for fp16) cheaper forms suffice:
//   exp and the division: the fast hardware forms (a few fp32 ulps);
//   log1p(z), 0 <= z <= 1: z q(z), with q a degree-5 polynomial fitted to
//     log1p(z) / z on [0, 1] by least squares at 4000 Chebyshev nodes,
//     weighted for relative error. Evaluated by Horner's rule in fp32 its
//     relative error is below 1e-5 (about 2^-16.6) over the whole interval,
//     small z included, and it takes no special-function instruction.
__device__ __forceinline__ float log1p_narrow(float z) {
  float q = -0.02333560399711132f;
  q = fmaf(q, z, 0.09986384958028793f);
  q = fmaf(q, z, -0.20883141458034515f);
  q = fmaf(q, z, 0.32475757598876953f);
  q = fmaf(q, z, -0.4993025064468384f);
  q = fmaf(q, z, 0.9999903440475464f);
  return z * q;
}
template <bool FAST>
__device__ __forceinline__ float gate_softplus(float x) {
  if constexpr (FAST) return fmaxf(x, 0.0f) + log1p_narrow(__expf(-fabsf(x)));
  else return softplus_f32(x);
}
template <bool FAST>
__device__ __forceinline__ float gate_sigmoid(float x) {
  if constexpr (FAST) {
    const float z = __expf(-fabsf(x));
    return __fdividef(x >= 0.0f ? 1.0f : z, 1.0f + z);
  } else {
    return sigmoid_f32(x);
  }
}

template <int TYPE>
struct GateElem;
template <>
struct GateElem<kGateF32> {
  using bits = uint32_t;
  static constexpr bool kFast = false;
  static constexpr int kPerVec = 4;
  __device__ static float load(bits x) { return __uint_as_float(x); }
  __device__ static bits store(float x) { return __float_as_uint(x); }
};
template <>
struct GateElem<kGateF16> {
  using bits = uint16_t;
  static constexpr bool kFast = true;
  static constexpr int kPerVec = 8;
  __device__ static float load(bits x) { return __half2float(__ushort_as_half(x)); }
  __device__ static bits store(float x) { return __half_as_ushort(__float2half_rn(x)); }
};
template <>
struct GateElem<kGateBF16> {
  using bits = uint16_t;
  static constexpr bool kFast = true;
  static constexpr int kPerVec = 8;
  __device__ static float load(bits x) { return bf16_bits_to_f32(x); }
  __device__ static bits store(float x) { return f32_to_bf16_bits(x); }
};

// decay (and beta) for elements [i0, i0 + count) of the flattened tensors.
template <int TYPE, bool BETA>
__device__ __forceinline__ void gate_elements(const typename GateElem<TYPE>::bits* a,
                                              const typename GateElem<TYPE>::bits* b,
                                              const float* dt_bias, const float* decay_scale,
                                              typename GateElem<TYPE>::bits* decay,
                                              typename GateElem<TYPE>::bits* beta, int64_t i0,
                                              int count, int H) {
  using E = GateElem<TYPE>;
  int h = static_cast<int>(i0 % H);
  for (int e = 0; e < count; ++e) {
    const int64_t i = i0 + e;
    const float x = E::load(a[i]) + __ldg(dt_bias + h);
    decay[i] = E::store(__ldg(decay_scale + h) * gate_softplus<E::kFast>(x));
    if constexpr (BETA) beta[i] = E::store(gate_sigmoid<E::kFast>(E::load(b[i])));
    h = h + 1 == H ? 0 : h + 1;
  }
}

// Vector path: n / kPerVec whole 16-byte vectors, all four tensors 16-byte
// aligned; the scalar remainder is done by the caller's tail launch. When
// HEADVEC (H a multiple of kPerVec and both per-head vectors 16-byte aligned),
// a vector's kPerVec elements are heads h0 .. h0 + kPerVec - 1 and their
// dt_bias and decay_scale come in as 16-byte loads. Each thread loads its next
// vector's a (and b) before it works on the current one.
template <int TYPE, bool BETA, bool HEADVEC>
__global__ void __launch_bounds__(256) gate_vec_kernel(const uint4* __restrict__ a,
                                                       const uint4* __restrict__ b,
                                                       const float* __restrict__ dt_bias,
                                                       const float* __restrict__ decay_scale,
                                                       uint4* __restrict__ decay,
                                                       uint4* __restrict__ beta, int64_t n_vec,
                                                       int H) {
  using E = GateElem<TYPE>;
  using bits = typename E::bits;
  constexpr int V = E::kPerVec;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  // head of this thread's first element, and how far it moves per stride
  int h0 = static_cast<int>((v * V) % H);
  const int h_step = static_cast<int>((stride * V) % H);
  uint4 av_next = make_uint4(0u, 0u, 0u, 0u), bv_next = av_next;
  if (v < n_vec) {
    av_next = __ldcs(a + v);
    if constexpr (BETA) bv_next = __ldcs(b + v);
  }
  for (; v < n_vec; v += stride, h0 = h0 + h_step >= H ? h0 + h_step - H : h0 + h_step) {
    const uint4 av = av_next;
    const uint4 bv = bv_next;
    if (v + stride < n_vec) {
      av_next = __ldcs(a + v + stride);
      if constexpr (BETA) bv_next = __ldcs(b + v + stride);
    }
    float dtb[V], dsc[V];
    if constexpr (HEADVEC) {
#pragma unroll
      for (int q = 0; q < V / 4; ++q) {
        const float4 t = __ldg(reinterpret_cast<const float4*>(dt_bias + h0) + q);
        const float4 u = __ldg(reinterpret_cast<const float4*>(decay_scale + h0) + q);
        dtb[4 * q] = t.x; dtb[4 * q + 1] = t.y; dtb[4 * q + 2] = t.z; dtb[4 * q + 3] = t.w;
        dsc[4 * q] = u.x; dsc[4 * q + 1] = u.y; dsc[4 * q + 2] = u.z; dsc[4 * q + 3] = u.w;
      }
    } else {
      int h = h0;
#pragma unroll
      for (int e = 0; e < V; ++e) {
        dtb[e] = __ldg(dt_bias + h);
        dsc[e] = __ldg(decay_scale + h);
        h = h + 1 == H ? 0 : h + 1;
      }
    }
    const bits* ae = reinterpret_cast<const bits*>(&av);
    const bits* be = reinterpret_cast<const bits*>(&bv);
    uint4 dv, btv;
    bits* de = reinterpret_cast<bits*>(&dv);
    bits* bte = reinterpret_cast<bits*>(&btv);
#pragma unroll
    for (int e = 0; e < V; ++e) {
      de[e] = E::store(dsc[e] * gate_softplus<E::kFast>(E::load(ae[e]) + dtb[e]));
      if constexpr (BETA) bte[e] = E::store(gate_sigmoid<E::kFast>(E::load(be[e])));
    }
    __stcs(decay + v, dv);
    if constexpr (BETA) __stcs(beta + v, btv);
  }
}

// Scalar path: elements [i_begin, n), one per thread over a grid-stride loop.
template <int TYPE, bool BETA>
__global__ void __launch_bounds__(256) gate_scalar_kernel(
    const typename GateElem<TYPE>::bits* __restrict__ a,
    const typename GateElem<TYPE>::bits* __restrict__ b, const float* __restrict__ dt_bias,
    const float* __restrict__ decay_scale, typename GateElem<TYPE>::bits* __restrict__ decay,
    typename GateElem<TYPE>::bits* __restrict__ beta, int64_t i_begin, int64_t n, int H) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = i_begin + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += stride)
    gate_elements<TYPE, BETA>(a, b, dt_bias, decay_scale, decay, beta, i, 1, H);
}

}  // namespace gdr
