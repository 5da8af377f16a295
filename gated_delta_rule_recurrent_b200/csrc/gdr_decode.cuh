// Decode kernel of the recurrent gated-delta-rule step for sm_100a.
//
// The arithmetic is the four steps of "lite_boost.ops.recurrent_gated_delta_rule"
// (MindSpore Lite API page, section 算法流程) and, when GATED, the gate of
// "com.microsoft.LinearAttentionGate" (README, section Description).
//
// Work decomposition. One CTA owns one (batch item b, value head h, 64-column
// slice of D_v) tile of the state: D_k rows x 64 columns. The tile lives in
// fp32 registers for all of the item's tokens and touches HBM twice: one
// coalesced bf16 load before the first token and one bf16 store after the
// last. A warp covers 32 rows of the tile: lane = (row group rl: 0..3) x
// (column group cg: 0..7); each thread holds rows [rl*8, rl*8+8) of its warp's
// 32 and columns [cg*8, cg*8+8) as 8x8 fp32 registers, so one warp-wide
// 16-byte load reads four full 128-byte row segments.
//
// Per token (after the decay, applied in place) the two column sums
// kv_mem = S^T k and p = S^T (q*scale) are formed together from the decayed
// state. The output then follows from
//   o = (S + k delta^T)^T q_s = p + delta * (k . q_s),
// the same quantity as step 4 with the sums reordered, so each token needs a
// single reduction: a reduce-scatter over the four row lanes of a warp (two
// xor-shuffle rounds), then one shared-memory combine across the warps.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdr {

constexpr int kSliceCols = 64;  // D_v columns per CTA
constexpr int kRowsPerThread = 8;
constexpr int kColsPerThread = 8;  // one 16-byte bf16x8 vector
constexpr int kMaxT = 8;           // decode only: at most 8 tokens per call

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
  float scale;
  int B, T, H_qk, H_v, D_v, pool_size;
  int group;     // H_v / H_qk
  int n_slices;  // D_v / kSliceCols
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

// Dynamic shared memory of one CTA, in floats.
template <int DK>
__host__ __device__ constexpr int decode_smem_floats(int T) {
  return 3 * T * DK              // k, q*scale, exp(g + gk) per token and row
         + (DK / 32) * 32 * 4    // per-warp partial sums
         + kSliceCols            // delta of the current token
         + 3 * kMaxT;            // beta, k.q_s and g per token
}

template <int DK, bool GATED>
__global__ void __launch_bounds__(DK) decode_kernel(const DecodeParams p) {
  constexpr int WARPS = DK / 32;
  constexpr int NT = DK;  // threads per CTA
  extern __shared__ float4 smem_f4[];
  float* smem = reinterpret_cast<float*>(smem_f4);

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int T = p.T;

  int blk = blockIdx.x;
  const int slice = blk % p.n_slices;
  blk /= p.n_slices;
  const int h = blk % p.H_v;
  const int b = blk / p.H_v;
  const int hq = h / p.group;
  const int col0 = slice * kSliceCols;

  const int s = p.state_indices[b];
  int L = p.seq_lengths[b];
  L = L < 0 ? 0 : (L > T ? T : L);
  if (s < 0 || s >= p.pool_size) L = 0;  // skipped item: zero output, no slot touched

  // out[b, h, :, col0 : col0 + 64]; padded tokens get +0.0 (16-byte stores).
  uint16_t* out_bh = p.out + (static_cast<size_t>(b) * p.H_v + h) * T * p.D_v + col0;
  for (int e = tid; e < (T - L) * (kSliceCols / 8); e += NT) {
    const int t = L + e / (kSliceCols / 8);
    const int v8 = e % (kSliceCols / 8);
    *reinterpret_cast<uint4*>(out_bh + static_cast<size_t>(t) * p.D_v + v8 * 8) =
        make_uint4(0u, 0u, 0u, 0u);
  }
  if (L == 0) return;

  // ---- state tile load (issued first so it is in flight during the prologue)
  const int cg = lane & 7;
  const int rl = lane >> 3;
  const int i0 = warp * 32 + rl * kRowsPerThread;
  uint16_t* tile = p.state_pool + ((static_cast<size_t>(s) * p.H_v + h) * DK) * p.D_v + col0 +
                   cg * kColsPerThread;
  uint4 raw[kRowsPerThread];
#pragma unroll
  for (int r = 0; r < kRowsPerThread; ++r)
    raw[r] = __ldcs(reinterpret_cast<const uint4*>(tile + static_cast<size_t>(i0 + r) * p.D_v));

  // ---- prologue: per-token vectors in shared memory
  float* sk = smem;               // [T][DK] k
  float* sq = sk + T * DK;        // [T][DK] q * scale
  float* sd = sq + T * DK;        // [T][DK] exp(g + gk)
  float* red = sd + T * DK;       // [WARPS][32][4]
  float* sdelta = red + WARPS * 128;
  float* s_beta = sdelta + kSliceCols;
  float* s_kq = s_beta + kMaxT;
  float* s_g = s_kq + kMaxT;

  if (tid < L) {
    float gt, bt;
    if constexpr (GATED) {
      const size_t ai = (static_cast<size_t>(b) * T + tid) * p.H_v + h;
      gt = p.decay_scale[h] * softplus_f32(bf16_bits_to_f32(p.gate_a[ai]) + p.dt_bias[h]);
      bt = sigmoid_f32(bf16_bits_to_f32(p.gate_b[ai]));
    } else {
      const size_t gi = (static_cast<size_t>(b) * p.H_v + h) * T + tid;
      gt = p.g[gi];
      bt = bf16_bits_to_f32(p.beta[gi]);
    }
    s_g[tid] = gt;
    s_beta[tid] = bt;
  }
  __syncthreads();
  {
    const size_t qk_off = (static_cast<size_t>(b) * p.H_qk + hq) * T * DK;
    const uint16_t* qb = p.query + qk_off;
    const uint16_t* kb = p.key + qk_off;
    const float* gkb = p.gk + (static_cast<size_t>(b) * p.H_v + h) * T * DK;
    for (int e = tid; e < L * DK; e += NT) {
      const int t = e / DK;
      sk[e] = bf16_bits_to_f32(kb[e]);
      sq[e] = bf16_bits_to_f32(qb[e]) * p.scale;
      sd[e] = expf(s_g[t] + gkb[e]);
    }
  }
  __syncthreads();
  for (int t = warp; t < L; t += WARPS) {
    float acc = 0.0f;
#pragma unroll
    for (int i = lane; i < DK; i += 32) acc = fmaf(sk[t * DK + i], sq[t * DK + i], acc);
    acc = warp_sum(acc);
    if (lane == 0) s_kq[t] = acc;
  }
  __syncthreads();

  float S[kRowsPerThread][kColsPerThread];
#pragma unroll
  for (int r = 0; r < kRowsPerThread; ++r) {
    const uint32_t w[4] = {raw[r].x, raw[r].y, raw[r].z, raw[r].w};
#pragma unroll
    for (int c2 = 0; c2 < 4; ++c2) {
      S[r][2 * c2] = bf16_lo(w[c2]);
      S[r][2 * c2 + 1] = bf16_hi(w[c2]);
    }
  }

  const bool bit4 = (lane >> 4) & 1;
  const bool bit3 = (lane >> 3) & 1;
  const uint16_t* v_bh = p.value + (static_cast<size_t>(b) * p.H_v + h) * T * p.D_v + col0;

  for (int t = 0; t < L; ++t) {
    const float* kt = sk + t * DK + i0;
    const float* qt = sq + t * DK + i0;
    const float* dt = sd + t * DK + i0;
    float kr[kRowsPerThread], qr[kRowsPerThread];
    float m[kColsPerThread], pp[kColsPerThread];
#pragma unroll
    for (int c = 0; c < kColsPerThread; ++c) m[c] = pp[c] = 0.0f;
#pragma unroll
    for (int r = 0; r < kRowsPerThread; ++r) {
      kr[r] = kt[r];
      qr[r] = qt[r];
      const float d = dt[r];
#pragma unroll
      for (int c = 0; c < kColsPerThread; ++c) {
        S[r][c] *= d;                       // step 1: decay row r
        m[c] = fmaf(S[r][c], kr[r], m[c]);  // step 2: kv_mem partial
        pp[c] = fmaf(S[r][c], qr[r], pp[c]);
      }
    }
    // Reduce-scatter over the 4 row lanes: xor 16 splits (kv_mem | p), xor 8
    // splits the 8 columns into halves. Lane (bit4, bit3, cg) ends with the
    // full warp sum of vector (bit4 ? p : kv_mem) at columns cg*8 + bit3*4 + 0..3.
    float x[kColsPerThread];
#pragma unroll
    for (int c = 0; c < kColsPerThread; ++c) {
      const float send = bit4 ? m[c] : pp[c];
      const float keep = bit4 ? pp[c] : m[c];
      x[c] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    float y[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float send = bit3 ? x[c] : x[c + 4];
      const float keep = bit3 ? x[c + 4] : x[c];
      y[c] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    *reinterpret_cast<float4*>(red + (warp * 32 + lane) * 4) = make_float4(y[0], y[1], y[2], y[3]);
    __syncthreads();
    if (tid < kSliceCols) {
      const int j = tid;
      const int lm = ((j >> 2) & 1) * 8 + (j >> 3);  // lane holding kv_mem of column j
      const int e = j & 3;
      float mem = 0.0f, pj = 0.0f;
#pragma unroll
      for (int w = 0; w < WARPS; ++w) {
        mem += red[(w * 32 + lm) * 4 + e];
        pj += red[(w * 32 + 16 + lm) * 4 + e];
      }
      const float vj = bf16_bits_to_f32(v_bh[static_cast<size_t>(t) * p.D_v + j]);
      const float delta = (vj - mem) * s_beta[t];  // step 3: (v - kv_mem) * beta
      sdelta[j] = delta;
      const float o = fmaf(delta, s_kq[t], pj);    // step 4: o = S_new^T q_s
      out_bh[static_cast<size_t>(t) * p.D_v + j] = f32_to_bf16_bits(o);
    }
    __syncthreads();
    float dl[kColsPerThread];
    {
      const float4 d0 = *reinterpret_cast<const float4*>(sdelta + cg * 8);
      const float4 d1 = *reinterpret_cast<const float4*>(sdelta + cg * 8 + 4);
      dl[0] = d0.x; dl[1] = d0.y; dl[2] = d0.z; dl[3] = d0.w;
      dl[4] = d1.x; dl[5] = d1.y; dl[6] = d1.z; dl[7] = d1.w;
    }
#pragma unroll
    for (int r = 0; r < kRowsPerThread; ++r)
#pragma unroll
      for (int c = 0; c < kColsPerThread; ++c) S[r][c] = fmaf(kr[r], dl[c], S[r][c]);  // step 3
  }

  // ---- state tile store: bf16, round-to-nearest-even, once per call
#pragma unroll
  for (int r = 0; r < kRowsPerThread; ++r) {
    uint4 o;
    o.x = pack_bf16x2(S[r][0], S[r][1]);
    o.y = pack_bf16x2(S[r][2], S[r][3]);
    o.z = pack_bf16x2(S[r][4], S[r][5]);
    o.w = pack_bf16x2(S[r][6], S[r][7]);
    __stcs(reinterpret_cast<uint4*>(tile + static_cast<size_t>(i0 + r) * p.D_v), o);
  }
}

}  // namespace gdr
