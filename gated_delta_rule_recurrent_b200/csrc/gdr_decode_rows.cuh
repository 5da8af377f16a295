// Single-token decode on a k-contiguous pool [pool, H_v, D_v, D_k]: the four
// steps of "lite_boost.ops.recurrent_gated_delta_rule" (MindSpore Lite API
// page, section 算法流程) for T = 1, on the state layout the page's 注
// section gives for the NPU operator's own use.
//
// In this layout row j of a head's state holds S[:, j], its D_k entries
// contiguous, so each step is row-local:
//   kv_j = sum_i d_i S[i, j] k_i          (decay d = exp(g + gk), step 1-2)
//   delta_j = beta (v_j - kv_j)            (step 3)
//   S'[i, j] = d_i S[i, j] + k_i delta_j  (step 3)
//   o_j = sum_i S'[i, j] q_i scale         (step 4)
// A group of D_k / 8 lanes owns one row, 8 entries (16 bytes) per lane; the two
// sums are shuffle reductions inside the group, nothing crosses a group, and
// nothing is staged in shared memory. A warp takes blocks of RB consecutive
// rows of one head (RB = 64: 8 KB at D_k = 64, one contiguous run of the
// pool), 32 / (D_k / 8) rows per pass, computing the head's per-entry vectors
// d, k and q once per block. Loads go out four passes at a time, and the next
// four are in flight while the current four compute.
// Every read and write is a coalesced 16-byte access, so the kernel is bound by
// HBM once enough warps are resident.
//
// Items whose slot is outside the pool, or whose length clamps to 0, get
// +0.0 outputs and leave the pool untouched; with a committed count of 0 the
// output is still formed from the updated state and the slot keeps its bits
// (the committed-count reading of the multi-token kernels at T = 1).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr_decode.cuh"

namespace gdr {

constexpr int kRowsThreads = 256;  // 8 warps per CTA
constexpr int kRowsGroup = 4;      // passes whose loads are issued together

// One pass: row `row` of the block (this lane's 8 entries in w, its value v):
// the new row over the old one when `commit`, and o_j to out_rows[row].
template <int LPR>
__device__ __forceinline__ void rows_pass(const uint4 w, const float v, const float (&d)[8],
                                          const float (&kf)[8], const float (&qf)[8], float beta,
                                          uint16_t* row_ptr, uint16_t* out_row, bool commit,
                                          bool leader) {
  const uint32_t sw[4] = {w.x, w.y, w.z, w.w};
  float sd[8];
  float kv = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    sd[2 * e] = d[2 * e] * bf16_lo(sw[e]);
    sd[2 * e + 1] = d[2 * e + 1] * bf16_hi(sw[e]);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) kv = fmaf(sd[e], kf[e], kv);
#pragma unroll
  for (int o = 1; o < LPR; o <<= 1) kv += __shfl_xor_sync(0xffffffffu, kv, o);
  const float delta = beta * (v - kv);
  float o_part = 0.0f;
  uint32_t nw[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float s0 = fmaf(kf[2 * e], delta, sd[2 * e]);
    const float s1 = fmaf(kf[2 * e + 1], delta, sd[2 * e + 1]);
    o_part = fmaf(s0, qf[2 * e], o_part);
    o_part = fmaf(s1, qf[2 * e + 1], o_part);
    nw[e] = pack_bf16x2(s0, s1);
  }
#pragma unroll
  for (int o = 1; o < LPR; o <<= 1) o_part += __shfl_xor_sync(0xffffffffu, o_part, o);
  if (commit) *reinterpret_cast<uint4*>(row_ptr) = make_uint4(nw[0], nw[1], nw[2], nw[3]);
  if (leader) *out_row = f32_to_bf16_bits(o_part);
}

// RB rows of a head per warp block (64, or 16 for batches too small to give
// every SM enough 64-row blocks).
template <int DK, bool GATED, int RB>
__global__ void __launch_bounds__(kRowsThreads) decode_rows_kernel(const DecodeParams p,
                                                                    const int n_blocks) {
  constexpr int LPR = DK / 8;                   // lanes per row: 8 or 16
  constexpr int RPP = 32 / LPR;                 // rows per pass: 4 or 2
  constexpr int PASSES = RB / RPP;              // 4 .. 32
  constexpr int G = PASSES < kRowsGroup ? PASSES : kRowsGroup;
  constexpr int NG = PASSES / G;                // groups of G passes
  static_assert(PASSES % G == 0, "whole groups of passes");
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR;                   // row of the pass
  const int li = lane % LPR;                    // entries i = 8 li .. 8 li + 7
  const int n_warps = static_cast<int>(gridDim.x * blockDim.x) >> 5;
  const int blocks_per_head = p.D_v / RB;

  for (int blk = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5); blk < n_blocks;
       blk += n_warps) {
    const int jb = blk % blocks_per_head;
    const int h = (blk / blocks_per_head) % p.H_v;
    const int b = blk / (blocks_per_head * p.H_v);
    const size_t bh = static_cast<size_t>(b) * p.H_v + h;
    uint16_t* out_rows = p.out + bh * p.D_v + jb * RB;  // token 0 (T = 1)
    const int s = p.state_indices[b];
    int L = p.seq_lengths[b];
    L = L < 0 ? 0 : (L > 1 ? 1 : L);
    if (s < 0 || s >= p.pool_size) L = 0;
    if (L == 0) {  // padded or skipped: +0.0 outputs, the slot untouched
      for (int r = lane; r < RB; r += 32) out_rows[r] = 0;
      continue;
    }
    const bool commit = (p.num_accepted != nullptr ? p.num_accepted[b] : 1) > 0;
    uint16_t* rows =
        p.state_pool + ((static_cast<size_t>(s) * p.H_v + h) * p.D_v + jb * RB) * DK + 8 * li;
    const uint16_t* vrow = p.value + bh * p.D_v + jb * RB;
    // the first group's rows are requested before the head's vectors are formed
    uint4 w[2][G];
    float v[2][G];
#pragma unroll
    for (int q = 0; q < G; ++q) {
      w[0][q] = *reinterpret_cast<const uint4*>(rows + static_cast<size_t>(q * RPP + sub) * DK);
      v[0][q] = bf16_bits_to_f32(vrow[q * RPP + sub]);
    }

    // the head's gate and per-entry vectors for this lane's 8 entries
    float g, beta;
    if constexpr (GATED) {
      const size_t ai = static_cast<size_t>(b) * p.H_v + h;  // [B, T = 1, H_v]
      g = p.decay_scale[h] * softplus_f32(bf16_bits_to_f32(p.gate_a[ai]) + p.dt_bias[h]);
      beta = sigmoid_f32(bf16_bits_to_f32(p.gate_b[ai]));
    } else {
      g = p.g[bh];
      beta = bf16_bits_to_f32(p.beta[bh]);
    }
    const size_t qk = (static_cast<size_t>(b) * p.H_qk + h / p.group) * DK + 8 * li;
    const uint4 kw = *reinterpret_cast<const uint4*>(p.key + qk);
    const uint4 qw = *reinterpret_cast<const uint4*>(p.query + qk);
    const float* gkp = p.gk + bh * DK + 8 * li;
    float d[8], kf[8], qf[8];
    {
      const uint32_t kk[4] = {kw.x, kw.y, kw.z, kw.w};
      const uint32_t qq[4] = {qw.x, qw.y, qw.z, qw.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        kf[2 * e] = bf16_lo(kk[e]);
        kf[2 * e + 1] = bf16_hi(kk[e]);
        qf[2 * e] = bf16_lo(qq[e]) * p.scale;
        qf[2 * e + 1] = bf16_hi(qq[e]) * p.scale;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) d[e] = expf(g + gkp[e]);  // exp(g) exp(gk) as one exponential
    }

    // groups of G passes: the next group's loads are in flight while one computes
#pragma unroll
    for (int gi = 0; gi < NG; ++gi) {
      const int cur = gi & 1;
      if (gi + 1 < NG) {
#pragma unroll
        for (int q = 0; q < G; ++q) {
          const int row = ((gi + 1) * G + q) * RPP + sub;
          w[cur ^ 1][q] = *reinterpret_cast<const uint4*>(rows + static_cast<size_t>(row) * DK);
          v[cur ^ 1][q] = bf16_bits_to_f32(vrow[row]);
        }
      }
#pragma unroll
      for (int q = 0; q < G; ++q) {
        const int row = (gi * G + q) * RPP + sub;
        rows_pass<LPR>(w[cur][q], v[cur][q], d, kf, qf, beta,
                       rows + static_cast<size_t>(row) * DK, out_rows + row, commit, li == 0);
      }
    }
  }
}

}  // namespace gdr
