// Decode kernel with the two whole-tile contractions on the tcgen05 tensor
// cores, for 128 x 128 tiles of a D_k = 128 state (D_v a multiple of 128),
// any token count, on a [pool, H_v, D_k, D_v] pool or a k-contiguous
// [pool, H_v, D_v, D_k] pool (VK; there the staged tile holds VS rows j of
// D_k entries, pass 1 reads it K-major, and pass 2 forms D2^T = [delta parts]
// [e parts]^T so that TMEM lane j holds row j of the new tile).
//
// Arithmetic: the chunked form of the four steps of
// "lite_boost.ops.recurrent_gated_delta_rule" (MindSpore Lite API page,
// section 算法流程) over the L valid tokens of one (item, value head), as in
// gdr_decode_chunk.cuh: with d_t = exp(g_t + gk_t), running products P_t and
// P_{s->t}, u_t = P_t k_t, w_t = P_t q^_t (q^ = q * scale),
//   kv_mem_t = S_0^T u_t + sum_{s<t} A_ts delta_s,
//   o_t      = S_0^T w_t + sum_{s<=t} B_ts delta_s,
//   delta_t  = beta_t (v_t - kv_mem_t),
//   S_n      = c o S_0 + sum_{s<n} e_s delta_s^T   (c = P_{n-1}, e_s = P_{s->n-1} k_s),
// n the committed token count. When GATED, g and beta come from the gate of
// "com.microsoft.LinearAttentionGate" (README, section Description).
//
// The two products that touch every state entry run as tcgen05 MMAs with the
// fp32 accumulator in tensor memory:
//   pass 1  D1 = S_0^T [u_hi u_lo w_hi w_lo]          M = 128 (column j),
//           N = 32 (4 parts x 8 tokens), K = 128 (row i); S_0 is read where
//           TMA left it (bf16, 128-byte swizzle, M-major);
//   pass 2  D2 = [e_hi e_hi e_lo 0] [delta_hi delta_lo delta_hi 0]^T
//           M = 128 (row i), N = 128 (column j), K = 32.
// Operands are bf16, so every fp32 vector x enters as two bf16 parts, x_hi =
// bf16(x) and x_lo = bf16(x - x_hi), which carry 16 significant bits; the
// tensor core forms the bf16 products exactly and sums them in fp32. Pass 2
// drops only e_lo * delta_lo, below 2^-16 of the term. The L x L sums A_ts,
// B_ts, the gate, the decays and the unit lower-triangular solve for delta
// stay on the CUDA cores.
//
// CTA: NG consumer groups of 4 warps and one producer warp (plus, for
// single-token calls, one sums warp per group), one CTA per SM, persistent
// over tiles blockIdx.x, + gridDim.x, ...; group g takes every NG-th tile.
// Thread r of a group (warp w = r / 32, so TMEM lanes 32 (w % 4) + lane) is
// row i = r of the tile in the row-wise steps and column j = r in the
// column-wise ones:
//   1. finalise (row i): decays, u, w, e, c, and its share of A and B (a warp
//      reduce-scatter into the warp's slot); the row's pass-1 and pass-2
//      operands go to the group's shared block;
//   2. an elected lane issues pass 1 (8 MMAs, K = 16 each) and commits it to
//      the group's mbarrier; threads 0..63 add the four warps' slots of A and
//      B in a fixed order (deterministic). For a single token A and B reduce
//      to B_00 = k . q^, and the group's sums warp forms it instead, so the
//      group skips the slots and a barrier;
//   3. solve (column j): reads its TMEM lane of D1 (kv_mem and o parts),
//      solves for delta, writes o, and writes its delta row of the pass-2 B
//      operand;
//   4. the elected lane issues pass 2 (2 MMAs); each thread then reads its
//      row of D2, adds c_i S_0[i, :] from the staged tile, rounds to bf16 and
//      writes the row back over S_0 in place; the elected thread stores the
//      tile to the slot with one TMA store and releases the stage once the
//      store has read it, after finalising the group's next tile (so the
//      store's read of the stage overlaps that work).
// The producer warp starts the copies of each tile as in the chunked kernel
// (one TMA box for the state, bulk copies for the k, q, gk and v rows of the
// valid tokens, 4-byte copies for the gate scalars).
//
// Every mbarrier wait is bounded; a wait that runs out sets a bit in the
// device error word and the kernel carries on with the same control flow, so
// every named barrier is reached by every thread of its group and the tensor
// memory is always freed.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr_decode.cuh"
#include "gdr_decode_chunk.cuh"
#include "gdr_ptx.cuh"
#include "gdr_umma.cuh"

namespace gdr {

constexpr int kTcDK = 128;            // rows of a tile (D_k)
constexpr int kTcVS = 128;            // columns of a tile
constexpr int kTcStateBytes = kTcDK * kTcVS * 2;
constexpr int kTcGroupThreads = 128;  // one thread per TMEM lane
#ifndef GDR_TC_GROUPS
#define GDR_TC_GROUPS 2
#endif
constexpr int kTcGroups = GDR_TC_GROUPS;
// groups, one sums warp per group (single-token calls), the producer
constexpr int kTcMaxThreads = kTcGroups * (kTcGroupThreads + 32) + 32;
constexpr int kTcN1 = 32;  // pass-1 columns: u_hi, u_lo, w_hi, w_lo, 8 tokens each
constexpr int kTcK2 = 32;  // pass-2 depth: (e_hi, d_hi), (e_hi, d_lo), (e_lo, d_hi), zeros
// TMEM columns: D2 of group g at 128 g, D1 of group g at 128 NG + 32 g.
constexpr int kTcTmemCols = kTcGroups * (kTcVS + kTcN1) <= 256 ? 256 : 512;
static_assert(kTcGroups * (kTcVS + kTcN1) <= 512, "TMEM holds 512 columns");

// Per-stage vector block (after the stage's state tile), T padded tokens.
struct TcLayout {
  int v, k, q, gk, raw, meta, ab, bytes;
};
__host__ __device__ inline TcLayout tc_layout(int T) {
  TcLayout s;
  s.v = 0;                         // bf16 [T][VS]  value rows of the slice
  s.k = s.v + T * kTcVS * 2;       // bf16 [T][DK]  key rows
  s.q = s.k + T * kTcDK * 2;       // bf16 [T][DK]  query rows
  s.gk = s.q + T * kTcDK * 2;      // fp32 [T][DK]  gk rows
  s.raw = s.gk + T * kTcDK * 4;    // u32 [8] g or a words, [8] beta or b words, dt_bias, decay_scale
  s.meta = s.raw + 80;             // int32 [4]     length, slot, committed tokens
  s.ab = s.meta + 16;              // fp32 [8][8] A_ts, then [8][8] B_ts (from a sums warp)
  s.bytes = (s.ab + 512 + 127) & ~127;
  return s;
}

// Per-group block (1024-byte aligned). The MMA operands, bf16, no swizzle,
// in 8 x 16-byte core matrices of 128 contiguous bytes:
//   B1  pass-1 B, N-major: 16 bytes = 8 tokens of one part at row i, at
//       part * 2048 + (i / 8) * 128 + (i % 8) * 16 (LBO 128 along K = i,
//       SBO 2048 between the 8-column groups of N);
//   E   e parts, K-major: 16 bytes = 8 tokens of K group kc at row i, at
//       (i / 8) * 512 + kc * 128 + (i % 8) * 16 (LBO 128 between the two K
//       groups of one MMA, SBO 512 between 8-row groups);
//   DL  delta parts, K-major: the same over columns j.
// Pass 2 takes E as A and DL as B on a [pool, H_v, D_k, D_v] pool, and the
// other way round on a k-contiguous one.
constexpr int kTcB1 = 0;
constexpr int kTcE = 8192;
constexpr int kTcDL = 16384;
constexpr int kTcPart = 24576;  // fp32 [4 warps][8][8] partial sums of A and B
constexpr int kTcA = 25600;     // fp32 [8][8] A_ts at [t][s], s < t
constexpr int kTcBm = 25856;    // fp32 [8][8] B_ts at [t][s], s <= t
constexpr int kTcC = 26112;     // fp32 [DK] c (k-contiguous pools: read across rows)
constexpr int kTcGroupBytes = 26624;

// Four mbarriers per stage (vectors landed, state landed, stage released, A
// and B summed by a sums warp) and one per group (its MMAs done).
__host__ __device__ inline int tc_smem_bytes(int T, int n_stages, int n_groups) {
  const int vec = (n_stages * tc_layout(T).bytes + 1023) & ~1023;
  return 1024 /* alignment slack */ + n_stages * kTcStateBytes + vec + n_groups * kTcGroupBytes +
         (4 * n_stages + n_groups) * 8 + 16 /* TMEM address, abort word (gdr_ptx.cuh) */;
}

// Eight fp32 values as bf16 (hi, lo) parts, packed in pairs: hi = bf16(x),
// lo = bf16(x - hi) (0 when hi is not finite).
__device__ __forceinline__ void split_bf16x8(const float (&x)[8], uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    h[p] = pack_bf16x2(x[2 * p], x[2 * p + 1]);
    const float h0 = bf16_lo(h[p]), h1 = bf16_hi(h[p]);
    const float r0 = fabsf(h0) < __int_as_float(0x7f800000) ? x[2 * p] - h0 : 0.0f;
    const float r1 = fabsf(h1) < __int_as_float(0x7f800000) ? x[2 * p + 1] - h1 : 0.0f;
    l[p] = pack_bf16x2(r0, r1);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// ---------------------------------------------------------------- row-wise: finalise

// Row i of a tile with L = LC tokens: writes the row's pass-1 operand (u, w)
// and pass-2 operand (e), and, when PAIRS, this warp's partial sums of A and
// B to slot wq (entry (r, col): B_{t=r, s=col} for col <= r, A_{t=col, s=r}
// for col > r; without PAIRS a sums warp forms them). The gate value g_t sits
// in lane t. Returns c_i = P_{n-1}[i] (0 when n = 0). With nv < LC only the
// first nv tokens are valid (n <= nv): u and w are zero past them, and the
// sums that involve a later token are left unspecified (never read).
// before_e() runs right before the e operand is written (a caller whose
// previous pass 2 may still be reading it waits there).
struct TcNoHook {
  __device__ __forceinline__ void operator()() const {}
};
template <int LC, bool PAIRS, class BeforeE = TcNoHook>
__device__ __forceinline__ float tc_finalize(const uint8_t* vb, const TcLayout& lay, uint8_t* gb,
                                             float g_lane, float scale, int i, int lane, int wq,
                                             int n, int nv = LC, BeforeE before_e = BeforeE()) {
  constexpr int DK = kTcDK;
  constexpr int NM = pow2_at_least(LC * LC);  // partial sums, padded for the reduce-scatter
  float g[LC];
#pragma unroll
  for (int t = 0; t < LC; ++t) g[t] = __shfl_sync(0xffffffffu, g_lane, t);
  const uint16_t* sk = reinterpret_cast<const uint16_t*>(vb + lay.k);
  const uint16_t* sq = reinterpret_cast<const uint16_t*>(vb + lay.q);
  const float* sgk = reinterpret_cast<const float*>(vb + lay.gk);
  float d[LC], kf[LC], qf[LC];
#pragma unroll
  for (int t = 0; t < LC; ++t) {
    d[t] = expf(g[t] + sgk[t * DK + i]);  // exp(g) * exp(gk) as one exponential
    kf[t] = bf16_bits_to_f32(sk[t * DK + i]);
    qf[t] = bf16_bits_to_f32(sq[t * DK + i]) * scale;
  }
  // u_t = P_t k_t and w_t = P_t q^_t; the committed state is the one after
  // token n - 1, so c = P_{n-1}
  float u[8], w[8];
  float P = 1.0f, c = 0.0f;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    u[t] = 0.0f;
    w[t] = 0.0f;
    if (t < LC) {
      P = t == 0 ? d[0] : P * d[t];
      if (t < nv) {
        u[t] = P * kf[t];
        w[t] = P * qf[t];
      }
      if (t == n - 1) c = P;
    }
  }
  uint4 hi, lo;
  uint8_t* b1 = gb + kTcB1 + (i >> 3) * 128 + (i & 7) * 16;
  split_bf16x8(u, hi, lo);
  *reinterpret_cast<uint4*>(b1) = hi;
  *reinterpret_cast<uint4*>(b1 + 2048) = lo;
  split_bf16x8(w, hi, lo);
  *reinterpret_cast<uint4*>(b1 + 4096) = hi;
  *reinterpret_cast<uint4*>(b1 + 6144) = lo;

  if constexpr (!PAIRS) {  // a sums warp forms A and B: only e_s = P_{s->n-1} k_s here
    float e[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      e[s] = 0.0f;
      if (s < LC && s < n) {
        float z = kf[s];
#pragma unroll
        for (int t = s + 1; t < LC; ++t)
          if (t < n) z *= d[t];
        e[s] = z;
      }
    }
    split_bf16x8(e, hi, lo);
    before_e();
    uint8_t* ep = gb + kTcE + (i >> 3) * 512 + (i & 7) * 16;
    *reinterpret_cast<uint4*>(ep) = hi;
    *reinterpret_cast<uint4*>(ep + 128) = hi;
    *reinterpret_cast<uint4*>(ep + 256) = lo;
    *reinterpret_cast<uint4*>(ep + 384) = make_uint4(0u, 0u, 0u, 0u);
    return c;
  }
  // e_s = P_{s->n-1} k_s (0 for s >= n) and the sums A_ts = k_s . P_{s->t} k_t,
  // B_ts = k_s . P_{s->t} q^_t over this row, by running products
  float mp[NM];
#pragma unroll
  for (int j = 0; j < NM; ++j) mp[j] = 0.0f;
  float e[8];
#pragma unroll
  for (int s = 0; s < 8; ++s) e[s] = 0.0f;
#pragma unroll
  for (int s = 0; s < LC; ++s) {
    float z = kf[s];
    float es = s == n - 1 ? z : 0.0f;
    mp[s * LC + s] = fmaf(z, qf[s], mp[s * LC + s]);
#pragma unroll
    for (int t = s + 1; t < LC; ++t) {
      z *= d[t];
      mp[s * LC + t] = fmaf(z, kf[t], mp[s * LC + t]);
      mp[t * LC + s] = fmaf(z, qf[t], mp[t * LC + s]);
      if (t == n - 1) es = z;
    }
    e[s] = es;
  }
  split_bf16x8(e, hi, lo);
  before_e();
  uint8_t* ep = gb + kTcE + (i >> 3) * 512 + (i & 7) * 16;
  *reinterpret_cast<uint4*>(ep) = hi;
  *reinterpret_cast<uint4*>(ep + 128) = hi;
  *reinterpret_cast<uint4*>(ep + 256) = lo;
  *reinterpret_cast<uint4*>(ep + 384) = make_uint4(0u, 0u, 0u, 0u);

  reduce_scatter<NM>(mp, lane);
  constexpr int NL = NM >= 32 ? NM / 32 : 1;
  if (reduce_scatter_writer<NM>(lane)) {
    const int base = reduce_scatter_base<NM>(lane);
    float* part = reinterpret_cast<float*>(gb + kTcPart) + wq * 64;
#pragma unroll
    for (int j = 0; j < NL; ++j) {
      const int f = base + j;
      if (f < LC * LC) part[(f / LC) * 8 + f % LC] = mp[j];
    }
  }
  return c;
}

template <bool PAIRS>
__device__ __forceinline__ float tc_finalize_any(int L, int n, const uint8_t* vb,
                                                 const TcLayout& lay, uint8_t* gb, float g_lane,
                                                 float scale, int i, int lane, int wq) {
  switch (L) {
    case 1: return tc_finalize<1, PAIRS>(vb, lay, gb, g_lane, scale, i, lane, wq, n);
    case 2: return tc_finalize<2, PAIRS>(vb, lay, gb, g_lane, scale, i, lane, wq, n);
    case 3: return tc_finalize<3, PAIRS>(vb, lay, gb, g_lane, scale, i, lane, wq, n);
    case 4: return tc_finalize<4, PAIRS>(vb, lay, gb, g_lane, scale, i, lane, wq, n);
    case 5: return tc_finalize<5, PAIRS>(vb, lay, gb, g_lane, scale, i, lane, wq, n);
    case 6: return tc_finalize<6, PAIRS>(vb, lay, gb, g_lane, scale, i, lane, wq, n);
    case 7: return tc_finalize<7, PAIRS>(vb, lay, gb, g_lane, scale, i, lane, wq, n);
    case 8: return tc_finalize<8, PAIRS>(vb, lay, gb, g_lane, scale, i, lane, wq, n);
    default: return 0.0f;
  }
}

// A and B from the four warps' slots, in warp order; thread r < 64 of the
// group takes entry r of the [8][8] grid.
__device__ __forceinline__ void tc_sum_parts(uint8_t* gb, int L, int r) {
  const int row = r >> 3, col = r & 7;
  if (r < 64 && row < L && col < L) {
    const float* part = reinterpret_cast<const float*>(gb + kTcPart);
    const float x = ((part[r] + part[64 + r]) + part[128 + r]) + part[192 + r];
    if (col > row) reinterpret_cast<float*>(gb + kTcA)[col * 8 + row] = x;  // A_{t = col, s = row}
    else reinterpret_cast<float*>(gb + kTcBm)[r] = x;                       // B_{t = row, s = col}
  }
}

// ---------------------------------------------------------------- the L x L sums

// A_ts = k_s . (P_{s->t} k_t) for s < t and B_ts = k_s . (P_{s->t} q^_t) for
// s <= t, over the DK rows of a tile with L = LC tokens, by one warp: each
// lane takes rows lane + 32 m and forms its share by running products, and a
// warp reduce-scatter leaves each sum in one lane, which writes it to `ab`
// (A at [t][s], then B at [t][s]). The gate value g_t sits in lane t.
template <int LC>
__device__ __forceinline__ void tc_pair_sums(const uint8_t* vb, const TcLayout& lay, float* ab,
                                             float g_lane, float scale, int lane) {
  constexpr int DK = kTcDK;
  constexpr int NM = pow2_at_least(LC * LC);  // padded for the reduce-scatter
  float g[LC];
#pragma unroll
  for (int t = 0; t < LC; ++t) g[t] = __shfl_sync(0xffffffffu, g_lane, t);
  const uint16_t* sk = reinterpret_cast<const uint16_t*>(vb + lay.k);
  const uint16_t* sq = reinterpret_cast<const uint16_t*>(vb + lay.q);
  const float* sgk = reinterpret_cast<const float*>(vb + lay.gk);
  // mp[s * LC + t] (s < t) holds A_ts, mp[t * LC + s] (s <= t) holds B_ts
  float mp[NM];
#pragma unroll
  for (int j = 0; j < NM; ++j) mp[j] = 0.0f;
#pragma unroll 1
  for (int i = lane; i < DK; i += 32) {
    float d[LC], kf[LC], qf[LC];
#pragma unroll
    for (int t = 0; t < LC; ++t) {
      d[t] = expf(g[t] + sgk[t * DK + i]);
      kf[t] = bf16_bits_to_f32(sk[t * DK + i]);
      qf[t] = bf16_bits_to_f32(sq[t * DK + i]) * scale;
    }
#pragma unroll
    for (int s = 0; s < LC; ++s) {
      float z = kf[s];  // P_{s->t} k_s by running products
      mp[s * LC + s] = fmaf(z, qf[s], mp[s * LC + s]);
#pragma unroll
      for (int t = s + 1; t < LC; ++t) {
        z *= d[t];
        mp[s * LC + t] = fmaf(z, kf[t], mp[s * LC + t]);
        mp[t * LC + s] = fmaf(z, qf[t], mp[t * LC + s]);
      }
    }
  }
  reduce_scatter<NM>(mp, lane);
  constexpr int NL = NM >= 32 ? NM / 32 : 1;
  if (reduce_scatter_writer<NM>(lane)) {
    const int base = reduce_scatter_base<NM>(lane);
#pragma unroll
    for (int j = 0; j < NL; ++j) {
      const int f = base + j;
      if (f < LC * LC) {
        const int r = f / LC, col = f % LC;
        if (col > r) ab[col * 8 + r] = mp[j];  // A_{t = col, s = r}
        else ab[64 + r * 8 + col] = mp[j];     // B_{t = r, s = col}
      }
    }
  }
}

__device__ __forceinline__ void tc_pair_sums_any(int L, const uint8_t* vb, const TcLayout& lay,
                                                 float* ab, float g_lane, float scale, int lane) {
  switch (L) {
    case 1: tc_pair_sums<1>(vb, lay, ab, g_lane, scale, lane); break;
    case 2: tc_pair_sums<2>(vb, lay, ab, g_lane, scale, lane); break;
    case 3: tc_pair_sums<3>(vb, lay, ab, g_lane, scale, lane); break;
    case 4: tc_pair_sums<4>(vb, lay, ab, g_lane, scale, lane); break;
    case 5: tc_pair_sums<5>(vb, lay, ab, g_lane, scale, lane); break;
    case 6: tc_pair_sums<6>(vb, lay, ab, g_lane, scale, lane); break;
    case 7: tc_pair_sums<7>(vb, lay, ab, g_lane, scale, lane); break;
    case 8: tc_pair_sums<8>(vb, lay, ab, g_lane, scale, lane); break;
    default: break;
  }
}

// ---------------------------------------------------------------- column-wise: solve

// Column j of a tile with L = LC tokens, from this thread's TMEM lane of D1:
// kv_mem and the S_0 part of o per token, the unit lower-triangular solve for
// delta, o to `out_t0` (token 0, column 0 of the tile's output), and the
// column's delta row of the pass-2 B operand (zeros past LC, or past nv when
// only the first nv tokens are valid). beta_t sits in lane t.
template <int LC>
__device__ __forceinline__ void tc_solve(const uint32_t (&x)[32], const uint8_t* vb,
                                         const TcLayout& lay, uint8_t* gb, const float* sa,
                                         const float* sb, float b_lane, int j, uint16_t* out_t0,
                                         int D_v, int nv = LC) {
  const uint16_t* sv = reinterpret_cast<const uint16_t*>(vb + lay.v);
  float dl[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) dl[t] = 0.0f;
#pragma unroll
  for (int t = 0; t < LC; ++t) {
    if (t >= nv) break;  // tokens past nv: no output, delta 0
    const float beta = __shfl_sync(0xffffffffu, b_lane, t);
    // kv_mem_t = S_0^T u_t + sum_{s<t} A_ts delta_s (step 2)
    float kv = __uint_as_float(x[t]) + __uint_as_float(x[8 + t]);
#pragma unroll
    for (int s = 0; s < t; ++s) kv = fmaf(sa[t * 8 + s], dl[s], kv);
    dl[t] = (bf16_bits_to_f32(sv[t * kTcVS + j]) - kv) * beta;  // step 3
    // o_t = S_0^T w_t + sum_{s<=t} B_ts delta_s (step 4)
    float o = __uint_as_float(x[16 + t]) + __uint_as_float(x[24 + t]);
#pragma unroll
    for (int s = 0; s <= t; ++s) o = fmaf(sb[t * 8 + s], dl[s], o);
    out_t0[static_cast<size_t>(t) * D_v + j] = f32_to_bf16_bits(o);
  }
  uint4 hi, lo;
  split_bf16x8(dl, hi, lo);
  uint8_t* dp = gb + kTcDL + (j >> 3) * 512 + (j & 7) * 16;
  *reinterpret_cast<uint4*>(dp) = hi;
  *reinterpret_cast<uint4*>(dp + 128) = lo;
  *reinterpret_cast<uint4*>(dp + 256) = hi;
  *reinterpret_cast<uint4*>(dp + 384) = make_uint4(0u, 0u, 0u, 0u);
}

__device__ __forceinline__ void tc_solve_any(int L, const uint32_t (&x)[32], const uint8_t* vb,
                                             const TcLayout& lay, uint8_t* gb, const float* sa,
                                             const float* sb, float b_lane, int j,
                                             uint16_t* out_t0, int D_v) {
  switch (L) {
    case 1: tc_solve<1>(x, vb, lay, gb, sa, sb, b_lane, j, out_t0, D_v); break;
    case 2: tc_solve<2>(x, vb, lay, gb, sa, sb, b_lane, j, out_t0, D_v); break;
    case 3: tc_solve<3>(x, vb, lay, gb, sa, sb, b_lane, j, out_t0, D_v); break;
    case 4: tc_solve<4>(x, vb, lay, gb, sa, sb, b_lane, j, out_t0, D_v); break;
    case 5: tc_solve<5>(x, vb, lay, gb, sa, sb, b_lane, j, out_t0, D_v); break;
    case 6: tc_solve<6>(x, vb, lay, gb, sa, sb, b_lane, j, out_t0, D_v); break;
    case 7: tc_solve<7>(x, vb, lay, gb, sa, sb, b_lane, j, out_t0, D_v); break;
    case 8: tc_solve<8>(x, vb, lay, gb, sa, sb, b_lane, j, out_t0, D_v); break;
    default: break;
  }
}

// ---------------------------------------------------------------- row-wise: new state

// Row i of S_n = c_i S_0[i, :] + D2[i, :], rounded to bf16 and written over
// S_0 in the staged (swizzled) tile, 32 columns per TMEM read.
// 64 columns per round: two TMEM reads in flight, and the round's 8 state
// chunks read from shared memory while they are.
__device__ __forceinline__ void tc_new_state_row(uint8_t* st, uint32_t d2_lane, float c, int i) {
  const unsigned long long cc = pk(c, c);
#pragma unroll 1  // two rounds as a loop: half the code, measured faster

  for (int k = 0; k < kTcVS / 64; ++k) {
    uint32_t acc[2][32];
    tmem_ld32(d2_lane + 64 * k, acc[0]);
    tmem_ld32(d2_lane + 64 * k + 32, acc[1]);
    uint4* ptr[8];
    uint4 s0[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      ptr[q] = reinterpret_cast<uint4*>(st + swz_offset<kTcDK>(i, 64 * k + 8 * q));
      s0[q] = *ptr[q];
    }
    tmem_wait_ld();
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint32_t sw[4] = {s0[q].x, s0[q].y, s0[q].z, s0[q].w};
      const uint32_t* a = &acc[q >> 2][8 * (q & 3)];
      uint32_t nw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 r = upk(fma2(cc, pk(bf16_lo(sw[e]), bf16_hi(sw[e])),
                                  pk(__uint_as_float(a[2 * e]), __uint_as_float(a[2 * e + 1]))));
        nw[e] = pack_bf16x2(r.x, r.y);
      }
      *ptr[q] = make_uint4(nw[0], nw[1], nw[2], nw[3]);
    }
  }
}

// ---------------------------------------------------------------- kernel

// Block: n_groups consumer groups (warps 0 .. 4 n_groups - 1), then, when
// SUMS, one sums warp per group, then the producer warp. Sums warp g takes
// group g's tiles in order, so it follows that group's stages fill by fill
// and none of its waits can see a phase two fills old either (SUMS serves
// single-token calls: there the sums are one dot product per tile, and
// taking them off the groups saves a barrier per tile; with several tokens
// the sums are the larger part of the row work and are better spread over the
// groups' four warps, one per scheduler). Each group owns n_stages / n_groups
// stages (n_stages a multiple of n_groups) and takes them in turn, so a stage
// passes only between the producer and one group, which has waited for the
// stage's previous fill before it waits for the next: no wait can see a phase
// two fills old. T8 marks the instance that T = 8 calls launch (the row and
// column code for L <= 4 and L <= 8 only); other multi-token calls take the
// instance with all eight token counts.
__device__ __forceinline__ int tc_stage(int j, int n_groups, int per_group) {
  return (j % n_groups) * per_group + (j / n_groups) % per_group;
}
__device__ __forceinline__ uint32_t tc_phase(int j, int n_groups, int per_group) {
  return static_cast<uint32_t>((j / n_groups) / per_group) & 1u;
}

// k-contiguous pool: row j of S_n^T, S_n^T[j, i] = c_i S_0^T[j, i] + D2^T[j, i],
// over the staged tile [D_k / 64][VS rows j][64] (c from shared memory).
__device__ __forceinline__ void tc_new_state_row_vk(uint8_t* st, uint32_t d2_lane, const float* c,
                                                    int j) {
#pragma unroll 1  // as tc_new_state_row
  for (int k = 0; k < kTcDK / 64; ++k) {
    uint32_t acc[2][32];
    tmem_ld32(d2_lane + 64 * k, acc[0]);
    tmem_ld32(d2_lane + 64 * k + 32, acc[1]);
    uint4* ptr[8];
    uint4 s0[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      ptr[q] = reinterpret_cast<uint4*>(st + swz_offset<kTcVS>(j, 64 * k + 8 * q));
      s0[q] = *ptr[q];
    }
    tmem_wait_ld();
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint32_t sw[4] = {s0[q].x, s0[q].y, s0[q].z, s0[q].w};
      const uint32_t* a = &acc[q >> 2][8 * (q & 3)];
      const ulonglong2* cq = reinterpret_cast<const ulonglong2*>(c + 64 * k + 8 * q);
      const ulonglong2 c01 = cq[0], c23 = cq[1];
      const unsigned long long cc[4] = {c01.x, c01.y, c23.x, c23.y};
      uint32_t nw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 r = upk(fma2(cc[e], pk(bf16_lo(sw[e]), bf16_hi(sw[e])),
                                  pk(__uint_as_float(a[2 * e]), __uint_as_float(a[2 * e + 1]))));
        nw[e] = pack_bf16x2(r.x, r.y);
      }
      *ptr[q] = make_uint4(nw[0], nw[1], nw[2], nw[3]);
    }
  }
}

template <bool GATED, bool VK, bool SUMS, bool T8>
__global__ void __launch_bounds__(kTcMaxThreads, 1)
    decode_chunk_tc_kernel(const __grid_constant__ CUtensorMap pool_map, const DecodeParams p,
                           const int n_tiles, const int n_stages) {
  constexpr int DK = kTcDK, VS = kTcVS;
  const int T = p.T;
  const TcLayout lay = tc_layout(T);

  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw_base = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + (((raw_base + 1023u) & ~1023u) - raw_base);
  uint8_t* vec_base = smem + n_stages * kTcStateBytes;
  uint8_t* grp_base = vec_base + ((n_stages * lay.bytes + 1023) & ~1023);
  const int n_groups = (static_cast<int>(blockDim.x >> 5) - 1) / (SUMS ? 5 : 4);
  const int per_group = n_stages / n_groups;
  uint64_t* bars = reinterpret_cast<uint64_t*>(grp_base + n_groups * kTcGroupBytes);
  const uint32_t vec0 = smem_addr(bars);          // k, q, gk, v rows and gate scalars landed
  const uint32_t sta0 = vec0 + 8 * n_stages;      // state tile landed
  const uint32_t empty0 = sta0 + 8 * n_stages;    // the group is done with the stage
  const uint32_t ab0 = empty0 + 8 * n_stages;     // the stage's A and B are summed (SUMS)
  const uint32_t mma0 = ab0 + 8 * n_stages;       // a group's MMAs are done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4 * n_stages + n_groups);
  volatile int* abort_word = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int first_sums = 4 * n_groups;  // SUMS: sums warps, one per group
  const int producer = SUMS ? first_sums + n_groups : first_sums;
  const int n_slices = p.D_v / VS;
  const int n_mine = (n_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                     static_cast<int>(gridDim.x);

  if (tid == 0) {
    for (int i = 0; i < n_stages; ++i) {
      mbar_init(vec0 + 8 * i, 32);  // one cp.async arrival per producer lane
      mbar_init(sta0 + 8 * i, 1);   // the producer's lane 0 (+ the TMA bytes)
      mbar_init(empty0 + 8 * i, 1); // the group's elected thread
      mbar_init(ab0 + 8 * i, 1);    // lane 0 of the group's sums warp (SUMS)
    }
    for (int g = 0; g < n_groups; ++g) mbar_init(mma0 + 8 * g, 1);  // one MMA commit
    *abort_word = 0;
    fence_mbar_init();
  }
  __syncwarp();
  if (warp == 0) {
    tmem_alloc(smem_addr(tmem_slot), kTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == producer) {
    // ================================================================ producer
    // lane i holds the slot, length and committed count of tile (j & ~31) + i;
    // the next 32 tiles' are loaded 32 tiles ahead
    auto load_index = [&](int jj, int& slot, int& len, int& acc) {
      slot = 0;
      len = 0;
      acc = 0;
      if (jj < n_mine) {
        const int bb = (blockIdx.x + jj * gridDim.x) / (n_slices * p.H_v);
        slot = p.state_indices[bb];
        len = p.seq_lengths[bb];
        acc = p.num_accepted != nullptr ? p.num_accepted[bb] : T;
      }
    };
    int cur_s, cur_L, cur_n, nxt_s, nxt_L, nxt_n;
    load_index(lane, cur_s, cur_L, cur_n);
    load_index(32 + lane, nxt_s, nxt_L, nxt_n);
    // tiles issued: all of them, unless a wait for a free stage fails or (test
    // builds) a tile is held back; from there on nothing is issued or signalled
    int n_issue = n_mine;
    bool failed = false;  // lane 0: a wait for a free stage ran out (then nothing more)
    for (int j = 0; j < n_mine; ++j) {
      if (test_hold_tile(blockIdx.x + j * gridDim.x)) {
        n_issue = j;
        break;
      }
      if (j > 0 && (j & 31) == 0) {
        cur_s = nxt_s;
        cur_L = nxt_L;
        cur_n = nxt_n;
        load_index(j + 32 + lane, nxt_s, nxt_L, nxt_n);
      }
      const int tile = blockIdx.x + j * gridDim.x;
      const int slice = tile % n_slices;
      const int h = (tile / n_slices) % p.H_v;
      const int b = tile / (n_slices * p.H_v);
      const int s = __shfl_sync(0xffffffffu, cur_s, j & 31);
      int L = __shfl_sync(0xffffffffu, cur_L, j & 31);
      L = L < 0 ? 0 : (L > T ? T : L);
      if (s < 0 || s >= p.pool_size) L = 0;
      int n_commit = __shfl_sync(0xffffffffu, cur_n, j & 31);
      n_commit = n_commit < 0 ? 0 : (n_commit > L ? L : n_commit);
      const int stage = tc_stage(j, n_groups, per_group);
      const uint32_t phase = tc_phase(j, n_groups, per_group);
      uint8_t* vb = vec_base + stage * lay.bytes;
      const uint32_t vbar = vec0 + 8 * stage;
      const uint32_t sbar = sta0 + 8 * stage;
      if (lane == 0 && !failed)
        failed = !mbar_wait_free(empty0 + 8 * stage, phase ^ 1, abort_word, kErrProducerWait);
      __syncwarp();
      if (__shfl_sync(0xffffffffu, failed, 0)) {  // the stage may still be in use
        if (n_issue == n_mine) n_issue = j;
        continue;
      }
      if (lane == 0) {
        int* meta = reinterpret_cast<int*>(vb + lay.meta);
        meta[0] = L;
        meta[1] = s;
        meta[2] = n_commit;
        if (L > 0) {
          // the L valid tokens' rows are contiguous in HBM: one copy each
          mbar_expect_tx(vbar, L * (DK * 8 + VS * 2));
          mbar_expect_tx(sbar, kTcStateBytes);
          const size_t qk_off = (static_cast<size_t>(b) * p.H_qk + h / p.group) * T * DK;
          const size_t gk_off = (static_cast<size_t>(b) * p.H_v + h) * T * DK;
          bulk_load(smem_addr(vb + lay.k), p.key + qk_off, L * DK * 2, vbar);
          bulk_load(smem_addr(vb + lay.q), p.query + qk_off, L * DK * 2, vbar);
          bulk_load(smem_addr(vb + lay.gk), p.gk + gk_off, L * DK * 4, vbar);
          const uint16_t* vsrc =
              p.value + (static_cast<size_t>(b) * p.H_v + h) * T * p.D_v + slice * VS;
          if (VS == p.D_v) {
            bulk_load(smem_addr(vb + lay.v), vsrc, L * VS * 2, vbar);
          } else {
            for (int t = 0; t < L; ++t)
              bulk_load(smem_addr(vb + lay.v + t * VS * 2), vsrc + static_cast<size_t>(t) * p.D_v,
                        VS * 2, vbar);
          }
          if constexpr (VK)  // VS rows j of D_k entries
            tma_load_3d(smem_addr(smem + stage * kTcStateBytes), &pool_map, 0,
                        (s * p.H_v + h) * p.D_v + slice * VS, 0, sbar);
          else  // D_k rows i of VS entries
            tma_load_3d(smem_addr(smem + stage * kTcStateBytes), &pool_map, 0,
                        (s * p.H_v + h) * DK, slice * VS / 64, sbar);
        }
        mbar_arrive(sbar);
      }
      // gate scalars: lane t fetches token t's pair; lane 31 the per-head values
      uint32_t* rawv = reinterpret_cast<uint32_t*>(vb + lay.raw);
      if (lane < L) {
        if constexpr (GATED) {
          const size_t ai = (static_cast<size_t>(b) * T + lane) * p.H_v + h;
          cp_async_4(smem_addr(rawv + lane), word_of(p.gate_a + ai));
          cp_async_4(smem_addr(rawv + 8 + lane), word_of(p.gate_b + ai));
        } else {
          const size_t gi = (static_cast<size_t>(b) * p.H_v + h) * T + lane;
          cp_async_4(smem_addr(rawv + lane), p.g + gi);
          cp_async_4(smem_addr(rawv + 8 + lane), word_of(p.beta + gi));
        }
      }
      if constexpr (GATED) {
        if (lane == 31 && L > 0) {
          cp_async_4(smem_addr(rawv + 16), p.dt_bias + h);
          cp_async_4(smem_addr(rawv + 17), p.decay_scale + h);
        }
      }
      cp_async_arrive_noinc(vbar);
    }
    // No copy may outlive the CTA: wait (bounded, not abandonable) for both
    // barriers of the last tile issued into every stage (the last n_stages
    // tiles issued fill each stage once).
    for (int k = (n_issue > n_stages ? n_issue - n_stages : 0); k < n_issue; ++k) {
      const int stg = tc_stage(k, n_groups, per_group);
      const uint32_t ph = tc_phase(k, n_groups, per_group);
      if (!mbar_wait_bounded(vec0 + 8 * stg, ph) || !mbar_wait_bounded(sta0 + 8 * stg, ph)) {
        if (lane == 0) flag_error(kErrDrainWait);
        break;
      }
    }
  } else if (SUMS && warp >= first_sums) {
    // ================================================================ the L x L sums
    bool dead = false;  // a wait failed: this warp signals no tile ready again
    for (int j = warp - first_sums; j < n_mine && !dead; j += n_groups) {
      const int tile = blockIdx.x + j * gridDim.x;
      const int h = (tile / n_slices) % p.H_v;
      const int b = tile / (n_slices * p.H_v);
      const int stage = tc_stage(j, n_groups, per_group);
      const uint8_t* vb = vec_base + stage * lay.bytes;
      const bool landed = mbar_wait_abandonable(vec0 + 8 * stage, tc_phase(j, n_groups, per_group),
                                                abort_word, kErrProducerWait);
      if (!__all_sync(0xffffffffu, landed)) {
        dead = true;
        break;
      }
      int L = reinterpret_cast<const int*>(vb + lay.meta)[0];
      L = L < 0 ? 0 : (L > T ? T : L);
      if (L > 0) {
        float gt = 0.0f;
        if (lane < L) {  // the gate of token `lane` (g only)
          const uint32_t* rawv = reinterpret_cast<const uint32_t*>(vb + lay.raw);
          if constexpr (GATED) {
            const size_t ai = (static_cast<size_t>(b) * T + lane) * p.H_v + h;
            const float dtb = __uint_as_float(rawv[16]);
            const float dsc = __uint_as_float(rawv[17]);
            gt = dsc * softplus_f32(bf16_in_word(rawv[lane], p.gate_a + ai) + dtb);
          } else {
            gt = __uint_as_float(rawv[lane]);
          }
        }
        tc_pair_sums<1>(vb, lay, reinterpret_cast<float*>(const_cast<uint8_t*>(vb) + lay.ab), gt,
                        p.scale, lane);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(ab0 + 8 * stage);
    }
  } else if (warp < first_sums) {
    // ================================================================ consumer groups
    const int group = warp >> 2;
    const int wq = warp & 3;
    const int r = tid - kTcGroupThreads * group;  // row i / column j / TMEM lane
    const bool elected = r == 0;
    const int bar_id = 1 + group;
    uint8_t* gb = grp_base + group * kTcGroupBytes;
    const uint32_t mbar = mma0 + 8 * group;
    const uint32_t lane_field = static_cast<uint32_t>(32 * wq) << 16;
    const uint32_t d2 = tmem_base + kTcVS * group;
    const uint32_t d1 = tmem_base + kTcVS * n_groups + kTcN1 * group;
    // operand descriptors at K step 0 (the state's depends on the stage)
    const uint64_t b1_desc = umma_desc(smem_addr(gb + kTcB1), 128, 2048, kUmmaInterleave);
    const uint64_t e_desc = umma_desc(smem_addr(gb + kTcE), 128, 512, kUmmaInterleave);
    const uint64_t dl_desc = umma_desc(smem_addr(gb + kTcDL), 128, 512, kUmmaInterleave);
    // pass 1: A = S_0^T (M = j), M-major as [pool, H_v, D_k, D_v] stages it,
    // K-major as [pool, H_v, D_v, D_k] does; pass 2: both operands K-major
    constexpr uint32_t idesc1 = umma_idesc_bf16<kTcVS, kTcN1, !VK, true>();
    constexpr uint32_t idesc2 = umma_idesc_bf16<kTcDK, kTcVS, false, false>();
    uint32_t mma_phase = 0;
    int held = -1;  // the stage whose new state is still being stored (elected thread)
    // A wait of the group failed (decided by a vote, so the whole group agrees):
    // from then on it commits no state and frees no stage.
    bool dead = false;

    for (int it = group; it < n_mine; it += n_groups) {
      const int tile = blockIdx.x + it * gridDim.x;
      const int slice = tile % n_slices;
      const int h = (tile / n_slices) % p.H_v;
      const int b = tile / (n_slices * p.H_v);
      const int stage = tc_stage(it, n_groups, per_group);
      const uint32_t phase = tc_phase(it, n_groups, per_group);
      uint8_t* st = smem + stage * kTcStateBytes;
      const uint8_t* vb = vec_base + stage * lay.bytes;

      bool ok_self =
          !dead && mbar_wait_abandonable(vec0 + 8 * stage, phase, abort_word, kErrConsumerWait);
      const int* meta = reinterpret_cast<const int*>(vb + lay.meta);
      // one value per warp (the finalise below shuffles); 0 where a lane's wait failed
      int L = __all_sync(0xffffffffu, ok_self) ? meta[0] : 0;
      L = L < 0 ? 0 : (L > T ? T : L);
      const int s = meta[1];
      if (s < 0 || s >= p.pool_size) L = 0;
      int n_commit = meta[2];
      n_commit = n_commit < 0 ? 0 : (n_commit > L ? L : n_commit);

      // out[b, h, t, slice * VS + j]; padded tokens get +0.0
      const size_t bh = static_cast<size_t>(b) * p.H_v + h;
      uint16_t* out_t0 = p.out + bh * T * p.D_v + slice * VS;
      for (int t = L; t < T; ++t) out_t0[static_cast<size_t>(t) * p.D_v + r] = 0;

      // ---- 1. finalise: row i = r
      float c_row = 0.0f, b_lane = 0.0f;
      if (L > 0) {
        float gt = 0.0f;
        if (lane < L) {  // the gate of token `lane`
          const uint32_t* rawv = reinterpret_cast<const uint32_t*>(vb + lay.raw);
          if constexpr (GATED) {
            const size_t ai = (static_cast<size_t>(b) * T + lane) * p.H_v + h;
            const float dtb = __uint_as_float(rawv[16]);
            const float dsc = __uint_as_float(rawv[17]);
            gt = dsc * softplus_f32(bf16_in_word(rawv[lane], p.gate_a + ai) + dtb);  // g
            b_lane = sigmoid_f32(bf16_in_word(rawv[8 + lane], p.gate_b + ai));      // beta
          } else {
            const size_t gi = (static_cast<size_t>(b) * p.H_v + h) * T + lane;
            gt = __uint_as_float(rawv[lane]);
            b_lane = bf16_in_word(rawv[8 + lane], p.beta + gi);
          }
        }
        // The code a call runs is kept small (instruction fetch is a leading
        // stall here): T = 8 kernels hold two finalise instances that cover
        // every length (L <= 4 and L <= 8; the stage holds 8 rows and the
        // tokens past L are masked) and one L <= 8 solve, single-token
        // kernels the L = 1 code, and only the other token counts take the
        // switch over all eight.
        if constexpr (T8) {
          if (L <= 4)
            c_row = tc_finalize<4, true>(vb, lay, gb, gt, p.scale, r, lane, wq, n_commit, L);
          else
            c_row = tc_finalize<8, true>(vb, lay, gb, gt, p.scale, r, lane, wq, n_commit, L);
        } else if constexpr (SUMS) {  // single-token calls: L = 1
          c_row = tc_finalize<1, false>(vb, lay, gb, gt, p.scale, r, lane, wq, n_commit);
        } else {
          c_row = tc_finalize_any<!SUMS>(L, n_commit, vb, lay, gb, gt, p.scale, r, lane, wq);
        }
        if constexpr (VK) reinterpret_cast<float*>(gb + kTcC)[r] = c_row;
      }
      fence_async_smem();
      if (elected && held >= 0) {  // the previous tile's store has read its stage by now
        bulk_wait_read_all();
        if (!dead) mbar_arrive(empty0 + 8 * held);
        held = -1;
      }
      ok_self = ok_self &&
                mbar_wait_abandonable(sta0 + 8 * stage, phase, abort_word, kErrConsumerWait);
      tc_fence_before();
      // operands and slots written; D1 free. The vote: the tile goes on only if
      // every thread of the group saw both its copies land.
      if (!named_barrier_and(bar_id, kTcGroupThreads, ok_self)) {
        dead = true;
        L = 0;
      }

      // ---- 2. pass 1 on the tensor cores; A and B on the CUDA cores
      if (L > 0) {
        if (wq == 0) {  // warp-uniform: one lane issues
          // M-major: LBO = the next 64 columns j, SBO = the next 8 rows i; K-major:
          // SBO = the next 8 rows j, K steps of 32 bytes inside a 128-byte row
          // and 64 entries i further on in the next [VS][64] block
          const uint64_t st_desc =
              VK ? umma_desc(smem_addr(st), 16, 1024, kUmmaSwizzle128)
                 : umma_desc(smem_addr(st), DK * 128, 1024, kUmmaSwizzle128);
          if (elect_one()) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < DK / 16; ++ks)
              umma_bf16(d1,
                        umma_desc_advance(st_desc, VK ? (ks >> 2) * (VS * 128) + (ks & 3) * 32
                                                      : ks * 2048),
                        umma_desc_advance(b1_desc, ks * 256), idesc1, ks > 0);
            umma_commit(mbar);
          }
          __syncwarp();
        }
        if constexpr (!SUMS) tc_sum_parts(gb, L, r);
      }
      bool sums_ok = true;
      if constexpr (SUMS) {
        // A and B from the sums warp (waited for every tile, so that no later
        // wait on this stage can see a phase two fills old)
        sums_ok = !dead &&
                  mbar_wait_abandonable(ab0 + 8 * stage, phase, abort_word, kErrConsumerWait);
        sums_ok = __all_sync(0xffffffffu, sums_ok);  // one decision per warp (the solve shuffles)
      } else {
        named_barrier(bar_id, kTcGroupThreads);  // A and B ready
      }

      // ---- 3. solve: column j = r
      if (L > 0) {
        if (!mbar_wait_bounded(mbar, mma_phase)) flag_error(kErrConsumerWait);
        mma_phase ^= 1u;
        tc_fence_after();
        uint32_t x[32];
        tmem_ld32(d1 + lane_field, x);
        tmem_wait_ld();
        const float* sa = SUMS ? reinterpret_cast<const float*>(vb + lay.ab)
                               : reinterpret_cast<const float*>(gb + kTcA);
        const float* sb = SUMS ? sa + 64 : reinterpret_cast<const float*>(gb + kTcBm);
        if (sums_ok) {
          if constexpr (T8) {
            tc_solve<8>(x, vb, lay, gb, sa, sb, b_lane, r, out_t0, p.D_v, L);
          } else if constexpr (SUMS) {
            tc_solve<1>(x, vb, lay, gb, sa, sb, b_lane, r, out_t0, p.D_v);
          } else {
            tc_solve_any(L, x, vb, lay, gb, sa, sb, b_lane, r, out_t0, p.D_v);
          }
        }
      }
      fence_async_smem();
      tc_fence_before();
      // delta operand written; D1 reads done. The vote: commit only if every
      // warp of the group had its A and B.
      if (!named_barrier_and(bar_id, kTcGroupThreads, sums_ok)) dead = true;

      // ---- 4. pass 2 and the new state, when any token is committed
      const bool commit = L > 0 && n_commit > 0 && !dead;  // else the slot keeps its bits
      if (commit) {
        if (wq == 0) {
          if (elect_one()) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < kTcK2 / 16; ++ks)
              // [pool, H_v, D_k, D_v]: D2 = E Dl^T (lane = row i); [pool, H_v,
              // D_v, D_k]: D2 = Dl E^T (lane = row j of the k-contiguous tile)
              umma_bf16(d2, umma_desc_advance(VK ? dl_desc : e_desc, ks * 256),
                        umma_desc_advance(VK ? e_desc : dl_desc, ks * 256), idesc2, ks > 0);
            umma_commit(mbar);
          }
          __syncwarp();
        }
        if (!mbar_wait_bounded(mbar, mma_phase)) flag_error(kErrConsumerWait);
        mma_phase ^= 1u;
        tc_fence_after();
        if constexpr (VK)
          tc_new_state_row_vk(st, d2 + lane_field, reinterpret_cast<const float*>(gb + kTcC), r);
        else
          tc_new_state_row(st, d2 + lane_field, c_row, r);
        fence_async_smem();
      }
      tc_fence_before();
      named_barrier(bar_id, kTcGroupThreads);  // new state staged; D2 reads done
      // the store runs while the group finalises its next tile; the stage is
      // released once the store has read it
      if (elected) {
        if (commit) {
          if constexpr (VK)
            tma_store_3d(&pool_map, 0, (s * p.H_v + h) * p.D_v + slice * VS, 0, smem_addr(st));
          else
            tma_store_3d(&pool_map, 0, (s * p.H_v + h) * DK, slice * VS / 64, smem_addr(st));
          bulk_commit_group();
        }
        held = stage;
      }
    }
    if (elected) {
      if (held >= 0) {
        bulk_wait_read_all();
        if (!dead) mbar_arrive(empty0 + 8 * held);
      }
      bulk_wait_all();
    }
  }

  // every warp arrives here: free the tensor memory once no thread can touch it
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTcTmemCols);
  }
}

}  // namespace gdr
