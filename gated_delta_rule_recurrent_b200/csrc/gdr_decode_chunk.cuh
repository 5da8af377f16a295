// Multi-token decode kernel (T >= 2) for sm_100a: all L tokens of an item in
// one pass over the state.
//
// Arithmetic: the four steps of "lite_boost.ops.recurrent_gated_delta_rule"
// (MindSpore Lite API page, section 算法流程), applied to tokens t = 0..L-1 of
// one (item, value head), and, when GATED, the gate of
// "com.microsoft.LinearAttentionGate" (README, section Description).
//
// Write d_t = exp(g_t + gk_t) (a D_k vector), D_t = diag(d_t), q^_t = q_t *
// scale, and for s <= t the decay products P_t = D_0 ... D_t and
// P_{s->t} = D_{s+1} ... D_t (the identity when s = t). Unrolling the
// recurrence S_t = D_t S_{t-1} + k_t delta_t^T from the loaded state S_0:
//
//   S_t            = P_t S_0 + sum_{s<=t} P_{s->t} k_s delta_s^T
//   kv_mem_t       = (D_t S_{t-1})^T k_t = S_0^T u_t + sum_{s<t} A_ts delta_s
//   o_t            = S_t^T q^_t          = S_0^T w_t + sum_{s<=t} B_ts delta_s
//   delta_t        = beta_t (v_t - kv_mem_t)
//
// with u_t = P_t k_t, w_t = P_t q^_t, A_ts = k_s . (P_{s->t} k_t) and
// B_ts = k_s . (P_{s->t} q^_t). The new state is S_L = c o S_0 + sum_s e_s
// delta_s^T with c = P_{L-1} (per row) and e_s = P_{s->L-1} k_s. These are the
// same sums as the token-by-token recurrence, regrouped; only the rounding
// order differs. The products P_{s->t} are built by running multiplication
// (never by division), so no intermediate can overflow when the decays are
// small.
//
// A tile is one (item b, value head h, VS-column slice) of the state. Each CTA
// walks tiles blockIdx.x, + gridDim.x, ... through a ring of shared-memory
// stages:
//
//   producer warp - starts the copies of a tile (one TMA box for the state,
//           128-byte swizzled; one 1-D bulk copy each for the k, q and gk
//           rows of the valid tokens, which are contiguous in HBM, and for
//           the value rows; 4-byte cp.async copies of the gate scalars). Its
//           lanes read the slots and lengths of the next 32 tiles ahead.
//   finaliser warps - take every tile in tile order once its copies have
//           landed; each turns its share of the D_k rows (one per lane) into
//           d, u, w, e and c and its partial sums of A and B (a warp
//           reduce-scatter into its own slot); they meet on a named barrier,
//           add the partial sums in a fixed warp order (deterministic) and
//           mark the tile ready.
//   consumer groups - a group of VS / 32 warps takes every NG-th tile; warp
//           w of the group owns columns [32 w, 32 w + 32) of the tile.
//           1. Pass 1: lane (row group rg = lane / 8, column lane cl = lane %
//              8) reads 4 columns of the row quads 4 m + rg of the bf16 state
//              and forms the column sums S_0^T u_t and S_0^T w_t with packed
//              fp32 pairs over (even row, odd row), at most four tokens per
//              sweep; a reduce-scatter over the row groups leaves each lane
//              the sums of one column.
//           2. Each lane solves the unit lower-triangular system for delta
//              in its column and writes o; four shuffles per token hand every
//              lane the deltas of its 4 columns.
//           3. Pass 2 reads the state again and writes S_L to the slot with
//              8-byte stores.
//
// No step waits on another token's reduction, so the latency of a tile is one
// pass of sums, an L x L solve and one pass of updates whatever L is.
//
// Every mbarrier wait is bounded; a wait that runs out sets a bit in the
// device error word and the kernel carries on with the same control flow.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr_decode.cuh"
#include "gdr_ptx.cuh"

namespace gdr {

constexpr int kChunkWarpCols = 32;      // columns per consumer warp: 8 lanes x 4
constexpr int kChunkFinalizers = 2;     // warps that turn landed tiles into row vectors
#ifndef GDR_CHUNK_MAX_THREADS
#define GDR_CHUNK_MAX_THREADS 352
#endif
// Block size cap: consumer groups, the finalisers and the producer. It also
// caps the registers ptxas may give a thread (up to 384 threads: 168; 480:
// 128). Two consumer groups with 168 registers run faster than three with
// 128: with fewer registers the shared-memory loads cannot run ahead of
// their uses.
constexpr int kChunkMaxThreads = GDR_CHUNK_MAX_THREADS;
#ifndef GDR_CHUNK_SWEEP_TOKENS
#define GDR_CHUNK_SWEEP_TOKENS 4
#endif
constexpr int kChunkMaxSubTokens = GDR_CHUNK_SWEEP_TOKENS;  // tokens per pass-1 sweep

// Rows of the state per consumer thread in the k-contiguous layout (VK): the
// per-row vectors a thread reads are shared by its rows.
#ifndef GDR_VK_ROWS
#define GDR_VK_ROWS 2
#endif
#ifndef GDR_VK_SWEEP_TOKENS
#define GDR_VK_SWEEP_TOKENS 4
#endif
constexpr int kVkRowsPerThread = GDR_VK_ROWS;
constexpr int kVkSweepTokens = GDR_VK_SWEEP_TOKENS;

// VK: the pool is [pool, H_v, D_v, D_k] (k contiguous) and the tile is VS
// rows j (value columns) x D_k; otherwise [pool, H_v, D_k, D_v] and the tile
// is D_k rows x VS columns.
template <int DK, int VS, bool VK = false>
struct ChunkShape {
  static constexpr int kWarpsPerTile = VK ? VS / (32 * kVkRowsPerThread) : VS / kChunkWarpCols;
  static constexpr int kStateBytes = DK * VS * 2;
  static_assert(DK == 64 || DK == 128, "D_k must be 64 or 128");
  static_assert(VS == 64 || VS == 128, "64- or 128-column tiles");
  static_assert(kWarpsPerTile >= 1 && kWarpsPerTile * (VK ? 32 * kVkRowsPerThread : 32) == VS,
                "a tile must be covered by whole consumer warps");
};

// Shared memory: n_stages state tiles (DK x VS bf16, 128-byte swizzled, each
// 1024-byte aligned for the swizzle), then n_stages vector blocks, then four
// mbarriers per stage. Offsets below are within one vector block, for T
// padded tokens. Per-row vectors are fp32 [T][DK] (token-major), so four
// consecutive rows of one token are one 16-byte read.
struct ChunkLayout {
  int v, k, q, e, u, w, c, part, a, bm, beta, raw, meta, bytes;
};

template <int DK, int VS>
__host__ __device__ inline ChunkLayout chunk_layout(int T) {
  ChunkLayout s;
  s.v = 0;                               // bf16 [T][VS]  value rows of the slice
  s.k = s.v + T * VS * 2;                // bf16 [T][DK]  key rows
  s.q = s.k + T * DK * 2;                // bf16 [T][DK]  query rows
  s.e = s.q + T * DK * 2;                // fp32 [T][DK]  e_s
  s.u = s.e + T * DK * 4;                // fp32 [T][DK]  gk rows as loaded, then u_t
  s.w = s.u + T * DK * 4;                // fp32 [T][DK]  w_t
  s.c = s.w + T * DK * 4;                // fp32 [DK]     c
  s.part = s.c + DK * 4;                 // fp32 [finalisers][8][8] partial sums of A and B
  s.a = s.part + kChunkFinalizers * 256; // fp32 [8][8]   A_ts at [t][s], s < t
  s.bm = s.a + 256;                      // fp32 [8][8]   B_ts at [t][s], s <= t
  s.beta = s.bm + 256;                   // fp32 [8]
  s.raw = s.beta + 32;                   // u32 [8] g or a words, [8] beta or b words, dt_bias, decay_scale
  s.meta = s.raw + 80;                   // int32 [4]      length, slot, committed tokens
  s.bytes = (s.meta + 16 + 15) & ~15;
  return s;
}

// Four mbarriers per stage: vectors landed, state landed, tile finalised
// (in tile order), stage released.
constexpr int kChunkBarriers = 4;
template <int DK, int VS>
__host__ __device__ inline int chunk_stage_bytes(int T) {
  return ChunkShape<DK, VS>::kStateBytes + chunk_layout<DK, VS>(T).bytes;
}
template <int DK, int VS>
__host__ __device__ inline int chunk_smem_bytes(int T, int n_stages) {
  return 1024 /* alignment slack */ + n_stages * chunk_stage_bytes<DK, VS>(T) +
         kChunkBarriers * n_stages * 8 + 16 /* the abort word (gdr_ptx.cuh) */;
}

// In-register butterfly reduce-scatter of N values (N a power of two) over the
// 32 lanes of a warp. On return lane holds n = max(N / 32, 1) totals in
// v[0 .. n), the totals of entries base + [0, n) with base from
// reduce_scatter_base<N>(lane). For N < 32 the same total sits in 32 / N
// lanes; the one with reduce_scatter_writer<N>(lane) stores it.
template <int N, int BIT>
__device__ __forceinline__ void reduce_scatter_level(float (&v)[N], int lane) {
  constexpr int n = N >> (BIT == 16 ? 0 : BIT == 8 ? 1 : BIT == 4 ? 2 : BIT == 2 ? 3 : 4);
  if constexpr (n >= 2) {
    constexpr int H = n / 2;
    const bool up = (lane & BIT) != 0;
#pragma unroll
    for (int i = 0; i < H; ++i) {
      const float send = up ? v[i] : v[i + H];
      const float keep = up ? v[i + H] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, BIT);
    }
  } else {
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], BIT);
  }
}

template <int N>
__device__ __forceinline__ void reduce_scatter(float (&v)[N], int lane) {
  reduce_scatter_level<N, 16>(v, lane);
  reduce_scatter_level<N, 8>(v, lane);
  reduce_scatter_level<N, 4>(v, lane);
  reduce_scatter_level<N, 2>(v, lane);
  reduce_scatter_level<N, 1>(v, lane);
}

template <int N>
__device__ __forceinline__ int reduce_scatter_base(int lane) {
  int base = 0, n = N;
#pragma unroll
  for (int bit = 16; bit >= 1; bit >>= 1) {
    if (n >= 2) {
      n >>= 1;
      if (lane & bit) base += n;
    }
  }
  return base;
}

template <int N>
__device__ __forceinline__ bool reduce_scatter_writer(int lane) {
  return N >= 32 ? true : (lane & (32 / N - 1)) == 0;
}

constexpr int pow2_at_least(int x) {
  int n = 1;
  while (n < x) n <<= 1;
  return n;
}

// bf16 state words of rows (i, i + 1), 4 columns each, as packed fp32 pairs
// over the two rows: x[c] = {S[i][c0 + c], S[i + 1][c0 + c]}.
__device__ __forceinline__ void row_pair_columns(const uint2 a, const uint2 b,
                                                 unsigned long long (&x)[4]) {
  x[0] = pk(bf16_lo(a.x), bf16_lo(b.x));
  x[1] = pk(bf16_hi(a.x), bf16_hi(b.x));
  x[2] = pk(bf16_lo(a.y), bf16_lo(b.y));
  x[3] = pk(bf16_hi(a.y), bf16_hi(b.y));
}

// Byte offsets, in a swizzled state tile, of columns [c0, c0 + 4) of rows
// 4 rg + r (r < 4). Rows 16 m + 4 rg + r sit 16 m * 128 bytes further on: the
// swizzle depends only on the row modulo 8, which does not change with m.
template <int DK>
__device__ __forceinline__ void quad_offsets(int rg, int c0, int (&off)[4]) {
#pragma unroll
  for (int r = 0; r < 4; ++r) off[r] = swz_offset<DK>(4 * rg + r, c0) + (c0 & 7) * 2;
}
constexpr int kQuadStep = 16 * 128;  // bytes from row quad m to m + 1 of a row group

// Which of a lane's 4 columns it solves for, by row group: the reduce-scatter
// first splits the columns by row-group bit 0, then by bit 1.
__device__ __forceinline__ int solved_column(int rg) { return 2 * (rg & 1) + (rg >> 1); }
// The row group that solves column j of a lane's 4 (the inverse map).
__device__ __forceinline__ int solver_group(int j) { return (j & 1) * 2 + (j >> 1); }

// ---------------------------------------------------------------- finalise

// Row vectors and this warp's partial sums of A and B for a tile with L = LC
// tokens, in the stage's vector block `vb`. Finaliser warp fw of NF takes rows
// fw * 32 + lane + 32 * NF * r; the gate value g_t sits in lane t (t < LC).
// The partial sums go to this warp's own [8][8] slot (entry (r, col):
// B_{t=r, s=col} for col <= r, A_{t=col, s=r} for col > r); chunk_sum_parts
// adds the slots in warp order.
template <int DK, int NF, int LC>
__device__ __forceinline__ void chunk_finalize(uint8_t* vb, const ChunkLayout& lay, float g_lane,
                                               float scale, int lane, int fw, int n) {
  constexpr int NM = pow2_at_least(LC * LC);  // partial sums, padded for the reduce-scatter
  float g[LC];
#pragma unroll
  for (int t = 0; t < LC; ++t) g[t] = __shfl_sync(0xffffffffu, g_lane, t);
  const uint16_t* sk = reinterpret_cast<const uint16_t*>(vb + lay.k);  // [T][DK]
  const uint16_t* sq = reinterpret_cast<const uint16_t*>(vb + lay.q);
  float* su = reinterpret_cast<float*>(vb + lay.u);
  float* sw = reinterpret_cast<float*>(vb + lay.w);
  float* se = reinterpret_cast<float*>(vb + lay.e);
  float* sc = reinterpret_cast<float*>(vb + lay.c);
  // mp[s * LC + t] (s < t) holds A_ts, mp[t * LC + s] (s <= t) holds B_ts
  float mp[NM];
#pragma unroll
  for (int j = 0; j < NM; ++j) mp[j] = 0.0f;
#pragma unroll 1
  for (int i = fw * 32 + lane; i < DK; i += 32 * NF) {
    float d[LC], kf[LC], qf[LC];
#pragma unroll
    for (int t = 0; t < LC; ++t) {
      d[t] = expf(g[t] + su[t * DK + i]);  // exp(g) * exp(gk) as one exponential
      kf[t] = bf16_bits_to_f32(sk[t * DK + i]);
      qf[t] = bf16_bits_to_f32(sq[t * DK + i]) * scale;
    }
    // The committed state is the one after token n - 1 (n = L unless the
    // call commits fewer tokens): c = P_{n-1}, e_s = P_{s->n-1} k_s for s < n
    // and 0 for s >= n.
    float P = 1.0f, c = 0.0f;
#pragma unroll
    for (int t = 0; t < LC; ++t) {
      P = t == 0 ? d[0] : P * d[t];
      su[t * DK + i] = P * kf[t];  // u_t over the gk entry just read
      sw[t * DK + i] = P * qf[t];
      if (t == n - 1) c = P;
    }
    sc[i] = c;
#pragma unroll
    for (int s = 0; s < LC; ++s) {
      float z = kf[s];  // P_{s->t} k_s by running products
      float e = s == n - 1 ? z : 0.0f;
      mp[s * LC + s] = fmaf(z, qf[s], mp[s * LC + s]);
#pragma unroll
      for (int t = s + 1; t < LC; ++t) {
        z *= d[t];
        mp[s * LC + t] = fmaf(z, kf[t], mp[s * LC + t]);
        mp[t * LC + s] = fmaf(z, qf[t], mp[t * LC + s]);
        if (t == n - 1) e = z;
      }
      se[s * DK + i] = e;
    }
  }
  reduce_scatter<NM>(mp, lane);
  constexpr int NL = NM >= 32 ? NM / 32 : 1;
  if (reduce_scatter_writer<NM>(lane)) {
    const int base = reduce_scatter_base<NM>(lane);
    float* part = reinterpret_cast<float*>(vb + lay.part) + fw * 64;
#pragma unroll
    for (int j = 0; j < NL; ++j) {
      const int f = base + j;
      if (f < LC * LC) part[(f / LC) * 8 + f % LC] = mp[j];
    }
  }
}

// A and B from the finalisers' partial sums, in warp order: warp fw of NF
// sums the entries [fw * 64 / NF, (fw + 1) * 64 / NF) of the [8][8] grid.
template <int NF>
__device__ __forceinline__ void chunk_sum_parts(uint8_t* vb, const ChunkLayout& lay, int L,
                                                int lane, int fw) {
  constexpr int PER = 64 / NF;
  if (lane < PER) {
    const int f = fw * PER + lane;
    const int r = f >> 3, col = f & 7;
    if (r < L && col < L) {
      const float* part = reinterpret_cast<const float*>(vb + lay.part);
      float x = part[f];
#pragma unroll
      for (int w = 1; w < NF; ++w) x += part[w * 64 + f];
      if (col > r) reinterpret_cast<float*>(vb + lay.a)[col * 8 + r] = x;  // A_{t = col, s = r}
      else reinterpret_cast<float*>(vb + lay.bm)[f] = x;                   // B_{t = r, s = col}
    }
  }
}

template <int DK, int NF>
__device__ __forceinline__ void chunk_finalize_any(int L, int n, uint8_t* vb,
                                                   const ChunkLayout& lay, float g_lane,
                                                   float scale, int lane, int fw) {
  switch (L) {
    case 1: chunk_finalize<DK, NF, 1>(vb, lay, g_lane, scale, lane, fw, n); break;
    case 2: chunk_finalize<DK, NF, 2>(vb, lay, g_lane, scale, lane, fw, n); break;
    case 3: chunk_finalize<DK, NF, 3>(vb, lay, g_lane, scale, lane, fw, n); break;
    case 4: chunk_finalize<DK, NF, 4>(vb, lay, g_lane, scale, lane, fw, n); break;
    case 5: chunk_finalize<DK, NF, 5>(vb, lay, g_lane, scale, lane, fw, n); break;
    case 6: chunk_finalize<DK, NF, 6>(vb, lay, g_lane, scale, lane, fw, n); break;
    case 7: chunk_finalize<DK, NF, 7>(vb, lay, g_lane, scale, lane, fw, n); break;
    case 8: chunk_finalize<DK, NF, 8>(vb, lay, g_lane, scale, lane, fw, n); break;
    default: break;
  }
}

// ---------------------------------------------------------------- consumers

// Pass-1 sweep over tokens [T0, T0 + LS) of a tile: the column sums
// S_0^T u_t and S_0^T w_t of this lane's solved column into ms[t], ps[t].
template <int DK, int LC, int T0, int LS>
__device__ __forceinline__ void chunk_sums(const uint8_t* st, const float* su, const float* sw,
                                           int c0, int rg, int lane, float (&ms)[LC],
                                           float (&ps)[LC]) {
  unsigned long long acc[2 * LS][4];
#pragma unroll
  for (int v = 0; v < 2 * LS; ++v)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[v][c] = 0ull;  // (+0.0f, +0.0f)
  int off[4];
  quad_offsets<DK>(rg, c0, off);
  const float* su_m = su + T0 * DK + 4 * rg;
  const float* sw_m = sw + T0 * DK + 4 * rg;
  const uint8_t* st_m = st;
#pragma unroll 1
  for (int m = 0; m < DK / 16; ++m, st_m += kQuadStep, su_m += 16, sw_m += 16) {
    unsigned long long x0[4], x1[4];
    row_pair_columns(*reinterpret_cast<const uint2*>(st_m + off[0]),
                     *reinterpret_cast<const uint2*>(st_m + off[1]), x0);
    row_pair_columns(*reinterpret_cast<const uint2*>(st_m + off[2]),
                     *reinterpret_cast<const uint2*>(st_m + off[3]), x1);
#pragma unroll
    for (int t = 0; t < LS; ++t) {
      const ulonglong2 uq = *reinterpret_cast<const ulonglong2*>(su_m + t * DK);
      const ulonglong2 wq = *reinterpret_cast<const ulonglong2*>(sw_m + t * DK);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        acc[t][c] = fma2(x0[c], uq.x, acc[t][c]);
        acc[LS + t][c] = fma2(x0[c], wq.x, acc[LS + t][c]);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        acc[t][c] = fma2(x1[c], uq.y, acc[t][c]);
        acc[LS + t][c] = fma2(x1[c], wq.y, acc[LS + t][c]);
      }
    }
  }
  // fold (even row, odd row), then reduce-scatter over the row groups: lane
  // bit 3 keeps columns {2, 3} or {0, 1}, lane bit 4 one of those two
  const bool b0 = (lane >> 3) & 1, b1 = (lane >> 4) & 1;
#pragma unroll
  for (int v = 0; v < 2 * LS; ++v) {
    float y[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float2 a = upk(acc[v][c]);
      y[c] = a.x + a.y;
    }
    float z[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float send = b0 ? y[j] : y[j + 2];
      const float keep = b0 ? y[j + 2] : y[j];
      z[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    const float send = b1 ? z[0] : z[1];
    const float keep = b1 ? z[1] : z[0];
    const float f = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    if (v < LS) ms[T0 + v] = f;
    else ps[T0 + v - LS] = f;
  }
}

// One tile with L = LC tokens, for one consumer warp (columns [c0, c0 + 4)
// of the tile in this lane): state tile `st`, vector block `vb`. `dst` points
// at row 0, column c0 of the slot's slice; `out_t0` at token 0, column 0 of
// the tile's output.
template <int DK, int VS, int LC>
__device__ __forceinline__ void chunk_consume(const uint8_t* st, const uint8_t* vb,
                                              const ChunkLayout& lay, int c0, int rg, int lane,
                                              uint16_t* dst, uint16_t* out_t0, int D_v,
                                              bool commit) {
  const float* su = reinterpret_cast<const float*>(vb + lay.u);
  const float* sw = reinterpret_cast<const float*>(vb + lay.w);
  const float* se = reinterpret_cast<const float*>(vb + lay.e);
  const float* sc = reinterpret_cast<const float*>(vb + lay.c);

  // ---- pass 1: column sums, at most four tokens per sweep of the state
  float ms[LC], ps[LC];
  chunk_sums<DK, LC, 0, (LC < kChunkMaxSubTokens ? LC : kChunkMaxSubTokens)>(st, su, sw, c0, rg,
                                                                            lane, ms, ps);
  if constexpr (LC > kChunkMaxSubTokens)
    chunk_sums<DK, LC, kChunkMaxSubTokens, LC - kChunkMaxSubTokens>(st, su, sw, c0, rg, lane, ms,
                                                                   ps);

  // ---- delta (unit lower-triangular solve) and o, for the solved column
  const int col = c0 + solved_column(rg);
  const float* sa = reinterpret_cast<const float*>(vb + lay.a);
  const float* sb = reinterpret_cast<const float*>(vb + lay.bm);
  const uint16_t* sv = reinterpret_cast<const uint16_t*>(vb + lay.v);
  const float* sbeta = reinterpret_cast<const float*>(vb + lay.beta);
  float dl[LC];
#pragma unroll
  for (int t = 0; t < LC; ++t) {
    float kv = ms[t];  // kv_mem_t = S_0^T u_t + sum_{s<t} A_ts delta_s
#pragma unroll
    for (int s = 0; s < t; ++s) kv = fmaf(sa[t * 8 + s], dl[s], kv);
    dl[t] = (bf16_bits_to_f32(sv[t * VS + col]) - kv) * sbeta[t];  // step 3
    float o = ps[t];  // o_t = S_0^T w_t + sum_{s<=t} B_ts delta_s (step 4)
#pragma unroll
    for (int s = 0; s <= t; ++s) o = fmaf(sb[t * 8 + s], dl[s], o);
    out_t0[static_cast<size_t>(t) * D_v + col] = f32_to_bf16_bits(o);
  }
  // every lane gathers the deltas of its 4 columns: {delta_s[c], delta_s[c]}
  const int cl = lane & 7;
  unsigned long long dd[LC][4];
#pragma unroll
  for (int s = 0; s < LC; ++s)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float x = __shfl_sync(0xffffffffu, dl[s], solver_group(j) * 8 + cl);
      dd[s][j] = pk(x, x);
    }

  // ---- pass 2: S_L = c o S_0 + sum_s e_s delta_s^T, bf16 once, to the slot
  if (!commit) return;
  int off[4];
  quad_offsets<DK>(rg, c0, off);
  const uint8_t* st_m = st;
  const float* sc_m = sc + 4 * rg;
  const float* se_m = se + 4 * rg;
  uint16_t* d0 = dst + static_cast<size_t>(4 * rg) * D_v;
  const size_t d_step = static_cast<size_t>(16) * D_v;
#pragma unroll 1
  for (int m = 0; m < DK / 16; ++m, st_m += kQuadStep, sc_m += 16, se_m += 16, d0 += d_step) {
    unsigned long long n0[4], n1[4];
    row_pair_columns(*reinterpret_cast<const uint2*>(st_m + off[0]),
                     *reinterpret_cast<const uint2*>(st_m + off[1]), n0);
    row_pair_columns(*reinterpret_cast<const uint2*>(st_m + off[2]),
                     *reinterpret_cast<const uint2*>(st_m + off[3]), n1);
    const ulonglong2 cq = *reinterpret_cast<const ulonglong2*>(sc_m);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      n0[c] = mul2(n0[c], cq.x);
      n1[c] = mul2(n1[c], cq.y);
    }
#pragma unroll
    for (int s = 0; s < LC; ++s) {
      const ulonglong2 eq = *reinterpret_cast<const ulonglong2*>(se_m + s * DK);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        n0[c] = fma2(eq.x, dd[s][c], n0[c]);
        n1[c] = fma2(eq.y, dd[s][c], n1[c]);
      }
    }
    float2 a[4], b[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      a[c] = upk(n0[c]);
      b[c] = upk(n1[c]);
    }
    __stcs(reinterpret_cast<uint2*>(d0),
           make_uint2(pack_bf16x2(a[0].x, a[1].x), pack_bf16x2(a[2].x, a[3].x)));
    __stcs(reinterpret_cast<uint2*>(d0 + D_v),
           make_uint2(pack_bf16x2(a[0].y, a[1].y), pack_bf16x2(a[2].y, a[3].y)));
    __stcs(reinterpret_cast<uint2*>(d0 + 2 * D_v),
           make_uint2(pack_bf16x2(b[0].x, b[1].x), pack_bf16x2(b[2].x, b[3].x)));
    __stcs(reinterpret_cast<uint2*>(d0 + 3 * D_v),
           make_uint2(pack_bf16x2(b[0].y, b[1].y), pack_bf16x2(b[2].y, b[3].y)));
  }
}

// ---------------------------------------------------------------- consumers, k-contiguous pool

// One tile with L = LC tokens in the VK layout: the staged tile holds VS rows
// j (value columns of the state) of D_k entries each, as [D_k / 64][VS][64]
// with the 128-byte swizzle. Thread `tj` of the group owns rows tj + r * VS /
// kVkRowsPerThread; its column sums over i, its solve and its update need no
// other thread. `dst` points at row 0 of the slot's slice; `out_t0` at token
// 0, column 0 of the tile's output.
template <int DK, int VS, int LC>
__device__ __forceinline__ void chunk_consume_vk(const uint8_t* st, const uint8_t* vb,
                                                 const ChunkLayout& lay, int tj, uint16_t* dst,
                                                 uint16_t* out_t0, int D_v, bool commit) {
  constexpr int R = kVkRowsPerThread;
  constexpr int RS = VS / R;  // row stride between a thread's rows
  const float* su = reinterpret_cast<const float*>(vb + lay.u);
  const float* sw = reinterpret_cast<const float*>(vb + lay.w);
  const float* se = reinterpret_cast<const float*>(vb + lay.e);
  const float* sc = reinterpret_cast<const float*>(vb + lay.c);
  // byte offset of (row tj + r RS, columns [8 c8, 8 c8 + 8)) is off[r] + c8-term:
  // the chunk index within a 128-byte segment is c8 % 8, swizzled by row % 8
  auto chunk = [&](int r, int c8) -> uint4 {
    const int j = tj + r * RS;
    return *reinterpret_cast<const uint4*>(st + swz_offset<VS>(j, 8 * c8));
  };
  // ---- pass 1: m_t = S_0^T u_t and p_t = S_0^T w_t for this thread's rows,
  // packed fp32 pairs over (i, i + 1), two accumulators per vector
  float ms[R][LC], ps[R][LC];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int t = 0; t < LC; ++t) ms[r][t] = ps[r][t] = 0.0f;
  constexpr int SW = LC < kVkSweepTokens ? LC : kVkSweepTokens;
#pragma unroll
  for (int t0 = 0; t0 < LC; t0 += SW) {  // sweeps of at most SW tokens
    unsigned long long acc[R][2 * SW][2];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int v = 0; v < 2 * SW; ++v) acc[r][v][0] = acc[r][v][1] = 0ull;
#pragma unroll 1
    for (int c8 = 0; c8 < DK / 8; ++c8) {
      unsigned long long x[R][4];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint4 w = chunk(r, c8);
        x[r][0] = pk(bf16_lo(w.x), bf16_hi(w.x));
        x[r][1] = pk(bf16_lo(w.y), bf16_hi(w.y));
        x[r][2] = pk(bf16_lo(w.z), bf16_hi(w.z));
        x[r][3] = pk(bf16_lo(w.w), bf16_hi(w.w));
      }
#pragma unroll
      for (int tt = 0; tt < SW; ++tt) {
        if (t0 + tt < LC) {
          const ulonglong2 u01 = *reinterpret_cast<const ulonglong2*>(su + (t0 + tt) * DK + 8 * c8);
          const ulonglong2 u23 =
              *reinterpret_cast<const ulonglong2*>(su + (t0 + tt) * DK + 8 * c8 + 4);
          const ulonglong2 w01 = *reinterpret_cast<const ulonglong2*>(sw + (t0 + tt) * DK + 8 * c8);
          const ulonglong2 w23 =
              *reinterpret_cast<const ulonglong2*>(sw + (t0 + tt) * DK + 8 * c8 + 4);
#pragma unroll
          for (int r = 0; r < R; ++r) {
            acc[r][tt][0] = fma2(x[r][0], u01.x, acc[r][tt][0]);
            acc[r][tt][1] = fma2(x[r][1], u01.y, acc[r][tt][1]);
            acc[r][tt][0] = fma2(x[r][2], u23.x, acc[r][tt][0]);
            acc[r][tt][1] = fma2(x[r][3], u23.y, acc[r][tt][1]);
            acc[r][SW + tt][0] = fma2(x[r][0], w01.x, acc[r][SW + tt][0]);
            acc[r][SW + tt][1] = fma2(x[r][1], w01.y, acc[r][SW + tt][1]);
            acc[r][SW + tt][0] = fma2(x[r][2], w23.x, acc[r][SW + tt][0]);
            acc[r][SW + tt][1] = fma2(x[r][3], w23.y, acc[r][SW + tt][1]);
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int tt = 0; tt < SW; ++tt) {
        if (t0 + tt < LC) {
          const float2 a0 = upk(acc[r][tt][0]), a1 = upk(acc[r][tt][1]);
          const float2 b0 = upk(acc[r][SW + tt][0]), b1 = upk(acc[r][SW + tt][1]);
          ms[r][t0 + tt] = (a0.x + a0.y) + (a1.x + a1.y);
          ps[r][t0 + tt] = (b0.x + b0.y) + (b1.x + b1.y);
        }
      }
  }

  // ---- delta (unit lower-triangular solve) and o, per row
  const float* sa = reinterpret_cast<const float*>(vb + lay.a);
  const float* sb = reinterpret_cast<const float*>(vb + lay.bm);
  const uint16_t* sv = reinterpret_cast<const uint16_t*>(vb + lay.v);
  const float* sbeta = reinterpret_cast<const float*>(vb + lay.beta);
  unsigned long long dd[R][LC];  // {delta_s[j], delta_s[j]}
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int j = tj + r * RS;
    float dl[LC];
#pragma unroll
    for (int t = 0; t < LC; ++t) {
      float kv = ms[r][t];  // kv_mem_t = S_0^T u_t + sum_{s<t} A_ts delta_s
#pragma unroll
      for (int s = 0; s < t; ++s) kv = fmaf(sa[t * 8 + s], dl[s], kv);
      dl[t] = (bf16_bits_to_f32(sv[t * VS + j]) - kv) * sbeta[t];  // step 3
      float o = ps[r][t];  // o_t = S_0^T w_t + sum_{s<=t} B_ts delta_s (step 4)
#pragma unroll
      for (int s = 0; s <= t; ++s) o = fmaf(sb[t * 8 + s], dl[s], o);
      out_t0[static_cast<size_t>(t) * D_v + j] = f32_to_bf16_bits(o);
      dd[r][t] = pk(dl[t], dl[t]);
    }
  }

  // ---- pass 2: S_L = c o S_0 + sum_s e_s delta_s^T, bf16 once, to the slot
  if (!commit) return;
#pragma unroll 1
  for (int c8 = 0; c8 < DK / 8; ++c8) {
    const ulonglong2 c01 = *reinterpret_cast<const ulonglong2*>(sc + 8 * c8);
    const ulonglong2 c23 = *reinterpret_cast<const ulonglong2*>(sc + 8 * c8 + 4);
    unsigned long long n[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const uint4 w = chunk(r, c8);
      n[r][0] = mul2(pk(bf16_lo(w.x), bf16_hi(w.x)), c01.x);
      n[r][1] = mul2(pk(bf16_lo(w.y), bf16_hi(w.y)), c01.y);
      n[r][2] = mul2(pk(bf16_lo(w.z), bf16_hi(w.z)), c23.x);
      n[r][3] = mul2(pk(bf16_lo(w.w), bf16_hi(w.w)), c23.y);
    }
#pragma unroll
    for (int s = 0; s < LC; ++s) {
      const ulonglong2 e01 = *reinterpret_cast<const ulonglong2*>(se + s * DK + 8 * c8);
      const ulonglong2 e23 = *reinterpret_cast<const ulonglong2*>(se + s * DK + 8 * c8 + 4);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        n[r][0] = fma2(e01.x, dd[r][s], n[r][0]);
        n[r][1] = fma2(e01.y, dd[r][s], n[r][1]);
        n[r][2] = fma2(e23.x, dd[r][s], n[r][2]);
        n[r][3] = fma2(e23.y, dd[r][s], n[r][3]);
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float2 a = upk(n[r][0]), b = upk(n[r][1]), c = upk(n[r][2]), d = upk(n[r][3]);
      __stcs(reinterpret_cast<uint4*>(dst + static_cast<size_t>(tj + r * RS) * DK + 8 * c8),
             make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(b.x, b.y), pack_bf16x2(c.x, c.y),
                        pack_bf16x2(d.x, d.y)));
    }
  }
}

template <int DK, int VS>
__device__ __forceinline__ void chunk_consume_vk_any(int L, const uint8_t* st, const uint8_t* vb,
                                                     const ChunkLayout& lay, int tj,
                                                     uint16_t* dst, uint16_t* out_t0, int D_v,
                                                     bool commit) {
  switch (L) {
    case 1: chunk_consume_vk<DK, VS, 1>(st, vb, lay, tj, dst, out_t0, D_v, commit); break;
    case 2: chunk_consume_vk<DK, VS, 2>(st, vb, lay, tj, dst, out_t0, D_v, commit); break;
    case 3: chunk_consume_vk<DK, VS, 3>(st, vb, lay, tj, dst, out_t0, D_v, commit); break;
    case 4: chunk_consume_vk<DK, VS, 4>(st, vb, lay, tj, dst, out_t0, D_v, commit); break;
    case 5: chunk_consume_vk<DK, VS, 5>(st, vb, lay, tj, dst, out_t0, D_v, commit); break;
    case 6: chunk_consume_vk<DK, VS, 6>(st, vb, lay, tj, dst, out_t0, D_v, commit); break;
    case 7: chunk_consume_vk<DK, VS, 7>(st, vb, lay, tj, dst, out_t0, D_v, commit); break;
    case 8: chunk_consume_vk<DK, VS, 8>(st, vb, lay, tj, dst, out_t0, D_v, commit); break;
    default: break;
  }
}

template <int DK, int VS>
__device__ __forceinline__ void chunk_consume_any(int L, const uint8_t* st, const uint8_t* vb,
                                                  const ChunkLayout& lay, int c0, int rg, int lane,
                                                  uint16_t* dst, uint16_t* out_t0, int D_v,
                                                  bool commit) {
  switch (L) {
    case 1: chunk_consume<DK, VS, 1>(st, vb, lay, c0, rg, lane, dst, out_t0, D_v, commit); break;
    case 2: chunk_consume<DK, VS, 2>(st, vb, lay, c0, rg, lane, dst, out_t0, D_v, commit); break;
    case 3: chunk_consume<DK, VS, 3>(st, vb, lay, c0, rg, lane, dst, out_t0, D_v, commit); break;
    case 4: chunk_consume<DK, VS, 4>(st, vb, lay, c0, rg, lane, dst, out_t0, D_v, commit); break;
    case 5: chunk_consume<DK, VS, 5>(st, vb, lay, c0, rg, lane, dst, out_t0, D_v, commit); break;
    case 6: chunk_consume<DK, VS, 6>(st, vb, lay, c0, rg, lane, dst, out_t0, D_v, commit); break;
    case 7: chunk_consume<DK, VS, 7>(st, vb, lay, c0, rg, lane, dst, out_t0, D_v, commit); break;
    case 8: chunk_consume<DK, VS, 8>(st, vb, lay, c0, rg, lane, dst, out_t0, D_v, commit); break;
    default: break;
  }
}

// ---------------------------------------------------------------- the kernel

// Block: NG groups of VS / 32 consumer warps, then kChunkFinalizers finaliser
// warps, then the producer warp; NG = (blockDim.x / 32 - 1 - kChunkFinalizers)
// / (VS / 32). Requires n_stages >= NG + 1: tiles are finalised in tile order,
// so a group never waits on a stage two phases ahead of it.
template <int DK, int VS, bool GATED, bool VK>
__global__ void __launch_bounds__(kChunkMaxThreads, 1)
    decode_chunk_kernel(const __grid_constant__ CUtensorMap pool_map, const DecodeParams p,
                        const int n_tiles, const int n_stages) {
  using Shape = ChunkShape<DK, VS, VK>;
  constexpr int CWT = Shape::kWarpsPerTile;
  constexpr int NF = kChunkFinalizers;
  const int T = p.T;
  const ChunkLayout lay = chunk_layout<DK, VS>(T);

  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw_base = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + (((raw_base + 1023u) & ~1023u) - raw_base);
  uint8_t* vec_base = smem + n_stages * Shape::kStateBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(vec_base + n_stages * lay.bytes);
  const uint32_t vec0 = smem_addr(bars);        // k, q, gk rows and gate scalars landed
  const uint32_t sta0 = vec0 + 8 * n_stages;    // state tile landed
  const uint32_t full0 = sta0 + 8 * n_stages;   // tile finalised (in tile order)
  const uint32_t empty0 = full0 + 8 * n_stages; // the group is done with the stage
  volatile int* abort_word = reinterpret_cast<volatile int*>(bars + 4 * n_stages);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int producer = static_cast<int>(blockDim.x >> 5) - 1;
  const int first_finalizer = producer - NF;
  const int n_groups = first_finalizer / CWT;
  const int n_slices = p.D_v / VS;
  const int n_mine = (n_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                     static_cast<int>(gridDim.x);

  if (tid == 0) {
    for (int i = 0; i < n_stages; ++i) {
      mbar_init(vec0 + 8 * i, 32);     // one cp.async arrival per producer lane
      mbar_init(sta0 + 8 * i, 1);      // the producer's lane 0 (+ the TMA bytes)
      mbar_init(full0 + 8 * i, NF);    // one arrival per finaliser warp
      mbar_init(empty0 + 8 * i, CWT);  // one arrival per warp of the group
    }
    *abort_word = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp >= first_finalizer && warp < producer) {
    // ================================================================ finalisers
    // Every tile in tile order: wait for its vectors (not for the state),
    // compute the gate and this warp's rows of u, w, e, c and partial sums of
    // A and B, and mark the tile finalised.
    // A finaliser that saw a wait fail signals no tile ready again, but keeps
    // meeting the other finaliser on the named barrier every tile.
    const int fw = warp - first_finalizer;
    bool dead = false;
    for (int j = 0; j < n_mine; ++j) {
      const int tile = blockIdx.x + j * gridDim.x;
      const int h = (tile / n_slices) % p.H_v;
      const int b = tile / (n_slices * p.H_v);
      const int stage = j % n_stages;
      uint8_t* vb = vec_base + stage * lay.bytes;
      const bool landed = !dead && mbar_wait_abandonable(vec0 + 8 * stage, (j / n_stages) & 1,
                                                         abort_word, kErrProducerWait);
      dead = !__all_sync(0xffffffffu, landed);
      int L = dead ? 0 : reinterpret_cast<const int*>(vb + lay.meta)[0];
      L = L < 0 ? 0 : (L > T ? T : L);
      const int n_commit = reinterpret_cast<const int*>(vb + lay.meta)[2];
      if (L > 0) {
        float gt = 0.0f;
        if (lane < L) {  // the gate of token `lane`
          const uint32_t* rawv = reinterpret_cast<const uint32_t*>(vb + lay.raw);
          float bt;
          if constexpr (GATED) {
            const size_t ai = (static_cast<size_t>(b) * T + lane) * p.H_v + h;
            const float dtb = __uint_as_float(rawv[16]);
            const float dsc = __uint_as_float(rawv[17]);
            gt = dsc * softplus_f32(bf16_in_word(rawv[lane], p.gate_a + ai) + dtb);  // g
            bt = sigmoid_f32(bf16_in_word(rawv[8 + lane], p.gate_b + ai));          // beta
          } else {
            const size_t gi = (static_cast<size_t>(b) * p.H_v + h) * T + lane;
            gt = __uint_as_float(rawv[lane]);
            bt = bf16_in_word(rawv[8 + lane], p.beta + gi);
          }
          if (fw == 0) reinterpret_cast<float*>(vb + lay.beta)[lane] = bt;
        }
        chunk_finalize_any<DK, NF>(L, n_commit, vb, lay, gt, p.scale, lane, fw);
      }
      named_barrier(1, 32 * NF);  // every finaliser takes the same path: no early exits
      if (L > 0) chunk_sum_parts<NF>(vb, lay, L, lane, fw);
      __syncwarp();
      if (lane == 0 && !dead) mbar_arrive(full0 + 8 * stage);
    }
    return;
  }

  if (warp == producer) {
    // ================================================================ producer
    // lane i holds the slot, length and committed count of tile (j & ~31) + i;
    // the next 32 tiles' are loaded 32 tiles ahead (no committed-count array:
    // every token is committed)
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
      const int stage = j % n_stages;
      const uint32_t phase = (j / n_stages) & 1;
      uint8_t* vb = vec_base + stage * lay.bytes;
      const uint32_t vbar = vec0 + 8 * stage;
      const uint32_t sbar = sta0 + 8 * stage;
      bool free_ok = true;
      if (lane == 0)
        free_ok = mbar_wait_abandonable(empty0 + 8 * stage, phase ^ 1, abort_word,
                                        kErrProducerWait);
      if (!__shfl_sync(0xffffffffu, free_ok, 0)) {
        n_issue = j;
        break;
      }
      if (lane == 0) {
        int* meta = reinterpret_cast<int*>(vb + lay.meta);
        meta[0] = L;
        meta[1] = s;
        meta[2] = n_commit;
        if (L > 0) {
          // the L valid tokens' rows are contiguous in HBM: one copy each
          mbar_expect_tx(vbar, L * (DK * 8 + VS * 2));
          mbar_expect_tx(sbar, Shape::kStateBytes);
          const size_t qk_off = (static_cast<size_t>(b) * p.H_qk + h / p.group) * T * DK;
          const size_t gk_off = (static_cast<size_t>(b) * p.H_v + h) * T * DK;
          bulk_load(smem_addr(vb + lay.k), p.key + qk_off, L * DK * 2, vbar);
          bulk_load(smem_addr(vb + lay.q), p.query + qk_off, L * DK * 2, vbar);
          bulk_load(smem_addr(vb + lay.u), p.gk + gk_off, L * DK * 4, vbar);
          const uint16_t* vsrc =
              p.value + (static_cast<size_t>(b) * p.H_v + h) * T * p.D_v + slice * VS;
          if (VS == p.D_v) {
            bulk_load(smem_addr(vb + lay.v), vsrc, L * VS * 2, vbar);
          } else {
            for (int t = 0; t < L; ++t)
              bulk_load(smem_addr(vb + lay.v + t * VS * 2), vsrc + static_cast<size_t>(t) * p.D_v,
                        VS * 2, vbar);
          }
          if constexpr (VK)  // VS rows of D_k entries
            tma_load_3d(smem_addr(smem + stage * Shape::kStateBytes), &pool_map, 0,
                        (s * p.H_v + h) * p.D_v + slice * VS, 0, sbar);
          else  // D_k rows of VS entries
            tma_load_3d(smem_addr(smem + stage * Shape::kStateBytes), &pool_map, 0,
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
    // barriers of the last tile issued into every stage.
    for (int k = (n_issue > n_stages ? n_issue - n_stages : 0); k < n_issue; ++k) {
      const uint32_t ph = (k / n_stages) & 1;
      if (!mbar_wait_bounded(vec0 + 8 * (k % n_stages), ph) ||
          !mbar_wait_bounded(sta0 + 8 * (k % n_stages), ph)) {
        if (lane == 0) flag_error(kErrDrainWait);
        break;
      }
    }
    return;
  }

  // ================================================================ consumers
  const int group = warp / CWT;
  if (group >= n_groups) return;  // (no such warps with the launch shapes used)
  const int gw = warp % CWT;
  const int rg = lane >> 3;
  const int c0 = gw * kChunkWarpCols + (lane & 7) * 4;  // first tile column of this lane
  const int col = c0 + solved_column(rg);               // the column this lane solves
  const int tj = gw * 32 + lane;                        // VK: first row of this thread
  bool dead = false;  // a wait of this warp failed: it commits and frees nothing more
  for (int it = group; it < n_mine; it += n_groups) {
    const int tile = blockIdx.x + it * gridDim.x;
    const int slice = tile % n_slices;
    const int h = (tile / n_slices) % p.H_v;
    const int b = tile / (n_slices * p.H_v);
    const int stage = it % n_stages;
    const uint32_t phase = (it / n_stages) & 1;
    const uint8_t* st = smem + stage * Shape::kStateBytes;
    const uint8_t* vb = vec_base + stage * lay.bytes;

    // finalised (in tile order), then the state tile itself: it was issued
    // before the tile was finalised, so its barrier is at this tile's phase
    bool ok_self =
        !dead && mbar_wait_abandonable(full0 + 8 * stage, phase, abort_word, kErrConsumerWait);
    ok_self = ok_self &&
              mbar_wait_abandonable(sta0 + 8 * stage, phase, abort_word, kErrConsumerWait);
    const bool ok = __all_sync(0xffffffffu, ok_self);
    dead = !ok;
    const int* meta = reinterpret_cast<const int*>(vb + lay.meta);
    int L = ok ? meta[0] : 0;
    L = L < 0 ? 0 : (L > T ? T : L);
    const int s = meta[1];
    if (s < 0 || s >= p.pool_size) L = 0;
    const bool commit = ok && meta[2] > 0;  // else the slot keeps its bits (pass 2 is skipped)

    // out[b, h, t, slice * VS + column]; padded tokens get +0.0
    const size_t bh = static_cast<size_t>(b) * p.H_v + h;
    uint16_t* out_t0 = p.out + bh * T * p.D_v + slice * VS;
    if constexpr (VK) {
#pragma unroll
      for (int r = 0; r < kVkRowsPerThread; ++r)
        for (int t = L; t < T; ++t)
          out_t0[static_cast<size_t>(t) * p.D_v + tj + r * (VS / kVkRowsPerThread)] = 0;
    } else {
      for (int t = L; t < T; ++t) out_t0[static_cast<size_t>(t) * p.D_v + col] = 0;
    }

    if (L > 0) {
      if constexpr (VK) {
        uint16_t* dst =
            p.state_pool + ((static_cast<size_t>(s) * p.H_v + h) * p.D_v + slice * VS) * DK;
        chunk_consume_vk_any<DK, VS>(L, st, vb, lay, tj, dst, out_t0, p.D_v, commit);
      } else {
        uint16_t* dst = p.state_pool + (static_cast<size_t>(s) * p.H_v + h) * DK * p.D_v +
                        slice * VS + c0;
        chunk_consume_any<DK, VS>(L, st, vb, lay, c0, rg, lane, dst, out_t0, p.D_v, commit);
      }
    }
    __syncwarp();
    if (lane == 0 && !dead) mbar_arrive(empty0 + 8 * stage);
  }
}

}  // namespace gdr
