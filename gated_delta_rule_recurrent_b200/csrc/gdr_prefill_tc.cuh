// Prefill: the recurrence of "lite_boost.ops.recurrent_gated_delta_rule"
// (MindSpore Lite API page, section 算法流程, steps 1-4) over long token
// counts, for D_k = 128 and D_v a multiple of 128 on a [pool, H_v, D_k, D_v]
// pool. The page's op is decode-only and sends prefill to a chunk-level op
// (section 注); the result is the same four steps run over every valid
// token, which this kernel computes chunk by chunk.
//
// A tile is one (item, value head, 128-column slice). Its state lives in
// tensor memory as fp32 for the whole sequence (TMEM lane i = state row i,
// 128 columns j), and touches HBM twice: one TMA load of the bf16 slot at the
// start, one TMA store of the rounded state after the last committed token.
// The tokens are taken in chunks of at most kPfChunk = 8, each in the chunked
// form of gdr_decode_chunk_tc.cuh (running products of the decays, so nothing
// overflows or divides; reading P):
//   pass 1  D1 = S^T [u_hi u_lo w_hi w_lo]   (tcgen05, M = 128 columns j,
//           N = 32, K = 128 rows i), with S given as two bf16 tiles, S_hi =
//           bf16(S) and S_lo = bf16(S - S_hi), in the TMA's 128-byte swizzled
//           layout: D1 = S_hi^T [..] + S_lo^T [..], 16 significant bits of S;
//   solve   per column j: kv_mem, delta (unit lower-triangular), o -> out;
//   pass 2  S <- c o S + E Delta^T: the TMEM rows are scaled by c (while
//           pass 1 runs) and pass 2 accumulates into them (tcgen05, M = 128
//           rows i, N = 128, K = 32);
//   then every thread reads its row of S back and writes S_hi and S_lo for
//   the next chunk's pass 1. After the chunk that ends at the committed
//   count n, S_hi is exactly bf16_rne(S_n): the elected thread stores it to
//   the slot with one TMA store (once per call and tile, as the page's
//   state_out; reading D).
// Chunks start at multiples of 8 tokens, and one more boundary sits at n when
// n < L (reading E), so the committed state is the state after token n - 1
// while outputs continue to token L - 1.
//
// CTA: two consumer groups of four warps (thread r of a group = TMEM lane r =
// row i in row-wise steps, column j in column-wise ones) and one producer
// warp per group, one CTA per SM, persistent over tiles; group g takes the
// CTA's tiles g, g + 2, ... The producer of a group loads the slot of each of
// its tiles into the group's S_hi tile and streams the tile's chunks (k, q,
// gk and v rows, gate scalars) through the group's ring of vector stages.
// Both sides derive the chunk schedule from the item's length and committed
// count, read from global memory, so neither depends on data that may not
// have landed.
//
// Waits follow the failure protocol of gdr_ptx.cuh: abandonable waits, a
// per-CTA abort word, votes over the group before a tile goes on, no signal
// after a failure, and a drain of started copies before the CTA exits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr_decode.cuh"
#include "gdr_decode_chunk_tc.cuh"
#include "gdr_ptx.cuh"
#include "gdr_umma.cuh"

namespace gdr {

constexpr int kPfChunk = 8;      // tokens per chunk (the chunked form's L <= 8)
constexpr int kPfGroups = 2;     // consumer groups per CTA
constexpr int kPfStages = 2;     // vector stages per group
constexpr int kPfThreads = kPfGroups * (kTcGroupThreads + 32);  // + a producer warp per group
constexpr int kPfTmemCols = 512;  // S (128 columns) per group at 128 g, D1 (32) at 256 + 32 g

// Shared memory (from a 1024-byte boundary): per group the S_hi and S_lo
// tiles, the group's operand block, its vector stages; then the barriers (per
// group: vector full / empty per stage, state full / empty, MMA done), the
// TMEM address and the abort word.
constexpr int kPfStateOff = 0;                                       // [g][hi, lo] 32 KB each
constexpr int kPfGroupOff = kPfStateOff + kPfGroups * 2 * kTcStateBytes;
constexpr int kPfVecOff = kPfGroupOff + kPfGroups * kTcGroupBytes;
constexpr int kPfBarsPerGroup = 2 * kPfStages + 3;
__host__ __device__ inline int pf_vec_bytes() { return tc_layout(kPfChunk).bytes; }
__host__ __device__ inline int pf_bars_off() {
  return kPfVecOff + kPfGroups * kPfStages * pf_vec_bytes();
}
__host__ __device__ inline int pf_smem_bytes() {
  return 1024 /* alignment slack */ + pf_bars_off() + kPfGroups * kPfBarsPerGroup * 8 + 16;
}

// The item's valid tokens L (0 when its slot is outside the pool) and
// committed count n, clamped as for decode calls.
__device__ __forceinline__ void pf_item(const DecodeParams& p, int b, int& L, int& n, int& s) {
  s = p.state_indices[b];
  L = p.seq_lengths[b];
  L = L < 0 ? 0 : (L > p.T ? p.T : L);
  if (s < 0 || s >= p.pool_size) L = 0;
  n = p.num_accepted != nullptr ? p.num_accepted[b] : L;
  n = n < 0 ? 0 : (n > L ? L : n);
}

// End of the chunk that starts at `pos`: the next multiple of kPfChunk, L, or
// the committed count n when it falls inside.
__device__ __forceinline__ int pf_chunk_end(int pos, int L, int n) {
  int end = pos + kPfChunk - pos % kPfChunk;
  end = end < L ? end : L;
  if (pos < n && n < end) end = n;
  return end;
}

// Row i of the tile in tensor memory from the staged bf16 state: S = c S_0.
__device__ __forceinline__ void pf_state_from_tile(uint32_t s_lane, const uint8_t* s_hi, float c,
                                                   int i) {
#pragma unroll
  for (int k = 0; k < kTcVS / 32; ++k) {
    uint32_t r[32];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 w = *reinterpret_cast<const uint4*>(s_hi + swz_offset<kTcDK>(i, 32 * k + 8 * q));
      const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        r[8 * q + 2 * e] = __float_as_uint(c * bf16_lo(wv[e]));
        r[8 * q + 2 * e + 1] = __float_as_uint(c * bf16_hi(wv[e]));
      }
    }
    tmem_st32(s_lane + 32 * k, r);
  }
  tmem_wait_st();
}

// Row i of the tile in tensor memory scaled by c.
__device__ __forceinline__ void pf_state_scale(uint32_t s_lane, float c) {
#pragma unroll
  for (int k = 0; k < kTcVS / 32; ++k) {
    uint32_t r[32];
    tmem_ld32(s_lane + 32 * k, r);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(c * __uint_as_float(r[e]));
    tmem_st32(s_lane + 32 * k, r);
  }
  tmem_wait_st();
}

// Row i of the tile from tensor memory into the swizzled S_hi (bf16 RNE) and,
// when LO, S_lo (the rounding remainder, bf16) tiles.
template <bool LO>
__device__ __forceinline__ void pf_state_to_tiles(uint32_t s_lane, uint8_t* s_hi, uint8_t* s_lo,
                                                  int i) {
#pragma unroll
  for (int k = 0; k < kTcVS / 32; ++k) {
    uint32_t r[32];
    tmem_ld32(s_lane + 32 * k, r);
    tmem_wait_ld();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float x[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(r[8 * q + e]);
      uint4 hi, lo;
      split_bf16x8(x, hi, lo);
      const int off = swz_offset<kTcDK>(i, 32 * k + 8 * q);
      *reinterpret_cast<uint4*>(s_hi + off) = hi;
      if constexpr (LO) *reinterpret_cast<uint4*>(s_lo + off) = lo;
    }
  }
}

// Row i of the S_lo tile cleared (the slot's bf16 state is exact in S_hi).
__device__ __forceinline__ void pf_zero_row(uint8_t* tile, int i) {
#pragma unroll
  for (int c = 0; c < kTcVS; c += 8)
    *reinterpret_cast<uint4*>(tile + swz_offset<kTcDK>(i, c)) = make_uint4(0u, 0u, 0u, 0u);
}

// Output rows [t_begin, t_end) of one tile's 128 columns set to +0.0, by the
// group's 128 threads (16-byte stores).
__device__ __forceinline__ void pf_zero_out(uint16_t* out_tile, int t_begin, int t_end, int D_v,
                                            int r) {
  for (int e = t_begin * 16 + r; e < t_end * 16; e += kTcGroupThreads) {
    const int t = e >> 4, c = (e & 15) * 8;
    *reinterpret_cast<uint4*>(out_tile + static_cast<size_t>(t) * D_v + c) =
        make_uint4(0u, 0u, 0u, 0u);
  }
}

template <bool GATED>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap pool_map, const DecodeParams p,
                      const int n_tiles) {
  constexpr int DK = kTcDK, VS = kTcVS;
  const int T = p.T;
  const TcLayout lay = tc_layout(kPfChunk);
  const int vec_bytes = lay.bytes;

  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw_base = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + (((raw_base + 1023u) & ~1023u) - raw_base);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + pf_bars_off());
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kPfGroups * kPfBarsPerGroup);
  volatile int* abort_word = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int n_slices = p.D_v / VS;
  const int n_mine = (n_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                     static_cast<int>(gridDim.x);
  // group g: consumer warps 4 g .. 4 g + 3, producer warp 4 kPfGroups + g
  const bool is_producer = warp >= 4 * kPfGroups;
  const int group = is_producer ? warp - 4 * kPfGroups : warp >> 2;
  uint8_t* s_hi = smem + kPfStateOff + group * 2 * kTcStateBytes;
  uint8_t* s_lo = s_hi + kTcStateBytes;
  uint8_t* gb = smem + kPfGroupOff + group * kTcGroupBytes;
  uint8_t* vec_base = smem + kPfVecOff + group * kPfStages * vec_bytes;
  const uint32_t gbar = smem_addr(bars + group * kPfBarsPerGroup);
  const uint32_t vfull0 = gbar;                      // a chunk's rows and scalars landed
  const uint32_t vempty0 = gbar + 8 * kPfStages;     // the group is done with a vector stage
  const uint32_t sfull = gbar + 16 * kPfStages;      // the slot's state landed in S_hi
  const uint32_t sempty = sfull + 8;                 // S_hi is free for the next tile's state
  const uint32_t mbar = sempty + 8;                  // the group's MMAs are done

  if (tid == 0) {
    for (int g = 0; g < kPfGroups; ++g) {
      const uint32_t b0 = smem_addr(bars + g * kPfBarsPerGroup);
      for (int v = 0; v < kPfStages; ++v) {
        mbar_init(b0 + 8 * v, 32);                  // one cp.async arrival per producer lane
        mbar_init(b0 + 8 * kPfStages + 8 * v, 1);   // the group's elected thread
      }
      mbar_init(b0 + 16 * kPfStages, 1);      // the producer's lane 0 (+ the TMA bytes)
      mbar_init(b0 + 16 * kPfStages + 8, 1);  // the group's elected thread
      mbar_init(b0 + 16 * kPfStages + 16, 1); // one MMA commit
    }
    *abort_word = 0;
    fence_mbar_init();
  }
  __syncwarp();
  if (warp == 0) {
    tmem_alloc(smem_addr(tmem_slot), kPfTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (is_producer) {
    // ================================================================ producer of group g
    int rec = 0, fills = 0;  // chunk records and state fills issued
    bool stop = false;
    for (int it = group; it < n_mine && !stop; it += kPfGroups) {
      const int tile = blockIdx.x + it * gridDim.x;
      if (test_hold_tile(tile)) break;
      const int slice = tile % n_slices;
      const int h = (tile / n_slices) % p.H_v;
      const int b = tile / (n_slices * p.H_v);
      int L, n, s;
      pf_item(p, b, L, n, s);
      if (L > 0) {  // the slot's state into S_hi, once S_hi is free
        bool ok = true;
        if (lane == 0)
          ok = mbar_wait_abandonable(sempty, (fills & 1) ^ 1, abort_word, kErrProducerWait);
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        if (lane == 0) {
          mbar_expect_tx(sfull, kTcStateBytes);
          tma_load_3d(smem_addr(s_hi), &pool_map, 0, (s * p.H_v + h) * DK, slice * VS / 64,
                      sfull);
          mbar_arrive(sfull);
        }
        ++fills;
      }
      int pos = 0;
      do {  // one record per chunk; an empty item has one record of no tokens
        const int end = L > 0 ? pf_chunk_end(pos, L, n) : 0;
        const int Lc = end - pos;
        const int stage = rec % kPfStages;
        const uint32_t vbar = vfull0 + 8 * stage;
        uint8_t* vb = vec_base + stage * vec_bytes;
        bool ok = true;
        if (lane == 0)
          ok = mbar_wait_abandonable(vempty0 + 8 * stage, ((rec / kPfStages) & 1) ^ 1, abort_word,
                                     kErrProducerWait);
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          stop = true;
          break;
        }
        if (lane == 0 && Lc > 0) {
          // the chunk's rows are contiguous in HBM: one copy each
          mbar_expect_tx(vbar, Lc * (DK * 8 + VS * 2));
          const size_t qk_off = ((static_cast<size_t>(b) * p.H_qk + h / p.group) * T + pos) * DK;
          const size_t gk_off = ((static_cast<size_t>(b) * p.H_v + h) * T + pos) * DK;
          bulk_load(smem_addr(vb + lay.k), p.key + qk_off, Lc * DK * 2, vbar);
          bulk_load(smem_addr(vb + lay.q), p.query + qk_off, Lc * DK * 2, vbar);
          bulk_load(smem_addr(vb + lay.gk), p.gk + gk_off, Lc * DK * 4, vbar);
          const uint16_t* vsrc =
              p.value + ((static_cast<size_t>(b) * p.H_v + h) * T + pos) * p.D_v + slice * VS;
          if (VS == p.D_v) {
            bulk_load(smem_addr(vb + lay.v), vsrc, Lc * VS * 2, vbar);
          } else {
            for (int t = 0; t < Lc; ++t)
              bulk_load(smem_addr(vb + lay.v + t * VS * 2), vsrc + static_cast<size_t>(t) * p.D_v,
                        VS * 2, vbar);
          }
        }
        // gate scalars: lane t fetches token pos + t's pair; lane 31 the per-head values
        uint32_t* rawv = reinterpret_cast<uint32_t*>(vb + lay.raw);
        if (lane < Lc) {
          if constexpr (GATED) {
            const size_t ai = (static_cast<size_t>(b) * T + pos + lane) * p.H_v + h;
            cp_async_4(smem_addr(rawv + lane), word_of(p.gate_a + ai));
            cp_async_4(smem_addr(rawv + 8 + lane), word_of(p.gate_b + ai));
          } else {
            const size_t gi = (static_cast<size_t>(b) * p.H_v + h) * T + pos + lane;
            cp_async_4(smem_addr(rawv + lane), p.g + gi);
            cp_async_4(smem_addr(rawv + 8 + lane), word_of(p.beta + gi));
          }
        }
        if constexpr (GATED) {
          if (lane == 31 && Lc > 0) {
            cp_async_4(smem_addr(rawv + 16), p.dt_bias + h);
            cp_async_4(smem_addr(rawv + 17), p.decay_scale + h);
          }
        }
        cp_async_arrive_noinc(vbar);
        ++rec;
        pos = end;
      } while (pos < L);
    }
    // No copy may outlive the CTA: wait (bounded, not abandonable) for the last
    // fill of every vector stage and for the last state fill.
    for (int k = (rec > kPfStages ? rec - kPfStages : 0); k < rec; ++k) {
      if (!mbar_wait_bounded(vfull0 + 8 * (k % kPfStages), (k / kPfStages) & 1)) {
        if (lane == 0) flag_error(kErrDrainWait);
        break;
      }
    }
    if (fills > 0 && !mbar_wait_bounded(sfull, (fills - 1) & 1))
      if (lane == 0) flag_error(kErrDrainWait);
  } else {
    // ================================================================ consumer group g
    const int wq = warp & 3;
    const int r = tid - kTcGroupThreads * group;  // row i / column j / TMEM lane
    const bool elected = r == 0;
    const int bar_id = 1 + group;
    const uint32_t lane_field = static_cast<uint32_t>(32 * wq) << 16;
    const uint32_t s_tm = tmem_base + kTcVS * group;  // the state, fp32
    const uint32_t d1 = tmem_base + kTcVS * kPfGroups + kTcN1 * group;
    const uint64_t b1_desc = umma_desc(smem_addr(gb + kTcB1), 128, 2048, kUmmaInterleave);
    const uint64_t e_desc = umma_desc(smem_addr(gb + kTcE), 128, 512, kUmmaInterleave);
    const uint64_t dl_desc = umma_desc(smem_addr(gb + kTcDL), 128, 512, kUmmaInterleave);
    // S tiles M-major: LBO = the next 64 columns j, SBO = the next 8 rows i
    const uint64_t hi_desc = umma_desc(smem_addr(s_hi), DK * 128, 1024, kUmmaSwizzle128);
    const uint64_t lo_desc = umma_desc(smem_addr(s_lo), DK * 128, 1024, kUmmaSwizzle128);
    constexpr uint32_t idesc1 = umma_idesc_bf16<kTcVS, kTcN1, true, true>();
    constexpr uint32_t idesc2 = umma_idesc_bf16<kTcDK, kTcVS, false, false>();
    uint32_t mma_phase = 0;
    int rec = 0, fills = 0;
    bool dead = false;  // a wait of the group failed (by vote): no commit, no signal
    bool storing = false;  // a TMA store may still be reading S_hi (elected thread)

    for (int it = group; it < n_mine; it += kPfGroups) {
      const int tile = blockIdx.x + it * gridDim.x;
      const int slice = tile % n_slices;
      const int h = (tile / n_slices) % p.H_v;
      const int b = tile / (n_slices * p.H_v);
      int L, n, s;
      pf_item(p, b, L, n, s);
      uint16_t* out_tile = p.out + (static_cast<size_t>(b) * p.H_v + h) * T * p.D_v + slice * VS;
      const int fill = fills;
      if (L > 0) ++fills;
      int pos = 0;
      do {
        const int end = L > 0 ? pf_chunk_end(pos, L, n) : 0;
        const int Lc = end - pos;
        const bool first = pos == 0 && L > 0;
        const bool last = end >= L;
        const bool commit_here = n > 0 && end == n;
        const int stage = rec % kPfStages;
        const uint8_t* vb = vec_base + stage * vec_bytes;
        bool ok_self = dead ? false
                            : mbar_wait_abandonable(vfull0 + 8 * stage, (rec / kPfStages) & 1,
                                                    abort_word, kErrConsumerWait);
        int Lw = __all_sync(0xffffffffu, ok_self) ? Lc : 0;  // one value per warp

        // ---- finalise: row i = r (decays, u, w, e, c, partial sums of A and B)
        float c_row = 0.0f, b_lane = 0.0f;
        if (Lw > 0) {
          float gt = 0.0f;
          if (lane < Lw) {
            const uint32_t* rawv = reinterpret_cast<const uint32_t*>(vb + lay.raw);
            if constexpr (GATED) {
              const size_t ai = (static_cast<size_t>(b) * T + pos + lane) * p.H_v + h;
              const float dtb = __uint_as_float(rawv[16]);
              const float dsc = __uint_as_float(rawv[17]);
              gt = dsc * softplus_f32(bf16_in_word(rawv[lane], p.gate_a + ai) + dtb);  // g
              b_lane = sigmoid_f32(bf16_in_word(rawv[8 + lane], p.gate_b + ai));      // beta
            } else {
              const size_t gi = (static_cast<size_t>(b) * p.H_v + h) * T + pos + lane;
              gt = __uint_as_float(rawv[lane]);
              b_lane = bf16_in_word(rawv[8 + lane], p.beta + gi);
            }
          }
          c_row = tc_finalize_any<true>(Lw, Lw, vb, lay, gb, gt, p.scale, r, lane, wq);
        }
        if (first) {
          ok_self = ok_self &&
                    mbar_wait_abandonable(sfull, fill & 1, abort_word, kErrConsumerWait);
          pf_zero_row(s_lo, r);
        }
        fence_async_smem();
        tc_fence_before();
        // operands written; D1 free; the vote: the chunk goes on only if every
        // thread saw its rows (and, first, the slot's state) land
        if (!named_barrier_and(bar_id, kTcGroupThreads, ok_self)) {
          dead = true;
          Lw = 0;
        }

        if (Lw > 0) {
          // ---- pass 1: D1 = S_hi^T B1 + S_lo^T B1
          if (wq == 0) {
            if (elect_one()) {
              tc_fence_after();
#pragma unroll
              for (int ks = 0; ks < DK / 16; ++ks)
                umma_bf16(d1, umma_desc_advance(hi_desc, ks * 2048),
                          umma_desc_advance(b1_desc, ks * 256), idesc1, ks > 0);
#pragma unroll
              for (int ks = 0; ks < DK / 16; ++ks)
                umma_bf16(d1, umma_desc_advance(lo_desc, ks * 2048),
                          umma_desc_advance(b1_desc, ks * 256), idesc1, true);
              umma_commit(mbar);
            }
            __syncwarp();
          }
          // the state in TMEM scaled by c while pass 1 runs (it reads only the tiles)
          tc_fence_after();
          if (first)
            pf_state_from_tile(s_tm + lane_field, s_hi, c_row, r);
          else
            pf_state_scale(s_tm + lane_field, c_row);
          tc_sum_parts(gb, Lw, r);
        }
        tc_fence_before();
        named_barrier(bar_id, kTcGroupThreads);  // A and B summed; the state scaled

        // ---- solve: column j = r; outputs of tokens pos .. end - 1
        if (Lw > 0) {
          if (!mbar_wait_bounded(mbar, mma_phase)) flag_error(kErrConsumerWait);
          mma_phase ^= 1u;
          tc_fence_after();
          uint32_t x[32];
          tmem_ld32(d1 + lane_field, x);
          tmem_wait_ld();
          tc_solve_any(Lw, x, vb, lay, gb, reinterpret_cast<const float*>(gb + kTcA),
                       reinterpret_cast<const float*>(gb + kTcBm), b_lane, r,
                       out_tile + static_cast<size_t>(pos) * p.D_v, p.D_v);
        }
        if (elected && storing && Lw > 0) {  // S_hi is rewritten below
          bulk_wait_read_all();
          storing = false;
        }
        fence_async_smem();
        tc_fence_before();
        named_barrier(bar_id, kTcGroupThreads);  // delta written; D1 and the stage read
        if (elected && !dead) mbar_arrive(vempty0 + 8 * stage);

        // ---- pass 2 into the state, then the state back into S_hi / S_lo
        const bool stage_lo = !last;           // the next chunk's pass 1 reads S_lo
        const bool need_tiles = !last || commit_here;
        if (Lw > 0) {
          if (wq == 0) {
            if (elect_one()) {
              tc_fence_after();
#pragma unroll
              for (int ks = 0; ks < kTcK2 / 16; ++ks)
                umma_bf16(s_tm, umma_desc_advance(e_desc, ks * 256),
                          umma_desc_advance(dl_desc, ks * 256), idesc2, true);
              umma_commit(mbar);
            }
            __syncwarp();
          }
          if (!mbar_wait_bounded(mbar, mma_phase)) flag_error(kErrConsumerWait);
          mma_phase ^= 1u;
          tc_fence_after();
          if (need_tiles) {
            if (stage_lo)
              pf_state_to_tiles<true>(s_tm + lane_field, s_hi, s_lo, r);
            else
              pf_state_to_tiles<false>(s_tm + lane_field, s_hi, s_lo, r);
          }
          fence_async_smem();
        }
        tc_fence_before();
        named_barrier(bar_id, kTcGroupThreads);  // new state staged; TMEM reads done
        if (elected && Lw > 0 && commit_here) {
          tma_store_3d(&pool_map, 0, (s * p.H_v + h) * DK, slice * VS / 64, smem_addr(s_hi));
          bulk_commit_group();
          storing = true;
        }
        if (last) {
          // padded tokens (and every token of an empty or skipped item): +0.0
          pf_zero_out(out_tile, L, T, p.D_v, r);
          if (L > 0 && elected) {  // S_hi is free once the store has read it
            if (storing) {
              bulk_wait_read_all();
              storing = false;
            }
            if (!dead) mbar_arrive(sempty);
          }
        }
        ++rec;
        pos = end;
      } while (pos < L);
    }
    if (elected) bulk_wait_all();
  }

  // every warp arrives here: free the tensor memory once no thread can touch it
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kPfTmemCols);
  }
}

}  // namespace gdr
