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
//   pass 2  S <- c o S + E Delta^T: the TMEM rows already hold c o S, and
//           pass 2 accumulates into them (tcgen05, M = 128 rows i, N = 128,
//           K = 32);
//   then every thread reads its row of S back and writes S_hi and S_lo for
//   the next chunk's pass 1, and writes the row back to tensor memory scaled
//   by the next chunk's c. After the chunk that ends at the committed count
//   n, S_hi is exactly bf16_rne(S_n): the elected thread stores it to the
//   slot with one TMA store (once per call and tile, as the page's
//   state_out; reading D).
// The consumer loop runs one record behind: the iteration that waits for and
// finalises chunk k (whose operands depend on the inputs only) then reads
// back the state chunk k - 1 left, scaling it by chunk k's c on the way, so
// one group barrier serves both. Chunks run with L = 8 code throughout (a
// shorter chunk masks the missing tokens), so the finalise and solve are
// compiled once.
// Chunks start at multiples of 8 tokens, and one more boundary sits at n when
// n < L (reading E), so the committed state is the state after token n - 1
// while outputs continue to token L - 1.
//
// CTA: two consumer groups of four warps (thread r of a group = TMEM lane r =
// row i in row-wise steps, column j in column-wise ones) and one producer
// warp per group, one CTA per SM, persistent over tiles; group g takes the
// CTA's tiles g, g + 2, ... The producer of a group streams each tile's
// chunks (k, q, gk and v rows, gate scalars) through the group's ring of
// vector stages, and loads the tile's slot into the group's S_hi tile right
// after its first chunk (the group frees S_hi of its previous tile only once
// it has that chunk).
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

// One tile's coordinates: item b, value head h, column slice, the item's
// slot s, valid tokens L, committed count n, and its output block.
struct PfTile {
  int b, h, slice, s, L, n;
  uint16_t* out;
};
__device__ __forceinline__ PfTile pf_tile(const DecodeParams& p, int tile, int n_slices) {
  PfTile t;
  t.slice = tile % n_slices;
  t.h = (tile / n_slices) % p.H_v;
  t.b = tile / (n_slices * p.H_v);
  pf_item(p, t.b, t.L, t.n, t.s);
  t.out = p.out + (static_cast<size_t>(t.b) * p.H_v + t.h) * p.T * p.D_v + t.slice * kTcVS;
  return t;
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

// Row i of the tile from tensor memory into the swizzled S_hi (bf16 RNE) and,
// when LO, S_lo (the rounding remainder, bf16) tiles; when SCALE, the row is
// written back to tensor memory multiplied by c (the next chunk's decay).
template <bool LO, bool SCALE>
__device__ __forceinline__ void pf_state_to_tiles(uint32_t s_lane, uint8_t* s_hi, uint8_t* s_lo,
                                                  int i, float c) {
  const unsigned long long cc = pk(c, c);
  const unsigned long long neg1 = pk(-1.0f, -1.0f);
#pragma unroll
  for (int k = 0; k < kTcVS / 32; ++k) {
    uint32_t r[32];
    tmem_ld32(s_lane + 32 * k, r);
    tmem_wait_ld();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = __uint_as_float(r[8 * q + 2 * e]);
        const float x1 = __uint_as_float(r[8 * q + 2 * e + 1]);
        hw[e] = pack_bf16x2(x0, x1);  // bf16 round to nearest even
        if constexpr (LO) {
          // the remainder x - bf16(x), exact in fp32, rounded to bf16
          const float2 rem = upk(fma2(pk(bf16_lo(hw[e]), bf16_hi(hw[e])), neg1, pk(x0, x1)));
          lw[e] = pack_bf16x2(rem.x, rem.y);
        }
      }
      const int off = swz_offset<kTcDK>(i, 32 * k + 8 * q);
      *reinterpret_cast<uint4*>(s_hi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      if constexpr (LO)
        *reinterpret_cast<uint4*>(s_lo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    if constexpr (SCALE) {
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const float2 v = upk(mul2(cc, pk(__uint_as_float(r[e]), __uint_as_float(r[e + 1]))));
        r[e] = __float_as_uint(v.x);
        r[e + 1] = __float_as_uint(v.y);
      }
      tmem_st32(s_lane + 32 * k, r);
    }
  }
  if constexpr (SCALE) tmem_wait_st();
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
        if (pos == 0 && L > 0) {
          // the slot's state into S_hi once S_hi is free: after the tile's first
          // record, which the group waits for before it frees S_hi of its
          // previous tile
          bool ok_s = true;
          if (lane == 0)
            ok_s = mbar_wait_abandonable(sempty, (fills & 1) ^ 1, abort_word, kErrProducerWait);
          if (!__shfl_sync(0xffffffffu, ok_s, 0)) {
            stop = true;
            break;
          }
          if (lane == 0) {
            mbar_expect_tx(sfull, kTcStateBytes);
            tma_load_3d(smem_addr(s_hi), &pool_map, 0, (s * p.H_v + h) * DK, slice * VS / 64,
                        sfull);
            mbar_arrive(sfull);
          }
          ++fills;
        }
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

    // Records are taken one behind: the iteration that prepares record k (waits
    // for its rows, finalises them) first reads back the state that record
    // k - 1 left in tensor memory into S_hi / S_lo, and, when k continues the
    // same tile, writes it back to tensor memory already scaled by k's decay c.
    // A tile's commit and wrap-up follow that read-back. One loop iteration
    // per record plus one to finish the last; the finalise and solve code sit
    // in the loop once.
    int it = group;  // the tile of the record being prepared
    int pos = 0;
    PfTile cur{}, prev{};
    if (it < n_mine) cur = pf_tile(p, blockIdx.x + it * gridDim.x, n_slices);
    int fill = 0;
    if (it < n_mine && cur.L > 0) ++fills;
    bool have_prev = false, prev_last = false, prev_commit = false;
    int prev_Lw = 0;
    // Pass 2 of the previous record is issued without a wait: this thread
    // waits for it before the next finalise writes the e operand that pass 2
    // reads (or, with no finalise, before the state is read back), so the
    // MMA runs under the finalise's first part.
    bool pending = false;
    auto wait_pass2 = [&]() {
      if (pending) {
        if (!mbar_wait_bounded(mbar, mma_phase)) flag_error(kErrConsumerWait);
        mma_phase ^= 1u;
        pending = false;
      }
    };
    while (it < n_mine || have_prev) {
      const bool has_cur = it < n_mine;
      int end = 0;
      bool first = false, last = false, commit_here = false;
      if (has_cur) {
        end = cur.L > 0 ? pf_chunk_end(pos, cur.L, cur.n) : 0;
        first = pos == 0 && cur.L > 0;
        last = end >= cur.L;
        commit_here = cur.n > 0 && end == cur.n;
      }
      const int stage = rec % kPfStages;
      const uint8_t* vb = vec_base + stage * vec_bytes;

      // ---- this record's rows: wait, then finalise row i = r (decays, u, w,
      // e, c, partial sums of A and B)
      bool ok_self = true;
      int Lw = 0;
      float c_row = 0.0f, b_lane = 0.0f;
      if (has_cur) {
        ok_self = dead ? false
                       : mbar_wait_abandonable(vfull0 + 8 * stage, (rec / kPfStages) & 1,
                                               abort_word, kErrConsumerWait);
        Lw = __all_sync(0xffffffffu, ok_self) ? end - pos : 0;  // one value per warp
        if (Lw > 0) {
          float gt = 0.0f;
          if (lane < Lw) {
            const uint32_t* rawv = reinterpret_cast<const uint32_t*>(vb + lay.raw);
            if constexpr (GATED) {
              const size_t ai = (static_cast<size_t>(cur.b) * T + pos + lane) * p.H_v + cur.h;
              const float dtb = __uint_as_float(rawv[16]);
              const float dsc = __uint_as_float(rawv[17]);
              gt = dsc * softplus_f32(bf16_in_word(rawv[lane], p.gate_a + ai) + dtb);  // g
              b_lane = sigmoid_f32(bf16_in_word(rawv[8 + lane], p.gate_b + ai));      // beta
            } else {
              const size_t gi = (static_cast<size_t>(cur.b) * p.H_v + cur.h) * T + pos + lane;
              gt = __uint_as_float(rawv[lane]);
              b_lane = bf16_in_word(rawv[8 + lane], p.beta + gi);
            }
          }
          c_row = tc_finalize<kPfChunk, true>(vb, lay, gb, gt, p.scale, r, lane, wq, Lw, Lw,
                                              wait_pass2);
        }
        if (first) pf_zero_row(s_lo, r);  // the slot's bf16 state is exact in S_hi
      }

      // ---- the previous record's state back into the tiles (and, within a
      // tile, into tensor memory scaled by this record's c)
      wait_pass2();
      if (have_prev && prev_Lw > 0) {
        tc_fence_after();
        if (!prev_last)
          pf_state_to_tiles<true, true>(s_tm + lane_field, s_hi, s_lo, r, c_row);
        else if (prev_commit)
          pf_state_to_tiles<false, false>(s_tm + lane_field, s_hi, s_lo, r, 0.0f);
      }
      fence_async_smem();
      tc_fence_before();
      // operands and state tiles written, TMEM reads done; the vote: this
      // record goes on only if every thread saw its rows land
      if (!named_barrier_and(bar_id, kTcGroupThreads, ok_self)) {
        dead = true;
        Lw = 0;
      }

      // ---- the previous record's commit, and the wrap-up of its tile
      if (have_prev) {
        if (elected && prev_Lw > 0 && prev_commit) {
          tma_store_3d(&pool_map, 0, (prev.s * p.H_v + prev.h) * DK, prev.slice * VS / 64,
                       smem_addr(s_hi));
          bulk_commit_group();
          storing = true;
        }
        if (prev_last) {
          // padded tokens (and every token of an empty or skipped item): +0.0
          pf_zero_out(prev.out, prev.L, T, p.D_v, r);
          if (prev.L > 0 && elected) {  // S_hi is free once the store has read it
            if (storing) {
              bulk_wait_read_all();
              storing = false;
            }
            if (!dead) mbar_arrive(sempty);
          }
        }
      }
      if (!has_cur) break;
      if (first) {  // the slot's state landed in S_hi, by vote
        const bool ok_state =
            !dead && mbar_wait_abandonable(sfull, fill & 1, abort_word, kErrConsumerWait);
        if (!named_barrier_and(bar_id, kTcGroupThreads, ok_state)) {
          dead = true;
          Lw = 0;
        }
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
        // a tile's first record: the state into TMEM as c S_0 while pass 1 runs
        // (it reads only the tiles); later records find it scaled already
        if (first) {
          tc_fence_after();
          pf_state_from_tile(s_tm + lane_field, s_hi, c_row, r);
        }
        tc_sum_parts(gb, Lw, r);
      }
      tc_fence_before();
      named_barrier(bar_id, kTcGroupThreads);  // A and B summed; the state in TMEM

      // ---- solve: column j = r; outputs of tokens pos .. end - 1
      if (Lw > 0) {
        if (!mbar_wait_bounded(mbar, mma_phase)) flag_error(kErrConsumerWait);
        mma_phase ^= 1u;
        tc_fence_after();
        uint32_t x[32];
        tmem_ld32(d1 + lane_field, x);
        tmem_wait_ld();
        tc_solve<kPfChunk>(x, vb, lay, gb, reinterpret_cast<const float*>(gb + kTcA),
                           reinterpret_cast<const float*>(gb + kTcBm), b_lane, r,
                           cur.out + static_cast<size_t>(pos) * p.D_v, p.D_v, Lw);
      }
      if (elected && storing && Lw > 0) {  // S_hi is rewritten by the next read-back
        bulk_wait_read_all();
        storing = false;
      }
      fence_async_smem();
      tc_fence_before();
      named_barrier(bar_id, kTcGroupThreads);  // delta written; D1 and the stage read
      if (elected && !dead) mbar_arrive(vempty0 + 8 * stage);

      // ---- pass 2 into the state
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
        pending = true;
      }

      have_prev = true;
      prev_Lw = Lw;
      prev_last = last;
      prev_commit = commit_here;
      prev = cur;
      ++rec;
      pos = end;
      if (pos >= cur.L) {  // the tile's last record: on to the group's next tile
        it += kPfGroups;
        pos = 0;
        if (it < n_mine) {
          cur = pf_tile(p, blockIdx.x + it * gridDim.x, n_slices);
          fill = fills;
          if (cur.L > 0) ++fills;
        }
      }
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
