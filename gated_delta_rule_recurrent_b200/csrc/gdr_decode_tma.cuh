// Persistent, warp-specialised single-token decode kernel for sm_100a (calls
// with T = 1, the common decode step; calls with T > 1 go to the kernel in
// gdr_decode_chunk.cuh).
//
// Arithmetic: the four steps of "lite_boost.ops.recurrent_gated_delta_rule"
// (MindSpore Lite API page, section 算法流程) and, when GATED, the gate of
// "com.microsoft.LinearAttentionGate" (README, section Description).
//
// A tile is one (item b, value head h, VS-column slice of D_v) block of the
// state: all D_k rows x VS bf16 columns of slot ssm_state_indices[b]; with
// VS = D_v it is the slot's whole contiguous head state. Each CTA walks tiles
// tile = blockIdx.x, + gridDim.x, ... through a ring of shared-memory stages,
// with two roles:
//
//   producer warp - starts the asynchronous copies of a tile (one TMA box for
//           the state, 128-byte swizzled; 1-D bulk copies of the value row
//           and of the k, q and gk rows; 4-byte cp.async copies of the gate
//           scalars) and, kLookahead tiles later, once they have landed
//           ("raw" barrier), turns them into what the consumers use: per row
//           the float4 {d k, d q*scale, d, k} with d = exp(g + gk), in owner
//           order, and per token k.(q*scale) and beta ("full" barrier). No
//           lane waits on global-memory latency.
//   consumer warps - each owns ALL D_k rows of a band of columns; lane (row
//           lane, column lane) holds R rows x 8 columns. Every reduction over
//           D_k is a warp shuffle, so consumer warps never synchronise with
//           each other and drift apart freely. The decay is folded into the
//           row vectors: kv_mem = S^T (d k) and p = S^T (d q*scale) in one
//           read of the bf16 rows; a reduce-scatter over the row lanes; delta;
//           o = p + delta * (k.q*scale), which is step 4's S_new^T (q*scale)
//           with the sums reordered; then a second read of the rows gives
//           S_new = d S + k delta^T, rounded to bf16 once and stored straight
//           to the slot with 16-byte streaming stores. A warp gives the stage
//           back ("empty" barrier) when it has read what it needs.
//
// HBM sees one bulk read and one write of every touched state tile, and a
// stage is held only while its tile is loaded and computed.
//
// Every mbarrier wait is bounded (a clock budget of a few seconds). A wait
// that runs out sets a bit in a device-global error word and the kernel goes
// on with the same control flow, so it always terminates; the host reads the
// word with gdr_device_error().
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr_decode.cuh"
#include "gdr_ptx.cuh"

namespace gdr {

// Tuning constants (compile-time; the defaults are the measured best).
#ifndef GDR_LOOKAHEAD
#define GDR_LOOKAHEAD 1
#endif
// The producer finalises tile j - kLookahead after starting the copies of tile j.
constexpr int kLookahead = GDR_LOOKAHEAD;
// The ring never waits on itself: the producer refills a stage only after the
// consumers finished the tile it held, which the producer finalised kLookahead
// issues after starting it.
constexpr int kMinStages = kLookahead + 1;

// R: state rows per thread (8 or 16); a lane always holds 8 columns.
template <int DK, int VS, int R>
struct TmaShape {
  static constexpr int kRows = R;
  static constexpr int kRowLanes = DK / kRows;      // lanes that split the D_k rows: 4, 8 or 16
  static constexpr int kColLanes = 32 / kRowLanes;  // lanes that split the band: 8, 4 or 2
  static constexpr int kWarpCols = kColLanes * 8;   // columns per consumer warp: 64, 32 or 16
  static constexpr int kConsumerWarps = VS / kWarpCols;
  static constexpr int kConsumers = kConsumerWarps * 32;
  static constexpr int kThreads = kConsumers + 32;  // + the producer warp
  static constexpr int kStateBytes = DK * VS * 2;
  // Per-token stride of the per-row arrays: each row lane's R entries are
  // padded to R + 4, so the row lanes of one quarter-warp read different banks.
  static constexpr int kTokStride = DK + 4 * kRowLanes;
  static_assert(DK == 64 || DK == 128, "D_k must be 64 or 128");
  static_assert(R == 8 || R == 16, "8 or 16 rows per thread");
  static_assert(kRowLanes >= 4 && kRowLanes <= 16, "4 to 16 row lanes");
  static_assert(VS % kWarpCols == 0 && kConsumerWarps >= 1 && kConsumerWarps <= 16,
                "one to sixteen consumer warps per tile");
};

// Row ownership. Row lane rl owns rows r * RL + row_perm(rl), r < R: the rows
// that one quarter-warp reads together then differ in bit 2 (8 row lanes) or
// in bits 1-2 (16 row lanes) of the row index, so with the 128-byte swizzle of
// the state tile their 16-byte reads fall in different banks.
template <int RL>
__host__ __device__ constexpr int row_perm(int rl) {
  return RL == 8 ? ((rl >> 1) | ((rl & 1) << 2))
                 : (RL == 16 ? (2 * (rl & 3) + ((rl >> 2) & 1) + 8 * (rl >> 3)) : rl);
}

// Where row i sits in "owner order": the R rows of row lane rl are stored
// contiguously at [rl * (R + 4), rl * (R + 4) + R), so per-row vectors load as
// vectors and the four padding entries stagger the row lanes across banks.
template <int RL, int R>
__host__ __device__ constexpr int owner_slot(int i) {
  const int x = i % RL;
  const int r = i / RL;
  const int rl = RL == 8 ? (((x & 3) << 1) | (x >> 2))
                         : (RL == 16 ? (4 * (((x >> 3) << 1) | (x & 1)) + ((x >> 1) & 3)) : x);
  return rl * (R + 4) + r;
}

// Byte offsets inside one stage, for T padded tokens.
struct StageLayout {
  int v, k, q, gk, rv, raw, beta, kq, meta, bytes;
};

// The producer turns the k, q and gk rows into float4 row vectors
// {d k, d q_s, d, k} in owner order (see owner_slot).
template <int DK, int VS, int R>
__host__ __device__ inline StageLayout stage_layout(int T) {
  StageLayout s;
  s.v = TmaShape<DK, VS, R>::kStateBytes;  // bf16 [T][VS]   value rows of the slice
  // per-row arrays: [T][TS] with TS = DK + 4 * row lanes; rows arrive in natural
  // order and the producer rewrites them in owner order (see owner_slot)
  constexpr int TS = TmaShape<DK, VS, R>::kTokStride;
  s.k = s.v + T * VS * 2;               // bf16 [T][TS]   key rows
  s.q = s.k + T * TS * 2;               // bf16 [T][TS]   query rows
  s.gk = s.q + T * TS * 2;              // fp32 [T][TS]   gk rows
  s.rv = s.gk + T * TS * 4;             // fp32x4 [T][TS] {d*k, d*q*scale, d, k}
  s.raw = s.rv + T * TS * 16;           // u32 [2][8]  gate scalar words
  s.beta = s.raw + 64;                  // fp32 [8]
  s.kq = s.beta + 32;                   // fp32 [8]       k . (q * scale)
  s.meta = s.kq + 32;                   // int32 [4]      length, slot, committed tokens
  s.bytes = (s.meta + 16 + 1023) & ~1023;
  return s;
}

// CTA-level area after the stages: three mbarriers per stage, then the abort
// word of the failure protocol (gdr_ptx.cuh).
__host__ __device__ inline int cta_extra_bytes(int n_stages) { return 3 * n_stages * 8 + 16; }

template <int DK, int VS, int R>
__host__ __device__ inline int tma_smem_bytes(int T, int n_stages) {
  return 1024 /* alignment slack */ + n_stages * stage_layout<DK, VS, R>(T).bytes +
         cta_extra_bytes(n_stages);
}

// ---------------------------------------------------------------- the kernel

template <int DK, int VS, int RR, bool GATED>
__global__ void __launch_bounds__(TmaShape<DK, VS, RR>::kThreads, 1)
    decode_tma_kernel(const __grid_constant__ CUtensorMap pool_map, const DecodeParams p,
                      const int n_tiles, const int n_stages) {
  using Shape = TmaShape<DK, VS, RR>;
  constexpr int CW = Shape::kConsumerWarps;
  constexpr int R = Shape::kRows;
  constexpr int RL = Shape::kRowLanes;
  constexpr int CL = Shape::kColLanes;
  constexpr int WCOLS = Shape::kWarpCols;
  constexpr int NV = 16 / RL;  // reduced values per lane after the reduce-scatter: 4, 2 or 1
  constexpr int TS = Shape::kTokStride;
  const int T = p.T;
  const StageLayout lay = stage_layout<DK, VS, RR>(T);

  // Stages start on a 1024-byte boundary of the shared window. The offset is
  // added to the __shared__ array itself so every access stays a shared-memory
  // access (no generic addressing).
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw_base = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + (((raw_base + 1023u) & ~1023u) - raw_base);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + n_stages * lay.bytes);
  const uint32_t raw0 = smem_addr(bars);         // copies landed
  const uint32_t full0 = raw0 + 8 * n_stages;    // producer finished the stage
  const uint32_t empty0 = full0 + 8 * n_stages;  // consumers are done reading the stage
  volatile int* abort_word = reinterpret_cast<volatile int*>(bars + 3 * n_stages);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int n_slices = p.D_v / VS;
  const int n_mine = (n_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                     static_cast<int>(gridDim.x);

  if (tid == 0) {
    for (int i = 0; i < n_stages; ++i) {
      mbar_init(raw0 + 8 * i, 32);    // one cp.async arrival per producer lane
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, CW);  // one arrival per consumer warp
    }
    *abort_word = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == CW) {
    // ================================================================ producer
    constexpr int E = DK / 32;  // row elements per lane in the finalise step
    // Tiles this warp issues: all of them, unless a wait fails (then it stops
    // issuing and signals nothing more) or, in a test build, a tile is held back
    // (then it stops issuing but still finalises the tiles already issued).
    int n_issue = n_mine;
    bool silent = false;
    // slot, length and committed count of the next tile to issue, loaded one
    // iteration ahead (no committed-count array: all tokens are committed)
    int nx_s = 0, nx_L = 0, nx_n = 0;
    if (n_mine > 0) {
      const int b0 = blockIdx.x / (p.H_v * n_slices);
      nx_s = p.state_indices[b0];
      nx_L = p.seq_lengths[b0];
      nx_n = p.num_accepted != nullptr ? p.num_accepted[b0] : T;
    }
    for (int j = 0; j < n_issue + kLookahead && !silent; ++j) {
      if (j < n_issue && test_hold_tile(blockIdx.x + j * gridDim.x)) n_issue = j;
      if (j < n_issue) {
        // ---- issue tile j: start every copy it needs
        const int tile = blockIdx.x + j * gridDim.x;
        const int slice = tile % n_slices;
        const int h = (tile / n_slices) % p.H_v;
        const int b = tile / (n_slices * p.H_v);
        const int s = nx_s;
        int L = nx_L;
        L = L < 0 ? 0 : (L > T ? T : L);
        if (s < 0 || s >= p.pool_size) L = 0;
        const int n_commit = nx_n < 0 ? 0 : (nx_n > L ? L : nx_n);
        if (j + 1 < n_mine) {
          const int bn = (tile + gridDim.x) / (n_slices * p.H_v);
          nx_s = p.state_indices[bn];
          nx_L = p.seq_lengths[bn];
          nx_n = p.num_accepted != nullptr ? p.num_accepted[bn] : T;
        }
        const int stage = j % n_stages;
        const uint32_t phase = (j / n_stages) & 1;
        uint8_t* st = smem + stage * lay.bytes;
        const uint32_t rawb = raw0 + 8 * stage;
        bool free_ok = true;
        if (lane == 0)
          free_ok = mbar_wait_abandonable(empty0 + 8 * stage, phase ^ 1, abort_word,
                                          kErrProducerWait);
        if (!__shfl_sync(0xffffffffu, free_ok, 0)) {
          silent = true;  // the stage may still be in use: start nothing more
          n_issue = j;
          break;
        }
        const int col0 = slice * VS;
        const int hq = h / p.group;
        if (lane == 0) {
          int* meta = reinterpret_cast<int*>(st + lay.meta);
          meta[0] = L;
          meta[1] = s;
          meta[2] = n_commit;
          if (L > 0) {
            mbar_expect_tx(rawb, Shape::kStateBytes + L * (VS * 2 + DK * 8));
            tma_load_3d(smem_addr(st), &pool_map, 0, (s * p.H_v + h) * DK, col0 / 64, rawb);
            const size_t qk_off = (static_cast<size_t>(b) * p.H_qk + hq) * T * DK;
            const size_t gk_off = (static_cast<size_t>(b) * p.H_v + h) * T * DK;
            for (int t = 0; t < L; ++t) {  // one row of each per token (padded stride)
              bulk_load(smem_addr(st + lay.k + t * TS * 2), p.key + qk_off + t * DK, DK * 2, rawb);
              bulk_load(smem_addr(st + lay.q + t * TS * 2), p.query + qk_off + t * DK, DK * 2,
                        rawb);
              bulk_load(smem_addr(st + lay.gk + t * TS * 4), p.gk + gk_off + t * DK, DK * 4, rawb);
            }
            const uint16_t* vsrc =
                p.value + (static_cast<size_t>(b) * p.H_v + h) * T * p.D_v + col0;
            for (int t = 0; t < L; ++t)
              bulk_load(smem_addr(st + lay.v + t * VS * 2), vsrc + static_cast<size_t>(t) * p.D_v,
                        VS * 2, rawb);
          }
        }
        // gate scalars: lane t fetches token t's pair; lane 31 the per-head vectors
        uint32_t* rawv = reinterpret_cast<uint32_t*>(st + lay.raw);
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
            cp_async_4(smem_addr(st + lay.beta), p.dt_bias + h);
            cp_async_4(smem_addr(st + lay.kq), p.decay_scale + h);
          }
        }
        cp_async_arrive_noinc(rawb);
      }
      if (j >= kLookahead && j - kLookahead < n_issue) {
        // ---- finalise tile j - kLookahead: its copies have landed
        const int jf = j - kLookahead;
        const int tile = blockIdx.x + jf * gridDim.x;
        const int h = (tile / n_slices) % p.H_v;
        const int b = tile / (n_slices * p.H_v);
        const int stage = jf % n_stages;
        const uint32_t phase = (jf / n_stages) & 1;
        uint8_t* st = smem + stage * lay.bytes;
        const bool landed = mbar_wait_abandonable(raw0 + 8 * stage, phase, abort_word,
                                                  kErrProducerWait);
        if (!__all_sync(0xffffffffu, landed)) {
          silent = true;  // copies not seen to land: this tile is never signalled ready
          break;
        }
        int L = reinterpret_cast<const int*>(st + lay.meta)[0];
        L = L < 0 ? 0 : (L > T ? T : L);
        const uint32_t* rawv = reinterpret_cast<const uint32_t*>(st + lay.raw);
        float* sbeta = reinterpret_cast<float*>(st + lay.beta);
        float* skq = reinterpret_cast<float*>(st + lay.kq);
        float* sgk = reinterpret_cast<float*>(st + lay.gk);
        float4* srv = reinterpret_cast<float4*>(st + lay.rv);
        const uint16_t* sk = reinterpret_cast<const uint16_t*>(st + lay.k);
        const uint16_t* sq = reinterpret_cast<const uint16_t*>(st + lay.q);
        float dtb = 0.0f, dsc = 0.0f;
        if constexpr (GATED) {
          if (L > 0) {
            dtb = sbeta[0];  // dt_bias[h] and decay_scale[h] landed in the beta/kq words
            dsc = skq[0];
          }
        }
        __syncwarp();
#pragma unroll 1
        for (int t = 0; t < L; ++t) {
          float gt, bt;
          if constexpr (GATED) {
            const size_t ai = (static_cast<size_t>(b) * T + t) * p.H_v + h;
            const float av = bf16_in_word(rawv[t], p.gate_a + ai);
            const float bv = bf16_in_word(rawv[8 + t], p.gate_b + ai);
            gt = dsc * softplus_f32(av + dtb);  // g = decay_scale * softplus(a + dt_bias)
            bt = sigmoid_f32(bv);               // beta = sigmoid(b)
          } else {
            const size_t gi = (static_cast<size_t>(b) * p.H_v + h) * T + t;
            gt = __uint_as_float(rawv[t]);
            bt = bf16_in_word(rawv[8 + t], p.beta + gi);
          }
          // Row vectors go to owner order (see owner_slot).
          float kq = 0.0f;
          float dv[E], kv[E], qv[E];
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const int i = lane + 32 * e;
            dv[e] = expf(gt + sgk[t * TS + i]);  // exp(g) * exp(gk) as one exponential
            kv[e] = bf16_bits_to_f32(sk[t * TS + i]);
            qv[e] = bf16_bits_to_f32(sq[t * TS + i]) * p.scale;
            kq = fmaf(kv[e], qv[e], kq);
          }
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const int o = t * TS + owner_slot<RL, R>(lane + 32 * e);
            srv[o] = make_float4(dv[e] * kv[e], dv[e] * qv[e], dv[e], kv[e]);
          }
          kq = warp_sum(kq);
          __syncwarp();
          if (lane == 0) {
            sbeta[t] = bt;
            skq[t] = kq;  // k . (q * scale)
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(full0 + 8 * stage);
      }
    }
    // Before the CTA may retire, the copies this warp started must have landed:
    // wait (bounded, not abandonable) for the raw phase of the last tile issued
    // into every stage.
    for (int k = (n_issue > n_stages ? n_issue - n_stages : 0); k < n_issue; ++k) {
      if (!mbar_wait_bounded(raw0 + 8 * (k % n_stages), (k / n_stages) & 1)) {
        flag_error(kErrDrainWait);
        break;
      }
    }
    return;
  }

  // ================================================================ consumers
  // lane = rl * CL + cg: row lane rl owns rows r * RL + row_perm(rl), r < R
  // (their per-row vectors sit at owner slots [rl * R, rl * R + R)); column
  // lane cg owns the 8 columns [cg * 8, cg * 8 + 8) of this warp's band.
  const int rl = lane / CL;
  const int cg = lane % CL;
  const int i0 = rl * (R + 4);      // first owner slot of this thread
  const int rp = row_perm<RL>(rl);  // row of slot i0 + r is r * RL + rp
  const int cband = warp * WCOLS;  // first tile column of this warp
  const int c0 = cband + cg * 8;   // first tile column of this thread
  // After the reduce-scatter, lane (b4, sub, cg) with sub = rl mod (RL / 2)
  // holds vector (b4 ? p : kv_mem) at band columns cg * 8 + sub * NV + [0, NV).
  const bool b4 = (lane >> 4) & 1;
  const int cred = cg * 8 + NV * (rl & (RL / 2 - 1));

  bool dead = false;  // a wait of this warp failed: it commits and frees nothing more
  for (int it = 0; it < n_mine; ++it) {
    const int tile = blockIdx.x + it * gridDim.x;
    const int slice = tile % n_slices;
    const int h = (tile / n_slices) % p.H_v;
    const int b = tile / (n_slices * p.H_v);
    const int stage = it % n_stages;
    const uint32_t phase = (it / n_stages) & 1;
    uint8_t* st = smem + stage * lay.bytes;

    const bool ok_self =
        !dead && mbar_wait_abandonable(full0 + 8 * stage, phase, abort_word, kErrConsumerWait);
    const bool ok = __all_sync(0xffffffffu, ok_self);
    dead = !ok;
    const int* meta = reinterpret_cast<const int*>(st + lay.meta);
    int L = ok ? meta[0] : 0;  // one load for the whole warp: every lane sees one value
    L = L < 0 ? 0 : (L > T ? T : L);
    L = L > 1 ? 1 : L;  // single-token calls
    const int s = meta[1];
    if (s < 0 || s >= p.pool_size) L = 0;
    const bool commit = ok && meta[2] > 0;  // else the call leaves the slot's bits as they are

    // out[b, h, :, slice * VS + cband : + WCOLS]; padded tokens get +0.0.
    uint16_t* out_band =
        p.out + (static_cast<size_t>(b) * p.H_v + h) * T * p.D_v + slice * VS + cband;
    for (int e = lane; e < (T - L) * (WCOLS / 8); e += 32) {
      const int t = L + e / (WCOLS / 8);
      const int v8 = e % (WCOLS / 8);
      *reinterpret_cast<uint4*>(out_band + static_cast<size_t>(t) * p.D_v + v8 * 8) =
          make_uint4(0u, 0u, 0u, 0u);
    }

    // No state is kept in registers: a warp reads its rows from the stage
    // once for the column sums and once more for the update, and streams each
    // new row to the pool straight from the update.
    uint16_t* dst = p.state_pool + (static_cast<size_t>(s) * p.H_v + h) * DK * p.D_v +
                    slice * VS + c0;  // + row * D_v
    if (L > 0) {
      const float4* srv = reinterpret_cast<const float4*>(st + lay.rv);
      const float* sbeta = reinterpret_cast<const float*>(st + lay.beta);
      const float* skq = reinterpret_cast<const float*>(st + lay.kq);
      const uint16_t* sv = reinterpret_cast<const uint16_t*>(st + lay.v);

      for (int t = 0; t < L; ++t) {
        // kv_mem = S_dec^T k = S^T (d k) and p = S^T (d q_s): the decay of
        // step 1 is folded into the row vectors.
        unsigned long long m2[4], p2[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) m2[c] = p2[c] = 0ull;  // (+0.0f, +0.0f)
        // (the rows are re-read from shared memory, so the loop need not be
        // unrolled: unrolling it fully only raises register use)
        {
#pragma unroll 2
          for (int r = 0; r < R; ++r) {
            const float2 rv0 = reinterpret_cast<const float2*>(srv + t * TS + i0 + r)[0];
            const unsigned long long dk2 = pk(rv0.x, rv0.x);  // {d k, d k}
            const unsigned long long dq2 = pk(rv0.y, rv0.y);  // {d q_s, d q_s}
            const uint4 w = *reinterpret_cast<const uint4*>(st + swz_offset<DK>(r * RL + rp, c0));
            const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const unsigned long long sr = pk(bf16_lo(wv[c]), bf16_hi(wv[c]));
              m2[c] = fma2(sr, dk2, m2[c]);  // steps 1-2: kv_mem partial
              p2[c] = fma2(sr, dq2, p2[c]);  // S_dec^T q_s partial
            }
          }
        }
        // Reduce-scatter over the row lanes: xor 16 splits (kv_mem | p), then
        // xor 8 (and 4 for 8 row lanes, and 2 for 16) halve the columns.
        float x[8];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float2 mv = upk(m2[c]);
          const float2 pv = upk(p2[c]);
          const float s0 = b4 ? mv.x : pv.x, s1 = b4 ? mv.y : pv.y;
          const float k0 = b4 ? pv.x : mv.x, k1 = b4 ? pv.y : mv.y;
          x[2 * c] = k0 + __shfl_xor_sync(0xffffffffu, s0, 16);
          x[2 * c + 1] = k1 + __shfl_xor_sync(0xffffffffu, s1, 16);
        }
        float y[4];
        {
          const bool bit = (lane >> 3) & 1;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float send = bit ? x[c] : x[c + 4];
            const float keep = bit ? x[c + 4] : x[c];
            y[c] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
          }
        }
        float red[NV];
        if constexpr (NV == 4) {
#pragma unroll
          for (int c = 0; c < 4; ++c) red[c] = y[c];
        } else {
          float z[2];
          const bool bit = (lane >> 2) & 1;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const float send = bit ? y[c] : y[c + 2];
            const float keep = bit ? y[c + 2] : y[c];
            z[c] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
          }
          if constexpr (NV == 2) {
            red[0] = z[0];
            red[1] = z[1];
          } else {
            const bool bit1 = (lane >> 1) & 1;
            const float send = bit1 ? z[0] : z[1];
            const float keep = bit1 ? z[1] : z[0];
            red[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
          }
        }
        // kv_mem lanes: delta = (v - kv_mem) * beta (step 3), then handed to the
        // p lane of the same columns, which writes o (step 4).
        float dlt[NV];
        {
          const float bt = sbeta[t];
          if constexpr (NV == 4) {
            const uint2 w = *reinterpret_cast<const uint2*>(sv + t * VS + cband + cred);
            dlt[0] = (bf16_lo(w.x) - red[0]) * bt;
            dlt[1] = (bf16_hi(w.x) - red[1]) * bt;
            dlt[2] = (bf16_lo(w.y) - red[2]) * bt;
            dlt[3] = (bf16_hi(w.y) - red[3]) * bt;
          } else if constexpr (NV == 2) {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(sv + t * VS + cband + cred);
            dlt[0] = (bf16_lo(w) - red[0]) * bt;
            dlt[1] = (bf16_hi(w) - red[1]) * bt;
          } else {
            dlt[0] = (bf16_bits_to_f32(sv[t * VS + cband + cred]) - red[0]) * bt;
          }
        }
#pragma unroll
        for (int c = 0; c < NV; ++c) {
          const float other = __shfl_xor_sync(0xffffffffu, dlt[c], 16);
          if (b4) dlt[c] = other;
        }
        if (b4) {
          const float kq = skq[t];  // p already carries the query scale
          uint16_t* dst = out_band + static_cast<size_t>(t) * p.D_v + cred;
          if constexpr (NV == 4) {
            *reinterpret_cast<uint2*>(dst) =
                make_uint2(pack_bf16x2(fmaf(dlt[0], kq, red[0]), fmaf(dlt[1], kq, red[1])),
                           pack_bf16x2(fmaf(dlt[2], kq, red[2]), fmaf(dlt[3], kq, red[3])));  // step 4
          } else if constexpr (NV == 2) {
            *reinterpret_cast<uint32_t*>(dst) =
                pack_bf16x2(fmaf(dlt[0], kq, red[0]), fmaf(dlt[1], kq, red[1]));  // step 4
          } else {
            *dst = f32_to_bf16_bits(fmaf(dlt[0], kq, red[0]));  // step 4
          }
        }
        // every lane gathers delta of its own 8 columns from the kv_mem lanes
        // (b4 = 0, sub = sb, cg) = lane sb * CL + cg
        float dl[8];
#pragma unroll
        for (int sb = 0; sb < RL / 2; ++sb)
#pragma unroll
          for (int c = 0; c < NV; ++c)
            dl[sb * NV + c] = __shfl_sync(0xffffffffu, dlt[c], sb * CL + cg);
        unsigned long long dl2[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) dl2[c] = pk(dl[2 * c], dl[2 * c + 1]);
        // steps 1 and 3: S_new = d S + k delta^T
        {
#pragma unroll 2
          for (int r = 0; r < R; ++r) {
            const float2 rv1 = reinterpret_cast<const float2*>(srv + t * TS + i0 + r)[1];
            const unsigned long long d2 = pk(rv1.x, rv1.x);  // {d, d}
            const unsigned long long k2 = pk(rv1.y, rv1.y);  // {k, k}
            const uint4 w = *reinterpret_cast<const uint4*>(st + swz_offset<DK>(r * RL + rp, c0));
            const float2 n0 = upk(fma2(pk(bf16_lo(w.x), bf16_hi(w.x)), d2, mul2(k2, dl2[0])));
            const float2 n1 = upk(fma2(pk(bf16_lo(w.y), bf16_hi(w.y)), d2, mul2(k2, dl2[1])));
            const float2 n2 = upk(fma2(pk(bf16_lo(w.z), bf16_hi(w.z)), d2, mul2(k2, dl2[2])));
            const float2 n3 = upk(fma2(pk(bf16_lo(w.w), bf16_hi(w.w)), d2, mul2(k2, dl2[3])));
            // bf16 round-to-nearest-even, once per call, straight to the slot
            if (commit)
              __stcs(reinterpret_cast<uint4*>(dst + static_cast<size_t>(r * RL + rp) * p.D_v),
                     make_uint4(pack_bf16x2(n0.x, n0.y), pack_bf16x2(n1.x, n1.y),
                                pack_bf16x2(n2.x, n2.y), pack_bf16x2(n3.x, n3.y)));
          }
        }
      }
    }
    // This warp has read everything it needs from the stage: give it back.
    __syncwarp();
    if (lane == 0 && !dead) mbar_arrive(empty0 + 8 * stage);
  }
}

}  // namespace gdr
