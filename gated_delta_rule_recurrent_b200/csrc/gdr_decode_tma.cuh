// Persistent, warp-specialised decode kernel for sm_100a.
//
// Arithmetic: the four steps of "lite_boost.ops.recurrent_gated_delta_rule"
// (MindSpore Lite API page, section 算法流程) and, when GATED, the gate of
// "com.microsoft.LinearAttentionGate" (README, section Description).
//
// Data flow. A tile is one (item b, value head h, VS-column slice of D_v) block
// of the state: DK rows x VS bf16 columns of slot ssm_state_indices[b]. Each
// CTA walks tiles tile = blockIdx.x, + gridDim.x, ... through a ring of
// shared-memory stages, with three roles:
//
//   producer warp - starts the asynchronous copies of a tile (a 2-D TMA load
//           of the state box; 1-D bulk copies of the value rows and of the k,
//           q and gk rows of the valid tokens; 4-byte cp.async copies of the
//           per-token gate scalars) and, kLookahead tiles later, once they
//           have landed ("raw" barrier), turns them into what the consumers
//           use: exp(g + gk) per row (written over gk), k.(q*scale) and beta
//           per token ("full" barrier). No lane waits on global-memory latency.
//   consumer warps - keep an 8x8 sub-tile in fp32 registers for all valid
//           tokens: decay in place; the column sums kv_mem = S^T k and
//           p = S^T q together; one CTA barrier per token to combine partial
//           sums across warps; delta; output o = scale * p +
//           delta * (k.q*scale), which is step 4's S_new^T (q*scale) with the
//           sums reordered; rank-1 update. Once done reading the input stage
//           they give it back to the producer ("empty" barrier), then write
//           the new tile as bf16 into a separate output buffer ("out_full").
//   storer warp - issues the TMA store of every output buffer and frees the
//           buffer ("out_empty") once the store has read it.
//
// Input stages therefore cycle at the pace of HBM latency plus compute; the
// store drain only holds the small output ring.
//
// HBM sees one bulk read and one bulk write of every touched state tile.
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

namespace gdr {

// Bits of the device error word.
constexpr unsigned kErrConsumerWait = 1u;
constexpr unsigned kErrProducerWait = 2u;
constexpr unsigned kErrDrainWait = 4u;
constexpr unsigned kErrStorerWait = 8u;

static __device__ unsigned int g_device_error = 0;

constexpr long long kWaitLimitCycles = 4000000000LL;  // ~2 s at 2 GHz

// Tuning constants (compile-time; the defaults are the measured best).
#ifndef GDR_LOOKAHEAD
#define GDR_LOOKAHEAD 2
#endif
#ifndef GDR_STORES_IN_FLIGHT
#define GDR_STORES_IN_FLIGHT 1
#endif
// The producer finalises tile j - kLookahead after starting the copies of tile j.
constexpr int kLookahead = GDR_LOOKAHEAD;
// TMA stores whose shared-memory reads may still be pending before the
// storer frees their output buffers.
constexpr int kStoresInFlight = GDR_STORES_IN_FLIGHT;
// Neither ring may wait on itself: the producer refills a stage only after the
// consumers finished its previous tile, which the producer finalised
// kLookahead issues later; an output buffer is freed one stored tile late.
constexpr int kMinStages = kLookahead + 1;
constexpr int kOutBuffers = kStoresInFlight + 1;
static_assert(kStoresInFlight >= 1 && kStoresInFlight <= 4, "release queue holds 1..4 stages");

template <int DK, int VS>
struct TmaShape {
  static constexpr int kRows = 8;              // state rows per thread
  static constexpr int kWarpRows = 4 * kRows;  // a warp covers 32 rows x 64 columns
  static constexpr int kWC = VS / 64;          // warp columns
  static constexpr int kWR = DK / kWarpRows;   // warp rows
  static constexpr int kConsumerWarps = kWC * kWR;
  static constexpr int kConsumers = kConsumerWarps * 32;
  static constexpr int kThreads = kConsumers + 64;  // + producer warp + storer warp
  static constexpr int kStateBytes = DK * VS * 2;
};

// Byte offsets inside one stage, for T padded tokens.
struct StageLayout {
  int v, k, q, sd, raw, beta, kq, meta, bytes;
};

template <int DK, int VS>
__host__ __device__ inline StageLayout stage_layout(int T) {
  StageLayout s;
  s.v = TmaShape<DK, VS>::kStateBytes;  // bf16 [T][VS]   value rows of the slice
  s.k = s.v + T * VS * 2;               // bf16 [T][DK]   key rows
  s.q = s.k + T * DK * 2;               // bf16 [T][DK]   query rows
  s.sd = s.q + T * DK * 2;              // fp32 [T][DK]   gk, then exp(g + gk)
  s.raw = s.sd + T * DK * 4;            // u32 [2][8]     gate scalar words
  s.beta = s.raw + 64;                  // fp32 [8]
  s.kq = s.beta + 32;                   // fp32 [8]       k . (q * scale)
  s.meta = s.kq + 32;                   // int32 [4]      length, slot, consumer failure
  s.bytes = (s.meta + 16 + 1023) & ~1023;
  return s;
}

// CTA-level area after the input stages: kOutBuffers output tiles with their
// (length, slot, failure) words, two buffers of per-warp partial sums, and the
// mbarriers (three per input stage, two per output buffer).
template <int DK, int VS>
__host__ __device__ inline int cta_extra_bytes(int n_stages) {
  using S = TmaShape<DK, VS>;
  return kOutBuffers * S::kStateBytes + kOutBuffers * 16 + 2 * S::kConsumerWarps * 32 * 4 * 4 +
         (3 * n_stages + 2 * kOutBuffers) * 8;
}

template <int DK, int VS>
__host__ __device__ inline int tma_smem_bytes(int T, int n_stages) {
  return 1024 /* alignment slack */ + n_stages * stage_layout<DK, VS>(T).bytes +
         cta_extra_bytes<DK, VS>(n_stages);
}

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase of parity `parity` to complete, for at most
// kWaitLimitCycles. Returns false when the budget ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) return false;
  }
  return true;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// 1-D bulk copy global -> shared; both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// 4-byte asynchronous copy global -> shared (both 4-byte aligned).
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// Arrive on `bar` once every cp.async this thread has issued so far has landed.
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int x, int y, uint32_t src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::
                   "l"(map),
               "r"(x), "r"(y), "r"(src)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Barrier over `n` threads that also returns the AND of `v` over them.
__device__ __forceinline__ bool named_bar_and(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void flag_error(unsigned bit) { atomicOr(&g_device_error, bit); }

// The bf16 at `p` is fetched as the aligned 32-bit word that holds it (that
// word never leaves the page of `p`, so the wider read cannot fault).
__device__ __forceinline__ const void* word_of(const uint16_t* p) {
  return reinterpret_cast<const void*>(reinterpret_cast<uintptr_t>(p) & ~uintptr_t(3));
}
__device__ __forceinline__ float bf16_in_word(uint32_t w, const uint16_t* p) {
  return (reinterpret_cast<uintptr_t>(p) & 2) ? bf16_hi(w) : bf16_lo(w);
}

// Packed pairs of fp32 (sm_100 f32x2 instructions: one issue slot for two
// IEEE round-to-nearest operations, bit-identical to two scalar ones).
__device__ __forceinline__ unsigned long long pk(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 upk(unsigned long long v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ void unpack_bf16x8(const uint4 w, float (&f)[8]) {
  f[0] = bf16_lo(w.x); f[1] = bf16_hi(w.x);
  f[2] = bf16_lo(w.y); f[3] = bf16_hi(w.y);
  f[4] = bf16_lo(w.z); f[5] = bf16_hi(w.z);
  f[6] = bf16_lo(w.w); f[7] = bf16_hi(w.w);
}

// ---------------------------------------------------------------- the kernel

constexpr int kConsumerBar = 1;  // named barrier of the consumer warps

template <int DK, int VS, bool GATED>
__global__ void __launch_bounds__(TmaShape<DK, VS>::kThreads, 1)
    decode_tma_kernel(const __grid_constant__ CUtensorMap pool_map, const DecodeParams p,
                      const int n_tiles, const int n_stages) {
  using Shape = TmaShape<DK, VS>;
  constexpr int NC = Shape::kConsumers;
  constexpr int CW = Shape::kConsumerWarps;
  constexpr int WC = Shape::kWC;
  constexpr int WR = Shape::kWR;
  constexpr int R = Shape::kRows;
  const int T = p.T;
  const StageLayout lay = stage_layout<DK, VS>(T);

  // Stages start on a 1024-byte boundary of the shared window. The offset is
  // added to the __shared__ array itself so every access stays a shared-memory
  // access (no generic addressing).
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw_base = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + (((raw_base + 1023u) & ~1023u) - raw_base);
  uint8_t* obuf = smem + n_stages * lay.bytes;                         // [kOut][DK][VS] bf16
  int* ometa = reinterpret_cast<int*>(obuf + kOutBuffers * Shape::kStateBytes);  // [kOut][4]
  float* red = reinterpret_cast<float*>(ometa + 4 * kOutBuffers);         // [2][CW][32][4]
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 2 * CW * 128);
  const uint32_t raw0 = smem_addr(bars);             // copies landed
  const uint32_t full0 = raw0 + 8 * n_stages;        // producer finished the stage
  const uint32_t empty0 = full0 + 8 * n_stages;      // consumers done reading the stage
  const uint32_t ofull0 = empty0 + 8 * n_stages;     // consumers wrote the output buffer
  const uint32_t oempty0 = ofull0 + 8 * kOutBuffers;  // the store has read the buffer

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int n_slices = p.D_v / VS;
  const int n_mine = (n_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                     static_cast<int>(gridDim.x);

  if (tid == 0) {
    for (int i = 0; i < n_stages; ++i) {
      mbar_init(raw0 + 8 * i, 32);  // one cp.async arrival per producer lane
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, CW);  // one arrival per consumer warp
    }
    for (int i = 0; i < kOutBuffers; ++i) {
      mbar_init(ofull0 + 8 * i, CW);
      mbar_init(oempty0 + 8 * i, 1);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == CW) {
    // ================================================================ producer
    constexpr int E = DK / 32;  // row elements per lane in the finalise step
    bool failed = false;
    // slot and length of the next tile to issue, loaded one iteration ahead
    int nx_s = 0, nx_L = 0;
    if (n_mine > 0) {
      const int b0 = blockIdx.x / (p.H_v * n_slices);
      nx_s = p.state_indices[b0];
      nx_L = p.seq_lengths[b0];
    }
    for (int j = 0; j < n_mine + kLookahead; ++j) {
      if (j < n_mine) {
        // ---- issue tile j: start every copy it needs
        const int tile = blockIdx.x + j * gridDim.x;
        const int slice = tile % n_slices;
        const int h = (tile / n_slices) % p.H_v;
        const int b = tile / (n_slices * p.H_v);
        const int s = nx_s;
        int L = nx_L;
        L = L < 0 ? 0 : (L > T ? T : L);
        if (s < 0 || s >= p.pool_size) L = 0;
        if (j + 1 < n_mine) {
          const int bn = (tile + gridDim.x) / (n_slices * p.H_v);
          nx_s = p.state_indices[bn];
          nx_L = p.seq_lengths[bn];
        }
        const int stage = j % n_stages;
        const uint32_t phase = (j / n_stages) & 1;
        uint8_t* st = smem + stage * lay.bytes;
        const uint32_t rawb = raw0 + 8 * stage;
        if (lane == 0 && !failed) {
          if (!mbar_wait_bounded(empty0 + 8 * stage, phase ^ 1)) {
            failed = true;
            flag_error(kErrProducerWait);
          }
        }
        __syncwarp();
        const int col0 = slice * VS;
        const int hq = h / p.group;
        if (lane == 0) {
          int* meta = reinterpret_cast<int*>(st + lay.meta);
          meta[0] = L;
          meta[1] = s;
          if (L > 0) {
            mbar_expect_tx(rawb, Shape::kStateBytes + L * (VS * 2 + DK * 8));
            tma_load_2d(smem_addr(st), &pool_map, col0, (s * p.H_v + h) * DK, rawb);
            const size_t qk_off = (static_cast<size_t>(b) * p.H_qk + hq) * T * DK;
            const size_t gk_off = (static_cast<size_t>(b) * p.H_v + h) * T * DK;
            bulk_load(smem_addr(st + lay.k), p.key + qk_off, L * DK * 2, rawb);
            bulk_load(smem_addr(st + lay.q), p.query + qk_off, L * DK * 2, rawb);
            bulk_load(smem_addr(st + lay.sd), p.gk + gk_off, L * DK * 4, rawb);
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
      if (j >= kLookahead) {
        // ---- finalise tile j - kLookahead: its copies have landed
        const int jf = j - kLookahead;
        const int tile = blockIdx.x + jf * gridDim.x;
        const int h = (tile / n_slices) % p.H_v;
        const int b = tile / (n_slices * p.H_v);
        const int stage = jf % n_stages;
        const uint32_t phase = (jf / n_stages) & 1;
        uint8_t* st = smem + stage * lay.bytes;
        if (!mbar_wait_bounded(raw0 + 8 * stage, phase)) flag_error(kErrProducerWait);
        int L = reinterpret_cast<const int*>(st + lay.meta)[0];
        L = L < 0 ? 0 : (L > T ? T : L);
        const uint32_t* rawv = reinterpret_cast<const uint32_t*>(st + lay.raw);
        float* sbeta = reinterpret_cast<float*>(st + lay.beta);
        float* skq = reinterpret_cast<float*>(st + lay.kq);
        float* sd = reinterpret_cast<float*>(st + lay.sd);
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
          float kq = 0.0f;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const int i = lane + 32 * e;
            sd[t * DK + i] = expf(gt + sd[t * DK + i]);  // exp(g) * exp(gk) as one exponential
            kq = fmaf(bf16_bits_to_f32(sk[t * DK + i]), bf16_bits_to_f32(sq[t * DK + i]), kq);
          }
          kq = warp_sum(kq);
          __syncwarp();
          if (lane == 0) {
            sbeta[t] = bt;
            skq[t] = kq * p.scale;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(full0 + 8 * stage);
      }
    }
    // Before the CTA may retire, the copies this warp started must have landed:
    // wait (bounded) for the last raw phase of every stage still in use.
    for (int k = (n_mine > n_stages ? n_mine - n_stages : 0); k < n_mine; ++k) {
      if (!mbar_wait_bounded(raw0 + 8 * (k % n_stages), (k / n_stages) & 1)) {
        flag_error(kErrDrainWait);
        break;
      }
    }
    return;
  }

  if (warp == CW + 1) {
    // ================================================================ storer
    if (lane != 0) return;
    // Output buffers whose TMA stores may still be reading them, oldest first.
    int pend[kStoresInFlight + 1] = {};
    int n_pend = 0;
    for (int it = 0; it < n_mine; ++it) {
      const int tile = blockIdx.x + it * gridDim.x;
      const int slice = tile % n_slices;
      const int h = (tile / n_slices) % p.H_v;
      const int ob = it % kOutBuffers;
      const uint32_t phase = (it / kOutBuffers) & 1;
      const bool ok = mbar_wait_bounded(ofull0 + 8 * ob, phase);
      if (!ok) flag_error(kErrStorerWait);
      const int L = ometa[4 * ob + 0];
      const int s = ometa[4 * ob + 1];
      if (ok && ometa[4 * ob + 2] == 0 && L > 0 && s >= 0 && s < p.pool_size) {
        tma_store_2d(&pool_map, slice * VS, (s * p.H_v + h) * DK,
                     smem_addr(obuf + ob * Shape::kStateBytes));
        bulk_commit();
#pragma unroll
        for (int q = 0; q <= kStoresInFlight; ++q)
          if (q == n_pend) pend[q] = ob;  // constant indices keep pend in registers
        ++n_pend;
        if (n_pend > kStoresInFlight) {
          // all but the newest kStoresInFlight stores have read their buffers
          bulk_wait_read<kStoresInFlight>();
          mbar_arrive(oempty0 + 8 * pend[0]);
#pragma unroll
          for (int q = 0; q < kStoresInFlight; ++q) pend[q] = pend[q + 1];
          --n_pend;
        }
      } else {
        // Nothing to store from this buffer. Free it, and every pending one
        // once its store has read it, so no buffer waits on a later store.
        bulk_wait_read<0>();
#pragma unroll
        for (int q = 0; q < kStoresInFlight; ++q)
          if (q < n_pend) mbar_arrive(oempty0 + 8 * pend[q]);
        n_pend = 0;
        mbar_arrive(oempty0 + 8 * ob);
      }
    }
    bulk_wait_all();
    return;
  }

  // ================================================================ consumers
  const int cw = warp;  // consumer warp 0 .. CW-1
  const int wr = cw / WC;
  const int wc = cw % WC;
  const int cg = lane & 7;
  const int rl = lane >> 3;
  const int i0 = wr * Shape::kWarpRows + rl * R;  // first state row of this thread
  const int c0 = wc * 64 + cg * kColsPerThread;   // first tile column of this thread
  const bool bit4 = (lane >> 4) & 1;
  const bool bit3 = (lane >> 3) & 1;
  const bool writes_out = (wr == 0) && (rl == 0);  // one thread per 8 columns
  const float scale = p.scale;

  for (int it = 0; it < n_mine; ++it) {
    const int tile = blockIdx.x + it * gridDim.x;
    const int slice = tile % n_slices;
    const int h = (tile / n_slices) % p.H_v;
    const int b = tile / (n_slices * p.H_v);
    const int col0 = slice * VS;
    const int stage = it % n_stages;
    const uint32_t phase = (it / n_stages) & 1;
    uint8_t* st = smem + stage * lay.bytes;

    // The barrier also orders this tile's first write of the partial-sum
    // buffers after every consumer's last read of them in the previous tile.
    const bool ok_self = mbar_wait_bounded(full0 + 8 * stage, phase);
    const bool ok = named_bar_and(kConsumerBar, NC, ok_self);
    if (!ok_self) flag_error(kErrConsumerWait);
    const int* meta = reinterpret_cast<const int*>(st + lay.meta);
    int L = ok ? meta[0] : 0;
    L = L < 0 ? 0 : (L > T ? T : L);
    const int s = meta[1];

    uint16_t* out_bh = p.out + (static_cast<size_t>(b) * p.H_v + h) * T * p.D_v + col0;
    for (int e = tid; e < (T - L) * (VS / 8); e += NC) {
      const int t = L + e / (VS / 8);
      const int v8 = e % (VS / 8);
      *reinterpret_cast<uint4*>(out_bh + static_cast<size_t>(t) * p.D_v + v8 * 8) =
          make_uint4(0u, 0u, 0u, 0u);
    }

    // S2[r][c] holds columns 2c and 2c+1 of row r as a packed fp32 pair.
    unsigned long long S2[R][kColsPerThread / 2];
    if (L > 0) {
      const uint16_t* tile_s = reinterpret_cast<const uint16_t*>(st);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float f[8];
        unpack_bf16x8(*reinterpret_cast<const uint4*>(tile_s + (i0 + r) * VS + c0), f);
#pragma unroll
        for (int c = 0; c < 4; ++c) S2[r][c] = pk(f[2 * c], f[2 * c + 1]);
      }
      const uint16_t* sk = reinterpret_cast<const uint16_t*>(st + lay.k);
      const uint16_t* sq = reinterpret_cast<const uint16_t*>(st + lay.q);
      const float* sd = reinterpret_cast<const float*>(st + lay.sd);
      const float* sbeta = reinterpret_cast<const float*>(st + lay.beta);
      const float* skq = reinterpret_cast<const float*>(st + lay.kq);
      const uint16_t* sv = reinterpret_cast<const uint16_t*>(st + lay.v);

      for (int t = 0; t < L; ++t) {
        float* buf = red + (t & 1) * (CW * 128);
        float kr[R], qr[R], dr[R];
#pragma unroll
        for (int r4 = 0; r4 < R; r4 += 4) {
          const uint2 kw = *reinterpret_cast<const uint2*>(sk + t * DK + i0 + r4);
          const uint2 qw = *reinterpret_cast<const uint2*>(sq + t * DK + i0 + r4);
          const float4 dw = *reinterpret_cast<const float4*>(sd + t * DK + i0 + r4);
          kr[r4 + 0] = bf16_lo(kw.x); kr[r4 + 1] = bf16_hi(kw.x);
          kr[r4 + 2] = bf16_lo(kw.y); kr[r4 + 3] = bf16_hi(kw.y);
          qr[r4 + 0] = bf16_lo(qw.x); qr[r4 + 1] = bf16_hi(qw.x);
          qr[r4 + 2] = bf16_lo(qw.y); qr[r4 + 3] = bf16_hi(qw.y);
          dr[r4 + 0] = dw.x; dr[r4 + 1] = dw.y; dr[r4 + 2] = dw.z; dr[r4 + 3] = dw.w;
        }
        unsigned long long m2[4], p2[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) m2[c] = p2[c] = 0ull;  // (+0.0f, +0.0f)
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const unsigned long long d2 = pk(dr[r], dr[r]);
          const unsigned long long k2 = pk(kr[r], kr[r]);
          const unsigned long long q2 = pk(qr[r], qr[r]);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            S2[r][c] = mul2(S2[r][c], d2);      // step 1: decay row r
            m2[c] = fma2(S2[r][c], k2, m2[c]);  // step 2: kv_mem partial
            p2[c] = fma2(S2[r][c], q2, p2[c]);  // S^T q partial (scale applied later)
          }
        }
        float m[kColsPerThread], pp[kColsPerThread];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float2 mv = upk(m2[c]);
          const float2 pv = upk(p2[c]);
          m[2 * c] = mv.x; m[2 * c + 1] = mv.y;
          pp[2 * c] = pv.x; pp[2 * c + 1] = pv.y;
        }
        // Reduce-scatter over the 4 row lanes: xor 16 splits (kv_mem | p), xor 8
        // splits the 8 columns into halves. Lane (bit4, bit3, cg) ends with the
        // warp sum of vector (bit4 ? p : kv_mem) at columns cg*8 + bit3*4 + 0..3.
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
        *reinterpret_cast<float4*>(buf + (cw * 32 + lane) * 4) = make_float4(y[0], y[1], y[2], y[3]);
        named_bar_sync(kConsumerBar, NC);
        // kv_mem of this thread's 8 columns: the sum over the warp rows of the
        // partials held by lanes (0, 0, cg) and (0, 1, cg) of each warp.
        float mem[kColsPerThread];
#pragma unroll
        for (int c = 0; c < kColsPerThread; ++c) mem[c] = 0.0f;
#pragma unroll
        for (int w = 0; w < WR; ++w) {
          const float* src = buf + ((w * WC + wc) * 32 + cg) * 4;
          const float4 lo = *reinterpret_cast<const float4*>(src);
          const float4 hi = *reinterpret_cast<const float4*>(src + 8 * 4);
          mem[0] += lo.x; mem[1] += lo.y; mem[2] += lo.z; mem[3] += lo.w;
          mem[4] += hi.x; mem[5] += hi.y; mem[6] += hi.z; mem[7] += hi.w;
        }
        float vv[kColsPerThread];
        unpack_bf16x8(*reinterpret_cast<const uint4*>(sv + t * VS + c0), vv);
        const float bt = sbeta[t];
        float dl[kColsPerThread];
#pragma unroll
        for (int c = 0; c < kColsPerThread; ++c) dl[c] = (vv[c] - mem[c]) * bt;  // step 3
        if (writes_out) {
          float pj[kColsPerThread];
#pragma unroll
          for (int c = 0; c < kColsPerThread; ++c) pj[c] = 0.0f;
#pragma unroll
          for (int w = 0; w < WR; ++w) {
            const float* src = buf + ((w * WC + wc) * 32 + 16 + cg) * 4;
            const float4 lo = *reinterpret_cast<const float4*>(src);
            const float4 hi = *reinterpret_cast<const float4*>(src + 8 * 4);
            pj[0] += lo.x; pj[1] += lo.y; pj[2] += lo.z; pj[3] += lo.w;
            pj[4] += hi.x; pj[5] += hi.y; pj[6] += hi.z; pj[7] += hi.w;
          }
          const float kq = skq[t];
          float o[kColsPerThread];
#pragma unroll
          for (int c = 0; c < kColsPerThread; ++c) o[c] = fmaf(dl[c], kq, pj[c] * scale);  // step 4
          uint4 ow;
          ow.x = pack_bf16x2(o[0], o[1]);
          ow.y = pack_bf16x2(o[2], o[3]);
          ow.z = pack_bf16x2(o[4], o[5]);
          ow.w = pack_bf16x2(o[6], o[7]);
          *reinterpret_cast<uint4*>(out_bh + static_cast<size_t>(t) * p.D_v + c0) = ow;
        }
        unsigned long long dl2[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) dl2[c] = pk(dl[2 * c], dl[2 * c + 1]);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const unsigned long long k2 = pk(kr[r], kr[r]);
#pragma unroll
          for (int c = 0; c < 4; ++c) S2[r][c] = fma2(k2, dl2[c], S2[r][c]);  // step 3: S += k delta^T
        }
      }
    }
    // This warp is done reading the input stage: the producer may refill it.
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * stage);

    // Write the new tile into the next output buffer once its last store has
    // read it, then hand it to the storer.
    const int ob = it % kOutBuffers;
    const uint32_t ophase = (it / kOutBuffers) & 1;
    bool ok_out = true;
    if (L > 0) {
      ok_out = mbar_wait_bounded(oempty0 + 8 * ob, ophase ^ 1);
      if (!ok_out) flag_error(kErrConsumerWait);
      uint16_t* out_tile = reinterpret_cast<uint16_t*>(obuf + ob * Shape::kStateBytes);
      // bf16, round-to-nearest-even, once per call
#pragma unroll
      for (int r = 0; r < R; ++r) {
        uint4 o;
        float2 v;
        v = upk(S2[r][0]); o.x = pack_bf16x2(v.x, v.y);
        v = upk(S2[r][1]); o.y = pack_bf16x2(v.x, v.y);
        v = upk(S2[r][2]); o.z = pack_bf16x2(v.x, v.y);
        v = upk(S2[r][3]); o.w = pack_bf16x2(v.x, v.y);
        *reinterpret_cast<uint4*>(out_tile + (i0 + r) * VS + c0) = o;
      }
      fence_proxy_async_smem();
    } else {
      // Nothing is written; still wait for the buffer so the (length, slot)
      // words below are not changed under a store that is reading them.
      ok_out = mbar_wait_bounded(oempty0 + 8 * ob, ophase ^ 1);
      if (!ok_out) flag_error(kErrConsumerWait);
    }
    if (tid == 0) {
      ometa[4 * ob + 0] = L;
      ometa[4 * ob + 1] = s;
      ometa[4 * ob + 2] = (ok && ok_out) ? 0 : 1;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(ofull0 + 8 * ob);
  }
}

}  // namespace gdr
