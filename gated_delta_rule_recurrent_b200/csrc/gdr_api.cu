// C ABI of libgdr (declared in include/gdr.h): host-side argument checks and
// kernel dispatch for the recurrent gated-delta-rule decode step.
//
// Everything here runs on the host before any launch. A failed check returns
// its status with nothing queued; device values (lengths, slot indices) are
// handled by the kernel without traps.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <string>

#include "gdr.h"
#include "gdr_decode.cuh"

namespace {

thread_local std::string g_last_error;

int fail(int status, const std::string& what) {
  g_last_error = what;
  return status;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

// Checks shared by both entry points. Returns GDR_OK or a failure status.
int check_dims(const gdr_dims* d) {
  if (d == nullptr) return fail(GDR_ERR_NULL, "dims is NULL");
  if (d->B < 0) return fail(GDR_ERR_DIMS, "B must be >= 0");
  if (d->T < 1 || d->T > gdr::kMaxT)
    return fail(GDR_ERR_DIMS, "T must be in [1, 8] (decode only)");
  if (d->H_qk < 1 || d->H_v < 1) return fail(GDR_ERR_DIMS, "H_qk and H_v must be >= 1");
  if (d->H_v % d->H_qk != 0) return fail(GDR_ERR_DIMS, "H_v must be a multiple of H_qk");
  if (d->D_k < 1 || d->D_v < 1) return fail(GDR_ERR_DIMS, "D_k and D_v must be >= 1");
  if (d->pool_size < 1) return fail(GDR_ERR_DIMS, "pool_size must be >= 1");
  if (d->D_k != 64 && d->D_k != 128)
    return fail(GDR_ERR_UNSUPPORTED, "D_k must be 64 or 128");
  if (d->D_v % gdr::kSliceCols != 0)
    return fail(GDR_ERR_UNSUPPORTED, "D_v must be a multiple of 64");
  // Grid size: B * H_v * (D_v / 64) CTAs must fit a 31-bit grid dimension.
  const long long ctas = static_cast<long long>(d->B) * d->H_v * (d->D_v / gdr::kSliceCols);
  if (ctas > 0x7fffffffLL) return fail(GDR_ERR_DIMS, "B * H_v * D_v / 64 exceeds 2^31 - 1");
  return GDR_OK;
}

template <int DK, bool GATED>
int launch(const gdr::DecodeParams& p, cudaStream_t stream) {
  const int smem_bytes = gdr::decode_smem_floats<DK>(p.T) * static_cast<int>(sizeof(float));
  const unsigned grid = static_cast<unsigned>(p.B) * p.H_v * p.n_slices;
  gdr::decode_kernel<DK, GATED><<<grid, DK, smem_bytes, stream>>>(p);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess)
    return fail(GDR_ERR_CUDA, std::string("kernel launch failed: ") + cudaGetErrorString(err));
  return GDR_OK;
}

int dispatch(const gdr::DecodeParams& p, int D_k, bool gated, cudaStream_t stream) {
  if (D_k == 64) return gated ? launch<64, true>(p, stream) : launch<64, false>(p, stream);
  return gated ? launch<128, true>(p, stream) : launch<128, false>(p, stream);
}

gdr::DecodeParams base_params(const gdr_dims* d, const gdr_bf16* query, const gdr_bf16* key,
                              const gdr_bf16* value, gdr_bf16* state_pool,
                              const int32_t* asl, const int32_t* idx, const float* gk,
                              float scale, gdr_bf16* out) {
  gdr::DecodeParams p{};
  p.query = query;
  p.key = key;
  p.value = value;
  p.gk = gk;
  p.state_pool = state_pool;
  p.out = out;
  p.seq_lengths = asl;
  p.state_indices = idx;
  p.scale = scale;
  p.B = d->B;
  p.T = d->T;
  p.H_qk = d->H_qk;
  p.H_v = d->H_v;
  p.D_v = d->D_v;
  p.pool_size = d->pool_size;
  p.group = d->H_v / d->H_qk;
  p.n_slices = d->D_v / gdr::kSliceCols;
  return p;
}

int check_common_pointers(const gdr_bf16* query, const gdr_bf16* key, const gdr_bf16* value,
                          gdr_bf16* state_pool, const int32_t* asl, const int32_t* idx,
                          const float* gk, gdr_bf16* out) {
  if (!query || !key || !value || !state_pool || !asl || !idx || !gk || !out)
    return fail(GDR_ERR_NULL, "a required tensor pointer is NULL");
  if (!aligned16(query) || !aligned16(key) || !aligned16(value) || !aligned16(gk) ||
      !aligned16(state_pool) || !aligned16(out))
    return fail(GDR_ERR_ALIGN,
                "query, key, value, gk, state_pool and out must be 16-byte aligned");
  return GDR_OK;
}

}  // namespace

extern "C" {

GDR_API int gdr_decode(const gdr_dims* dims, const gdr_bf16* query, const gdr_bf16* key,
                       const gdr_bf16* value, const gdr_bf16* beta, gdr_bf16* state_pool,
                       const int32_t* actual_seq_lengths, const int32_t* ssm_state_indices,
                       const float* g, const float* gk, const int32_t* num_accepted_tokens,
                       float scale_value, gdr_bf16* out, gdr_stream_t stream) {
  (void)num_accepted_tokens;  // does not enter the arithmetic
  int rc = check_dims(dims);
  if (rc != GDR_OK) return rc;
  if (dims->B == 0) return GDR_OK;
  rc = check_common_pointers(query, key, value, state_pool, actual_seq_lengths,
                             ssm_state_indices, gk, out);
  if (rc != GDR_OK) return rc;
  if (!beta || !g) return fail(GDR_ERR_NULL, "beta and g must not be NULL");
  gdr::DecodeParams p = base_params(dims, query, key, value, state_pool, actual_seq_lengths,
                                    ssm_state_indices, gk, scale_value, out);
  p.beta = beta;
  p.g = g;
  return dispatch(p, dims->D_k, false, reinterpret_cast<cudaStream_t>(stream));
}

GDR_API int gdr_gate_fused(const gdr_dims* dims, const gdr_bf16* query, const gdr_bf16* key,
                           const gdr_bf16* value, const gdr_bf16* a, const gdr_bf16* b,
                           const float* dt_bias, const float* decay_scale, gdr_bf16* state_pool,
                           const int32_t* actual_seq_lengths, const int32_t* ssm_state_indices,
                           const float* gk, const int32_t* num_accepted_tokens,
                           float scale_value, gdr_bf16* out, gdr_stream_t stream) {
  (void)num_accepted_tokens;
  int rc = check_dims(dims);
  if (rc != GDR_OK) return rc;
  if (dims->B == 0) return GDR_OK;
  rc = check_common_pointers(query, key, value, state_pool, actual_seq_lengths,
                             ssm_state_indices, gk, out);
  if (rc != GDR_OK) return rc;
  if (!a || !b || !dt_bias || !decay_scale)
    return fail(GDR_ERR_NULL, "a, b, dt_bias and decay_scale must not be NULL");
  gdr::DecodeParams p = base_params(dims, query, key, value, state_pool, actual_seq_lengths,
                                    ssm_state_indices, gk, scale_value, out);
  p.gate_a = a;
  p.gate_b = b;
  p.dt_bias = dt_bias;
  p.decay_scale = decay_scale;
  return dispatch(p, dims->D_k, true, reinterpret_cast<cudaStream_t>(stream));
}

GDR_API const char* gdr_status_string(int status) {
  switch (status) {
    case GDR_OK: return "GDR_OK";
    case GDR_ERR_NULL: return "GDR_ERR_NULL";
    case GDR_ERR_DIMS: return "GDR_ERR_DIMS";
    case GDR_ERR_ALIGN: return "GDR_ERR_ALIGN";
    case GDR_ERR_UNSUPPORTED: return "GDR_ERR_UNSUPPORTED";
    case GDR_ERR_CUDA: return "GDR_ERR_CUDA";
    default: return "unknown status";
  }
}

GDR_API const char* gdr_last_error(void) { return g_last_error.c_str(); }

GDR_API int gdr_abi_version(void) { return 1; }

}  // extern "C"
