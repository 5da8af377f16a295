/*
 * gdr.h - C ABI of libgdr: the recurrent gated-delta-rule decode step on
 * NVIDIA B200 (sm_100a).
 *
 * The operation is the one defined on the MindSpore Lite API page
 * "lite_boost.ops.recurrent_gated_delta_rule" (signature; section 算法流程,
 * steps 1-4; section 参数 for shapes and dtypes; section 返回 for outputs). For
 * every batch item b, value head h and token t < actual_seq_lengths[b], in
 * token order:
 *
 *   1. decay         S = S * exp(g[b,h,t]) * exp(gk[b,h,t,i])   (row i of D_k)
 *   2. memory read   kv_mem = S^T k                              (length D_v)
 *   3. delta update  S = S + k (x) ((v - kv_mem) * beta[b,h,t])
 *   4. output        o = S^T (q * scale_value), stored as bfloat16
 *
 * gdr_gate_fused additionally computes the gate in front of step 1, as the
 * "com.microsoft.LinearAttentionGate" README defines it (section Description):
 * g = decay_scale[h] * softplus(a[b,t,h] + dt_bias[h]), beta = sigmoid(b[b,t,h]).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.   Every tensor pointer is DEVICE memory owned by the caller, dense,
 *           row-major in the shape order given. The library allocates nothing,
 *           never synchronises, and returns as soon as the work is queued on
 *           `stream` (a cudaStream_t; NULL means the legacy default stream).
 *           The current CUDA device must be the one that holds the tensors.
 * bf16.     gdr_bf16 is the raw bit pattern of an IEEE-style bfloat16.
 * State.    state_pool is [pool_size, H_v, D_k, D_v] bf16 (row = D_k,
 *           column = D_v, D_v contiguous); ssm_state_indices[b] names the slot
 *           item b reads and writes. The pool is updated IN PLACE: the page's
 *           `state_out` is the same buffer. Slots no item names are untouched.
 *           The state is carried in fp32 across the tokens of a call and
 *           rounded to bf16 (round-to-nearest-even) once, after the item's last
 *           valid token. Slot indices of one call must be distinct (two items
 *           writing one slot race).
 * Lengths.  actual_seq_lengths[b] is clamped to [0, T]. Tokens t >= length are
 *           padding: their inputs are not read, out[b,:,t,:] is +0.0, the state
 *           does not change. An item whose slot index lies outside
 *           [0, pool_size) is skipped the same way (all-zero out, no slot
 *           touched); the library never traps on device values.
 * Heads.    H_v must be a multiple of H_qk; value head h reads query/key head
 *           h / (H_v / H_qk) (grouped / multi-query heads).
 * Aliasing. Inputs must not overlap `out` or `state_pool`.
 * Sizes.    1 <= T <= 8 (decode only); D_k in {64, 128}; D_v a positive
 *           multiple of 64; H_qk, H_v, pool_size >= 1; B >= 0 (B == 0 queues
 *           nothing and returns GDR_OK).
 * Alignment: query, key, value, gk, state_pool and out must be 16-byte aligned.
 * Errors.   Every check runs on the host before anything is queued; a failed
 *           check returns its status and queues nothing. GDR_ERR_CUDA reports a
 *           launch failure. gdr_last_error() describes the most recent failure
 *           of the calling thread.
 * Tensor memory. The kernels for D_k = 128 with D_v a multiple of 128, and the
 *           prefill kernel, run one CTA per SM and take 512 columns of that
 *           SM's tensor memory (TMEM) for the length of a launch; they free it
 *           before they exit. The allocation waits until the columns are free
 *           (the hardware offers no form that gives up), so a caller must not
 *           run another kernel that holds TMEM on the same SMs at the same time,
 *           for example a tcgen05 GEMM on another stream. Calls queued on one
 *           stream are always safe.
 */
#ifndef GDR_H_
#define GDR_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(_WIN32)
#define GDR_API
#else
#define GDR_API __attribute__((visibility("default")))
#endif

/* Raw bfloat16 bits. */
typedef uint16_t gdr_bf16;

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st* gdr_stream_t;

/* Layout of state_pool. */
typedef enum gdr_state_layout {
  /* [pool_size, H_v, D_k, D_v]: the op page's state layout (参数: state), D_v
   * contiguous. The default. */
  GDR_LAYOUT_KV = 0,
  /* [pool_size, H_v, D_v, D_k]: the NPU operator's internal layout (注), D_k
   * contiguous; the same state, transposed per head. */
  GDR_LAYOUT_VK = 1
} gdr_state_layout;

/* Sizes of one call. B batch items, T padded tokens per item, H_qk query/key
 * heads, H_v value heads, D_k key width (state rows), D_v value width (state
 * columns), pool_size slots in state_pool, layout a gdr_state_layout (0 when
 * the struct is zero-initialised). */
typedef struct gdr_dims {
  int32_t B;
  int32_t T;
  int32_t H_qk;
  int32_t H_v;
  int32_t D_k;
  int32_t D_v;
  int32_t pool_size;
  int32_t layout;
} gdr_dims;

typedef enum gdr_status {
  GDR_OK = 0,
  GDR_ERR_NULL = 1,        /* a required pointer is NULL */
  GDR_ERR_DIMS = 2,        /* a size is out of range or inconsistent */
  GDR_ERR_ALIGN = 3,       /* a tensor is not 16-byte aligned */
  GDR_ERR_UNSUPPORTED = 4, /* valid sizes this build has no kernel for */
  GDR_ERR_CUDA = 5         /* the CUDA runtime reported an error */
} gdr_status;

/*
 * gdr_decode - one decode call of the op on "lite_boost.ops.recurrent_gated_delta_rule"
 * (signature and section 算法流程). Argument order follows the page.
 *
 *   query               [B, H_qk, T, D_k] bf16  (multiplied by scale_value)
 *   key                 [B, H_qk, T, D_k] bf16
 *   value               [B, H_v,  T, D_v] bf16
 *   beta                [B, H_v,  T]      bf16
 *   state_pool          [pool_size, H_v, D_k, D_v] bf16 (dims->layout = GDR_LAYOUT_KV)
 *                       or [pool_size, H_v, D_v, D_k] (GDR_LAYOUT_VK), read and
 *                       written in place
 *   actual_seq_lengths  [B] int32, valid tokens per item
 *   ssm_state_indices   [B] int32, pool slot per item
 *   g                   [B, H_v, T]       fp32
 *   gk                  [B, H_v, T, D_k]  fp32
 *   num_accepted_tokens [B] int32 or NULL: n = clamp(num_accepted_tokens[b], 0, L)
 *                       leading tokens of item b are committed. Outputs of all L
 *                       valid tokens are computed; the slot receives the state
 *                       after token n - 1 and keeps its bits when n = 0. NULL
 *                       commits all L (the page gives only the purpose,
 *                       speculative decoding; this is the library's reading)
 *   scale_value         the page's query scale (1.0 is its default)
 *   out                 [B, H_v, T, D_v]  bf16, fully written
 *   stream              CUDA stream the work is queued on
 *
 * Returns a gdr_status.
 */
GDR_API int gdr_decode(const gdr_dims* dims, const gdr_bf16* query, const gdr_bf16* key,
                       const gdr_bf16* value, const gdr_bf16* beta, gdr_bf16* state_pool,
                       const int32_t* actual_seq_lengths, const int32_t* ssm_state_indices,
                       const float* g, const float* gk, const int32_t* num_accepted_tokens,
                       float scale_value, gdr_bf16* out, gdr_stream_t stream);

/*
 * gdr_gate_fused - gdr_decode with the LinearAttentionGate computed in the
 * kernel ("com.microsoft.LinearAttentionGate", sections Description and
 * Inputs): per token and value head, in fp32,
 *   g    = decay_scale[h] * softplus(a[b,t,h] + dt_bias[h])
 *   beta = sigmoid(b[b,t,h])
 * The gate values stay in fp32 registers; nothing narrows them.
 *
 *   a, b         [B, T, H_v] bf16 (heads on the last axis)
 *   dt_bias      [H_v] fp32
 *   decay_scale  [H_v] fp32 (for gated DeltaNet, -exp(A_log))
 * Every other argument is as for gdr_decode; there is no g and no beta.
 * Returns a gdr_status.
 */
GDR_API int gdr_gate_fused(const gdr_dims* dims, const gdr_bf16* query, const gdr_bf16* key,
                           const gdr_bf16* value, const gdr_bf16* a, const gdr_bf16* b,
                           const float* dt_bias, const float* decay_scale, gdr_bf16* state_pool,
                           const int32_t* actual_seq_lengths, const int32_t* ssm_state_indices,
                           const float* gk, const int32_t* num_accepted_tokens,
                           float scale_value, gdr_bf16* out, gdr_stream_t stream);

/*
 * gdr_prefill - the op's recurrence over a long prompt: the four steps of
 * "lite_boost.ops.recurrent_gated_delta_rule" (section 算法流程) for every
 * valid token, in token order. The page's op is decode-only and sends prefill
 * to a chunk-level op (section 注); this entry point computes the same
 * result for any token count, with the arguments of gdr_decode.
 *
 * Arguments, layouts, ownership and the treatment of lengths, slots and
 * committed counts are those of gdr_decode, except:
 *   T                   any T >= 1 (the padded token count of the call);
 *   sizes               D_k = 128, D_v a multiple of 128, dims->layout =
 *                       GDR_LAYOUT_KV; other sizes return GDR_ERR_UNSUPPORTED;
 *   precision           the state is carried in fp32 across all L valid tokens
 *                       of an item and rounded to bf16 once, as in gdr_decode;
 *                       inside a chunk of 8 tokens the tensor-core products
 *                       read the state as bf16 hi + lo parts (16 significant
 *                       bits) and the per-token vectors likewise;
 *   num_accepted_tokens as for gdr_decode: the slot receives the state after
 *                       the first n tokens, the outputs of all L tokens are
 *                       computed.
 * Tensor memory: a launch takes all 512 columns of each SM it runs on for its
 * duration (see gdr_decode's kernels: one CTA per SM, freed before exit), so
 * it must not share an SM with another kernel that holds tensor memory.
 * Returns a gdr_status.
 */
GDR_API int gdr_prefill(const gdr_dims* dims, const gdr_bf16* query, const gdr_bf16* key,
                        const gdr_bf16* value, const gdr_bf16* beta, gdr_bf16* state_pool,
                        const int32_t* actual_seq_lengths, const int32_t* ssm_state_indices,
                        const float* g, const float* gk, const int32_t* num_accepted_tokens,
                        float scale_value, gdr_bf16* out, gdr_stream_t stream);

/*
 * gdr_prefill_gated - gdr_prefill with the LinearAttentionGate computed in
 * the kernel, as for gdr_gate_fused ("com.microsoft.LinearAttentionGate",
 * section Description): a, b [B, T, H_v] bf16, dt_bias and decay_scale [H_v]
 * fp32 in place of g and beta. Returns a gdr_status.
 */
GDR_API int gdr_prefill_gated(const gdr_dims* dims, const gdr_bf16* query, const gdr_bf16* key,
                              const gdr_bf16* value, const gdr_bf16* a, const gdr_bf16* b,
                              const float* dt_bias, const float* decay_scale,
                              gdr_bf16* state_pool, const int32_t* actual_seq_lengths,
                              const int32_t* ssm_state_indices, const float* gk,
                              const int32_t* num_accepted_tokens, float scale_value,
                              gdr_bf16* out, gdr_stream_t stream);

/* Element types of the standalone gate's a, b, decay and beta. */
typedef enum gdr_dtype {
  GDR_DTYPE_F32 = 0,  /* float32, one of the gate page's types (Type constraints) */
  GDR_DTYPE_F16 = 1,  /* float16, the other one */
  GDR_DTYPE_BF16 = 2  /* bfloat16, the decode op's storage type (an extension) */
} gdr_dtype;

/*
 * gdr_linear_attention_gate - the LinearAttentionGate op on its own
 * ("com.microsoft.LinearAttentionGate", sections Description, Inputs, Outputs
 * and Type constraints). For every element, in float32:
 *   decay = decay_scale[h] * softplus(a + dt_bias[h])
 *   beta  = sigmoid(b)                      (only when beta is requested)
 * narrowed to `dtype` on store (round to nearest even). h is the index on the
 * last axis; every leading axis is folded into `rows`.
 *
 *   a            [rows, H] of `dtype`
 *   b            [rows, H] of `dtype`, or NULL; read only when beta is requested
 *   dt_bias      [H] fp32
 *   decay_scale  [H] fp32 (for gated DeltaNet, -exp(A_log))
 *   decay        [rows, H] of `dtype`, written
 *   beta         [rows, H] of `dtype`, written; NULL when beta is not requested
 *   rows, H      rows >= 0, 1 <= H
 *   dtype        a gdr_dtype
 *   stream       CUDA stream the work is queued on
 *
 * All pointers are device memory owned by the caller; any alignment works
 * (16-byte aligned tensors take the vector path). Errors, checked on the host
 * before anything is queued: GDR_ERR_NULL if a, dt_bias, decay_scale or decay is
 * NULL, or if beta is requested without b (the page's rule); GDR_ERR_DIMS for
 * rows < 0, H < 1 or rows * H >= 2^62; GDR_ERR_UNSUPPORTED for an unknown
 * dtype. rows = 0 queues nothing. Returns a gdr_status.
 */
GDR_API int gdr_linear_attention_gate(const void* a, const void* b, const float* dt_bias,
                                      const float* decay_scale, void* decay, void* beta,
                                      int64_t rows, int32_t H, int dtype, gdr_stream_t stream);

/* Static English name of a gdr_status value ("GDR_OK", ...); "unknown status"
 * for other values. Never NULL. */
GDR_API const char* gdr_status_string(int status);

/* Description of the most recent failed call made by the calling thread
 * (which check failed, or the CUDA error string); "" if none failed yet. The
 * pointer stays valid until the thread's next call into the library. */
GDR_API const char* gdr_last_error(void);

/* Device-side error word of the current device, OR-ed over every kernel run
 * since the last reset: bit 0 = a consumer's wait for a ready tile ran out of
 * time, bit 1 = a wait on the producing side (a free stage, or landed copies
 * to prepare) ran out of time, bit 2 = the final wait for in-flight copies ran
 * out of time. A wait that runs out never
 * hangs the kernel: it flags the word and the kernel finishes, and the outputs
 * of that call are invalid. Writes the word to *flags and clears it when
 * `reset` is nonzero. SYNCHRONISES the device (a blocking copy). No
 * counterpart on the pages: every bounded wait of the kernels reports here. */
GDR_API int gdr_device_error(uint32_t* flags, int reset);

/* Kernel families of the library (gdr_launch_info.kernel). */
typedef enum gdr_kernel {
  GDR_KERNEL_NONE = 0,
  GDR_KERNEL_SINGLE_TOKEN = 1,     /* one token per call, CUDA cores */
  GDR_KERNEL_CHUNKED = 2,          /* several tokens, CUDA cores */
  GDR_KERNEL_TENSOR_CORE = 3,      /* D_k = 128, D_v a multiple of 128, several tokens */
  GDR_KERNEL_TENSOR_CORE_ONE = 4,  /* the same kernel's form for one token per call */
  GDR_KERNEL_GATE = 5,             /* the standalone gate */
  GDR_KERNEL_PREFILL = 6,          /* gdr_prefill / gdr_prefill_gated */
  GDR_KERNEL_ROWS = 7              /* one token on a k-contiguous pool, one row per lane group */
} gdr_kernel;

/* One kernel launch: its family, the key width, the column width of a tile
 * (the rows of a warp's block for GDR_KERNEL_ROWS; 0 for the gate), whether
 * the gate is fused, the pool layout, and the launch shape (blocks, threads
 * per block, dynamic shared memory, pipeline stages). */
typedef struct gdr_launch_info {
  int32_t kernel;
  int32_t D_k;
  int32_t tile_cols;
  int32_t gated;
  int32_t layout;
  int32_t grid;
  int32_t threads;
  int32_t smem_bytes;
  int32_t stages;
} gdr_launch_info;

/* The most recent kernel launch the calling thread made through the library
 * (kernel = GDR_KERNEL_NONE before the first one, and for a call that queued
 * nothing, such as B = 0). Host-only; no counterpart on the pages: it lets a
 * caller or a test see which kernel and tile width the dispatcher chose.
 * Returns GDR_ERR_NULL for a NULL `info`, else GDR_OK. */
GDR_API int gdr_last_launch(gdr_launch_info* info);

/* The decode kernel forms the dispatcher can choose, as (kernel, D_k,
 * tile_cols, gated, layout); the launch-shape fields are 0. gdr_kernel_form
 * fills form `i`, 0 <= i < gdr_kernel_form_count(), and returns GDR_ERR_DIMS
 * for any other i. Host-only, needs no GPU; no counterpart on the pages. */
GDR_API int gdr_kernel_form_count(void);
GDR_API int gdr_kernel_form(int i, gdr_launch_info* info);

/* Library ABI version, currently 6 (2 added gdr_linear_attention_gate, 3 the
 * layout field of gdr_dims, 4 gdr_last_launch and the kernel forms, 5
 * gdr_prefill and gdr_prefill_gated, 6 the GDR_KERNEL_ROWS form). */
GDR_API int gdr_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H_ */
