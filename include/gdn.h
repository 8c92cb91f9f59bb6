/*
 * gdn.h -- C ABI of libgdn.so, a B200 (sm_100a) implementation of the Gated DeltaNet
 * linear-attention layer of the Qwen3-Next hybrid stack.
 *
 * Sources for what is computed:
 *   - layer constants: "Qwen3-Coder-Next" model card (llm-atlas), raw config.json fields
 *     (linear_conv_kernel_dim 4, linear_num_key_heads 16, linear_num_value_heads 32,
 *     linear_key_head_dim = linear_value_head_dim = 128, rms_norm_eps 1e-6, hidden_act silu);
 *   - the token mixer: hyper.ai story on Qwen3-Next in Transformers, Gated DeltaNet paragraph
 *     (QKV plus a Z projection, causal convolution for local context, beta gating the update
 *     strength, kv_mem as the prior knowledge read from the recurrent state, linear cost through
 *     a recurrent state update, zero-centred RMSNorm);
 *   - state size independent of the sequence: Qwen3.5 teardown (rkmt.cn), section 3.2;
 *   - fp32 recurrent state by default, chunked FLA kernels with chunk 64 as prior art:
 *     "Qwen3-Next" SGLang cookbook, section 3.2 Configuration Tips.
 * Per token t of a sequence (value head h reads key head h / (Hv/Hk)):
 *   y     = silu(causal depthwise conv_K(x))          (x = [q | k | v] projections)
 *   q     = q~ / sqrt(|q~|^2 + l2_eps) * q_scale,   k = k~ / sqrt(|k~|^2 + l2_eps)
 *   S_t   = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   alpha_t = exp(g_t)
 *   o_t   = S_t q_t
 *   out_t = o_t / sqrt(mean(o_t^2) + norm_eps) * w * silu(z_t)       (when z is given)
 *
 * General rules for every call:
 *   - Pointers are DEVICE pointers owned by the caller unless a comment says "host".  The
 *     library allocates no device memory of its own, except where an entry point says so
 *     (gdn_chunk_prefill_static_ws: a static array).  Its multi-stream paths create CUDA
 *     streams and events once per host thread and device and keep them; debug settings
 *     (gdn_debug_set) and an attached trace are per host thread; no other state survives a
 *     call.
 *   - Tensors are dense, row-major, contiguous and 16-byte aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *   - Return value: GDN_OK, or a negative gdn_status.  On argument errors nothing is launched
 *     and no memory is touched.  GDN_ERR_CUDA reports a failed launch (cudaGetLastError).
 *   - Supported shapes: head_dim 128, conv_kernel 4, num_v_heads a multiple of num_k_heads.
 *     Other values return GDN_ERR_UNSUPPORTED.
 *   - Activations use one dtype per call (gdn_dtype); the recurrent state is always fp32
 *     [.., Hv, d_v, d_k] with row = value index.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDN_ABI_VERSION 2

typedef enum gdn_status {
  GDN_OK = 0,
  GDN_ERR_INVALID_ARG = -1, /* null/misaligned pointer, negative size, bad cu_seqlens shape;
                               on the device: a slot index outside its pool */
  GDN_ERR_UNSUPPORTED = -2, /* shape or dtype this build does not implement */
  GDN_ERR_CUDA = -3,        /* a CUDA runtime call or kernel launch failed */
  GDN_ERR_TIMEOUT = -4,     /* written to dev_status by a device wait that ran out */
  GDN_ERR_WORKSPACE = -5,   /* workspace missing or smaller than *_workspace_size() */
  GDN_ERR_BOUNDS = -6       /* bounds-check build only (libgdn_checked.so, compiled with
                               -DGDN_BOUNDS_CHECK): a kernel index check failed and the access
                               was skipped; never reported by the normal build */
} gdn_status;

typedef enum gdn_dtype { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

/* Layer shape.  Qwen3-Next: {16, 32, 128, 4, 1.0f, 1e-6f, 1e-6f}. */
typedef struct gdn_dims {
  int32_t num_k_heads; /* Hk: query/key heads */
  int32_t num_v_heads; /* Hv: value heads (state heads), multiple of Hk */
  int32_t head_dim;    /* d = d_k = d_v (128) */
  int32_t conv_kernel; /* K, causal conv width (4) */
  float q_scale;       /* multiplies the L2-normalised q (1.0) */
  float l2_eps;        /* inside the square root of the q/k L2 norm (1e-6) */
  float norm_eps;      /* inside the square root of the gated RMSNorm (1e-6) */
} gdn_dims;

/* Conv channel count Cc = (2*Hk + Hv) * d, in the order [q (Hk*d) | k (Hk*d) | v (Hv*d)]. */
int64_t gdn_conv_channels(const gdn_dims* dims);

/* Human-readable text of a status code (static string, never NULL). */
const char* gdn_status_string(int status);

/*
 * gdn_conv1d_update -- causal depthwise conv (width K, no bias) + SiLU over packed sequences.
 * Source: the causal convolution of the hyper.ai Gated DeltaNet paragraph; width from
 * linear_conv_kernel_dim in the Qwen3-Coder-Next raw config.json fields.
 *   x          [T, Cc]       input rows of all sequences, packed
 *   y          [T, Cc]       out: y[t,c] = silu(sum_i w[c,i] * x_{t-K+1+i}[c]); may not alias x
 *   conv_w     [Cc, K]       tap K-1 multiplies the current token
 *   cu_seqlens [N+1] int32   device; 0 = cu[0] <= cu[1] <= ... <= cu[N] = T
 *   conv_state_in  [N, K-1, Cc] nullable (= zeros): row j holds x_{j-K+1} of the sequence
 *   conv_state_out [N, K-1, Cc] nullable: last K-1 rows of [state_in ; x_seq]; may equal
 *                  conv_state_in (in-place update).
 * T = 1 per sequence is the decode-time update.
 */
int gdn_conv1d_update(const gdn_dims* dims, gdn_dtype dtype, const void* x, void* y,
                      const void* conv_w, const int32_t* cu_seqlens, int32_t num_seqs,
                      int32_t num_tokens, const void* conv_state_in, void* conv_state_out,
                      void* stream);

/*
 * gdn_gated_rmsnorm -- y = o / sqrt(mean(o^2) + eps) * w * silu(z), per row of `dim`.
 * Source: the z projection and zero-centred RMSNorm of the hyper.ai Gated DeltaNet
 * paragraph; eps from rms_norm_eps (Qwen3-Coder-Next raw config.json fields).  `w` is the
 * effective weight (a zero-centred parameterisation passes 1 + w); NULL means ones.
 *   o, z, y [rows, dim] (y may equal o), w [dim]; dim a multiple of 8, at most 1024.
 */
int gdn_gated_rmsnorm(gdn_dtype dtype, const void* o, const void* z, const void* w, float eps,
                      int32_t rows, int32_t dim, void* y, void* stream);

/*
 * gdn_chunk_prefill -- the whole layer over packed variable-length sequences, chunked.
 * Source: the recurrence in the file header; chunked (WY / UT transform) evaluation as in the
 * FLA kernels named in the "Qwen3-Next" SGLang cookbook, section 3.2 (this build uses its own
 * chunk size).  bf16 runs on tcgen05 tensor cores; fp32 runs an fp32 SIMT recurrence.
 *   x        [T, Cc]          pre-conv q|k|v projections
 *   conv_w   [Cc, K]          nullable: conv + SiLU switched off (x used as is)
 *   beta     [T, Hv] fp32     update strength
 *   g        [T, Hv] fp32     log alpha (<= 0)
 *   z        [T, Hv, d]       nullable: gated RMSNorm switched off (out = o)
 *   norm_w   [d]              nullable: ones
 *   cu_seqlens [N+1] int32    device, as for gdn_conv1d_update
 *   S0       [N, Hv, d, d] fp32  nullable: zero initial states
 *   SN       [N, Hv, d, d] fp32  nullable: final states (may equal S0)
 *   conv0    [N, K-1, Cc]     nullable: zero conv history
 *   convN    [N, K-1, Cc]     nullable: final conv history (may equal conv0)
 *   out      [T, Hv, d]
 *   workspace, workspace_bytes: device scratch of at least
 *            gdn_chunk_prefill_workspace_size(dims, dtype, N, T) bytes, 256-byte aligned.
 *   dev_status  int32, nullable: set to GDN_ERR_TIMEOUT if a device wait ran out (the caller
 *            zeroes it and reads it after synchronising).
 */
size_t gdn_chunk_prefill_workspace_size(const gdn_dims* dims, gdn_dtype dtype, int32_t num_seqs,
                                        int32_t num_tokens);
int gdn_chunk_prefill(const gdn_dims* dims, gdn_dtype dtype, const void* x, const void* conv_w,
                      const float* beta, const float* g, const void* z, const void* norm_w,
                      const int32_t* cu_seqlens, int32_t num_seqs, int32_t num_tokens,
                      const float* S0, float* SN, const void* conv0, void* convN, void* out,
                      void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * gdn_chunk_prefill_states -- gdn_chunk_prefill that also returns the recurrent state after
 * every chunk (128 tokens, the last chunk of a sequence possibly shorter).
 * Source: the "Qwen3-Next" SGLang cookbook, section 3.2: the radix cache of the hybrid GDN
 * layers keeps states at branching points, with a page size that divides or is divided by the
 * kernel's chunk; a prefill that emits the chunk-boundary states supplies them.
 *   chunk_states [C, Hv, d, d] fp32 (layout as SN), C = sum over sequences of ceil(L_n / 128);
 *     entry c is the state after chunk c, chunks numbered sequence by sequence (sequence n's
 *     chunk j, covering its tokens [128 j, min(128 (j + 1), L_n)), is c = j + sum_{m<n}
 *     ceil(L_m / 128)); required when num_tokens > 0, 16-byte aligned.  The entry of a
 *     sequence's last chunk equals its final state.
 * bf16 only (GDN_ERR_UNSUPPORTED for GDN_F32).  Every other argument, the workspace size and
 * the status codes are those of gdn_chunk_prefill.  The extra cost is the write of C Hv d^2 fp32.
 */
int gdn_chunk_prefill_states(const gdn_dims* dims, gdn_dtype dtype, const void* x,
                             const void* conv_w, const float* beta, const float* g,
                             const void* z, const void* norm_w, const int32_t* cu_seqlens,
                             int32_t num_seqs, int32_t num_tokens, const float* S0, float* SN,
                             const void* conv0, void* convN, void* out, float* chunk_states,
                             void* workspace, size_t workspace_bytes, int32_t* dev_status,
                             void* stream);

/*
 * gdn_chunk_prefill_pages -- gdn_chunk_prefill_states for a cache page of 64 or 128 tokens.
 * Source: the "Qwen3-Next" SGLang cookbook, section 3.2, radix cache for the hybrid layers: its
 * example serves with --page-size 64, and the page size must divide the linear-attention
 * kernel's chunk or be a multiple of it; with this library's 128-token chunk, pages of 64 need
 * the state in the middle of every chunk as well.
 *   page_size     64 or 128 (GDN_ERR_UNSUPPORTED otherwise).  128: the result of
 *                 gdn_chunk_prefill_states.
 *   page_states   [P, Hv, d, d] fp32, P = sum over sequences of ceil(L_n / page_size): entry p is
 *                 the state after page p, pages numbered sequence by sequence (sequence n's page
 *                 j covers its tokens [page_size j, min(page_size (j + 1), L_n))); the entry of a
 *                 sequence's last page equals its final state.  Required when num_tokens > 0.
 * With 64, the chain adds for each chunk of more than 64 tokens the state after its first 64:
 * e^(G_63) S_c + K[0:64]^T diag(e^(G_63 - G_i)) U[0:64] (the chunk's own U, fp32 accumulation).
 * bf16 only.  Other arguments, the workspace size and the status codes: gdn_chunk_prefill.
 */
int gdn_chunk_prefill_pages(const gdn_dims* dims, gdn_dtype dtype, const void* x,
                            const void* conv_w, const float* beta, const float* g, const void* z,
                            const void* norm_w, const int32_t* cu_seqlens, int32_t num_seqs,
                            int32_t num_tokens, const float* S0, float* SN, const void* conv0,
                            void* convN, void* out, int32_t page_size, float* page_states,
                            void* workspace, size_t workspace_bytes, int32_t* dev_status,
                            void* stream);

/*
 * gdn_chunk_prefill_host -- gdn_chunk_prefill (bf16) with the per-token tensors in host memory.
 * Source: as gdn_chunk_prefill.  The packed batch is cut into segments of about segment_tokens
 * tokens, ending at sequence ends or 128-token chunk boundaries of a sequence; the copy of one
 * segment's inputs to the device, the layer on the previous segment and the copy of the output
 * before that back to the host overlap on the library's two copy streams and `stream`.  A
 * sequence cut between segments carries its fp32 state and conv history from one to the next,
 * so the result equals one gdn_chunk_prefill call on device copies of the same inputs.
 *   x [T, Cc], beta, g [T, Hv] fp32, z [T, Hv, d] (nullable), out [T, Hv, d]: HOST memory
 *     (page-locked for the copies to overlap; pageable memory works, serialised).
 *   cu_seqlens_host [N+1] int32: HOST memory, cu[0] = 0, non-decreasing, cu[N] = T.
 *   conv_w, norm_w, S0, SN, conv0, convN, dev_status: device, as gdn_chunk_prefill.
 *   segment_tokens: a multiple of 128, or 0 for the library's choice (T / 8 rounded up to 128,
 *     at least 512).
 *   workspace: device, gdn_chunk_prefill_host_workspace_size() bytes, 256-byte aligned (it
 *     holds device copies of the per-token tensors).
 * Asynchronous on `stream`: the host buffers may be reused, and out read, once `stream` has
 * reached the point of the call.  This holds on error returns too: copies queued before the
 * error still read or write the host buffers, and `stream` waits for them.  Not for stream
 * capture (the copy streams are the library's).
 * Status codes as gdn_chunk_prefill; GDN_ERR_UNSUPPORTED unless Hv = 2 Hk and Hv % 4 == 0.
 * gdn_chunk_prefill_host_plan writes the segments (first sequence, sequences, first token,
 * tokens; four int32 each) into `segments` and returns their number (or a status < 0;
 * GDN_ERR_WORKSPACE when max_segments is too small; segments may be NULL to count).
 */
int32_t gdn_chunk_prefill_host_plan(const int32_t* cu_seqlens_host, int32_t num_seqs,
                                    int32_t num_tokens, int32_t segment_tokens,
                                    int32_t* segments, int32_t max_segments);
size_t gdn_chunk_prefill_host_workspace_size(const gdn_dims* dims, const int32_t* cu_seqlens_host,
                                             int32_t num_seqs, int32_t num_tokens,
                                             int32_t segment_tokens);
int gdn_chunk_prefill_host(const gdn_dims* dims, const void* x, const void* conv_w,
                           const float* beta, const float* g, const void* z, const void* norm_w,
                           const int32_t* cu_seqlens_host, int32_t num_seqs, int32_t num_tokens,
                           const float* S0, float* SN, const void* conv0, void* convN, void* out,
                           int32_t segment_tokens, void* workspace, size_t workspace_bytes,
                           int32_t* dev_status, void* stream);

/*
 * gdn_chunk_prefill_slots -- gdn_chunk_prefill whose initial and final states live in a state
 * pool shared with gdn_decode_step: sequence n reads and overwrites row slot_idx[n] of the pools.
 * Source: the "Qwen3-Next" SGLang cookbook, section 3.2 (the mamba state cache of the hybrid GDN
 * layers, one cached state per request slot, fp32 by default).
 *   slot_idx  [N] int32 device, nullable (= identity); the slots of one call must be distinct.
 *   num_slots rows of the pools (>= N when slot_idx is NULL).  The kernels check every slot
 *             against it: a sequence whose slot lies outside [0, num_slots) starts from zero
 *             states, writes no state and sets dev_status to GDN_ERR_INVALID_ARG (its outputs
 *             are computed from the zero states); no pool row outside the range is touched.
 *   S_pool    [slots, Hv, d, d] fp32, in/out, required when N > 0.
 *   conv_pool [slots, K-1, Cc] (activation dtype), in/out, nullable: zero conv history, none kept.
 * Every other argument, the workspace size and the status codes are those of gdn_chunk_prefill;
 * the result equals gdn_chunk_prefill with S0 = SN = S_pool[slot_idx] and conv0 = convN =
 * conv_pool[slot_idx], pool rows outside slot_idx untouched.
 */
int gdn_chunk_prefill_slots(const gdn_dims* dims, gdn_dtype dtype, const void* x,
                            const void* conv_w, const float* beta, const float* g, const void* z,
                            const void* norm_w, const int32_t* cu_seqlens, int32_t num_seqs,
                            int32_t num_tokens, const int32_t* slot_idx, int32_t num_slots,
                            float* S_pool, void* conv_pool, void* out, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * gdn_decode_step -- one token for each of B sequences; conv and recurrent state in place.
 * Source: as gdn_chunk_prefill with T = 1 per sequence; states resident in a slot pool, fp32
 * recurrent state as the "Qwen3-Next" SGLang cookbook's default --mamba-ssm-dtype.
 *   x [B, Cc], beta/g [B, Hv] fp32, z [B, Hv, d] nullable, conv_w [Cc, K] (required),
 *   norm_w [d] nullable, conv_state [slots, K-1, Cc] in/out, S [slots, Hv, d, d] fp32 in/out,
 *   slot_idx [B] int32 device, nullable (= identity); slots of one call must be distinct.
 *   num_slots  rows of conv_state and S (>= B when slot_idx is NULL).  A sequence whose slot lies
 *     outside [0, num_slots) is skipped on the device: no state access, its out rows are not
 *     written, and dev_status (int32, nullable) is set to GDN_ERR_INVALID_ARG.
 *   out [B, Hv, d].
 * One pass over the state: it is read once and written once.
 */
int gdn_decode_step(const gdn_dims* dims, gdn_dtype dtype, const void* x, const void* conv_w,
                    const float* beta, const float* g, const void* z, const void* norm_w,
                    void* conv_state, float* S, const int32_t* slot_idx, int32_t num_slots,
                    int32_t batch, void* out, int32_t* dev_status, void* stream);

/*
 * gdn_block_prefill -- the token mixer of a Gated DeltaNet decoder layer: input projections,
 * gates, gdn_chunk_prefill and the output projection, bf16 activations and weights.
 * Source: the hyper.ai Qwen3-Next paragraph (QKV and a separate Z projection around the gated
 * delta rule) and the Qwen3-Coder-Next config table (hidden_size 2048).  The gate formulas are
 * not on the pages; this library reads them as beta = sigmoid(b), g = log(alpha) =
 * -exp(A_log) * softplus(a + dt_bias) per value head.
 *   h [T, H]; w_qkv [H, Cc], w_z [H, Hv d], w_ba [H, 2 Hv] (columns: b for the Hv heads, then
 *   a), all row-major (input x output); a_log, dt_bias [Hv] fp32; w_out [Hv d, H]; y [T, H].
 *   conv_w, norm_w, cu_seqlens, S0, SN, conv0, convN, dev_status: as gdn_chunk_prefill.
 *   workspace: at least gdn_block_prefill_workspace_size() bytes, 256-byte aligned.
 * The four projections run on the library's own tcgen05 GEMM (bf16 operands, fp32
 * accumulation in TMEM): the [b | a] projection computes the gates in its epilogue (beta and g
 * never leave the GEMM as b and a); the q|k|v, z and output projections round to bf16.
 * GDN_ERR_UNSUPPORTED when 2 Hv > 64 (the gate GEMM's tile width).
 */
size_t gdn_block_prefill_workspace_size(const gdn_dims* dims, int32_t hidden, int32_t num_seqs,
                                        int32_t num_tokens);
int gdn_block_prefill(const gdn_dims* dims, int32_t hidden, const void* h, const void* w_qkv,
                      const void* w_z, const void* w_ba, const float* a_log, const float* dt_bias,
                      const void* conv_w, const void* norm_w, const void* w_out,
                      const int32_t* cu_seqlens, int32_t num_seqs, int32_t num_tokens,
                      const float* S0, float* SN, const void* conv0, void* convN, void* y,
                      void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * gdn_decode_multi -- k tokens for each of B sequences in one call: the verification step of
 * speculative decoding with multi-token prediction.
 * Source: the "Qwen3-Next" SGLang cookbook, section 4.2.4 (MTP / NEXTN speculative decoding,
 * 4 draft tokens per step).  The result is that of k calls of gdn_decode_step on tokens
 * 0..k-1 in order (the same fp32 arithmetic per token): outputs of every token, conv and
 * recurrent state after token k-1.  The state rows are read and written once for all k tokens.
 *   x [B, k, Cc], beta/g [B, k, Hv] fp32, z [B, k, Hv, d] nullable, out [B, k, Hv, d];
 *   conv_w, norm_w, conv_state, S (fp32), slot_idx, num_slots, dev_status as gdn_decode_step;
 *   0 <= k <= 8
 *   (GDN_ERR_UNSUPPORTED above 8; k = 0 or B = 0 launch nothing).
 *   snapshots [B, k, Hv, d, d] fp32, nullable: the recurrent state after each token, indexed by
 *     position in the call (not by slot), for a caller that accepts only the first m tokens
 *     (it restores snapshot m - 1; the conv history after m tokens is the last 3 rows of the
 *     old history followed by x[b, 0..m-1]).
 */
int gdn_decode_multi(const gdn_dims* dims, gdn_dtype dtype, const void* x, const void* conv_w,
                     const float* beta, const float* g, const void* z, const void* norm_w,
                     void* conv_state, float* S, const int32_t* slot_idx, int32_t num_slots,
                     int32_t batch, int32_t tokens, void* out, float* snapshots,
                     int32_t* dev_status, void* stream);

/*
 * gdn_decode_step_bf16_state -- gdn_decode_step with the recurrent state stored in bf16.
 * Source: the "Qwen3-Next" SGLang cookbook, section 3.2: --mamba-ssm-dtype selects bf16 or fp32
 * (the default) for the recurrent state of the GDN layers.  Each step reads the bf16 state,
 * does all arithmetic in fp32 exactly as gdn_decode_step, and rounds the new state to bf16
 * (round to nearest even) once when it is written back: half the state bytes of the fp32 call.
 *   S [slots, Hv, d, d] bf16 in/out (16-byte aligned); every other argument, the layout, the
 *   ownership and the status codes are those of gdn_decode_step.
 */
int gdn_decode_step_bf16_state(const gdn_dims* dims, gdn_dtype dtype, const void* x,
                               const void* conv_w, const float* beta, const float* g,
                               const void* z, const void* norm_w, void* conv_state, void* S,
                               const int32_t* slot_idx, int32_t num_slots, int32_t batch,
                               void* out, int32_t* dev_status, void* stream);

/*
 * gdn_chunk_prefill_static_ws -- gdn_chunk_prefill for callers that cannot allocate device
 * memory.  No counterpart on the source pages: this is a deployment aid of this library.
 * Some callers have no way to obtain a device workspace: extensions loaded into a host
 * framework that owns every device allocation and lends none to plugins, C programs without a
 * caching allocator, and latency-critical loops that must not pay the implicit device
 * synchronisation of cudaMalloc/cudaFree.  This entry point takes the same arguments as
 * gdn_chunk_prefill minus workspace/workspace_bytes and allocates nothing: its scratch is a
 * file-scope device array of GDN_STATIC_WORKSPACE_BYTES (64 MiB) inside libgdn.so, which every
 * GPU that loads the library holds until the process exits.
 *   - Sizes whose gdn_chunk_prefill_workspace_size() exceeds GDN_STATIC_WORKSPACE_BYTES return
 *     GDN_ERR_WORKSPACE and launch nothing (for the Qwen3-Next shape, one sequence of up to
 *     1,791 tokens, or fewer tokens spread over more sequences).
 *   - The first call on each device looks the array's device address up (cudaGetSymbolAddress,
 *     with that device current) and caches it; make that first call before any stream capture.
 *     The cached address belongs to the device context of that first call: do not call this
 *     entry point again after a cudaDeviceReset (or any reset of the primary context) in the
 *     same process.
 *   - All calls share the one array and it keeps the previous call's contents (nothing in it
 *     needs to start at zero).  Calls that overlap on the GPU (different streams, or different
 *     host threads on one device) race on it and must be serialised by the caller.
 * Other arguments, results and status codes are those of gdn_chunk_prefill.
 */
#define GDN_STATIC_WORKSPACE_BYTES (64u << 20)
int gdn_chunk_prefill_static_ws(const gdn_dims* dims, gdn_dtype dtype, const void* x,
                                const void* conv_w, const float* beta, const float* g,
                                const void* z, const void* norm_w, const int32_t* cu_seqlens,
                                int32_t num_seqs, int32_t num_tokens, const float* S0, float* SN,
                                const void* conv0, void* convN, void* out, int32_t* dev_status,
                                void* stream);

/*
 * Launch tracing (host-side measurement aid, not on the compute path).  While a trace is
 * attached to the calling host thread, every kernel the library launches from that thread is
 * bracketed by two CUDA events recorded on the launch stream.  After synchronising, read the
 * per-launch device times.  A trace holds up to 4096 launches; further ones are not recorded.
 * Launches made while the stream is being captured into a CUDA graph get their two events as
 * event-record nodes of that graph: each replay records them again, so after a replay (and a
 * synchronisation) gdn_trace_get returns the times of that replay's launches.
 */
typedef struct gdn_trace gdn_trace;
int gdn_trace_create(gdn_trace** out);         /* host object, owned by the caller */
int gdn_trace_destroy(gdn_trace* trace);
int gdn_trace_attach(gdn_trace* trace);        /* NULL detaches; per host thread */
int gdn_trace_reset(gdn_trace* trace);
int gdn_trace_count(const gdn_trace* trace);   /* launches recorded */
/* name: static kernel name; ms: device time of launch i (synchronises on its end event). */
int gdn_trace_get(gdn_trace* trace, int32_t i, const char** name, float* ms);
/* Start and end of launch i in ms after the start of launch 0 of the same trace (launches on
 * different streams overlap on this common time line).  Synchronises on both end events. */
int gdn_trace_span(gdn_trace* trace, int32_t i, float* start_ms, float* end_ms);

/*
 * gdn_debug_set -- debug and test controls, not needed for normal use.  The settings apply to
 * the calls the calling host thread makes afterwards (the library copies *opts); NULL restores
 * the defaults (all fields zero).  Workspace sizes depend on segment_chunks: query them with
 * the same settings as the call.
 *   wait_limit_us  bound of every device wait of the prefill kernels, in microseconds (0: 2 s).
 *                  A wait that runs out writes GDN_ERR_TIMEOUT to dev_status, lets the copies
 *                  and products it has in flight land, frees its TMEM and ends its CTA.
 *   segment_chunks length in 128-token chunks of the segments the bf16 prefill pipelines over
 *                  its streams (0: the library's choice, 64 from 512 chunks on, else one).
 *   chain_split    d_v blocks per state in the sequential chain kernel: 1, 2 or 4 (0: the
 *                  library's choice).
 *   fault          GDN_FAULT_NONE, or GDN_FAULT_SKIP_CHAIN_LOAD: the first CTA of the chain
 *                  kernel does not issue the load of chunk fault_chunk's W tile (chunk index of
 *                  the call's table, sequence by sequence), so its bounded wait for that tile
 *                  runs out.  Used to test the timeout path with no GPU fault: the call then
 *                  reports GDN_ERR_TIMEOUT in dev_status and its outputs are undefined.
 *   fault_chunk    see fault.
 *   timestamps     device pointer (uint64, 1024 entries) or NULL: the kernels of the bf16
 *                  prefill that support it record %globaltimer stamps of their phases there
 *                  (first CTA only), for profiling the pipeline of a persistent kernel.
 * Returns GDN_OK, or GDN_ERR_INVALID_ARG for an out-of-range field (settings unchanged).
 */
#define GDN_FAULT_NONE 0
#define GDN_FAULT_SKIP_CHAIN_LOAD 1
typedef struct gdn_debug_options {
  uint32_t wait_limit_us;
  int32_t segment_chunks;
  int32_t chain_split;
  int32_t fault;
  int32_t fault_chunk;
  uint64_t* timestamps;
} gdn_debug_options;
int gdn_debug_set(const gdn_debug_options* opts);

/*
 * gdn_debug_wait_probe -- test aid for the bounded device waits: launches one CTA that waits
 * on an mbarrier nothing will complete, with the given limit in microseconds (<= 10^6), and
 * writes GDN_ERR_TIMEOUT to dev_status when the wait gives up.  No fault, trap or hang.
 */
int gdn_debug_wait_probe(int32_t* dev_status, uint32_t limit_us, void* stream);

int gdn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
