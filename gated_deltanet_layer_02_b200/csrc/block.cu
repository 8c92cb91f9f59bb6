// block.cu -- the whole Gated DeltaNet token mixer of a decoder layer: input projections, the
// gates, the layer (gdn_chunk_prefill) and the output projection.
//
// Source: the hyper.ai Qwen3-Next paragraph (QKV and a separate Z projection around the gated
// delta rule, beta gating the update strength) and the llm-atlas Qwen3-Coder-Next config table
// (hidden_size 2048, 16 key / 32 value heads of 128).  The pages do not give the gate formulas;
// the reading here is beta = sigmoid(b) and g = log(alpha) = -exp(A_log) * softplus(a + dt_bias)
// per value head, with b and a the two halves of a [H, 2 Hv] projection (the same form as the
// synthetic g of the layer workloads, -exp(.) * softplus(.)).
//
// The projections run on this library's tcgen05 GEMM (gemm.cu): the [b | a] projection with
// the gates in its epilogue, the other three as plain bf16 GEMMs with fp32 accumulation.
#include <cuda_runtime.h>

#include "args.cuh"
#include "common.cuh"

namespace gdn_host {
cudaError_t gemm_bf16(const void* A, const void* B, void* C, int M, int N, int K,
                      int32_t* status, cudaStream_t s);
cudaError_t gemm_bf16_gates(const void* A, const void* B, int M, int Hv, int K,
                            const float* a_log, const float* dt_bias, float* beta, float* g,
                            int32_t* status, cudaStream_t s);
}  // namespace gdn_host

namespace {

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

struct BlockWs {
  size_t x, z, beta, g, o, layer, total;
};

BlockWs block_ws(const gdn_dims* d, int N, int T) {
  const size_t Cc = (size_t)(2 * d->num_k_heads + d->num_v_heads) * d->head_dim;
  const size_t Hv = d->num_v_heads, hd = d->head_dim;
  BlockWs w{};
  size_t o = 0;
  w.x = o; o = align256(o + (size_t)T * Cc * 2);
  w.z = o; o = align256(o + (size_t)T * Hv * hd * 2);
  w.beta = o; o = align256(o + (size_t)T * Hv * 4);
  w.g = o; o = align256(o + (size_t)T * Hv * 4);
  w.o = o; o = align256(o + (size_t)T * Hv * hd * 2);
  w.layer = o;
  o += gdn_chunk_prefill_workspace_size(d, GDN_BF16, N, T);
  w.total = o;
  return w;
}

}  // namespace

extern "C" {

size_t gdn_block_prefill_workspace_size(const gdn_dims* dims, int32_t hidden, int32_t num_seqs,
                                        int32_t num_tokens) {
  if (!dims || hidden <= 0 || num_seqs < 0 || num_tokens < 0) return 0;
  if (gdn_chunk_prefill_workspace_size(dims, GDN_BF16, num_seqs, num_tokens) == 0) return 0;
  return block_ws(dims, num_seqs, num_tokens).total;
}

int gdn_block_prefill(const gdn_dims* dims, int32_t hidden, const void* h, const void* w_qkv,
                      const void* w_z, const void* w_ba, const float* a_log, const float* dt_bias,
                      const void* conv_w, const void* norm_w, const void* w_out,
                      const int32_t* cu_seqlens, int32_t num_seqs, int32_t num_tokens,
                      const float* S0, float* SN, const void* conv0, void* convN, void* y,
                      void* workspace, size_t workspace_bytes, int32_t* dev_status,
                      void* stream) {
  if (!dims || hidden <= 0 || hidden % 8 != 0 || num_seqs < 0 || num_tokens < 0 ||
      (num_seqs == 0 && num_tokens > 0))
    return GDN_ERR_INVALID_ARG;
  const size_t need = gdn_block_prefill_workspace_size(dims, hidden, num_seqs, num_tokens);
  if (need == 0) return GDN_ERR_INVALID_ARG;
  if (num_tokens > 0 && (!h || !w_qkv || !w_z || !w_ba || !a_log || !dt_bias || !w_out || !y))
    return GDN_ERR_INVALID_ARG;
  if (num_seqs > 0 && !cu_seqlens) return GDN_ERR_INVALID_ARG;
  if (dims->num_v_heads != 2 * dims->num_k_heads) return GDN_ERR_UNSUPPORTED;  // the bf16 layer
  const void* ptrs[] = {h, w_qkv, w_z, w_ba, a_log, dt_bias, conv_w, norm_w, w_out, y, workspace};
  for (const void* p : ptrs)
    if (p && (reinterpret_cast<uintptr_t>(p) & 15u)) return GDN_ERR_INVALID_ARG;
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return GDN_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < need) return GDN_ERR_WORKSPACE;
  if (num_seqs == 0 || num_tokens == 0) {
    // no tokens: the layer still carries the states through
    return gdn_chunk_prefill(dims, GDN_BF16, nullptr, conv_w, nullptr, nullptr, nullptr, norm_w,
                             cu_seqlens, num_seqs, 0, S0, SN, conv0, convN, nullptr,
                             static_cast<uint8_t*>(workspace) + block_ws(dims, num_seqs, 0).layer,
                             workspace_bytes - block_ws(dims, num_seqs, 0).layer, dev_status,
                             stream);
  }
  if (2 * dims->num_v_heads > 64) return GDN_ERR_UNSUPPORTED;  // the gates GEMM's tile width
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const BlockWs l = block_ws(dims, num_seqs, num_tokens);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  const int T = num_tokens, H = hidden, Hv = dims->num_v_heads, d = dims->head_dim;
  const int Cc = (2 * dims->num_k_heads + Hv) * d;
  void* x = w + l.x;
  void* z = w + l.z;
  float* beta = reinterpret_cast<float*>(w + l.beta);
  float* g = reinterpret_cast<float*>(w + l.g);
  void* o = w + l.o;
  gdn_host::trace_begin("gemm_qkv", s);
  cudaError_t e = gdn_host::gemm_bf16(h, w_qkv, x, T, Cc, H, dev_status, s);
  gdn_host::trace_end(s);
  if (e == cudaSuccess) {
    gdn_host::trace_begin("gemm_z", s);
    e = gdn_host::gemm_bf16(h, w_z, z, T, Hv * d, H, dev_status, s);
    gdn_host::trace_end(s);
  }
  if (e == cudaSuccess) {
    gdn_host::trace_begin("gemm_ba_gates", s);
    e = gdn_host::gemm_bf16_gates(h, w_ba, T, Hv, H, a_log, dt_bias, beta, g, dev_status, s);
    gdn_host::trace_end(s);
  }
  if (e != cudaSuccess) return GDN_ERR_CUDA;
  int rc = gdn_chunk_prefill(dims, GDN_BF16, x, conv_w, beta, g, z, norm_w, cu_seqlens, num_seqs,
                             T, S0, SN, conv0, convN, o, w + l.layer, workspace_bytes - l.layer,
                             dev_status, stream);
  if (rc != GDN_OK) return rc;
  gdn_host::trace_begin("gemm_out", s);
  e = gdn_host::gemm_bf16(o, w_out, y, T, H, Hv * d, dev_status, s);
  gdn_host::trace_end(s);
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // extern "C"
