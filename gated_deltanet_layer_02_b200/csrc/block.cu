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
// The projections are plain bf16 GEMMs with fp32 accumulation and run in cuBLAS, which is
// loaded when this entry point is first used (libgdn.so does not link it).
#include <cublas_v2.h>
#include <cuda_runtime.h>
#include <dlfcn.h>

#include <mutex>

#include "args.cuh"
#include "common.cuh"

namespace gdn {

// beta = sigmoid(b), g = -exp(A_log) softplus(a + dt_bias); ba rows are [b (Hv) | a (Hv)].
__global__ void block_gates_kernel(const float* __restrict__ ba, const float* __restrict__ a_log,
                                   const float* __restrict__ dt_bias, int T, int Hv,
                                   float* __restrict__ beta, float* __restrict__ g) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= T * Hv) return;
  const int t = i / Hv, h = i % Hv;
  const float b = ba[(size_t)t * 2 * Hv + h];
  const float a = ba[(size_t)t * 2 * Hv + Hv + h] + dt_bias[h];
  beta[i] = 1.f / (1.f + expf(-b));
  const float sp = a > 20.f ? a : log1pf(expf(a));  // softplus
  g[i] = -expf(a_log[h]) * sp;
}

}  // namespace gdn

namespace {

// The few cuBLAS entry points used here, resolved at run time (types from cublas_api.h).
using cublasHandle = cublasHandle_t;
using PfnCreate = cublasStatus_t (*)(cublasHandle_t*);
using PfnSetStream = cublasStatus_t (*)(cublasHandle_t, cudaStream_t);
using PfnGemmEx = cublasStatus_t (*)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int,
                                     int, int, const void*, const void*, cudaDataType_t, int,
                                     const void*, cudaDataType_t, int, const void*, void*,
                                     cudaDataType_t, int, cublasComputeType_t, cublasGemmAlgo_t);

struct Blas {
  bool tried = false, ok = false;
  PfnCreate create = nullptr;
  PfnSetStream set_stream = nullptr;
  PfnGemmEx gemm = nullptr;
};

Blas& blas() {
  static Blas b;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (!b.tried) {
    b.tried = true;
    void* h = dlopen("libcublas.so.12", RTLD_NOW | RTLD_NOLOAD);  // already in the process
    if (!h) h = dlopen("libcublas.so.12", RTLD_NOW | RTLD_LOCAL);
    if (!h) h = dlopen("libcublas.so", RTLD_NOW | RTLD_LOCAL);
    if (h) {
      b.create = reinterpret_cast<PfnCreate>(dlsym(h, "cublasCreate_v2"));
      b.set_stream = reinterpret_cast<PfnSetStream>(dlsym(h, "cublasSetStream_v2"));
      b.gemm = reinterpret_cast<PfnGemmEx>(dlsym(h, "cublasGemmEx"));
      b.ok = b.create && b.set_stream && b.gemm;
    }
  }
  return b;
}

// one handle per device and host thread (created on first use)
cublasHandle handle_for_current_device() {
  constexpr int kMaxDev = 64;
  static thread_local cublasHandle t_handle[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
  if (!t_handle[dev] && blas().create(&t_handle[dev]) != CUBLAS_STATUS_SUCCESS)
    t_handle[dev] = nullptr;
  return t_handle[dev];
}

// Row-major C[M][N] (bf16 or fp32) = A[M][K] B[K][N] (bf16), fp32 accumulation: in cuBLAS's
// column-major view C^T = B^T A^T.
int gemm_rm(cublasHandle hd, int M, int N, int K, const void* A, const void* B, void* C,
            bool c_fp32) {
  const float one = 1.f, zero = 0.f;
  return blas().gemm(hd, CUBLAS_OP_N, CUBLAS_OP_N, N, M, K, &one, B, CUDA_R_16BF, N, A,
                     CUDA_R_16BF, K, &zero, C, c_fp32 ? CUDA_R_32F : CUDA_R_16BF, N,
                     CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS;
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

struct BlockWs {
  size_t x, z, ba, beta, g, o, layer, total;
};

BlockWs block_ws(const gdn_dims* d, int N, int T) {
  const size_t Cc = (size_t)(2 * d->num_k_heads + d->num_v_heads) * d->head_dim;
  const size_t Hv = d->num_v_heads, hd = d->head_dim;
  BlockWs w{};
  size_t o = 0;
  w.x = o; o = align256(o + (size_t)T * Cc * 2);
  w.z = o; o = align256(o + (size_t)T * Hv * hd * 2);
  w.ba = o; o = align256(o + (size_t)T * 2 * Hv * 4);
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
  if (!blas().ok) return GDN_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cublasHandle hd = handle_for_current_device();
  if (!hd || blas().set_stream(hd, s) != CUBLAS_STATUS_SUCCESS) return GDN_ERR_CUDA;
  const BlockWs l = block_ws(dims, num_seqs, num_tokens);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  const int T = num_tokens, H = hidden, Hv = dims->num_v_heads, d = dims->head_dim;
  const int Cc = (2 * dims->num_k_heads + Hv) * d;
  void* x = w + l.x;
  void* z = w + l.z;
  float* ba = reinterpret_cast<float*>(w + l.ba);
  float* beta = reinterpret_cast<float*>(w + l.beta);
  float* g = reinterpret_cast<float*>(w + l.g);
  void* o = w + l.o;
  gdn_host::trace_begin("block_in_proj", s);
  int rc = gemm_rm(hd, T, Cc, H, h, w_qkv, x, false);
  if (!rc) rc = gemm_rm(hd, T, Hv * d, H, h, w_z, z, false);
  if (!rc) rc = gemm_rm(hd, T, 2 * Hv, H, h, w_ba, ba, true);
  gdn_host::trace_end(s);
  if (rc) return GDN_ERR_CUDA;
  gdn_host::trace_begin("block_gates", s);
  gdn::block_gates_kernel<<<(T * Hv + 255) / 256, 256, 0, s>>>(ba, a_log, dt_bias, T, Hv, beta, g);
  gdn_host::trace_end(s);
  if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
  rc = gdn_chunk_prefill(dims, GDN_BF16, x, conv_w, beta, g, z, norm_w, cu_seqlens, num_seqs, T,
                         S0, SN, conv0, convN, o, w + l.layer, workspace_bytes - l.layer,
                         dev_status, stream);
  if (rc != GDN_OK) return rc;
  gdn_host::trace_begin("block_out_proj", s);
  rc = gemm_rm(hd, T, H, Hv * d, o, w_out, y, false);
  gdn_host::trace_end(s);
  return rc ? GDN_ERR_CUDA : GDN_OK;
}

}  // extern "C"
