// conv1d.cu -- causal depthwise conv (width 4) + SiLU over packed sequences, and the final
// conv history of each sequence.
//
// Source: the causal convolution in the hyper.ai Gated DeltaNet paragraph; width 4 is
// linear_conv_kernel_dim of the Qwen3-Coder-Next raw config.json fields; SiLU is hidden_act.
// Each thread owns 8 channels (one 16-byte vector) and a run of kRun consecutive tokens, keeping
// the 3-token history in registers; sequence boundaries inside a run restart the history from
// the caller's conv state.  Reads and writes are 16-byte vectors, consecutive threads on
// consecutive channels, so every warp access is one contiguous 256/512-byte segment.
#include "args.cuh"
#include "common.cuh"

namespace gdn {

constexpr int kRun = 16;  // tokens per thread

template <typename T>
__device__ __forceinline__ void load_hist(const T* x, const T* state_in, int Cc, int c, int n,
                                          int seq_start, int t, float (&h)[3][8]) {
  // h[j] = input of token t-3+j of sequence n (state rows before its start)
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const int row = t - 3 + j;
    if (row >= seq_start) {
      load8(x + (size_t)row * Cc + c, h[j]);
    } else if (state_in) {
      const int sr = 3 + (row - seq_start);  // 0..2
      load8(state_in + ((size_t)n * 3 + sr) * Cc + c, h[j]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) h[j][e] = 0.f;
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(128) conv1d_silu_kernel(const T* __restrict__ x, T* __restrict__ y,
                                                          const T* __restrict__ w,
                                                          const int32_t* __restrict__ cu, int N,
                                                          int T_total, int Cc,
                                                          const T* __restrict__ state_in) {
  const int c = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
  const int t0 = blockIdx.y * kRun;
  if (c >= Cc || t0 >= T_total) return;
  float wv[4][8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    // w is [Cc][4]: the 8 channels' taps are 32 consecutive elements
#pragma unroll
    for (int i = 0; i < 4; ++i) wv[i][e] = to_f(w[(size_t)(c + e) * 4 + i]);
  }
  int n = seq_of_token(cu, N, t0);
  int s = __ldg(cu + n), e_end = __ldg(cu + n + 1);
  float h[3][8];
  load_hist(x, state_in, Cc, c, n, s, t0, h);
  const int t1 = min(T_total, t0 + kRun);
  for (int t = t0; t < t1; ++t) {
    if (t >= e_end) {  // next non-empty sequence starts here
      while (t >= e_end) {
        ++n;
        s = e_end;
        e_end = __ldg(cu + n + 1);
      }
      load_hist(x, state_in, Cc, c, n, s, t, h);
    }
    float xv[8], out[8];
    load8(x + (size_t)t * Cc + c, xv);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float a = wv[0][k] * h[0][k] + wv[1][k] * h[1][k] + wv[2][k] * h[2][k] + wv[3][k] * xv[k];
      out[k] = silu_f(a);
      h[0][k] = h[1][k];
      h[1][k] = h[2][k];
      h[2][k] = xv[k];
    }
    store8(y + (size_t)t * Cc + c, out);
  }
}

// Last 3 rows of [state_in ; x_seq] for every sequence.  One thread per (sequence, 8 channels);
// it reads everything it needs before writing, so state_out may equal state_in.
template <typename T>
__global__ void __launch_bounds__(128) conv_state_out_kernel(const T* __restrict__ x,
                                                             const int32_t* __restrict__ cu, int N,
                                                             int Cc, const T* state_in,
                                                             T* state_out,
                                                             const int32_t* __restrict__ slot,
                                                             int num_slots, int32_t* status) {
  const int c = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
  const int n = blockIdx.y;
  if (c >= Cc || n >= N) return;
  const int s = __ldg(cu + n), L = __ldg(cu + n + 1) - s;
  if (!GDN_IN_BOUNDS(s >= 0 && L >= 0, status)) return;
  const int srow = state_row(slot, n, num_slots);
  if (srow < 0) {  // slot out of range: no access to the pool
    if (c == 0) report_status(status, GDN_ERR_INVALID_ARG);
    return;
  }
  const size_t row = (size_t)srow * 3;
  float r[3][8];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const int e = L + j;  // index into [state rows 0..2, x rows 0..L-1]
    if (e >= 3) {
      load8(x + (size_t)(s + e - 3) * Cc + c, r[j]);
    } else if (state_in) {
      load8(state_in + (row + e) * Cc + c, r[j]);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) r[j][k] = 0.f;
    }
  }
#pragma unroll
  for (int j = 0; j < 3; ++j) store8(state_out + (row + j) * Cc + c, r[j]);
}

}  // namespace gdn

namespace gdn_host {

template <typename T>
static cudaError_t conv1d_impl(const void* x, void* y, const void* w, const int32_t* cu, int N,
                               int T_total, int Cc, const void* st_in, void* st_out,
                               cudaStream_t s) {
  if (T_total > 0) {
    dim3 grid((Cc / 8 + 127) / 128, (T_total + gdn::kRun - 1) / gdn::kRun);
    trace_begin("conv1d_silu", s);
    gdn::conv1d_silu_kernel<T><<<grid, 128, 0, s>>>(
        static_cast<const T*>(x), static_cast<T*>(y), static_cast<const T*>(w), cu, N, T_total, Cc,
        static_cast<const T*>(st_in));
    trace_end(s);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (st_out && N > 0) {
    dim3 grid((Cc / 8 + 127) / 128, N);
    trace_begin("conv_state_out", s);
    gdn::conv_state_out_kernel<T><<<grid, 128, 0, s>>>(static_cast<const T*>(x), cu, N, Cc,
                                                       static_cast<const T*>(st_in),
                                                       static_cast<T*>(st_out), nullptr, N,
                                                       nullptr);
    trace_end(s);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

cudaError_t launch_conv1d(bool bf16, const void* x, void* y, const void* w, const int32_t* cu,
                          int N, int T_total, int Cc, const void* st_in, void* st_out,
                          cudaStream_t s) {
  return bf16 ? conv1d_impl<__nv_bfloat16>(x, y, w, cu, N, T_total, Cc, st_in, st_out, s)
              : conv1d_impl<float>(x, y, w, cu, N, T_total, Cc, st_in, st_out, s);
}

cudaError_t launch_conv_state_out(bool bf16, const void* x, const int32_t* cu, int N, int Cc,
                                  const void* st_in, void* st_out, const int32_t* slot,
                                  int num_slots, int32_t* status, cudaStream_t s) {
  if (!st_out || N == 0) return cudaSuccess;
  dim3 grid((Cc / 8 + 127) / 128, N);
  trace_begin("conv_state_out", s);
  if (bf16)
    gdn::conv_state_out_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), cu, N, Cc,
        static_cast<const __nv_bfloat16*>(st_in), static_cast<__nv_bfloat16*>(st_out), slot, num_slots, status);
  else
    gdn::conv_state_out_kernel<float><<<grid, 128, 0, s>>>(static_cast<const float*>(x), cu, N,
                                                           Cc, static_cast<const float*>(st_in),
                                                           static_cast<float*>(st_out), slot, num_slots,
                                                           status);
  trace_end(s);
  return cudaGetLastError();
}

}  // namespace gdn_host
