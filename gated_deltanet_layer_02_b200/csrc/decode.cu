// decode.cu -- one decode token per sequence: conv-state shift + conv + SiLU, L2 norms of q and
// k, one read-modify-write pass over the fp32 recurrent state, z-gated RMSNorm.
//
// Source: the recurrence of the hyper.ai Gated DeltaNet paragraph as read in gdn.h (beta gates
// the update, kv_mem = alpha S k is the read-out of the stored knowledge), with the fp32 state
// of the "Qwen3-Next" SGLang cookbook, section 3.2 (--mamba-ssm-dtype default).
//
// Per state row r (value index) of value head h, with alpha = exp(g), kq = k.q:
//   kv  = alpha * (S_r . k)                 (kv_mem)
//   u   = beta * (v_r - kv)
//   o_r = alpha * (S_r . q) + u * kq        (= S'_r . q)
//   S'_r = alpha * S_r + u * k
// so each state element is read once and written once.  One CTA per (sequence, key head)
// handles that key head's R = Hv/Hk value heads; each warp streams whole rows (a lane owns 4
// consecutive columns, 512 contiguous bytes per warp load) with kRowBatch rows in flight, and
// reduces the two dot products with warp shuffles.
#include "args.cuh"
#include "common.cuh"

namespace gdn {

constexpr int kDecodeThreads = 128;  // four warps: four CTAs per SM at 128 registers
constexpr int kMaxR = 8;

// Four consecutive state elements of a lane: fp32 (16 bytes) or bf16 (8 bytes, the serving
// option of a bf16 recurrent state: arithmetic stays fp32, the new state is rounded to nearest
// even once per step).  Loads stay raw until used, so that the bf16 state keeps as many bytes
// in flight (twice the rows) in the same registers.  Streaming loads and stores: the state is
// touched once per step.
template <typename TS>
struct StateIO;
template <>
struct StateIO<float> {
  using Raw = float4;
  static constexpr int kRows = 8;  // rows per batch and warp
  static __device__ __forceinline__ Raw load(const float* p) {
    return __ldcs(reinterpret_cast<const float4*>(p));
  }
  static __device__ __forceinline__ float4 f4(Raw r) { return r; }
  static __device__ __forceinline__ void store(float* p, float4 v) {
    __stcs(reinterpret_cast<float4*>(p), v);
  }
};
template <>
struct StateIO<__nv_bfloat16> {
  using Raw = uint2;
  static constexpr int kRows = 16;
  static __device__ __forceinline__ Raw load(const __nv_bfloat16* p) {
    return __ldcs(reinterpret_cast<const uint2*>(p));
  }
  static __device__ __forceinline__ float4 f4(Raw u) {
    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, float4 v) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t*>(&lo);
    u.y = *reinterpret_cast<const uint32_t*>(&hi);
    __stcs(reinterpret_cast<uint2*>(p), u);
  }
};

template <typename T, typename TS>
__global__ void __launch_bounds__(kDecodeThreads, 4) decode_kernel(DecodeArgs a) {
  constexpr int d = kHeadDim;
  const int b = blockIdx.x / a.Hk;
  const int hk = blockIdx.x % a.Hk;
  const int R = a.Hv / a.Hk;
  const int Cc = (2 * a.Hk + a.Hv) * d;
  const int slot = state_row(a.slot_idx, b, a.num_slots);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (slot < 0) {  // slot out of range: the sequence is skipped, its outputs are not written
    if (tid == 0) report_status(a.status, GDN_ERR_INVALID_ARG);
    return;
  }

  __shared__ float y_s[(2 + kMaxR) * d];  // q | k | v_0..v_{R-1} after conv
  __shared__ float o_s[kMaxR * d];
  __shared__ float red_s[4];

  const T* x = static_cast<const T*>(a.x) + (size_t)b * Cc;
  const T* w = static_cast<const T*>(a.conv_w);
  T* cs = static_cast<T*>(a.conv_state) + (size_t)slot * 3 * Cc;

  // the first batch of state rows does not depend on q and k: its loads go out before the conv
  using IO = StateIO<TS>;
  constexpr int kRowBatch = IO::kRows;
  const int rows_per_warp = R * d / (kDecodeThreads / 32);
  const int nbatch = rows_per_warp / kRowBatch;
  TS* S = static_cast<TS*>(a.S);
  auto row_ptr = [&](int gr) {
    const int hr = gr / d, v = gr % d;
    return S + (((size_t)slot * a.Hv + hk * R + hr) * d + v) * d + 4 * lane;
  };
  typename IO::Raw sv[kRowBatch], sn[kRowBatch];
#pragma unroll
  for (int i = 0; i < kRowBatch; ++i) sv[i] = IO::load(row_ptr(warp * rows_per_warp + i));

  // ---- conv + SiLU with in-place history shift: 2 channels per item
  const int items = (2 + R) * d / 2;
  for (int it = tid; it < items; it += kDecodeThreads) {
    const int gch = it * 2;              // position inside y_s
    const int grp = gch / d, off = gch % d;
    int c;
    if (grp == 0) c = hk * d + off;
    else if (grp == 1) c = a.Hk * d + hk * d + off;
    else c = 2 * a.Hk * d + (hk * R + grp - 2) * d + off;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float s0 = to_f(cs[c + e]), s1 = to_f(cs[Cc + c + e]), s2 = to_f(cs[2 * Cc + c + e]);
      const T xt = x[c + e];
      const T* wr = w + (size_t)(c + e) * 4;
      const float acc = to_f(wr[0]) * s0 + to_f(wr[1]) * s1 + to_f(wr[2]) * s2 + to_f(wr[3]) * to_f(xt);
      y_s[gch + e] = silu_f(acc);
      cs[c + e] = from_f<T>(s1);
      cs[Cc + c + e] = from_f<T>(s2);
      cs[2 * Cc + c + e] = xt;
    }
  }
  __syncthreads();
  // ---- |q|^2, |k|^2, q.k
  if (warp < 3) {
    float acc = 0.f;
    for (int i = lane; i < d; i += 32) {
      const float qv = y_s[i], kv = y_s[d + i];
      acc += warp == 0 ? qv * qv : (warp == 1 ? kv * kv : qv * kv);
    }
    acc = warp_sum(acc);
    if (lane == 0) red_s[warp] = acc;
  }
  __syncthreads();
  const float rq = a.q_scale * rsqrtf(red_s[0] + a.l2_eps);
  const float rk = rsqrtf(red_s[1] + a.l2_eps);
  const float kq = red_s[2] * rq * rk;
  float kreg[4], qreg[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    kreg[j] = y_s[d + 4 * lane + j] * rk;
    qreg[j] = y_s[4 * lane + j] * rq;
  }

  // ---- state pass: R*d rows split over the warps, two batches of rows in flight
  for (int bt = 0; bt < nbatch; ++bt) {
    const int r0 = warp * rows_per_warp + bt * kRowBatch;
    if (bt + 1 < nbatch) {
#pragma unroll
      for (int i = 0; i < kRowBatch; ++i) sn[i] = IO::load(row_ptr(r0 + kRowBatch + i));
    }
    float dk[kRowBatch], dq[kRowBatch];
#pragma unroll
    for (int i = 0; i < kRowBatch; ++i) {
      const float4 f = IO::f4(sv[i]);
      dk[i] = f.x * kreg[0] + f.y * kreg[1] + f.z * kreg[2] + f.w * kreg[3];
      dq[i] = f.x * qreg[0] + f.y * qreg[1] + f.z * qreg[2] + f.w * qreg[3];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int i = 0; i < kRowBatch; ++i) {
        dk[i] += __shfl_xor_sync(0xffffffffu, dk[i], o);
        dq[i] += __shfl_xor_sync(0xffffffffu, dq[i], o);
      }
    }
#pragma unroll
    for (int i = 0; i < kRowBatch; ++i) {
      const int gr = r0 + i, hr = gr / d, v = gr % d;
      const int h = hk * R + hr;
      const float alpha = expf(__ldg(a.g + (size_t)b * a.Hv + h));
      const float beta = __ldg(a.beta + (size_t)b * a.Hv + h);
      const float vv = y_s[(2 + hr) * d + v];
      const float u = beta * (vv - alpha * dk[i]);
      if (lane == 0) o_s[hr * d + v] = alpha * dq[i] + u * kq;
      const float4 f = IO::f4(sv[i]);
      float4 nv;
      nv.x = alpha * f.x + u * kreg[0];
      nv.y = alpha * f.y + u * kreg[1];
      nv.z = alpha * f.z + u * kreg[2];
      nv.w = alpha * f.w + u * kreg[3];
      IO::store(row_ptr(gr), nv);
    }
#pragma unroll
    for (int i = 0; i < kRowBatch; ++i) sv[i] = sn[i];
  }
  __syncthreads();
  // ---- gated RMSNorm (or plain output), one warp per value head
  T* out = static_cast<T*>(a.out);
  for (int hr = warp; hr < R; hr += kDecodeThreads / 32) {
    const int h = hk * R + hr;
    float ov[4], ss = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      ov[j] = o_s[hr * d + 4 * lane + j];
      ss += ov[j] * ov[j];
    }
    if (a.z) {
      ss = warp_sum(ss);
      const float inv = rsqrtf(ss / d + a.norm_eps);
      const T* zr = static_cast<const T*>(a.z) + ((size_t)b * a.Hv + h) * d;
      const T* nw = static_cast<const T*>(a.norm_w);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = 4 * lane + j;
        ov[j] = ov[j] * inv * (nw ? to_f(nw[c]) : 1.f) * silu_f(to_f(zr[c]));
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) out[((size_t)b * a.Hv + h) * d + 4 * lane + j] = from_f<T>(ov[j]);
  }
}

// ---------------------------------------------------------------------------- multi-token
// k tokens per sequence in one launch (verification of k speculative draft tokens): the state
// rows are read once, take the k updates in registers and are written once; every token uses
// exactly the arithmetic of decode_kernel, so the results equal k calls of the one-token step.
// With `snaps` set, the state after every token is stored as well ([B, k, Hv, d, d] fp32), so
// that a caller that accepts only the first m tokens can take snapshot m - 1.  Dynamic shared
// memory: per token (2 + R) d conv outputs, R d outputs and three norms.
constexpr int kMaxTokens = 8;

template <typename T>
__global__ void __launch_bounds__(kDecodeThreads) decode_multi_kernel(DecodeArgs a, int k,
                                                                      float* snaps) {
  constexpr int d = kHeadDim;
  const int b = blockIdx.x / a.Hk;
  const int hk = blockIdx.x % a.Hk;
  const int R = a.Hv / a.Hk;
  const int Cc = (2 * a.Hk + a.Hv) * d;
  const int slot = state_row(a.slot_idx, b, a.num_slots);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (slot < 0) {  // slot out of range: the sequence is skipped, its outputs are not written
    if (tid == 0) report_status(a.status, GDN_ERR_INVALID_ARG);
    return;
  }
  extern __shared__ float dsm[];
  float* y_s = dsm;                          // [k][(2 + R) d]: q | k | v_0..v_{R-1}
  float* o_s = y_s + k * (2 + R) * d;        // [k][R d]
  float* red_s = o_s + k * R * d;            // [k][3]: |q|^2, |k|^2, q.k

  const T* w = static_cast<const T*>(a.conv_w);
  T* cs = static_cast<T*>(a.conv_state) + (size_t)slot * 3 * Cc;
  using IO = StateIO<float>;
  constexpr int kRowBatch = IO::kRows;
  const int rows_per_warp = R * d / (kDecodeThreads / 32);
  const int nbatch = rows_per_warp / kRowBatch;
  float* S = static_cast<float*>(a.S);
  auto row_off = [&](int gr) {
    const int hr = gr / d, v = gr % d;
    return (((size_t)slot * a.Hv + hk * R + hr) * d + v) * d + 4 * lane;
  };
  float4 sv[kRowBatch];
#pragma unroll
  for (int i = 0; i < kRowBatch; ++i) sv[i] = IO::load(S + row_off(warp * rows_per_warp + i));

  // ---- conv + SiLU over the k tokens, history in registers, final history written back
  const int items = (2 + R) * d / 2;
  for (int it = tid; it < items; it += kDecodeThreads) {
    const int gch = it * 2;
    const int grp = gch / d, off = gch % d;
    int c;
    if (grp == 0) c = hk * d + off;
    else if (grp == 1) c = a.Hk * d + hk * d + off;
    else c = 2 * a.Hk * d + (hk * R + grp - 2) * d + off;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float s0 = to_f(cs[c + e]), s1 = to_f(cs[Cc + c + e]), s2 = to_f(cs[2 * Cc + c + e]);
      const T* wr = w + (size_t)(c + e) * 4;
      T xt = T();
      for (int t = 0; t < k; ++t) {
        xt = static_cast<const T*>(a.x)[((size_t)b * k + t) * Cc + c + e];
        const float acc = to_f(wr[0]) * s0 + to_f(wr[1]) * s1 + to_f(wr[2]) * s2 + to_f(wr[3]) * to_f(xt);
        y_s[t * (2 + R) * d + gch + e] = silu_f(acc);
        s0 = s1;
        s1 = s2;
        s2 = to_f(xt);
      }
      cs[c + e] = from_f<T>(s0);
      cs[Cc + c + e] = from_f<T>(s1);
      cs[2 * Cc + c + e] = xt;
    }
  }
  __syncthreads();
  // ---- |q|^2, |k|^2, q.k per token
  for (int job = warp; job < 3 * k; job += kDecodeThreads / 32) {
    const int t = job / 3, kind = job % 3;
    const float* yt = y_s + t * (2 + R) * d;
    float acc = 0.f;
    for (int i = lane; i < d; i += 32) {
      const float qv = yt[i], kv = yt[d + i];
      acc += kind == 0 ? qv * qv : (kind == 1 ? kv * kv : qv * kv);
    }
    acc = warp_sum(acc);
    if (lane == 0) red_s[t * 3 + kind] = acc;
  }
  __syncthreads();

  // ---- state pass: each batch of rows takes the k updates in registers
  for (int bt = 0; bt < nbatch; ++bt) {
    const int r0 = warp * rows_per_warp + bt * kRowBatch;
    for (int t = 0; t < k; ++t) {
      const float* yt = y_s + t * (2 + R) * d;
      const float rq = a.q_scale * rsqrtf(red_s[t * 3] + a.l2_eps);
      const float rk = rsqrtf(red_s[t * 3 + 1] + a.l2_eps);
      const float kq = red_s[t * 3 + 2] * rq * rk;
      float kreg[4], qreg[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        kreg[j] = yt[d + 4 * lane + j] * rk;
        qreg[j] = yt[4 * lane + j] * rq;
      }
      float dk[kRowBatch], dq[kRowBatch];
#pragma unroll
      for (int i = 0; i < kRowBatch; ++i) {
        const float4 f = sv[i];
        dk[i] = f.x * kreg[0] + f.y * kreg[1] + f.z * kreg[2] + f.w * kreg[3];
        dq[i] = f.x * qreg[0] + f.y * qreg[1] + f.z * qreg[2] + f.w * qreg[3];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
        for (int i = 0; i < kRowBatch; ++i) {
          dk[i] += __shfl_xor_sync(0xffffffffu, dk[i], o);
          dq[i] += __shfl_xor_sync(0xffffffffu, dq[i], o);
        }
      }
#pragma unroll
      for (int i = 0; i < kRowBatch; ++i) {
        const int gr = r0 + i, hr = gr / d, v = gr % d;
        const int h = hk * R + hr;
        const float alpha = expf(__ldg(a.g + ((size_t)b * k + t) * a.Hv + h));
        const float beta = __ldg(a.beta + ((size_t)b * k + t) * a.Hv + h);
        const float vv = yt[(2 + hr) * d + v];
        const float u = beta * (vv - alpha * dk[i]);
        if (lane == 0) o_s[(t * R + hr) * d + v] = alpha * dq[i] + u * kq;
        const float4 f = sv[i];
        float4 nv;
        nv.x = alpha * f.x + u * kreg[0];
        nv.y = alpha * f.y + u * kreg[1];
        nv.z = alpha * f.z + u * kreg[2];
        nv.w = alpha * f.w + u * kreg[3];
        sv[i] = nv;
        if (snaps)
          IO::store(snaps + ((((size_t)b * k + t) * a.Hv + h) * d + v) * d + 4 * lane, nv);
      }
    }
#pragma unroll
    for (int i = 0; i < kRowBatch; ++i) IO::store(S + row_off(r0 + i), sv[i]);
    if (bt + 1 < nbatch) {
#pragma unroll
      for (int i = 0; i < kRowBatch; ++i) sv[i] = IO::load(S + row_off(r0 + kRowBatch + i));
    }
  }
  __syncthreads();
  // ---- gated RMSNorm (or plain output) per token, one warp per (token, value head)
  T* out = static_cast<T*>(a.out);
  for (int job = warp; job < k * R; job += kDecodeThreads / 32) {
    const int t = job / R, hr = job % R;
    const int h = hk * R + hr;
    float ov[4], ss = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      ov[j] = o_s[(t * R + hr) * d + 4 * lane + j];
      ss += ov[j] * ov[j];
    }
    if (a.z) {
      ss = warp_sum(ss);
      const float inv = rsqrtf(ss / d + a.norm_eps);
      const T* zr = static_cast<const T*>(a.z) + (((size_t)b * k + t) * a.Hv + h) * d;
      const T* nw = static_cast<const T*>(a.norm_w);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = 4 * lane + j;
        ov[j] = ov[j] * inv * (nw ? to_f(nw[c]) : 1.f) * silu_f(to_f(zr[c]));
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
      out[(((size_t)b * k + t) * a.Hv + h) * d + 4 * lane + j] = from_f<T>(ov[j]);
  }
}

}  // namespace gdn

namespace gdn_host {

cudaError_t launch_decode(bool bf16, bool state_bf16, const gdn::DecodeArgs& a,
                          cudaStream_t s) {
  if (a.B == 0) return cudaSuccess;
  const dim3 grid(a.B * a.Hk), block(gdn::kDecodeThreads);
  trace_begin(state_bf16 ? "decode_step_bf16_state" : "decode_step", s);
  if (bf16 && state_bf16)
    gdn::decode_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, block, 0, s>>>(a);
  else if (bf16)
    gdn::decode_kernel<__nv_bfloat16, float><<<grid, block, 0, s>>>(a);
  else if (state_bf16)
    gdn::decode_kernel<float, __nv_bfloat16><<<grid, block, 0, s>>>(a);
  else
    gdn::decode_kernel<float, float><<<grid, block, 0, s>>>(a);
  trace_end(s);
  return cudaGetLastError();
}

cudaError_t launch_decode_multi(bool bf16, const gdn::DecodeArgs& a, int k, float* snaps,
                                cudaStream_t s) {
  if (a.B == 0 || k == 0) return cudaSuccess;
  const int R = a.Hv / a.Hk;
  const size_t smem = ((size_t)k * (2 + 2 * R) * gdn::kHeadDim + 3 * k) * sizeof(float);
  static bool attr = false;
  if (!attr) {  // the largest request: kMaxTokens tokens, kMaxR value heads per key head
    const int most = (gdn::kMaxTokens * (2 + 2 * gdn::kMaxR) * gdn::kHeadDim + 3 * gdn::kMaxTokens) *
                     (int)sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(gdn::decode_multi_kernel<__nv_bfloat16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gdn::decode_multi_kernel<float>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, most);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const dim3 grid(a.B * a.Hk), block(gdn::kDecodeThreads);
  trace_begin("decode_multi", s);
  if (bf16)
    gdn::decode_multi_kernel<__nv_bfloat16><<<grid, block, smem, s>>>(a, k, snaps);
  else
    gdn::decode_multi_kernel<float><<<grid, block, smem, s>>>(a, k, snaps);
  trace_end(s);
  return cudaGetLastError();
}

}  // namespace gdn_host
