// prefill_f32.cu -- fp32 prefill: the token-by-token recurrence on CUDA cores in fp32.
//
// Source: the recurrence of the hyper.ai Gated DeltaNet paragraph as read in gdn.h.  This is
// the precision path (fp32 activations, max-abs error ~1e-6 against an fp64 evaluation); the
// bf16 path runs the chunked tensor-core kernels in prefill_tc.cu.
//
// One CTA per (sequence, value head), 256 threads.  Threads 0..127 own channel j of q, k and v
// (conv history in registers); each warp owns 16 state rows (a lane holds 4 consecutive
// columns of each row in registers), so the state never leaves the SM between tokens.
#include "args.cuh"
#include "common.cuh"

namespace gdn {


__global__ void __launch_bounds__(256) recurrent_f32_kernel(RecArgs a) {
  constexpr int d = kHeadDim, kRows = 16;
  const int n = blockIdx.x / a.Hv, h = blockIdx.x % a.Hv;
  const int hk = h / (a.Hv / a.Hk);
  const int Cc = (2 * a.Hk + a.Hv) * d;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cq = hk * d, ck = a.Hk * d + hk * d, cv = 2 * a.Hk * d + h * d;
  __shared__ float q_s[d], k_s[d], v_s[d], o_s[d];
  __shared__ float red_q[4], red_k[4], red_o[8];

  const int s = __ldg(a.cu + n), e = __ldg(a.cu + n + 1);
  const int srow = state_row(a.slot, n, a.num_slots);  // -1: slot out of range, no state access
  if (srow < 0 && tid == 0 && h == 0) report_status(a.status, GDN_ERR_INVALID_ARG);
  // conv history (threads < 128): rows t-3, t-2, t-1 of channel tid of q, k, v
  float hq[3] = {0, 0, 0}, hkk[3] = {0, 0, 0}, hv[3] = {0, 0, 0};
  float wq[4], wk[4], wv[4];
  if (tid < d) {
    if (a.conv0 && srow >= 0) {
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        const float* row = a.conv0 + ((size_t)srow * 3 + j) * Cc;
        hq[j] = row[cq + tid];
        hkk[j] = row[ck + tid];
        hv[j] = row[cv + tid];
      }
    }
    if (a.conv_w) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        wq[i] = a.conv_w[(size_t)(cq + tid) * 4 + i];
        wk[i] = a.conv_w[(size_t)(ck + tid) * 4 + i];
        wv[i] = a.conv_w[(size_t)(cv + tid) * 4 + i];
      }
    }
  }
  // state rows of this warp
  float st[kRows][4];
  const size_t sbase = ((size_t)(srow < 0 ? 0 : srow) * a.Hv + h) * d * d;
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int v = warp * kRows + r;
    if (a.S0 && srow >= 0) {
      float4 p = *reinterpret_cast<const float4*>(a.S0 + sbase + (size_t)v * d + 4 * lane);
      st[r][0] = p.x; st[r][1] = p.y; st[r][2] = p.z; st[r][3] = p.w;
    } else {
      st[r][0] = st[r][1] = st[r][2] = st[r][3] = 0.f;
    }
  }

  for (int t = s; t < e; ++t) {
    // ---- conv + SiLU, partial squares
    if (tid < d) {
      const float* xr = a.x + (size_t)t * Cc;
      const float xq = xr[cq + tid], xk = xr[ck + tid], xv = xr[cv + tid];
      float yq, yk, yv;
      if (a.conv_w) {
        yq = silu_f(wq[0] * hq[0] + wq[1] * hq[1] + wq[2] * hq[2] + wq[3] * xq);
        yk = silu_f(wk[0] * hkk[0] + wk[1] * hkk[1] + wk[2] * hkk[2] + wk[3] * xk);
        yv = silu_f(wv[0] * hv[0] + wv[1] * hv[1] + wv[2] * hv[2] + wv[3] * xv);
      } else {
        yq = xq; yk = xk; yv = xv;
      }
      hq[0] = hq[1]; hq[1] = hq[2]; hq[2] = xq;
      hkk[0] = hkk[1]; hkk[1] = hkk[2]; hkk[2] = xk;
      hv[0] = hv[1]; hv[1] = hv[2]; hv[2] = xv;
      q_s[tid] = yq;
      k_s[tid] = yk;
      v_s[tid] = yv;
      const float sq = warp_sum(yq * yq), sk = warp_sum(yk * yk);
      if (lane == 0) { red_q[warp] = sq; red_k[warp] = sk; }
    }
    __syncthreads();
    const float rq = a.q_scale / sqrtf(red_q[0] + red_q[1] + red_q[2] + red_q[3] + a.l2_eps);
    const float rk = 1.0f / sqrtf(red_k[0] + red_k[1] + red_k[2] + red_k[3] + a.l2_eps);
    float kr[4], qr[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      kr[j] = k_s[4 * lane + j] * rk;
      qr[j] = q_s[4 * lane + j] * rq;
    }
    const float alpha = expf(a.g[(size_t)t * a.Hv + h]);
    const float beta = a.beta[(size_t)t * a.Hv + h];
    // ---- state update of this warp's rows
    float osq = 0.f;
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int v = warp * kRows + r;
#pragma unroll
      for (int j = 0; j < 4; ++j) st[r][j] *= alpha;
      float kv = st[r][0] * kr[0] + st[r][1] * kr[1] + st[r][2] * kr[2] + st[r][3] * kr[3];
      kv = warp_sum(kv);
      const float u = beta * (v_s[v] - kv);
#pragma unroll
      for (int j = 0; j < 4; ++j) st[r][j] += u * kr[j];
      float o = st[r][0] * qr[0] + st[r][1] * qr[1] + st[r][2] * qr[2] + st[r][3] * qr[3];
      o = warp_sum(o);
      if (lane == 0) o_s[v] = o;
      osq += o * o;
    }
    if (lane == 0) red_o[warp] = osq;
    __syncthreads();
    // ---- output (gated RMSNorm when z is given)
    if (tid < d) {
      float o = o_s[tid];
      if (a.z) {
        float ss = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) ss += red_o[w];
        const float inv = 1.0f / sqrtf(ss / d + a.norm_eps);
        const float zz = a.z[((size_t)t * a.Hv + h) * d + tid];
        o = o * inv * (a.norm_w ? a.norm_w[tid] : 1.f) * silu_f(zz);
      }
      a.out[((size_t)t * a.Hv + h) * d + tid] = o;
    }
  }
  if (a.SN && srow >= 0) {
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int v = warp * kRows + r;
      *reinterpret_cast<float4*>(a.SN + sbase + (size_t)v * d + 4 * lane) =
          make_float4(st[r][0], st[r][1], st[r][2], st[r][3]);
    }
  }
}

}  // namespace gdn

namespace gdn_host {

cudaError_t launch_recurrent_f32(const gdn::RecArgs& a, cudaStream_t s) {
  if (a.N == 0) return cudaSuccess;
  trace_begin("recurrent_f32", s);
  gdn::recurrent_f32_kernel<<<a.N * a.Hv, 256, 0, s>>>(a);
  trace_end(s);
  return cudaGetLastError();
}

}  // namespace gdn_host
