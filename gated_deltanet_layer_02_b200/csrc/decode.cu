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
// handles that key head's R = Hv/Hk value heads.  A warp streams four rows at a time (a row
// quad), eight lanes per row: a lane holds 16 elements of its row, and the two dot products
// reduce in three shuffle steps inside each group of eight lanes.  Every aligned 128-byte line
// of a row is read by one group of eight lanes with one 16-byte load each.
#include "args.cuh"
#include "common.cuh"
#include "tc.cuh"

namespace gdn {

constexpr int kDecodeThreads = 128;  // four warps: four CTAs per SM at 128 registers
constexpr int kMaxR = 8;

// Sixteen elements of a row held by one lane (s = lane & 7, its place in the row's group):
// fp32 columns 4 s + 32 m + e (m = 0..3, e = 0..3), or bf16 columns 8 s + 64 m + e (m = 0, 1,
// e = 0..7) for the serving option of a bf16 recurrent state (arithmetic stays fp32, the new
// state is rounded to nearest even once per step).  Loads stay raw until used, so that the
// bf16 state keeps as many bytes in flight (twice the rows) in the same registers.  Streaming
// loads and stores: the state is touched once per step.
template <typename TS>
struct RowPart;
template <>
struct RowPart<float> {
  static constexpr int kQuads = 2;  // row quads per batch and warp (8 rows)
  struct Raw {
    float4 v[4];
  };
  static __device__ __forceinline__ int col(int s, int j) { return 4 * s + 32 * (j >> 2) + (j & 3); }
  static __device__ __forceinline__ void load(Raw& r, const float* row, int s) {
#pragma unroll
    for (int m = 0; m < 4; ++m) r.v[m] = __ldcs(reinterpret_cast<const float4*>(row + 4 * s + 32 * m));
  }
  static __device__ __forceinline__ void unpack(const Raw& r, float (&f)[16]) {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      f[4 * m] = r.v[m].x;
      f[4 * m + 1] = r.v[m].y;
      f[4 * m + 2] = r.v[m].z;
      f[4 * m + 3] = r.v[m].w;
    }
  }
  static __device__ __forceinline__ void store(float* row, int s, const float (&f)[16]) {
#pragma unroll
    for (int m = 0; m < 4; ++m)
      __stcs(reinterpret_cast<float4*>(row + 4 * s + 32 * m),
             make_float4(f[4 * m], f[4 * m + 1], f[4 * m + 2], f[4 * m + 3]));
  }
};
template <>
struct RowPart<__nv_bfloat16> {
  static constexpr int kQuads = 4;  // 16 rows
  struct Raw {
    uint4 v[2];
  };
  static __device__ __forceinline__ int col(int s, int j) { return 8 * s + 64 * (j >> 3) + (j & 7); }
  static __device__ __forceinline__ void load(Raw& r, const __nv_bfloat16* row, int s) {
#pragma unroll
    for (int m = 0; m < 2; ++m) r.v[m] = __ldcs(reinterpret_cast<const uint4*>(row + 8 * s + 64 * m));
  }
  static __device__ __forceinline__ void unpack(const Raw& r, float (&f)[16]) {
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const uint32_t w[4] = {r.v[m].x, r.v[m].y, r.v[m].z, r.v[m].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 p = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
        f[8 * m + 2 * e] = p.x;
        f[8 * m + 2 * e + 1] = p.y;
      }
    }
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* row, int s, const float (&f)[16]) {
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 p = __floats2bfloat162_rn(f[8 * m + 2 * e], f[8 * m + 2 * e + 1]);
        w[e] = *reinterpret_cast<const uint32_t*>(&p);
      }
      __stcs(reinterpret_cast<uint4*>(row + 8 * s + 64 * m), make_uint4(w[0], w[1], w[2], w[3]));
    }
  }
};

// One token's update of one row (the lane's 16 elements f, in place); returns o_r (in every
// lane of the row's group).  kn, qn: the lane's elements of the normalised k and q.  The one-
// and k-token kernels both call this, so that their results agree bit for bit.
__device__ __forceinline__ float row_update(float (&f)[16], const float (&kn)[16],
                                            const float (&qn)[16], float alpha, float beta,
                                            float vv, float kq) {
  // packed fp32 pairs (FFMA2): two element pairs per accumulator
  float2 dk2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  float2 dq2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    const float2 fj = make_float2(f[j], f[j + 1]);
    const int p = (j >> 1) & 1;
    dk2[p] = __ffma2_rn(fj, make_float2(kn[j], kn[j + 1]), dk2[p]);
    dq2[p] = __ffma2_rn(fj, make_float2(qn[j], qn[j + 1]), dq2[p]);
  }
  float dk = (dk2[0].x + dk2[0].y) + (dk2[1].x + dk2[1].y);
  float dq = (dq2[0].x + dq2[0].y) + (dq2[1].x + dq2[1].y);
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) {
    dk += __shfl_xor_sync(0xffffffffu, dk, o);
    dq += __shfl_xor_sync(0xffffffffu, dq, o);
  }
  const float u = beta * (vv - alpha * dk);
  const float2 a2 = make_float2(alpha, alpha), u2 = make_float2(u, u);
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    const float2 r = __ffma2_rn(u2, make_float2(kn[j], kn[j + 1]),
                                __fmul2_rn(a2, make_float2(f[j], f[j + 1])));
    f[j] = r.x;
    f[j + 1] = r.y;
  }
  return fmaf(alpha, dq, u * kq);
}

// One step of the causal conv (width 4, history s0 oldest .. s2 newest, input xv) and the SiLU;
// the one- and k-token kernels both call it, with the products in this fixed order.
__device__ __forceinline__ float conv_silu(const float (&w)[4], float s0, float s1, float s2,
                                           float xv) {
  return silu_f(fmaf(w[3], xv, fmaf(w[2], s2, fmaf(w[1], s1, w[0] * s0))));
}

// Input channel of position gch of the conv outputs of key head hk (q | k | v_0..v_{R-1}).
__device__ __forceinline__ int channel_of(int gch, int hk, int R, int Hk) {
  const int grp = gch / kHeadDim, off = gch % kHeadDim;
  if (grp == 0) return hk * kHeadDim + off;
  if (grp == 1) return Hk * kHeadDim + hk * kHeadDim + off;
  return 2 * Hk * kHeadDim + (hk * R + grp - 2) * kHeadDim + off;
}

template <typename T, typename TS>
__global__ void __launch_bounds__(kDecodeThreads, 4) decode_kernel(DecodeArgs a) {
  constexpr int d = kHeadDim;
  const int b = blockIdx.x / a.Hk;
  const int hk = blockIdx.x % a.Hk;
  const int R = a.Hv / a.Hk;
  const int Cc = (2 * a.Hk + a.Hv) * d;
  const int slot = state_row(a.slot_idx, b, a.num_slots);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grp = lane >> 3, sub = lane & 7;
  if (slot < 0) {  // slot out of range: the sequence is skipped, its outputs are not written
    if (tid == 0) report_status(a.status, GDN_ERR_INVALID_ARG);
    return;
  }

  __shared__ float y_s[(2 + kMaxR) * d];  // q | k | v_0..v_{R-1} after conv
  __shared__ float o_s[kMaxR * d];
  __shared__ float red_s[4];
  __shared__ float2 ab_s[kMaxR];          // (alpha, beta) per value head

  const T* x = static_cast<const T*>(a.x) + (size_t)b * Cc;
  const T* w = static_cast<const T*>(a.conv_w);
  T* cs = static_cast<T*>(a.conv_state) + (size_t)slot * 3 * Cc;

  // the first batch of state rows does not depend on q and k: its loads go out before the conv
  using RP = RowPart<TS>;
  constexpr int kQ = RP::kQuads;
  constexpr int kBatch = 4 * kQ;
  const int rows_per_warp = R * d / (kDecodeThreads / 32);
  const int nbatch = rows_per_warp / kBatch;
  TS* S = static_cast<TS*>(a.S);
  auto row_ptr = [&](int gr) {  // gr: row of the CTA's R d rows
    return S + ((size_t)slot * a.Hv + hk * R) * d * d + (size_t)gr * d;
  };
  typename RP::Raw cur[kQ], nxt[kQ];
#pragma unroll
  for (int q = 0; q < kQ; ++q) RP::load(cur[q], row_ptr(warp * rows_per_warp + 4 * q + grp), sub);

  if (tid < R) {
    const int h = hk * R + tid;
    ab_s[tid] = make_float2(expf(a.g[(size_t)b * a.Hv + h]), a.beta[(size_t)b * a.Hv + h]);
  }
  // ---- conv + SiLU with in-place history shift: 2 channels per item
  const int items = (2 + R) * d / 2;
  for (int it = tid; it < items; it += kDecodeThreads) {
    const int gch = it * 2;  // position inside y_s
    const int c = channel_of(gch, hk, R, a.Hk);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float s0 = to_f(cs[c + e]), s1 = to_f(cs[Cc + c + e]), s2 = to_f(cs[2 * Cc + c + e]);
      const T xt = x[c + e];
      const T* wr = w + (size_t)(c + e) * 4;
      const float wf[4] = {to_f(wr[0]), to_f(wr[1]), to_f(wr[2]), to_f(wr[3])};
      y_s[gch + e] = conv_silu(wf, s0, s1, s2, to_f(xt));
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
  float kn[16], qn[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    kn[j] = y_s[d + RP::col(sub, j)] * rk;
    qn[j] = y_s[RP::col(sub, j)] * rq;
  }

  // ---- state pass: the warp's rows in batches of kQ row quads, the next batch in flight
  for (int bt = 0; bt < nbatch; ++bt) {
    const int r0 = warp * rows_per_warp + bt * kBatch;
    if (bt + 1 < nbatch) {
#pragma unroll
      for (int q = 0; q < kQ; ++q) RP::load(nxt[q], row_ptr(r0 + kBatch + 4 * q + grp), sub);
    }
#pragma unroll
    for (int q = 0; q < kQ; ++q) {
      const int gr = r0 + 4 * q + grp, hr = gr / d;
      const float2 ab = ab_s[hr];
      float f[16];
      RP::unpack(cur[q], f);
      const float o = row_update(f, kn, qn, ab.x, ab.y, y_s[(2 + hr) * d + gr % d], kq);
      if (sub == 0) o_s[gr] = o;
      RP::store(row_ptr(gr), sub, f);
    }
#pragma unroll
    for (int q = 0; q < kQ; ++q) cur[q] = nxt[q];
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
// exactly the arithmetic of decode_kernel (the same row_update, the same normalised q and k
// products), so the results equal k calls of the one-token step.  Per-token constants (the
// normalised q and k, alpha, beta) are set up once in shared memory before the state pass.
// With `snaps` set, the state after every token is stored as well ([B, k, Hv, d, d] fp32), so
// that a caller that accepts only the first m tokens can take snapshot m - 1.
// The rows stream through shared memory: each warp keeps kMultiStages batches of 8 rows (4 KB,
// contiguous in the state) in flight as bulk copies (cp.async.bulk, no registers held while
// they are in flight), so that the k token updates of one batch overlap the loads of the next
// ones; the new rows go back to HBM from registers.  Dynamic shared memory: the warps' stages
// and their mbarriers, then per token (2 + R) d conv outputs (q and k normalised in place),
// R d outputs, three norms and R (alpha, beta) pairs.
constexpr int kMaxTokens = 8;
constexpr int kMultiStages = 2;
constexpr int kMultiBatchBytes = 8 * kHeadDim * 4;  // 8 rows of fp32
constexpr size_t kMultiRingBytes =
    (size_t)(kDecodeThreads / 32) * kMultiStages * kMultiBatchBytes + 128;  // + mbarriers

__host__ __device__ constexpr size_t multi_smem_floats(int k, int R) {
  return (size_t)k * (2 + 2 * R) * kHeadDim + 3 * k + 2 * k * R;
}
__host__ __device__ constexpr size_t multi_smem_bytes(int k, int R) {
  return kMultiRingBytes + (multi_smem_floats(k, R) + 1) * sizeof(float);
}

template <typename T>
__global__ void __launch_bounds__(kDecodeThreads, 4) decode_multi_kernel(DecodeArgs a, int k,
                                                                         float* snaps) {
  constexpr int d = kHeadDim;
  const int b = blockIdx.x / a.Hk;
  const int hk = blockIdx.x % a.Hk;
  const int R = a.Hv / a.Hk;
  const int Cc = (2 * a.Hk + a.Hv) * d;
  const int slot = state_row(a.slot_idx, b, a.num_slots);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grp = lane >> 3, sub = lane & 7;
  if (slot < 0) {  // slot out of range: the sequence is skipped, its outputs are not written
    if (tid == 0) report_status(a.status, GDN_ERR_INVALID_ARG);
    return;
  }
  extern __shared__ __align__(128) uint8_t dsm_raw[];
  uint8_t* ring = dsm_raw + (size_t)warp * kMultiStages * kMultiBatchBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(dsm_raw + kMultiRingBytes - 128) + warp * kMultiStages;
  float* dsm = reinterpret_cast<float*>(dsm_raw + kMultiRingBytes);
  float* y_s = dsm;                          // [k][(2 + R) d]: q | k | v_0..v_{R-1}
  float* o_s = y_s + k * (2 + R) * d;        // [k][R d]
  float* red_s = o_s + k * R * d;            // [k][3]: |q|^2, |k|^2, q.k
  float2* ab_s = reinterpret_cast<float2*>(red_s + 3 * k + (k & 1));  // [k][R]

  const T* w = static_cast<const T*>(a.conv_w);
  T* cs = static_cast<T*>(a.conv_state) + (size_t)slot * 3 * Cc;
  using RP = RowPart<float>;
  constexpr int kQ = RP::kQuads;
  constexpr int kBatch = 4 * kQ;
  const int rows_per_warp = R * d / (kDecodeThreads / 32);
  const int nbatch = rows_per_warp / kBatch;
  float* S = static_cast<float*>(a.S);
  auto row_off = [&](int gr) { return ((size_t)slot * a.Hv + hk * R) * d * d + (size_t)gr * d; };
  // the first stages of this warp's rows go out before the conv (they do not depend on it)
  auto issue = [&](int bt) {  // lane 0: batch bt of the warp into its stage
    const int st = bt % kMultiStages;
    mbar_arrive_expect_tx(bars + st, kMultiBatchBytes);
    bulk_load(ring + st * kMultiBatchBytes, S + row_off(warp * rows_per_warp + bt * kBatch),
              kMultiBatchBytes, bars + st);
  };
  if (lane == 0) {
    for (int st = 0; st < kMultiStages; ++st) mbar_init(bars + st, 1);
    fence_barrier_init();
    for (int bt = 0; bt < kMultiStages && bt < nbatch; ++bt) issue(bt);
  }
  __syncwarp();

  for (int i = tid; i < k * R; i += kDecodeThreads) {
    const int t = i / R, h = hk * R + i % R;
    const size_t gi = ((size_t)b * k + t) * a.Hv + h;
    ab_s[i] = make_float2(expf(a.g[gi]), a.beta[gi]);
  }
  // ---- conv + SiLU over the k tokens, history in registers, final history written back.
  // Every load of an item goes out before its first step (one memory latency per item).
  const int items = (2 + R) * d / 2;
  const T* xb = static_cast<const T*>(a.x) + (size_t)b * k * Cc;
  for (int it = tid; it < items; it += kDecodeThreads) {
    const int gch = it * 2;
    const int c = channel_of(gch, hk, R, a.Hk);
    T xs[kMaxTokens][2];
#pragma unroll
    for (int t = 0; t < kMaxTokens; ++t) {
#pragma unroll
      for (int e = 0; e < 2; ++e) xs[t][e] = t < k ? xb[(size_t)t * Cc + c + e] : T();
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float s0 = to_f(cs[c + e]), s1 = to_f(cs[Cc + c + e]), s2 = to_f(cs[2 * Cc + c + e]);
      const T* wr = w + (size_t)(c + e) * 4;
      const float wf[4] = {to_f(wr[0]), to_f(wr[1]), to_f(wr[2]), to_f(wr[3])};
      T xt = T();
#pragma unroll
      for (int t = 0; t < kMaxTokens; ++t) {
        if (t < k) {
          xt = xs[t][e];
          y_s[t * (2 + R) * d + gch + e] = conv_silu(wf, s0, s1, s2, to_f(xt));
          s0 = s1;
          s1 = s2;
          s2 = to_f(xt);
        }
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
  // ---- q and k normalised in place, and k.q of the normalised vectors (the values the
  // one-token kernel forms in registers, by the same expressions)
  for (int i = tid; i < k * 2 * d; i += kDecodeThreads) {
    const int t = i / (2 * d), c = i % (2 * d);
    const float rq = a.q_scale * rsqrtf(red_s[t * 3] + a.l2_eps);
    const float rk = rsqrtf(red_s[t * 3 + 1] + a.l2_eps);
    y_s[t * (2 + R) * d + c] *= c < d ? rq : rk;
    if (c == 0) red_s[t * 3 + 2] = red_s[t * 3 + 2] * rq * rk;  // read by no other thread here
  }
  __syncthreads();

  // ---- state pass: each batch of row quads takes the k updates in registers
  int issued = min(kMultiStages, nbatch), bt = 0;
  bool ok = true;
  for (; bt < nbatch; ++bt) {
    const int r0 = warp * rows_per_warp + bt * kBatch;
    const int st = bt % kMultiStages;
    ok = mbar_wait(bars + st, (bt / kMultiStages) & 1);
    if (!__all_sync(0xffffffffu, ok)) break;
    float f[kQ][16];
#pragma unroll
    for (int q = 0; q < kQ; ++q) {
      const float* src = reinterpret_cast<const float*>(ring + st * kMultiBatchBytes) +
                         (4 * q + grp) * d + 4 * sub;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float4 v = *reinterpret_cast<const float4*>(src + 32 * m);
        f[q][4 * m] = v.x, f[q][4 * m + 1] = v.y, f[q][4 * m + 2] = v.z, f[q][4 * m + 3] = v.w;
      }
    }
    __syncwarp();  // every lane has read the stage: it takes batch bt + kMultiStages next
    if (lane == 0 && issued < nbatch) {
      fence_proxy_async_smem();
      issue(issued++);
    }
    for (int t = 0; t < k; ++t) {
      const float* yt = y_s + t * (2 + R) * d;
      const float kq = red_s[t * 3 + 2];
      float kn[16], qn[16];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float4 kv = *reinterpret_cast<const float4*>(yt + d + 4 * sub + 32 * m);
        const float4 qv = *reinterpret_cast<const float4*>(yt + 4 * sub + 32 * m);
        kn[4 * m] = kv.x, kn[4 * m + 1] = kv.y, kn[4 * m + 2] = kv.z, kn[4 * m + 3] = kv.w;
        qn[4 * m] = qv.x, qn[4 * m + 1] = qv.y, qn[4 * m + 2] = qv.z, qn[4 * m + 3] = qv.w;
      }
#pragma unroll
      for (int q = 0; q < kQ; ++q) {
        const int gr = r0 + 4 * q + grp, hr = gr / d;
        const float2 ab = ab_s[t * R + hr];
        const float o = row_update(f[q], kn, qn, ab.x, ab.y, yt[(2 + hr) * d + gr % d], kq);
        if (sub == 0) o_s[t * R * d + gr] = o;
        if (snaps)
          RP::store(snaps + (((size_t)b * k + t) * a.Hv + hk * R) * d * d + (size_t)gr * d, sub,
                    f[q]);
      }
    }
#pragma unroll
    for (int q = 0; q < kQ; ++q) RP::store(S + row_off(r0 + 4 * q + grp), sub, f[q]);
  }
  if (bt < nbatch) {
    // a wait ran out: report it, let the copies still in flight land (bounded), leave the rest
    if (lane == 0) {
      report_status(a.status, GDN_ERR_TIMEOUT);
      for (int b2 = bt; b2 < issued; ++b2)
        mbar_wait(bars + b2 % kMultiStages, (b2 / kMultiStages) & 1);
    }
    __syncwarp();
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
  const size_t smem = gdn::multi_smem_bytes(k, R);
  static bool attr = false;
  if (!attr) {  // the largest request: kMaxTokens tokens, kMaxR value heads per key head
    const int most = (int)gdn::multi_smem_bytes(gdn::kMaxTokens, gdn::kMaxR);
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
