// prefill_tc.cu -- chunked Gated DeltaNet prefill on tcgen05 tensor cores (bf16 operands, fp32
// accumulation in TMEM, fp32 recurrent state).
//
// Source: the recurrence of the hyper.ai Gated DeltaNet paragraph (as read in gdn.h), evaluated
// in chunks with the WY / UT-transform form used by the FLA kernels that the "Qwen3-Next"
// SGLang cookbook names in section 3.2 (chunk 64 there; 128 here, one tcgen05 M=128 tile).
// Per value head and chunk of L <= 128 tokens (G = cumulative log decay inside the chunk):
//   A_ij = beta_i exp(G_i - G_j) k_i.k_j (j < i),  T = (I + A)^-1
//   W = T diag(beta) diag(e^G) K,   U~ = T diag(beta) V
//   U = U~ - W S^T,   O = diag(e^G) Q S^T + P U,   P_ij = e^(G_i - G_j) q_i.k_j (j <= i)
//   S <- e^(G_L) S + U^T diag(e^(G_L - G)) K
// Padded rows of a partial chunk carry k = q = v = 0, beta = 0, g = 0, which changes nothing.
//
// Kernels (in order, programmatic dependent launch between them; optionally pipelined):
//   schedule   one CTA: chunk table (sequence, first token, length) from cu_seqlens.
//   qkv        per (chunk, 128-channel slice): conv + SiLU + L2 norms -> bf16 Q, K, V tiles.
//   prep       per (chunk, value head): gates, K K^T on tcgen05, the 128x128 inverse (four
//              32x32 in-warp row substitutions joined on tcgen05 in two levels), then W and U~.
//   chain      per (sequence, value head, d_v block): the sequential part; S^T lives in TMEM
//              (fp32); per chunk: X = W S_b^T (tcgen05), U = U~ - X, S^T += K^T diag(.) U.
//   out        per (chunk, value head): P from Q K^T, O = e^G Q S^T + P U (TMEM A operands),
//              z-gated RMSNorm epilogue, bf16 output.
// Workspace tiles are plain row-major [128][128] bf16; TMA loads them with 128-byte swizzle.
#include "args.cuh"
#include "common.cuh"
#include "tc.cuh"

#include <cudaTypedefs.h>

#include <algorithm>
#include <utility>
#include <cstdlib>

namespace gdn {

constexpr int kC = 128;  // chunk length (tokens)
constexpr int kD = 128;  // head dim
constexpr uint32_t kTile = 16384;  // one [128][64] bf16 row tile



// ------------------------------------------------------------------------------ schedule
__global__ void chunk_schedule_kernel(const int32_t* __restrict__ cu, int N, int T,
                                      Workspace ws, const __nv_bfloat16* conv0,
                                      __nv_bfloat16* convN, const int32_t* slot, int num_slots,
                                      int Cc, int32_t* status) {
  // single CTA: prefix sums over sequences (in blocks of blockDim) of their 128-token chunks
  // and of their 64-token pages, then the chunk entries written in parallel
  __shared__ int carry, carry_p;
  __shared__ int part[1024], part_p[1024];
  if (threadIdx.x == 0) carry = carry_p = 0;
  __syncthreads();
  for (int base = 0; base < N; base += blockDim.x) {
    const int n = base + threadIdx.x;
    int cnt = 0, pages = 0;
    // bounds-check build: a sequence whose cu_seqlens entries are out of order or past T gets
    // no chunks (and GDN_ERR_BOUNDS)
    if (n < N && GDN_IN_BOUNDS(cu[n] >= 0 && cu[n + 1] >= cu[n] && cu[n + 1] <= T, status)) {
      cnt = (cu[n + 1] - cu[n] + kC - 1) / kC;
      pages = (cu[n + 1] - cu[n] + 63) / 64;
    }
    part[threadIdx.x] = cnt;
    part_p[threadIdx.x] = pages;
    __syncthreads();
    for (int off = 1; off < (int)blockDim.x; off <<= 1) {  // inclusive scans
      const bool in = threadIdx.x >= (unsigned)off;
      const int v = in ? part[threadIdx.x - off] : 0, vp = in ? part_p[threadIdx.x - off] : 0;
      __syncthreads();
      part[threadIdx.x] += v;
      part_p[threadIdx.x] += vp;
      __syncthreads();
    }
    if (n < N) {
      ws.seq_first[n] = carry + part[threadIdx.x] - cnt;
      ws.page_first[n] = carry_p + part_p[threadIdx.x] - pages;
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) {
      carry += part[threadIdx.x];
      carry_p += part_p[threadIdx.x];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    ws.seq_first[N] = carry;
    ws.page_first[N] = carry_p;
  }
  __syncthreads();  // seq_first (global, written by this CTA) is visible to all its threads
  // chunk entries: chunk k belongs to the last sequence n with seq_first[n] <= k
  const int total = carry;
  for (int k = threadIdx.x; k < total; k += blockDim.x) {
    int lo = 0, hi = N;  // seq_first[lo] <= k < seq_first[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (ws.seq_first[mid] <= k) lo = mid; else hi = mid;
    }
    ChunkInfo info;
    info.n = lo;
    info.t0 = cu[lo] + (k - ws.seq_first[lo]) * kC;
    info.L = min(kC, cu[lo + 1] - info.t0);
    info.pad = k - ws.seq_first[lo];
    ws.chunks[k] = info;
  }
  // final conv history of empty sequences (the q/k/v kernel writes the others): the initial one
  if (convN) {
    for (int n = 0; n < N; ++n) {
      if (cu[n + 1] != cu[n]) continue;
      const int srow = state_row(slot, n, num_slots);
      if (srow < 0) {
        if (threadIdx.x == 0) report_status(status, GDN_ERR_INVALID_ARG);
        continue;
      }
      const size_t row = (size_t)srow * 3 * Cc;
      for (int k = threadIdx.x; k < 3 * Cc; k += blockDim.x)
        convN[row + k] = conv0 ? conv0[row + k] : __float2bfloat16(0.f);
    }
  }
}


// --------------------------------------------------------------------------------- q/k/v
__device__ __forceinline__ void unpack8(const uint4& u, float (&v)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// silu(x) = x * sigmoid(x), sigmoid(x) = (1 + tanh(x / 2)) / 2: one transcendental per element.
__device__ __forceinline__ float silu_fast(float x) {
  const float h = 0.5f * x;
  return fmaf(h, tanh_approx(h), h);
}

// One CTA per (chunk, 128-channel group of the conv input): causal conv (width 4) + SiLU, and
// for q and k the L2 norm of every (token, head) row.  The chunk's input rows, with the 3
// preceding rows, arrive by TMA as two [131][64] boxes (128-byte swizzle); for the first chunk
// of a sequence the 3 preceding rows are replaced by the caller's conv state (or zeros).
// 128 threads: 16 column vectors x 8 runs of 16 tokens; the 16 threads of a row share a
// half-warp, so the norm is a 4-step shuffle.  At most 96 registers: five CTAs per SM.  Outputs are bf16 [128][128] tiles per (chunk,
// head): Q -> Qw, K -> Kw, V -> Uw (read by gdn_prep, which overwrites it with U~).  Rows past
// the chunk's length are written as zeros.
constexpr int kXRows = kC + 3;
constexpr uint32_t kXBox = 17408;  // one [131][64] bf16 box, rounded up to 1024 bytes
constexpr uint32_t kQkvSmem = 2 * kXBox + 1024 + 64;

__global__ void __launch_bounds__(128, 5) gdn_qkv_kernel(PrefillArgs a,
                                                         const __grid_constant__ CUtensorMap mapX) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + 2 * kXBox);
  const int grp = blockIdx.x, c = a.c0 + blockIdx.y;
  pdl_wait();  // the chunk table, and the end of every reader of the previous call's tiles
  if (c >= a.ws.seq_first[a.N]) return;
  const ChunkInfo ci = a.ws.chunks[c];
  if (!GDN_IN_BOUNDS(ci.n >= 0 && ci.n < a.N && ci.t0 >= 0 && ci.L > 0 && ci.L <= kC &&
                         ci.t0 + ci.L <= a.T, a.status))
    return;
  const int tid = threadIdx.x, vec = tid & 15, run = tid >> 4;
  const int Hk = a.Hk, Hv = a.Hv;
  const int Cc = (2 * Hk + Hv) * kD;
  const int kind = grp < Hk ? 0 : (grp < 2 * Hk ? 1 : 2);
  const int head = kind == 0 ? grp : (kind == 1 ? grp - Hk : grp - 2 * Hk);
  const int ch = grp * kD + vec * 8;
  const int seq_start = __ldg(a.cu + ci.n);
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
    mbar_arrive_expect_tx(bar, 2 * kXRows * 128);
    tma_load_2d(sm, &mapX, bar, grp * kD, ci.t0 - 3);
    tma_load_2d(sm + kXBox, &mapX, bar, grp * kD + 64, ci.t0 - 3);
  }
  __syncthreads();  // the barrier is initialised before any thread waits on it
  __nv_bfloat16* dst = (kind == 0 ? a.ws.Qw + ((size_t)c * Hk + head) * kC * kD
                      : kind == 1 ? a.ws.Kw + ((size_t)c * Hk + head) * kC * kD
                                  : a.ws.Uw + ((size_t)c * Hv + head) * kC * kD) + vec * 8;
  float2 wv[4][4];  // taps x channel pairs
  if (a.conv_w) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      uint2 u = *reinterpret_cast<const uint2*>(a.conv_w + (size_t)(ch + e) * 4);
      const __nv_bfloat162* hw = reinterpret_cast<const __nv_bfloat162*>(&u);
      const float2 f0 = __bfloat1622float2(hw[0]), f1 = __bfloat1622float2(hw[1]);
      const float t[4] = {f0.x, f0.y, f1.x, f1.y};
#pragma unroll
      for (int k = 0; k < 4; ++k) {  // halved: the conv then yields h = x / 2 for the SiLU
        if (e & 1) wv[k][e >> 1].y = 0.5f * t[k]; else wv[k][e >> 1].x = 0.5f * t[k];
      }
    }
  }
  uint8_t* box = sm + (vec >> 3) * kXBox;
  const uint32_t chunk = vec & 7;
  auto row_ptr = [&](int r) { return reinterpret_cast<uint4*>(box + sw128_off(r, chunk)); };
  const bool ok = mbar_wait(bar, 0, a.wait_ns);
  pdl_trigger();
  if (!ok) {
    if (tid == 0) report_status(a.status, GDN_ERR_TIMEOUT);
    return;
  }
  // state-pool row of the sequence (-1: its slot is out of range, no pool access)
  const int srow = state_row(a.slot, ci.n, a.num_slots);
  if (srow < 0 && tid == 0) report_status(a.status, GDN_ERR_INVALID_ARG);
  // first chunk of a sequence: the 3 rows before it come from the conv state (or are zero)
  if (ci.t0 == seq_start && run == 0) {
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (a.conv0 && srow >= 0)
        v = *reinterpret_cast<const uint4*>(a.conv0 + ((size_t)srow * 3 + j) * Cc + ch);
      *row_ptr(j) = v;
    }
  }
  __syncthreads();
  // last chunk of its sequence: the final conv history is the box's rows L .. L+2 (the three
  // inputs before the sequence end, conv state rows included when L < 3)
  if (a.convN && srow >= 0 && run == 0 && ci.t0 + ci.L == __ldg(a.cu + ci.n + 1)) {
#pragma unroll
    for (int j = 0; j < 3; ++j)
      *reinterpret_cast<uint4*>(a.convN + ((size_t)srow * 3 + j) * Cc + ch) =
          *row_ptr(ci.L + j);
  }
  const int i0 = run * 16;
  float2 hst[3][4];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    float v8[8];
    unpack8(*row_ptr(i0 + j), v8);
#pragma unroll
    for (int p = 0; p < 4; ++p) hst[j][p] = make_float2(v8[2 * p], v8[2 * p + 1]);
  }
  const float sc_mul = kind == 0 ? a.q_scale : 1.0f;
#pragma unroll 4
  for (int u = 0; u < 16; ++u) {
    const int i = i0 + u;
    float xv[8], y[8];
    unpack8(*row_ptr(i + 3), xv);
    float2 y2[4];
    if (a.conv_w) {
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float2 xp = make_float2(xv[2 * p], xv[2 * p + 1]);
        float2 hh = __fmul2_rn(wv[3][p], xp);  // h = conv / 2
        hh = __ffma2_rn(wv[2][p], hst[2][p], hh);
        hh = __ffma2_rn(wv[1][p], hst[1][p], hh);
        hh = __ffma2_rn(wv[0][p], hst[0][p], hh);
        // silu(x) = x sigmoid(x) = h + h tanh(h), h = x / 2
        y2[p] = __ffma2_rn(hh, make_float2(tanh_approx(hh.x), tanh_approx(hh.y)), hh);
        hst[0][p] = hst[1][p];
        hst[1][p] = hst[2][p];
        hst[2][p] = xp;
      }
    } else {
#pragma unroll
      for (int p = 0; p < 4; ++p) y2[p] = make_float2(xv[2 * p], xv[2 * p + 1]);
    }
    if (kind < 2) {
      float2 s2 = __fmul2_rn(y2[0], y2[0]);
#pragma unroll
      for (int p = 1; p < 4; ++p) s2 = __ffma2_rn(y2[p], y2[p], s2);
      float ss = s2.x + s2.y;
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float sc = sc_mul * rsqrtf(ss + a.l2_eps);
#pragma unroll
      for (int p = 0; p < 4; ++p) y2[p] = __fmul2_rn(y2[p], make_float2(sc, sc));
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      y[2 * p] = y2[p].x;
      y[2 * p + 1] = y2[p].y;
    }
    if (i >= ci.L) {
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] = 0.f;
    }
    store8(dst + (size_t)i * kD, y);
  }
}

// ---------------------------------------------------------------------------------- prep
// One CTA per (chunk, value head), 8 warps, two CTAs per SM.  K and V arrive by TMA from the
// tiles gdn_qkv wrote.  Gates -> K K^T (tcgen05) -> A -> two 64x64 forward substitutions (CUDA
// cores) -> Y = N T_h, Z' = T_h Y diag(beta) (tcgen05) -> T diag(beta) -> W and U~ (tcgen05).
// smem map (bytes from the 1024-aligned base)
constexpr uint32_t kPrepKs = 0;        // K (TMA) -> K^ = diag(e^G) K, in place
constexpr uint32_t kPrepR1 = 32768;    // D -> T_h -> T diag(beta), row-major bf16
constexpr uint32_t kPrepR2 = 65536;    // N (16 KB) + compact Y1 (16 KB) / Y' (8 KB) -> V (TMA)
constexpr uint32_t kPrepEnd = 98304;
constexpr uint32_t kPrepSmem = kPrepEnd + 1024 + 2048;
// TMEM columns (256 allocated)
constexpr uint32_t kColGram = 0, kColY = 128, kColZ = 192, kColW = 0, kColU = 128;
constexpr uint32_t kColL = 128, kColY1 = 0, kColZ1 = 0;  // 32 -> 64 join (L1: packed bf16)

// tcgen05.mma with the A operand in TMEM (row i in lane i, two bf16 per 32-bit column; one
// K step of 16 = 8 columns) and B in shared memory.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void zero_row_chunk(uint8_t* tile, uint32_t row, uint32_t chunk) {
  *reinterpret_cast<uint4*>(tile + sw128_off(row, chunk)) = make_uint4(0, 0, 0, 0);
}

// Barriers and small arrays of a prep CTA, above the tiles.
struct PrepCtl {
  float* G_s;       // [128]
  float* B_s;       // [128]
  float* wt_s;      // [8] warp totals
  float* F_s;       // [128] column factors
  uint64_t* bar_k;  // K landed
  uint64_t* bar_v;  // V landed
  uint64_t* bar;    // MMA completions (six per unit)
  uint64_t* bar_w;  // W products done
  uint32_t* tslot;  // TMEM address
  int* unit;        // next work unit (persistent workers)
  __device__ explicit PrepCtl(uint8_t* sm) {
    G_s = reinterpret_cast<float*>(sm + kPrepEnd);
    B_s = G_s + kC;
    wt_s = B_s + kC;
    F_s = wt_s + 8;
    bar_k = reinterpret_cast<uint64_t*>(F_s + kC);
    bar_v = bar_k + 1;
    bar = bar_k + 2;
    bar_w = bar_k + 3;
    tslot = reinterpret_cast<uint32_t*>(bar_k + 4);
    unit = reinterpret_cast<int*>(tslot + 1);
  }
  __device__ void init() const {  // one thread; a __syncthreads must follow before any wait
    mbar_init(bar_k, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar, 1);
    mbar_init(bar_w, 1);
    fence_barrier_init();
  }
};

// One (chunk c, value head h) unit of prep on a CTA whose barriers are initialised and whose 256
// TMEM columns are allocated.  `par` is the parity of this unit on bar_k, bar_v and bar_w (one
// completion each per unit; bar completes six times, so its parity starts at 0 every unit).
// Returns false after a wait ran out (the status word is set).
__device__ __forceinline__ bool prep_unit(const PrefillArgs& a, const CUtensorMap& mapK,
                                          const CUtensorMap& mapV, const CUtensorMap& mapW,
                                          int c, int h, uint8_t* sm, uint32_t tmem,
                                          uint32_t par) {
  const PrepCtl ctl(sm);
  float* G_s = ctl.G_s;
  float* B_s = ctl.B_s;
  float* wt_s = ctl.wt_s;
  float* F_s = ctl.F_s;
  uint64_t* bar_k = ctl.bar_k;
  uint64_t* bar_v = ctl.bar_v;
  uint64_t* bar = ctl.bar;
  uint64_t* bar_w = ctl.bar_w;
  const ChunkInfo ci = a.ws.chunks[c];
  if (!GDN_IN_BOUNDS(ci.t0 >= 0 && ci.L > 0 && ci.L <= kC && ci.t0 + ci.L <= a.T, a.status))
    return false;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int quarter = warp & 3, wg = warp >> 2;
  const int Hv = a.Hv;
  const int hk = h / (Hv / a.Hk);

  // thread 128 (a warp that does not scan the gates) waits for the q/k/v tiles of the previous
  // kernel and starts the K load; the gates below overlap that kernel's tail
  if (tid == 128) {
    pdl_wait();
    const int rowK = (c * a.Hk + hk) * kC;
    mbar_arrive_expect_tx(bar_k, 2 * kTile);
    tma_load_2d(sm + kPrepKs, &mapK, bar_k, 0, rowK);
    tma_load_2d(sm + kPrepKs + kTile, &mapK, bar_k, 64, rowK);
    // V is loaded once the joins have released its buffer; bring it into L2 meanwhile
    const int rowV = (c * Hv + h) * kC;
    tma_prefetch_2d(&mapV, 0, rowV);
    tma_prefetch_2d(&mapV, 64, rowV);
  }
  // ---------------- gates: G = inclusive cumsum of g inside the chunk, beta
  if (warp < 4) {
    const int i = warp * 32 + lane;
    const bool valid = i < ci.L;
    float gv = valid ? __ldg(a.g + (size_t)(ci.t0 + i) * Hv + h) : 0.f;
    const float bv = valid ? __ldg(a.beta + (size_t)(ci.t0 + i) * Hv + h) : 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, gv, o);
      if (lane >= o) gv += y;
    }
    if (lane == 31) wt_s[warp] = gv;
    B_s[i] = bv;
    G_s[i] = gv;  // warp-local prefix; completed below
  }
  __syncthreads();
  if (warp < 4) {
    const int i = warp * 32 + lane;
    float pre = 0.f;
    for (int w = 0; w < warp; ++w) pre += wt_s[w];
    const float gv = G_s[i] + pre;
    G_s[i] = gv;
    a.ws.Gw[((size_t)c * Hv + h) * kC + i] = gv;
  }
  __syncthreads();
  // column factors exp(G_m - G_j), m = last column of j's 32-column chunk (exponent <= 0)
  if (tid < kC) F_s[tid] = __expf(G_s[tid | 31] - G_s[tid]);
  __syncthreads();
  tc_fence_after();
  const uint32_t sKs = smem_u32(sm + kPrepKs);
  const uint32_t lane_addr = tmem_at(tmem, quarter * 32, 0);
  uint32_t phase = 0;
  bool ok = true;
  // ---------------- gram K K^T
  if (tid == 0) {
    ok = mbar_wait(bar_k, par, a.wait_ns);
    tc_fence_after();
    if (ok) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem + kColGram, desc_kmajor(sKs, kk, kTile), desc_kmajor(sKs, kk, kTile),
                 idesc_bf16(128, 128, false, false), kk > 0);
      mma_commit(bar);
    }
  }
  if (__syncthreads_or(!ok)) goto done;
  ok = mbar_wait(bar, phase, a.wait_ns);
  phase ^= 1;
  if (__syncthreads_or(!ok)) goto done;
  tc_fence_after();
  {
  // ---------------- A from the gram: thread row i, column half wg (two 32-column chunks).
  // The diagonal 32x32 blocks stay in the registers of the warps that invert them (row block q
  // in column half q / 2: warps 0, 1, 6, 7).  The blocks (1,0) and (3,2) go to TMEM as the
  // bf16 A operand L1 of the 32 -> 64 join; rows 64..127 x columns 0..63 go to the bf16 tile N
  // of the 64 -> 128 join.  Everything above the diagonal is zero.
  const int i = quarter * 32 + lane;
  const bool solver = (quarter >> 1) == wg;  // warp-uniform
  float adiag[32];
  {
    const float Gi = G_s[i], bi = B_s[i];
    uint8_t* Nt = sm + kPrepR2;
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int j0 = wg * 64 + cc * 32;
      const int bj = j0 >> 5;  // column block (warp-uniform)
      if (bj > quarter) continue;
      float v[32];
      tmem_ld32(lane_addr + kColGram + j0, v);
      if (bj < quarter) {
        // every j < every i: exp(G_i - G_j) = exp(G_i - G_m) exp(G_m - G_j), m = j0 + 31,
        // both exponents <= 0
        const float rf = bi * __expf(Gi - G_s[j0 + 31]);
        tmem_ld_wait();
        float av[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) av[e] = rf * F_s[j0 + e] * v[e];
        if (wg == 0 && quarter >= 2) {
          // N: rows 64..127, columns 0..63 (bf16, K-major)
#pragma unroll
          for (int q = 0; q < 4; ++q) st_row8_bf16(Nt, kTile, i, (j0 >> 3) + q, av + 8 * q);
        } else {
          // (1,0) or (3,2): L1 row, packed bf16 pairs at K = j0 .. j0 + 31 of 128
          float pk[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) pk[e] = 0.f;
          const int g = (j0 >> 1) >> 5;  // 32-column group of the packed K range
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[((j0 >> 1) & 31) + e] = __uint_as_float(pack_bf16x2(av[2 * e], av[2 * e + 1]));
          float zz[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) zz[e] = 0.f;
          tmem_st32(lane_addr + kColL + g * 32, pk);
          tmem_st32(lane_addr + kColL + (g ^ 1) * 32, zz);
        }
      } else {
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int j = j0 + e;
          adiag[e] = lower_decay(j < i, Gi, G_s[j], bi * v[e]);
        }
      }
    }
    if (wg == 0 && quarter < 2) {
#pragma unroll
      for (int q = 0; q < 8; ++q) zero_row_chunk(Nt, i, q);  // N rows 0..63 are zero
    }
    if (warp == 2 || warp == 4) {
      // L1 rows 64..95 (warp 2) and 0..31 (warp 4) are zero
      float zz[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) zz[e] = 0.f;
      tmem_st32(lane_addr + kColL, zz);
      tmem_st32(lane_addr + kColL + 32, zz);
    }
  }
  // ---------------- the four 32x32 diagonal inverses, one warp each, row i in lane i % 32:
  // T_qq = (I + A_qq)^-1 row by row, T[l] = e_l - sum_{j<l} A[l][j] T[j]; row j is broadcast by
  // shuffle once it is final (A[l][j] = 0 for j >= l, so every lane may take every step).
  float trow[32];
  uint8_t* Dt = sm + kPrepR1;  // D = blockdiag(T_00, T_11, T_22, T_33), row-major bf16
  if (solver) {
#pragma unroll
    for (int e = 0; e < 32; ++e) trow[e] = (e == lane) ? 1.f : 0.f;
#pragma unroll
    for (int j = 0; j < 31; ++j) {
      const float2 cj = make_float2(-adiag[j], -adiag[j]);
#pragma unroll
      for (int e = 0; e <= j; e += 2) {
        if (e + 1 <= j) {
          const float x0 = __shfl_sync(0xffffffffu, trow[e], j);
          const float x1 = __shfl_sync(0xffffffffu, trow[e + 1], j);
          const float2 o = __ffma2_rn(cj, make_float2(x0, x1), make_float2(trow[e], trow[e + 1]));
          trow[e] = o.x;
          trow[e + 1] = o.y;
        } else {
          const float x0 = __shfl_sync(0xffffffffu, trow[e], j);
          trow[e] = fmaf(cj.x, x0, trow[e]);
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) st_row8_bf16(Dt, kTile, i, quarter * 4 + q, trow + 8 * q);
#pragma unroll
    for (int q = 0; q < 4; ++q) zero_row_chunk(Dt + wg * kTile, i, ((quarter & 1) ? 0 : 4) + q);
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) zero_row_chunk(Dt + wg * kTile, i, q);
    // meanwhile K^ = diag(e^G) K in place (the gram has consumed K): one row per thread
    const int row = ((warp - 2) & 3) * 32 + lane;  // warps 2..5 -> rows 0..127
    const float gam = __expf(G_s[row]);
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const uint32_t off = (q >> 3) * kTile + sw128_off(row, q & 7);
      uint4 u = *reinterpret_cast<const uint4*>(sm + kPrepKs + off);
      __nv_bfloat162* hv = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(hv[e]);
        hv[e] = __floats2bfloat162_rn(f.x * gam, f.y * gam);
      }
      *reinterpret_cast<uint4*>(sm + kPrepKs + off) = u;
    }
  }
  tmem_st_wait();
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  // ---------------- 32 -> 64:  T_64 = D - D L1 D   (Y1 = L1 D, Z1 = D Y1; (L1 D)^2 = 0 inside
  // each 64 block).  L1 is non-zero in the K ranges 0..31 and 64..95 only.
  const uint32_t sD = smem_u32(Dt);
  uint8_t* Yc = sm + kPrepR2 + kTile;  // Y1 rows 32..63 and 96..127, compacted: [64][128] bf16
  if (tid == 0) {
    tc_fence_after();
    constexpr uint32_t id = idesc_bf16(128, 128, false, true);
    const int ks[4] = {0, 1, 4, 5};
#pragma unroll
    for (int t = 0; t < 4; ++t)
      mma_bf16_ts(tmem + kColY1, tmem + kColL + ks[t] * 8, desc_mnmajor(sD, ks[t], kTile), id,
                  t > 0);
    mma_commit(bar);
  }
  ok = mbar_wait(bar, phase, a.wait_ns);
  phase ^= 1;
  if (__syncthreads_or(!ok)) goto done;
  tc_fence_after();
  if (quarter & 1) {
    // rows 32..63 -> compact rows 0..31, rows 96..127 -> 32..63 (swizzle phase kept: row & 7)
    const int cr = quarter == 1 ? i - 32 : i - 64;
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      float v[32];
      tmem_ld32(lane_addr + kColY1 + wg * 64 + cc * 32, v);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) st_row8_bf16(Yc, 8192, cr, wg * 8 + cc * 4 + q, v + 8 * q);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    tc_fence_after();
    constexpr uint32_t id = idesc_bf16(128, 128, false, true);
    const uint32_t sYc = smem_u32(Yc);
    const int ks[4] = {2, 3, 6, 7};
#pragma unroll
    for (int t = 0; t < 4; ++t)
      mma_bf16(tmem + kColZ1, desc_kmajor(sD, ks[t], kTile), desc_mnmajor(sYc, t, 8192), id,
               t > 0);
    mma_commit(bar);
  }
  ok = mbar_wait(bar, phase, a.wait_ns);
  phase ^= 1;
  if (__syncthreads_or(!ok)) goto done;
  tc_fence_after();
  if ((quarter == 1 && wg == 0) || (quarter == 3 && wg == 1)) {
    // -Z1 into the (1,0) and (3,2) blocks: D becomes T_h = blockdiag(T_64, T_64')
    const int c0 = quarter == 1 ? 0 : 64;
    float v[32];
    tmem_ld32(lane_addr + kColZ1 + c0, v);
    tmem_ld_wait();
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] = -v[e];
#pragma unroll
    for (int q = 0; q < 4; ++q) st_row8_bf16(Dt, kTile, i, (c0 >> 3) + q, v + 8 * q);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  // ---------------- 64 -> 128:  T = T_h - T_h N T_h diag... (N = rows 64..127, cols 0..63)
  // ---- Y = N T_h (M=128, N=64, K=64): B = T_h rows 0..63, columns 0..63 (MN-major)
  if (tid == 0) {
    tc_fence_after();
    const uint32_t sN = smem_u32(sm + kPrepR2);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tmem + kColY, desc_kmajor(sN, kk, kTile), desc_mnmajor(sD, kk, kTile),
               idesc_bf16(128, 64, false, true), kk > 0);
    mma_commit(bar);
  }
  ok = mbar_wait(bar, phase, a.wait_ns);
  phase ^= 1;
  if (__syncthreads_or(!ok)) goto done;
  tc_fence_after();
  // ---- Y' = Y diag(beta) restricted to rows 64..127, cols 0..63 -> bf16 [64][64]
  if (quarter >= 2) {
    const int half = wg;
    float v[32];
    tmem_ld32(lane_addr + kColY + half * 32, v);
    tmem_ld_wait();
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] *= B_s[half * 32 + e];
    uint8_t* Yt = sm + kPrepR2 + kTile;
#pragma unroll
    for (int q = 0; q < 4; ++q) st_row8_bf16(Yt, kTile, i - 64, half * 4 + q, v + 8 * q);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  // ---- Z' = T_h[:, 64..127] Y' (M=128, N=64, K=64): A = T_h's second column tile (K-major)
  if (tid == 0) {
    tc_fence_after();
    const uint32_t sY = smem_u32(sm + kPrepR2 + kTile);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tmem + kColZ, desc_kmajor(sD + kTile, kk, kTile), desc_mnmajor(sY, kk, kTile),
               idesc_bf16(128, 64, false, true), kk > 0);
    mma_commit(bar);
  }
  ok = mbar_wait(bar, phase, a.wait_ns);
  phase ^= 1;
  if (__syncthreads_or(!ok)) goto done;
  tc_fence_after();
  // ---- V into R2 (N and Y' are consumed) while T diag(beta) is written over T_h:
  //   diagonal 32-blocks from the fp32 rows of the solver warps, the (1,0), (3,2) blocks from
  //   -Z1 (TMEM), the lower-left 64x64 block from -Z' (which already carries diag(beta))
  if (tid == 0) {
    pdl_wait();  // returns at once: thread 128 has seen the previous kernel complete
    const int rowV = (c * Hv + h) * kC;
    mbar_arrive_expect_tx(bar_v, 2 * kTile);
    tma_load_2d(sm + kPrepR2, &mapV, bar_v, 0, rowV);
    tma_load_2d(sm + kPrepR2 + kTile, &mapV, bar_v, 64, rowV);
  }
  if (solver) {
#pragma unroll
    for (int e = 0; e < 32; ++e) trow[e] *= B_s[quarter * 32 + e];
#pragma unroll
    for (int q = 0; q < 4; ++q) st_row8_bf16(Dt, kTile, i, quarter * 4 + q, trow + 8 * q);
  }
  if ((quarter == 1 && wg == 1) || (quarter == 3 && wg == 0)) {
    const int c0 = quarter == 1 ? 0 : 64;
    float v[32];
    tmem_ld32(lane_addr + kColZ1 + c0, v);
    tmem_ld_wait();
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] = -v[e] * B_s[c0 + e];
#pragma unroll
    for (int q = 0; q < 4; ++q) st_row8_bf16(Dt, kTile, i, (c0 >> 3) + q, v + 8 * q);
  }
  if (quarter >= 2) {
    // lower-left block: -Z'
    const int half = wg;
    float v[32];
    tmem_ld32(lane_addr + kColZ + half * 32, v);
    tmem_ld_wait();
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] = -v[e];
#pragma unroll
    for (int q = 0; q < 4; ++q) st_row8_bf16(Dt, kTile, i, half * 4 + q, v + 8 * q);
  }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  // ---- W = T diag(beta) K^ (issued at once), U~ = T diag(beta) V (once V has landed);
  // separate commits, so that W is read out while U~ is computed
  if (tid == 0) {
    tc_fence_after();
    const uint32_t sTB = smem_u32(sm + kPrepR1), sK = smem_u32(sm + kPrepKs),
                   sV = smem_u32(sm + kPrepR2);
    constexpr uint32_t id = idesc_bf16(128, 128, false, true);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_bf16(tmem + kColW, desc_kmajor(sTB, kk, kTile), desc_mnmajor(sK, kk, kTile), id, kk > 0);
    mma_commit(bar_w);
    pdl_trigger();
    ok = mbar_wait(bar_v, par, a.wait_ns);
    tc_fence_after();
    if (ok) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem + kColU, desc_kmajor(sTB, kk, kTile), desc_mnmajor(sV, kk, kTile), id, kk > 0);
      mma_commit(bar);
    } else {
      mbar_wait(bar_w, par, a.wait_ns);  // let the W products finish before the CTA gives up its TMEM
    }
  }
  if (__syncthreads_or(!ok)) goto done;
  // ---- W, then U~ -> bf16 swizzled tiles (W over K^, U~ over V) -> TMA stores
  {
    const int i = quarter * 32 + lane, half = wg;
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      ok = mbar_wait(m == 0 ? bar_w : bar, m == 0 ? par : phase, a.wait_ns);
      if (__syncthreads_or(!ok)) goto done;
      tc_fence_after();
      uint8_t* tile = sm + (m == 0 ? kPrepKs : kPrepR2);
      const uint32_t col = (m == 0 ? kColW : kColU) + half * 64;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float v[32];
        tmem_ld32(lane_addr + col + cc * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) st_row8_bf16(tile, kTile, i, half * 8 + cc * 4 + q, v + 8 * q);
      }
      fence_proxy_async_smem();
      __syncthreads();
      if (tid == 0) {
        const int row = (c * Hv + h) * kC;
        const CUtensorMap* map = m == 0 ? &mapW : &mapV;
        tma_store_2d(map, tile, 0, row);
        tma_store_2d(map, tile + kTile, 64, row);
        bulk_commit();
      }
    }
    if (tid == 0) bulk_wait_reads();  // the writes complete before the kernel is seen to end
  }
done:
  // every exit reaches this point on all threads (each early exit follows a block-wide vote)
  const bool all_ok = !__syncthreads_or(!ok);
  if (tid == 0 && !all_ok) {
    report_status(a.status, GDN_ERR_TIMEOUT);
    bulk_wait_reads();  // a store already issued still reads shared memory
  }
  return all_ok;
}

__global__ void __launch_bounds__(256, 2) gdn_prep_kernel(PrefillArgs a,
                                                          const __grid_constant__ CUtensorMap mapK,
                                                          const __grid_constant__ CUtensorMap mapV,
                                                          const __grid_constant__ CUtensorMap mapW) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const PrepCtl ctl(sm);
  const int c = a.c0 + blockIdx.x;
  const int h = blockIdx.y;
  if (c >= a.ws.seq_first[a.N]) {
    pdl_wait();
    return;
  }
  if (threadIdx.x == 128) ctl.init();
  if (threadIdx.x < 32) tmem_alloc(ctl.tslot, 256);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *ctl.tslot;
  prep_unit(a, mapK, mapV, mapW, c, h, sm, tmem, 0);
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) tmem_dealloc(tmem, 256);
}

// --------------------------------------------------------------------------------- chain
// One CTA per (sequence, value head, d_v block).  Thread t owns TMEM lane t % 128 (d_k row of S^T,
// token row of X) and, with 256 threads (d_v blocks of 64 or 128), the column half t / 128.  A launch covers the chunks of its sequence inside [c0, c1): the state
// enters from S0 (or zero) when the sequence starts there, else from carry_in, and leaves to SN
// when the sequence ends there, else to carry_out.  Shared memory: W tile(s), one K tile and one
// bf16 operand tile that holds S_b^T for X and then U^ for the state update (X has consumed S_b
// by the time U^ is written).  It stays near 100 KB so that a prep or out CTA fits beside it.
// With MID (64-token pages), a second operand tile holds the first half of the chunk's U^ for
// the state in the middle of the chunk, and a third TMEM region accumulates it.
template <int DV, bool MID = false, int WS = (DV > 64 ? 1 : 2)>
struct ChainCfg {
  static_assert(DV == 32 || DV == 64 || DV == 128, "d_v block");
  static_assert(WS == 1 || WS == 2, "W stages");
  static constexpr int kThreads = DV >= 64 ? 256 : 128;
  static constexpr int kCPT = DV * 128 / kThreads;              // value columns per thread
  static constexpr uint32_t kOpTiles = DV > 64 ? 2 : 1;         // 64-col tiles of S_b / U^
  static constexpr uint32_t kWStages = WS;                      // W tiles in flight
  static constexpr uint32_t kK = kWStages * 2 * kTile;          // K tile pair
  static constexpr uint32_t kOp = kK + 2 * kTile;               // S_b^T, then U^
  static constexpr uint32_t kOpMid = kOp + kOpTiles * kTile;    // first-half U^ (MID)
  static constexpr uint32_t kEnd = kOpMid + (MID ? kOpTiles * kTile : 0);
  static constexpr uint32_t kSmem = kEnd + 1024 + 256;
  static constexpr uint32_t kTmemCols = MID ? (DV == 32 ? 128 : DV == 64 ? 256 : 512)
                                            : 2 * DV;           // S^T | X (| S_mid^T)
};

// The chain of CTA `bid` = (sequence, value head, d_v block).
template <int DV, bool MID>
__device__ __forceinline__ void chain_body(const PrefillArgs& a, const CUtensorMap& mapW,
                                           const CUtensorMap& mapK, const CUtensorMap& mapS,
                                           const CUtensorMap& mapU, int bid, uint8_t* sm) {
  using Cfg = ChainCfg<DV, MID>;
  // From a d_v block of 64 on (without mid-chunk states), S_c and U leave for the workspace as
  // TMA stores of the bf16 operand tiles (whole 128-byte rows, instead of 16-byte pieces of 128
  // rows from every thread), and the decay of the state update goes onto K (the operand tile
  // then holds U itself): S^T += (diag(e^(G_L - G)) K)^T U.
  constexpr bool kTmaOut = DV >= 64 && !MID;
  // the chain's own threads (the first Cfg::kThreads of the block) synchronise on barrier 1
#define CSYNC() bar_sync_n(1, Cfg::kThreads)
#define CSYNC_OR(x) bar_or_n(1, Cfg::kThreads, (x))
  uint64_t* bar_w = reinterpret_cast<uint64_t*>(sm + Cfg::kEnd);  // [kWStages]
  uint64_t* bar_k = bar_w + 2;
  uint64_t* bar_mma = bar_k + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar_mma + 1);

  const int nsplit = a.nsplit;
  const int blk = bid % nsplit;
  const int h = (bid / nsplit) % a.Hv;
  const int n = bid / (nsplit * a.Hv);
  const int hk = h / (a.Hv / a.Hk);
  const int tid = threadIdx.x, warp = tid >> 5;
  pdl_wait();  // W, U~, G of this call, and the carry of the previous launch
  const int s_first = a.ws.seq_first[n], s_end = a.ws.seq_first[n + 1];
  if (!GDN_IN_BOUNDS(s_first >= 0 && s_end >= s_first && s_end <= a.T / kC + a.N, a.status))
    return;
  const int first = max(s_first, a.c0);
  const int nch = min(s_end, a.c1) - first;
  // an empty sequence belongs to the launch whose range holds its position in the chunk table
  const bool mine = nch > 0 || (s_first == s_end && a.c0 <= s_first && s_first < a.c1);
  if (!mine) return;  // uniform over the CTA, before any barrier or TMEM is set up
  const bool from_carry = s_first < a.c0;
  const bool to_carry = s_end > a.c1;
  const int v0 = blk * DV;

  if (tid == 0) {
    mbar_init(bar_w, 1);
    mbar_init(bar_w + 1, 1);
    mbar_init(bar_k, 1);
    mbar_init(bar_mma, 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tslot, Cfg::kTmemCols);
  CSYNC();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t colS = 0, colX = DV, colM = 2 * DV;
  constexpr int kCPT = Cfg::kCPT, kGroups = kCPT / 32;
  const uint32_t lane_addr = tmem_at(tmem, (warp & 3) * 32, 0);
  const int k_row = tid & 127;  // TMEM lane = d_k index for S^T, = token index for X
  const int cs = (tid >> 7) * kCPT;  // first column of this thread inside the d_v block
  const int srow = state_row(a.slot, n, a.num_slots);  // -1: slot out of range
  if (srow < 0 && tid == 0) report_status(a.status, GDN_ERR_INVALID_ARG);
  const size_t sbase = ((size_t)(srow < 0 ? 0 : srow) * a.Hv + h) * kD * kD;
  // state outputs after chunks (and, with MID, after the first 64 tokens of a chunk): entry of
  // the state after chunk j of this sequence, and of the one in its middle
  const int page_first = MID ? a.ws.page_first[n] : 0;
  auto end_entry = [&](int c, int L) {
    return MID ? page_first + 2 * (c - s_first) + (L > 64 ? 1 : 0) : c;
  };

  // ---- S^T initial value: lane k, column v  (state layout [v][k])
  {
    const float* src = from_carry ? a.carry_in + (size_t)h * kD * kD
                                  : (a.S0 && srow >= 0 ? a.S0 + sbase : nullptr);
#pragma unroll
    for (int gi = 0; gi < kGroups; ++gi) {
      float v[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int vv = v0 + cs + gi * 32 + e;
        v[e] = src ? src[(size_t)vv * kD + k_row] : 0.f;
      }
      tmem_st32(lane_addr + colS + cs + gi * 32, v);
    }
    tmem_st_wait();
  }
  // thread 0's count of loads issued and waited for, to drain them after a failed wait; a W
  // load left out on purpose (debug fault injection: the first chain CTA skips the load of chunk
  // a.fault_chunk, so that its bounded wait runs out) is never waited for in the drain
  int w_issued = 0, w_done = 0, k_issued = 0, k_done = 0, w_skipped = -1;
  auto issue_w = [&](int ci) {
    const int c = first + ci;
    if (bid == 0 && c == a.fault_chunk) {
      w_skipped = ci;
      return;
    }
    const int st = Cfg::kWStages == 1 ? 0 : (ci & 1);
    uint8_t* dst = sm + st * 2 * kTile;
    mbar_arrive_expect_tx(bar_w + st, 2 * kTile);
    const int row = (c * a.Hv + h) * kC;
    tma_load_2d(dst, &mapW, bar_w + st, 0, row);
    tma_load_2d(dst + kTile, &mapW, bar_w + st, 64, row);
  };
  auto issue_k = [&](int ci) {
    const int c = first + ci;
    uint8_t* dst = sm + Cfg::kK;
    mbar_arrive_expect_tx(bar_k, 2 * kTile);
    const int row = (c * a.Hk + hk) * kC;
    tma_load_2d(dst, &mapK, bar_k, 0, row);
    tma_load_2d(dst + kTile, &mapK, bar_k, 64, row);
  };
  bool mma_pending = false;
  if (tid == 0 && nch > 0) {
    issue_w(0);
    issue_k(0);
    w_issued = k_issued = 1;
  }
  uint32_t mma_phase = 0;
  bool ok = true;
  int failed = 0;
  uint8_t* OP = sm + Cfg::kOp;
  // per-token inputs of a chunk (row = k_row): U~ slice (packed bf16), G_i, G_last
  constexpr int kVec = kCPT / 8;
  uint4 ut_cur[kVec], ut_nxt[kVec];
  float Gi_cur = 0.f, Gl_cur = 0.f, Gi_nxt = 0.f, Gl_nxt = 0.f;
  float Gm_cur = 0.f, Gm_nxt = 0.f;  // G after token 63 (MID)
  int L_cur = 0, L_nxt = 0;          // tokens in the chunk (state outputs)
  auto load_chunk_rows = [&](int ci, uint4 (&ut)[kVec], float& Gi, float& Gl, float& Gm,
                             int& L) {
    const int c = first + ci;
    const float* Gc = a.ws.Gw + ((size_t)c * a.Hv + h) * kC;
    Gi = Gc[k_row];
    Gl = Gc[kC - 1];
    if (MID) Gm = Gc[63];
    if (a.chunk_states) L = a.ws.chunks[c].L;
    const uint4* src = reinterpret_cast<const uint4*>(
        a.ws.Uw + (((size_t)c * a.Hv + h) * kC + k_row) * kD + v0 + cs);
#pragma unroll
    for (int q = 0; q < kVec; q += 2) load32(src + q, ut[q], ut[q + 1]);  // 32-byte aligned
  };
  if (nch > 0) load_chunk_rows(0, ut_cur, Gi_cur, Gl_cur, Gm_cur, L_cur);
  for (int ci = 0; ci < nch; ++ci) {
    const int c = first + ci;
    const int wst = Cfg::kWStages == 1 ? 0 : (ci & 1);
    const uint32_t wphase = Cfg::kWStages == 1 ? (ci & 1) : ((ci >> 1) & 1);
    __syncwarp();  // warp 0 reconverges before its TMEM loads
    if (Cfg::kWStages == 2 && tid == 0 && ci + 1 < nch) {
      issue_w(ci + 1);
      ++w_issued;
    }
    // ---- S_b (bf16) -> operand tile (the only step X waits for).  With 32 columns per
    // thread the rest of the S bookkeeping runs while X is computed; with 64 it stays here
    // (register budget).
    constexpr bool kOverlap = kCPT <= 32;
    const float gam = __expf(Gl_cur);
    __nv_bfloat16* Srow = a.ws.Sw + (((size_t)c * a.Hv + h) * kD + k_row) * kD + v0 + cs;
    float sreg[kGroups][32];
    float smid[MID ? kGroups : 1][32];  // e^(G_63) S_c^T, the decayed part of the middle state
#pragma unroll
    for (int gi = 0; gi < kGroups; ++gi) {
      tmem_ld32(lane_addr + colS + cs + gi * 32, sreg[gi]);
      tmem_ld_wait();
      if constexpr (MID) {
        const float gm = __expf(Gm_cur);
#pragma unroll
        for (int e = 0; e < 32; ++e) smid[gi][e] = gm * sreg[gi][e];
      }

#pragma unroll
      for (int q = 0; q < 4; ++q)
        st_row8_bf16(OP, kTile, k_row, (cs + gi * 32 + 8 * q) >> 3, sreg[gi] + 8 * q);
      if constexpr (!kOverlap) {
        if constexpr (!kTmaOut) {
          store16(Srow + gi * 32, sreg[gi]);
          store16(Srow + gi * 32 + 16, sreg[gi] + 16);
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) sreg[gi][e] *= gam;
        tmem_st32(lane_addr + colS + cs + gi * 32, sreg[gi]);
      }
    }
    if constexpr (!kOverlap) tmem_st_wait();
    fence_proxy_async_smem();
    tc_fence_before();
    CSYNC();
    const int row_cv = (c * a.Hv + h) * kC;  // first workspace row of (chunk, value head)
    if (kTmaOut && tid == 0) {  // S_c (bf16) to the workspace from the operand tile
#pragma unroll
      for (uint32_t t = 0; t < Cfg::kOpTiles; ++t)
        tma_store_2d(&mapS, OP + t * kTile, v0 + 64 * t, row_cv);
      bulk_commit();
    }
    // ---- X = W S_b^T  (M = 128 tokens, N = DV, K = d_k)
    if (tid == 0) {
      ok = mbar_wait(bar_w + wst, wphase, a.wait_ns);
      tc_fence_after();
      if (ok) {
        ++w_done;
        const uint32_t sW = smem_u32(sm + wst * 2 * kTile), sS = smem_u32(OP);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + colX, desc_kmajor(sW, kk, kTile), desc_mnmajor(sS, kk, kTile),
                   idesc_bf16(128, DV, false, true), kk > 0);
        mma_commit(bar_mma);
        mma_pending = true;
      }
    }
    // while X runs: S_c to the workspace, S^T *= e^(G_last) in TMEM, next chunk's rows
    if constexpr (kOverlap) {
#pragma unroll
      for (int gi = 0; gi < kGroups; ++gi) {
        if constexpr (!kTmaOut) {
          store16(Srow + gi * 32, sreg[gi]);
          store16(Srow + gi * 32 + 16, sreg[gi] + 16);
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) sreg[gi][e] *= gam;
        tmem_st32(lane_addr + colS + cs + gi * 32, sreg[gi]);
      }
      tmem_st_wait();
    }
    if constexpr (kTmaOut) {
      // K^ = diag(e^(G_L - G)) K in place, once K has landed: this thread's token row, the
      // 64 d_k columns of its half (two threads per row)
      const bool k_ok = mbar_wait(bar_k, ci & 1, a.wait_ns);
      ok = ok && k_ok;
      if (k_ok) {
        const float dec = __expf(Gl_cur - Gi_cur);
        uint8_t* kt = sm + Cfg::kK + (tid >> 7) * kTile;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          uint4* p = reinterpret_cast<uint4*>(kt + sw128_off(k_row, q));
          uint4 u = *p;
          __nv_bfloat162* hv = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(hv[e]);
            hv[e] = __floats2bfloat162_rn(f.x * dec, f.y * dec);
          }
          *p = u;
        }
      }
    }
    if (ci + 1 < nch) load_chunk_rows(ci + 1, ut_nxt, Gi_nxt, Gl_nxt, Gm_nxt, L_nxt);
    if ((failed = CSYNC_OR(!ok))) break;
    ok = mbar_wait(bar_mma, mma_phase, a.wait_ns);
    if (kTmaOut && tid == 0) bulk_wait_reads();  // the S_c store has read the operand tile
    if ((failed = CSYNC_OR(!ok))) break;
    mma_phase ^= 1;
    mma_pending = false;
    tc_fence_after();
    // X has consumed W (single W buffer: the next chunk's W may come in now)
    if (Cfg::kWStages == 1 && tid == 0 && ci + 1 < nch) {
      issue_w(ci + 1);
      ++w_issued;
    }
    // ---- U = U~ - X; U^ = diag(e^(G_L - G)) U -> operand tile (U to the workspace afterwards)
    float ureg[kOverlap ? kCPT : 8];
    __nv_bfloat16* Urow = a.ws.Uw + (((size_t)c * a.Hv + h) * kC + k_row) * kD + v0 + cs;
    {
      const float dec = __expf(Gl_cur - Gi_cur);
      // MID: the first 64 tokens of U, decayed to token 63, for the state in the middle of the
      // chunk (rows 64..127 of that operand are never read)
      const float decm = MID && k_row < 64 ? __expf(Gm_cur - Gi_cur) : 0.f;
#pragma unroll
      for (int gi = 0; gi < kGroups; ++gi) {
        float v[32];
        tmem_ld32(lane_addr + colX + cs + gi * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int vq = (gi * 32 + 8 * q) >> 3;  // 8-column group inside this thread's slice
          const __nv_bfloat162* uh = reinterpret_cast<const __nv_bfloat162*>(&ut_cur[vq]);
          float* u8 = kOverlap ? ureg + vq * 8 : ureg;
          float h8[8];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const float2 f = __bfloat1622float2(uh[e2]);
            u8[2 * e2] = f.x - v[8 * q + 2 * e2];
            u8[2 * e2 + 1] = f.y - v[8 * q + 2 * e2 + 1];
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) h8[e] = kTmaOut ? u8[e] : u8[e] * dec;
          st_row8_bf16(OP, kTile, k_row, (cs >> 3) + vq, h8);
          if (MID && k_row < 64) {
#pragma unroll
            for (int e = 0; e < 8; ++e) h8[e] = u8[e] * decm;
            st_row8_bf16(sm + Cfg::kOpMid, kTile, k_row, (cs >> 3) + vq, h8);
          }
          if constexpr (!kOverlap && !kTmaOut) {
            float w8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w8[e] = u8[e];
            store8(Urow + vq * 8, w8);
          }
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    CSYNC();
    if (kTmaOut && tid == 0) {  // U (bf16) to the workspace from the operand tile
#pragma unroll
      for (uint32_t t = 0; t < Cfg::kOpTiles; ++t)
        tma_store_2d(&mapU, OP + t * kTile, v0 + 64 * t, row_cv);
      bulk_commit();
    }
    // ---- S^T += K^T U^  (M = d_k, N = DV, K = tokens); with kTmaOut: K^^T U
    if (tid == 0) {
      ok = mbar_wait(bar_k, ci & 1, a.wait_ns);
      tc_fence_after();
      if (ok) {
        ++k_done;
        const uint32_t sK = smem_u32(sm + Cfg::kK), sU = smem_u32(OP);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + colS, desc_mnmajor(sK, kk, kTile), desc_mnmajor(sU, kk, kTile),
                   idesc_bf16(128, DV, true, true), 1);
        if (MID && L_cur > 64) {
          // S_mid^T = e^(G_63) S_c^T + K[0:64]^T U^mid: the product over tokens 0..63 here,
          // the decayed state added at the readout
          const uint32_t sUm = smem_u32(sm + Cfg::kOpMid);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + colM, desc_mnmajor(sK, kk, kTile), desc_mnmajor(sUm, kk, kTile),
                     idesc_bf16(128, DV, true, true), kk > 0);
        }
        mma_commit(bar_mma);
        mma_pending = true;
      }
    }
    // while the state update runs: U to the workspace
    if constexpr (kOverlap && !kTmaOut) {
#pragma unroll
      for (int q = 0; q < kCPT / 16; ++q) store16(Urow + q * 16, ureg + q * 16);
    }
    if ((failed = CSYNC_OR(!ok))) break;
    ok = mbar_wait(bar_mma, mma_phase, a.wait_ns);
    if (kTmaOut && tid == 0) bulk_wait_reads();  // the U store has read the operand tile
    if ((failed = CSYNC_OR(!ok))) break;
    mma_phase ^= 1;
    mma_pending = false;
    tc_fence_after();
    if (a.chunk_states) {
      // the state after chunk c (fp32, layout [v][k]), for prefix and branch caching
      float* cst = a.chunk_states +
                   (((size_t)end_entry(c, L_cur) * a.Hv + h) * kD + v0 + cs) * kD + k_row;
#pragma unroll
      for (int gi = 0; gi < kGroups; ++gi) {
        float v[32];
        tmem_ld32(lane_addr + colS + cs + gi * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) cst[(gi * 32 + e) * kD] = v[e];
      }
      if (MID && L_cur > 64) {
        // and the state after the chunk's first 64 tokens (the entry before the chunk end's)
        float* mst = cst - (size_t)a.Hv * kD * kD;
#pragma unroll
        for (int gi = 0; gi < kGroups; ++gi) {
          float v[32];
          tmem_ld32(lane_addr + colM + cs + gi * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) mst[(gi * 32 + e) * kD] = v[e] + smid[MID ? gi : 0][e];
        }
      }
    }
    // the update has consumed K and the operand tile
    if (tid == 0 && ci + 1 < nch) {
      issue_k(ci + 1);
      ++k_issued;
    }
#pragma unroll
    for (int q = 0; q < kVec; ++q) ut_cur[q] = ut_nxt[q];
    Gi_cur = Gi_nxt;
    Gl_cur = Gl_nxt;
    Gm_cur = Gm_nxt;
    L_cur = L_nxt;
  }
  float* dst = to_carry ? a.carry_out + (size_t)h * kD * kD
                        : (a.SN && srow >= 0 ? a.SN + sbase : nullptr);
  if (!failed && dst) {
#pragma unroll
    for (int gi = 0; gi < kGroups; ++gi) {
      float v[32];
      tmem_ld32(lane_addr + colS + cs + gi * 32, v);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) dst[(size_t)(v0 + cs + gi * 32 + e) * kD + k_row] = v[e];
    }
  }
  if (failed && tid == 0) {
    report_status(a.status, GDN_ERR_TIMEOUT);
    // give loads and products still in flight a bounded time to land before the CTA's shared
    // memory and TMEM are released
    for (int j = w_done; j < w_issued; ++j)
      if (j != w_skipped)
        mbar_wait(bar_w + (Cfg::kWStages == 1 ? 0 : (j & 1)),
                Cfg::kWStages == 1 ? (j & 1) : ((j >> 1) & 1), a.wait_ns);
    for (int j = k_done; j < k_issued; ++j) mbar_wait(bar_k, j & 1, a.wait_ns);
    if (mma_pending) mbar_wait(bar_mma, mma_phase, a.wait_ns);
  }
  if (kTmaOut && tid == 0) bulk_wait_all();  // the workspace stores are complete
  tc_fence_before();
  CSYNC();
  if (warp == 0) tmem_dealloc(tmem, Cfg::kTmemCols);
#undef CSYNC
#undef CSYNC_OR
}

template <int DV, bool MID>
__global__ void __launch_bounds__(ChainCfg<DV>::kThreads, 1) gdn_chain_kernel(PrefillArgs a,
                                                           const __grid_constant__ CUtensorMap mapW,
                                                           const __grid_constant__ CUtensorMap mapK,
                                                           const __grid_constant__ CUtensorMap mapS,
                                                           const __grid_constant__ CUtensorMap mapU) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  pdl_trigger();
  chain_body<DV, MID>(a, mapW, mapK, mapS, mapU, blockIdx.x, sm);
}

// --------------------------------------------------------------------------- out, persistent
// The output step as a persistent, warp-specialised kernel: each CTA takes a contiguous range of
// (chunk, value head) units and pipelines them over two shared-memory stages, so that the tiles
// of the next unit load while the current one computes, and the epilogue of one unit overlaps
// the products of the next.
//   warps 0-3  (group A) per unit: P = mask(e^(G_i - G_j)) Q K^T and Q^ = diag(e^G) Q, written
//              to TMEM as bf16 A operands (thread = token row, all 128 columns)
//   warps 4-7  (group B) per unit: gated RMSNorm epilogue of O from one of two TMEM buffers,
//              z and the chunk entry loaded into registers one unit ahead, bf16 rows out
//   warp 8     TMA loads of Q, K and U into the unit's stage, as soon as the stage is free
//   warp 9     tcgen05.mma: Q K^T; once it has completed, the TMA load of S^T into K's place;
//              then O = Q^ S^T + P U into TMEM buffer (unit % 2)
// Stage s (96 KB): Q | K, then S^T | U.  It is free again when the unit's O products complete
// (group A has read Q before it released P and Q^).  Every hand-over is an mbarrier (TMA
// transactions, tcgen05.commit, or 128 thread arrivals), and every wait is bounded; a wait that
// runs out sets the abort flag, which the other roles' waits also observe.
constexpr int kOutPThreads = 320;
constexpr uint32_t kOpStage = 98304;                        // Q | K-then-S^T | U
constexpr uint32_t kOpQ = 0, kOpKS = 32768, kOpU = 65536;   // offsets inside a stage
constexpr uint32_t kOpEnd = 2 * kOpStage;                   // 196608
constexpr uint32_t kOutPSmem = kOpEnd + 1024 + 2048;
constexpr uint32_t kColPQ0 = 0, kColO0 = 256;  // P|Q^ buffer b at 128 b, O buffer b at 256 + 128 b

struct OutPCtl {
  uint64_t* qk_full;      // [2]
  uint64_t* u_full;       // [2]
  uint64_t* s_full;       // [2]
  uint64_t* stage_empty;  // [2]
  uint64_t* gram_done;    // [2]
  uint64_t* pq_ready;     // [2]
  uint64_t* o_full;       // [2]
  uint64_t* o_empty;      // [2]
  uint64_t* drain;        // products in flight after an abort
  uint32_t* tslot;
  int* abort;
  float* G_s;             // [128] gates of the unit group A works on
  float* F_s;             // [128] column factors
  float* w_s;             // [128] norm weight
  __device__ explicit OutPCtl(uint8_t* sm) {
    uint64_t* b = reinterpret_cast<uint64_t*>(sm + kOpEnd);
    qk_full = b;
    u_full = b + 2;
    s_full = b + 4;
    stage_empty = b + 6;
    gram_done = b + 8;
    pq_ready = b + 10;
    o_full = b + 12;
    o_empty = b + 14;
    drain = b + 16;
    tslot = reinterpret_cast<uint32_t*>(b + 17);
    abort = reinterpret_cast<int*>(tslot + 1);
    G_s = reinterpret_cast<float*>(sm + kOpEnd + 256);
    F_s = G_s + kC;
    w_s = F_s + kC;
  }
};

// Bounded wait that also gives up once another role has set the abort flag.
__device__ __forceinline__ bool wait_role(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_timer_ns() - t0 > limit_ns) return false;
    __nanosleep(32);
  }
}

__global__ void __launch_bounds__(kOutPThreads, 1) gdn_out_persistent_kernel(
    PrefillArgs a, const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
    const __grid_constant__ CUtensorMap mapS, const __grid_constant__ CUtensorMap mapU) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const OutPCtl ctl(sm);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Hv = a.Hv;
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(ctl.qk_full + b, 1);
      mbar_init(ctl.u_full + b, 1);
      mbar_init(ctl.s_full + b, 1);
      mbar_init(ctl.stage_empty + b, 1);
      mbar_init(ctl.o_full + b, 1);
      mbar_init(ctl.o_empty + b, 128);
      mbar_init(ctl.gram_done + b, 1);
      mbar_init(ctl.pq_ready + b, 128);
    }
    mbar_init(ctl.drain, 1);
    *ctl.abort = 0;
    fence_barrier_init();
  }
  if (warp == 8) tmem_alloc(ctl.tslot, 512);
  if (tid >= 128 && tid < 256)
    ctl.w_s[tid - 128] = a.norm_w ? __bfloat162float(a.norm_w[tid - 128]) : 1.f;
  pdl_wait();  // the chain's S^T and U (and, before it, every earlier kernel of the call)
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *ctl.tslot;
  volatile int* abort = ctl.abort;
  // this CTA's units: a contiguous range of the (chunk, value head) units of the launch, so
  // that the two value heads of a key head (same Q and K tiles) follow each other
  const int nchunks = min(a.c1, a.ws.seq_first[a.N]) - a.c0;
  const int nunits = max(nchunks, 0) * Hv;
  const int per = (nunits + gridDim.x - 1) / gridDim.x;
  const int u0 = blockIdx.x * per, u1 = min(nunits, u0 + per);
  const int count = max(u1 - u0, 0);
  bool ok = true;
  // debug stamps (first CTA, first 32 units): [role * 64 + 2 i (+1)] = start / end of unit i
  uint64_t* stamps = (a.stamps && blockIdx.x == 0) ? a.stamps : nullptr;
  auto stamp = [&](int role, int i, int end) {
    if (stamps && i < 32) stamps[role * 64 + 2 * i + end] = global_timer_ns();
  };
  int last_qk[2] = {-1, -1};  // producer: last unit loaded into each stage
  int last_s = -1;            // MMA role: last unit whose S^T load it issued

  if (warp == 8) {
    // ------------------------------------------------------------------- TMA producer
    if (lane == 0) {
      for (int i = 0; i < count && ok; ++i) {
        const int u = u0 + i, c = a.c0 + u / Hv, h = u % Hv, hk = h / (Hv / a.Hk);
        const int st = i & 1;
        if (i >= 2) ok = wait_role(ctl.stage_empty + st, ((i >> 1) - 1) & 1, abort, a.wait_ns);
        if (!ok) break;
        uint8_t* stage = sm + st * kOpStage;
        stamp(0, i, 0);
        const int rowQK = (c * a.Hk + hk) * kC, rowV = (c * Hv + h) * kC;
        mbar_arrive_expect_tx(ctl.qk_full + st, 4 * kTile);
        tma_load_2d(stage + kOpQ, &mapQ, ctl.qk_full + st, 0, rowQK);
        tma_load_2d(stage + kOpQ + kTile, &mapQ, ctl.qk_full + st, 64, rowQK);
        tma_load_2d(stage + kOpKS, &mapK, ctl.qk_full + st, 0, rowQK);
        tma_load_2d(stage + kOpKS + kTile, &mapK, ctl.qk_full + st, 64, rowQK);
        mbar_arrive_expect_tx(ctl.u_full + st, 2 * kTile);
        tma_load_2d(stage + kOpU, &mapU, ctl.u_full + st, 0, rowV);
        tma_load_2d(stage + kOpU + kTile, &mapU, ctl.u_full + st, 64, rowV);
        // S^T is loaded into K's place once Q K^T has run; bring it into L2 meanwhile
        tma_prefetch_2d(&mapS, 0, rowV);
        tma_prefetch_2d(&mapS, 64, rowV);
        last_qk[st] = i;
      }
      if (!ok) *abort = 1;
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------------- MMA issue
    // Q K^T of unit i + 1 goes out before O of unit i (two P|Q^ buffers), so that group A works
    // on the next unit while the current one's products run
    if (lane == 0) {
      auto gram = [&](int i) -> bool {
        const int st = i & 1;
        if (!wait_role(ctl.qk_full + st, (i >> 1) & 1, abort, a.wait_ns)) return false;
        stamp(1, i, 0);
        tc_fence_after();
        const uint32_t sQ = smem_u32(sm + st * kOpStage + kOpQ);
        const uint32_t sK = smem_u32(sm + st * kOpStage + kOpKS);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + kColPQ0 + st * 128, desc_kmajor(sQ, kk, kTile),
                   desc_kmajor(sK, kk, kTile), idesc_bf16(128, 128, false, false), kk > 0);
        mma_commit(ctl.gram_done + st);
        return true;
      };
      if (count > 0) ok = gram(0);
      for (int i = 0; i < count && ok; ++i) {
        const int u = u0 + i, c = a.c0 + u / Hv, h = u % Hv;
        const int st = i & 1;
        // K of unit i is consumed once its product completes: S^T into its place at once
        ok = wait_role(ctl.gram_done + st, (i >> 1) & 1, abort, a.wait_ns);
        if (!ok) break;
        const int rowV = (c * Hv + h) * kC;
        uint8_t* ks = sm + st * kOpStage + kOpKS;
        mbar_arrive_expect_tx(ctl.s_full + st, 2 * kTile);
        tma_load_2d(ks, &mapS, ctl.s_full + st, 0, rowV);
        tma_load_2d(ks + kTile, &mapS, ctl.s_full + st, 64, rowV);
        last_s = i;
        // the next unit's product, so that group A can start on it
        if (i + 1 < count && !(ok = gram(i + 1))) break;
        ok = wait_role(ctl.pq_ready + st, (i >> 1) & 1, abort, a.wait_ns) &&
             wait_role(ctl.s_full + st, (i >> 1) & 1, abort, a.wait_ns) &&
             wait_role(ctl.u_full + st, (i >> 1) & 1, abort, a.wait_ns) &&
             (i < 2 || wait_role(ctl.o_empty + st, ((i >> 1) - 1) & 1, abort, a.wait_ns));
        if (!ok) break;
        stamp(1, i, 1);
        tc_fence_after();
        const uint32_t sKS = smem_u32(ks), sU = smem_u32(sm + st * kOpStage + kOpU);
        const uint32_t colO = kColO0 + st * 128, colPQ = kColPQ0 + st * 128;
        constexpr uint32_t id = idesc_bf16(128, 128, false, true);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + colO, tmem + colPQ + 64 + kk * 8, desc_mnmajor(sKS, kk, kTile), id,
                      kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + colO, tmem + colPQ + kk * 8, desc_mnmajor(sU, kk, kTile), id, 1);
        mma_commit(ctl.o_full + st);
        mma_commit(ctl.stage_empty + st);
      }
      if (!ok) *abort = 1;
    }
  } else if (warp < 4) {
    // ------------------------------------------------ group A: P and Q^ into TMEM, row tid
    const int i_row = tid;
    const uint32_t lane_addr = tmem_at(tmem, warp * 32, 0);
    float g_next = 0.f;
    if (count > 0) {
      const int c = a.c0 + u0 / Hv, h = u0 % Hv;
      g_next = a.ws.Gw[((size_t)c * Hv + h) * kC + i_row];
    }
    for (int i = 0; i < count; ++i) {
      const int st = i & 1;
      // gates of this unit into shared memory (loaded one unit ahead), column factors
      bar_sync_n(1, 128);  // the previous unit's readers of G_s / F_s are done
      ctl.G_s[i_row] = g_next;
      if (i + 1 < count) {
        const int u = u0 + i + 1, c = a.c0 + u / Hv, h = u % Hv;
        g_next = a.ws.Gw[((size_t)c * Hv + h) * kC + i_row];
      }
      bar_sync_n(1, 128);
      ctl.F_s[i_row] = __expf(ctl.G_s[i_row | 31] - ctl.G_s[i_row]);
      // one decision for the whole group (its named barriers need all 128 threads)
      const bool got = wait_role(ctl.gram_done + st, (i >> 1) & 1, abort, a.wait_ns);
      if (bar_or_n(1, 128, !got)) {
        ok = false;
        break;
      }
      if (i_row == 0) stamp(2, i, 0);
      tc_fence_after();
      const float Gi = ctl.G_s[i_row];
      const int rq = i_row >> 5;  // row block of this thread (warp-uniform)
      const uint32_t colPQ = kColPQ0 + st * 128;
      // P block jb (bf16 pairs) goes to columns 16 jb.., over fp32 gram columns this thread has
      // already read (the gram block jb starts at column 32 jb); loops kept rolled so that the
      // code stays small (four roles share each SM sub-partition's instruction cache)
#pragma unroll 1
      for (int jb = 0; jb < 4; ++jb) {
        const int j0 = jb * 32;
        uint32_t p16[16];
        if (jb > rq) {
#pragma unroll
          for (int e = 0; e < 16; ++e) p16[e] = 0u;
        } else {
          float v[32];
          tmem_ld32(lane_addr + colPQ + j0, v);
          tmem_ld_wait();
          if (jb < rq) {
            // every j < every i: exp(G_i - G_j) = exp(G_i - G_m) exp(G_m - G_j), m = j0 + 31
            const float rf = __expf(Gi - ctl.G_s[j0 + 31]);
            const float4* F4 = reinterpret_cast<const float4*>(ctl.F_s + j0);
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
              const float4 f = F4[e4];
              p16[2 * e4] = pack_bf16x2(rf * f.x * v[4 * e4], rf * f.y * v[4 * e4 + 1]);
              p16[2 * e4 + 1] = pack_bf16x2(rf * f.z * v[4 * e4 + 2], rf * f.w * v[4 * e4 + 3]);
            }
          } else {
            const float4* G4 = reinterpret_cast<const float4*>(ctl.G_s + j0);
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
              const float4 gj = G4[e4];
              const int j = j0 + 4 * e4;
              p16[2 * e4] = pack_bf16x2(lower_decay(j <= i_row, Gi, gj.x, v[4 * e4]),
                                        lower_decay(j + 1 <= i_row, Gi, gj.y, v[4 * e4 + 1]));
              p16[2 * e4 + 1] = pack_bf16x2(lower_decay(j + 2 <= i_row, Gi, gj.z, v[4 * e4 + 2]),
                                            lower_decay(j + 3 <= i_row, Gi, gj.w, v[4 * e4 + 3]));
            }
          }
        }
        tmem_st16(lane_addr + colPQ + jb * 16, p16);
      }
      if (i_row == 96) stamp(4, i, 0);
      // Q^ = e^(G_i) Q row into columns 64.. (the gram columns there are read by now)
      const float eg = __expf(Gi);
      const uint8_t* Qs = sm + st * kOpStage + kOpQ;
#pragma unroll 1
      for (int qb = 0; qb < 4; ++qb) {
        uint32_t q16[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c16 = qb * 4 + q;  // 16-byte chunk of the row (8 elements)
          const uint4 u4 =
              *reinterpret_cast<const uint4*>(Qs + (c16 >> 3) * kTile + sw128_off(i_row, c16 & 7));
          const __nv_bfloat162* hq = reinterpret_cast<const __nv_bfloat162*>(&u4);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(hq[e]);
            q16[q * 4 + e] = pack_bf16x2(f.x * eg, f.y * eg);
          }
        }
        tmem_st16(lane_addr + colPQ + 64 + qb * 16, q16);
      }
      if (i_row == 96) stamp(4, i, 1);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(ctl.pq_ready + st);  // Q of the stage is read, P and Q^ are in TMEM
      if (i_row == 0) stamp(2, i, 1);
    }
    if (!ok) *abort = 1;
  } else {
    // ----------------------------------------------- group B: gated RMSNorm epilogue, row
    const int i_row = tid - 128;
    const uint32_t lane_addr = tmem_at(tmem, (warp & 3) * 32, 0);
    const bool out32 = (reinterpret_cast<uintptr_t>(a.out) & 31u) == 0;
    const bool z32 = (reinterpret_cast<uintptr_t>(a.z) & 31u) == 0;
    uint4 zreg[16];
    // chunk entries two units ahead, z rows one unit ahead (two dependent loads otherwise)
    auto entry = [&](int i) {
      ChunkInfo e{};
      if (i < count) e = a.ws.chunks[a.c0 + (u0 + i) / Hv];
      return e;
    };
    ChunkInfo ci_next = entry(0), ci_next2 = entry(1);
    auto prefetch = [&](int i) {  // z row of unit i (its chunk entry is ci_next)
      const int h = (u0 + i) % Hv;
      if (a.z && i_row < ci_next.L) {
        const uint4* zp =
            reinterpret_cast<const uint4*>(a.z + ((size_t)(ci_next.t0 + i_row) * Hv + h) * kD);
        if (z32) {  // whole sectors when z allows it
#pragma unroll
          for (int q = 0; q < 16; q += 2) load32_nc(zp + q, zreg[q], zreg[q + 1]);
        } else {
#pragma unroll
          for (int q = 0; q < 16; ++q) zreg[q] = __ldg(zp + q);
        }
      }
    };
    if (count > 0) prefetch(0);
    for (int i = 0; i < count; ++i) {
      const int u = u0 + i, h = u % Hv;
      const ChunkInfo ci = ci_next;
      ci_next = ci_next2;
      ci_next2 = entry(i + 2);
      const int st = i & 1;
      ok = wait_role(ctl.o_full + st, (i >> 1) & 1, abort, a.wait_ns);
      if (!ok) break;
      if (i_row == 0) stamp(3, i, 0);
      tc_fence_after();
      const uint32_t colO = kColO0 + st * 128;
      float inv = 1.f;
      // loops kept rolled (the code stays small: four roles share each SM sub-partition's
      // instruction cache); the z words of column block q are picked by selects
      if (a.z) {
        float ss = 0.f;
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          float v[32];
          if (q == 0 && i_row == 0) stamp(5, i, 0);
          tmem_ld32(lane_addr + colO + q * 32, v);
          tmem_ld_wait();
          if (q == 0 && i_row == 0) stamp(5, i, 1);
#pragma unroll
          for (int e = 0; e < 32; ++e) ss = fmaf(v[e], v[e], ss);
        }
        inv = rsqrtf(ss / kD + a.norm_eps);
      }
      __nv_bfloat16* dst = a.out + ((size_t)(ci.t0 + i_row) * Hv + h) * kD;
      const bool valid = i_row < ci.L;
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        float v[32];
        tmem_ld32(lane_addr + colO + q * 32, v);
        tmem_ld_wait();
        if (a.z) {
          uint4 zq[4];
#pragma unroll
          for (int r = 0; r < 4; ++r)
            zq[r] = q == 0 ? zreg[r] : q == 1 ? zreg[4 + r] : q == 2 ? zreg[8 + r] : zreg[12 + r];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const __nv_bfloat162* zh = reinterpret_cast<const __nv_bfloat162*>(&zq[r]);
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
              const float2 zf = __bfloat1622float2(zh[e2]);
              const int e = r * 8 + e2 * 2;
              v[e] = v[e] * inv * ctl.w_s[q * 32 + e] * silu_fast(zf.x);
              v[e + 1] = v[e + 1] * inv * ctl.w_s[q * 32 + e + 1] * silu_fast(zf.y);
            }
          }
        }
        if (valid) {
          if (out32) {  // 32-byte stores (whole sectors) when the output allows them
            store16(dst + q * 32, v);
            store16(dst + q * 32 + 16, v + 16);
          } else {
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              float o8[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) o8[e] = v[r * 8 + e];
              store8(dst + q * 32 + r * 8, o8);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(ctl.o_empty + st);
      if (i_row == 0) stamp(3, i, 1);
      if (i + 1 < count) prefetch(i + 1);
    }
    if (!ok) *abort = 1;
  }
  // every role has left its loop; without an abort, group B has seen the last products
  // complete and every load was consumed
  __syncthreads();
  if (*abort) {
    if (tid == 0) report_status(a.status, GDN_ERR_TIMEOUT);
    if (tid == 32 * 9) {  // every product and S^T load issued so far lands first
      mma_commit(ctl.drain);
      mbar_wait(ctl.drain, 0, a.wait_ns);
      if (last_s >= 0) mbar_wait(ctl.s_full + (last_s & 1), (last_s >> 1) & 1, a.wait_ns);
    }
    if (tid == 32 * 8) {  // and every load of the producer
      for (int b = 0; b < 2; ++b)
        if (last_qk[b] >= 0) {
          mbar_wait(ctl.qk_full + b, (last_qk[b] >> 1) & 1, a.wait_ns);
          mbar_wait(ctl.u_full + b, (last_qk[b] >> 1) & 1, a.wait_ns);
        }
    }
    __syncthreads();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) tmem_dealloc(tmem, 512);
}

}  // namespace gdn

// =================================================================================== host
namespace gdn_host {

using gdn::kC;
using gdn::kD;

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Launch with programmatic stream serialisation: the kernel may start while the previous kernel
// in the stream drains, and waits for it with griddepcontrol.wait before touching its outputs.
template <typename... KArgs, typename... Args>
static cudaError_t launch_k(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (pdl && !trace_attached()) ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Software pipeline over the chunk table.  The chunk range [0, NCmax) (NCmax = T/128 + N, an
// upper bound on the chunks the table can hold) is cut into `nseg` segments of `seg` chunks.
// Segment k's q/k/v + prep run while the chain works on segment k-1 and out on segment k-2, so
// the sequential chain overlaps the parallel kernels instead of following them.  The parallel
// kernels already fill every SM (two CTAs each, bound by shared memory), so the overlap only
// pays where the chain is long: by default the table is cut only from 512 chunks on, into
// segments of 64 (of 128 from 1024 chunks on: at 262,144 tokens, 9.84 ms per call against 9.92
// with 64).  The debug option segment_chunks sets the segment length (a value at or above the
// chunk count gives a single launch of each kernel).
struct SegPlan {
  int nseg, seg;
};
constexpr int kPipelineChunks = 512;  // chunk count from which a call is pipelined

static SegPlan seg_plan(int N, int T) {
  const int NC = T / kC + N;
  if (T == 0 || NC <= 1) return {1, NC > 0 ? NC : 1};
  int target = debug_opts().segment_chunks;
  if (target <= 0) target = NC >= 2 * kPipelineChunks ? 128 : (NC >= kPipelineChunks ? 64 : NC);
  int nseg = (NC + target - 1) / target;
  if (nseg < 1) nseg = 1;
  const int seg = (NC + nseg - 1) / nseg;
  nseg = (NC + seg - 1) / seg;
  return {nseg, seg};
}

struct WsLayout {
  size_t chunks, seq_first, page_first, Qw, Kw, Ww, Uw, Sw, Gw, carry, total;
};

static WsLayout ws_layout(int N, int T, int Hk, int Hv) {
  const size_t NC = (size_t)T / kC + (size_t)N + 1;
  const size_t tile = (size_t)kC * kD * 2;
  const SegPlan p = seg_plan(N, T);
  WsLayout l{};
  size_t o = 0;
  l.chunks = o; o = align_up(o + NC * sizeof(gdn::ChunkInfo), 1024);
  l.seq_first = o; o = align_up(o + (size_t)(N + 1) * 4, 1024);
  l.page_first = o; o = align_up(o + (size_t)(N + 1) * 4, 1024);
  l.Qw = o; o = align_up(o + NC * Hk * tile, 1024);
  l.Kw = o; o = align_up(o + NC * Hk * tile, 1024);
  l.Ww = o; o = align_up(o + NC * Hv * tile, 1024);
  l.Uw = o; o = align_up(o + NC * Hv * tile, 1024);
  l.Sw = o; o = align_up(o + NC * Hv * tile, 1024);
  l.Gw = o; o = align_up(o + NC * Hv * kC * 4, 1024);
  // one fp32 [Hv][d][d] state per segment boundary (at most one sequence crosses each)
  l.carry = o; o = align_up(o + (size_t)(p.nseg - 1) * Hv * kD * kD * 4, 1024);
  l.total = o;
  return l;
}

size_t prefill_tc_workspace(int N, int T, int Hk, int Hv) { return ws_layout(N, T, Hk, Hv).total; }

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D map over a [rows][128] bf16 matrix, box [128 rows][64 cols], 128-byte swizzle.
static bool make_map(CUtensorMap* m, const void* base, size_t rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kC};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over the conv input x [T][Cc] bf16: box [128 + 3 rows][64 cols], 128-byte swizzle.
static bool make_map_x(CUtensorMap* m, const void* base, int T, int Cc) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)Cc, (cuuint64_t)T};
  cuuint64_t strides[1] = {(cuuint64_t)Cc * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)gdn::kXRows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DV, bool MID>
static cudaError_t launch_chain(const gdn::PrefillArgs& a, const CUtensorMap& mW,
                                const CUtensorMap& mK, const CUtensorMap& mS,
                                const CUtensorMap& mU, cudaStream_t s, bool pdl) {
  using Cfg = gdn::ChainCfg<DV, MID>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(gdn::gdn_chain_kernel<DV, MID>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  trace_begin("gdn_chain", s);
  cudaError_t e = launch_k(pdl, gdn::gdn_chain_kernel<DV, MID>, dim3(a.N * a.Hv * a.nsplit),
                           dim3(Cfg::kThreads), Cfg::kSmem, s, a, mW, mK, mS, mU);
  trace_end(s);
  return e;
}

// d_v blocks per chain state.  More blocks shorten each chunk step of the chain (fewer columns
// per CTA) but hold more SMs: a chain CTA leaves no room for an output CTA on its SM.  A call
// that runs as one launch of each kernel wants the shortest chain (up to 4 blocks, while the
// chains fill fewer than the SMs); a pipelined call (from 512 chunks on) overlaps the chain with
// the parallel kernels of later segments and takes at most 2 blocks (measured at 262,144 tokens,
// 16/32 heads: 9.84 ms per call with 2 blocks, 10.06 with 4, 12.99 with 1).
int choose_nsplit(int N, int T, int Hv) {
  const int forced = debug_opts().chain_split;
  if (forced == 1 || forced == 2 || forced == 4) return forced;
  const int units = N * Hv;
  if (units >= 148) return 1;
  if (units * 2 >= 148) return 2;
  return T / kC + N >= kPipelineChunks ? 2 : 4;
}

// Helper streams of the pipeline, per device and host thread (a capture on one thread never
// sees another thread's launches).  Consecutive segments alternate between two front streams
// (q/k/v + prep) and two out streams, so that the next segment's CTAs fill the SMs while the
// last wave of the previous one drains.  The chain stream gets the highest priority: it is the
// critical path, and its CTAs should take a free SM slot before the next prep or out CTA.
struct PipeStreams {
  static constexpr int kWays = 2;
  bool ready = false;
  cudaStream_t P[kWays] = {}, O[kWays] = {}, C = nullptr;
  cudaEvent_t fork = nullptr, evP = nullptr, evC = nullptr;
  cudaEvent_t join[2 * kWays + 1] = {};
};

static cudaError_t pipe_streams(PipeStreams** out) {
  constexpr int kMaxDev = 64;
  static thread_local PipeStreams t_pipe[kMaxDev];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  PipeStreams& ps = t_pipe[dev];
  if (!ps.ready) {
    int least = 0, greatest = 0;
    if ((e = cudaDeviceGetStreamPriorityRange(&least, &greatest)) != cudaSuccess) return e;
    for (int i = 0; i < PipeStreams::kWays; ++i)
      if ((e = cudaStreamCreateWithPriority(&ps.P[i], cudaStreamNonBlocking, least)) !=
              cudaSuccess ||
          (e = cudaStreamCreateWithPriority(&ps.O[i], cudaStreamNonBlocking, least)) !=
              cudaSuccess)
        return e;
    if ((e = cudaStreamCreateWithPriority(&ps.C, cudaStreamNonBlocking, greatest)) != cudaSuccess)
      return e;
    if ((e = cudaEventCreateWithFlags(&ps.fork, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&ps.evP, cudaEventDisableTiming)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&ps.evC, cudaEventDisableTiming)) != cudaSuccess)
      return e;
    for (cudaEvent_t& ev : ps.join)
      if ((e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming)) != cudaSuccess) return e;
    ps.ready = true;
  }
  *out = &ps;
  return cudaSuccess;
}

cudaError_t launch_prefill_tc(gdn::PrefillArgs a, void* workspace, cudaStream_t s) {
  const WsLayout l = ws_layout(a.N, a.T, a.Hk, a.Hv);
  const SegPlan plan = seg_plan(a.N, a.T);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  a.ws.chunks = reinterpret_cast<gdn::ChunkInfo*>(w + l.chunks);
  a.ws.seq_first = reinterpret_cast<int32_t*>(w + l.seq_first);
  a.ws.page_first = reinterpret_cast<int32_t*>(w + l.page_first);
  a.ws.Qw = reinterpret_cast<__nv_bfloat16*>(w + l.Qw);
  a.ws.Kw = reinterpret_cast<__nv_bfloat16*>(w + l.Kw);
  a.ws.Ww = reinterpret_cast<__nv_bfloat16*>(w + l.Ww);
  a.ws.Uw = reinterpret_cast<__nv_bfloat16*>(w + l.Uw);
  a.ws.Sw = reinterpret_cast<__nv_bfloat16*>(w + l.Sw);
  a.ws.Gw = reinterpret_cast<float*>(w + l.Gw);
  const size_t NC = (size_t)a.T / kC + (size_t)a.N + 1;
  float* carry = reinterpret_cast<float*>(w + l.carry);
  const size_t carry_stride = (size_t)a.Hv * kD * kD;
  CUtensorMap mQ, mK, mW, mU, mS, mX;
  const int Cc = (2 * a.Hk + a.Hv) * kD;
  if (a.T > 0 && !make_map_x(&mX, a.x, a.T, Cc)) return cudaErrorInvalidValue;
  if (!make_map(&mQ, a.ws.Qw, NC * a.Hk * kC) || !make_map(&mK, a.ws.Kw, NC * a.Hk * kC) ||
      !make_map(&mW, a.ws.Ww, NC * a.Hv * kC) || !make_map(&mU, a.ws.Uw, NC * a.Hv * kC) ||
      !make_map(&mS, a.ws.Sw, NC * a.Hv * kC))
    return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(gdn::gdn_prep_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         gdn::kPrepSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gdn::gdn_qkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               gdn::kQkvSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gdn::gdn_out_persistent_kernel,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, gdn::kOutPSmem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  int num_sms = 0;
  {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e;
  trace_begin("chunk_schedule", s);
  // one CTA; its width only needs to cover the sequences of one pass of the scan
  const int sched_work = std::max(a.N, a.T / kC);
  const int sched_threads = sched_work <= 32 ? 32 : (sched_work <= 256 ? 256 : 1024);
  gdn::chunk_schedule_kernel<<<1, sched_threads, 0, s>>>(
      a.cu, a.N, a.T, a.ws, a.conv0, a.convN, a.slot, a.num_slots, Cc, a.status);
  trace_end(s);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  // one segment's kernels on the given streams; `pdl` where each follows the previous kernel
  // of the same stream with no other dependency in between
  auto launch_parallel_front = [&](const gdn::PrefillArgs& sa, cudaStream_t st,
                                   bool pdl) -> cudaError_t {
    const unsigned nc = (unsigned)(sa.c1 - sa.c0);
    trace_begin("gdn_qkv", st);
    cudaError_t e2 = launch_k(pdl, gdn::gdn_qkv_kernel, dim3(2 * sa.Hk + sa.Hv, nc), dim3(128),
                              gdn::kQkvSmem, st, sa, mX);
    trace_end(st);
    if (e2 != cudaSuccess) return e2;
    trace_begin("gdn_prep", st);
    e2 = launch_k(pdl, gdn::gdn_prep_kernel, dim3(nc, sa.Hv), dim3(256), gdn::kPrepSmem, st, sa, mK,
                  mU, mW);
    trace_end(st);
    return e2;
  };
  auto launch_chain_any = [&](gdn::PrefillArgs sa, cudaStream_t st, bool pdl) -> cudaError_t {
    if (sa.page64) {
      switch (sa.nsplit) {
        case 4: return launch_chain<32, true>(sa, mW, mK, mS, mU, st, pdl);
        case 2: return launch_chain<64, true>(sa, mW, mK, mS, mU, st, pdl);
        default: sa.nsplit = 1; return launch_chain<128, true>(sa, mW, mK, mS, mU, st, pdl);
      }
    }
    switch (sa.nsplit) {
      case 4: return launch_chain<32, false>(sa, mW, mK, mS, mU, st, pdl);
      case 2: return launch_chain<64, false>(sa, mW, mK, mS, mU, st, pdl);
      default: sa.nsplit = 1; return launch_chain<128, false>(sa, mW, mK, mS, mU, st, pdl);
    }
  };
  auto launch_out = [&](const gdn::PrefillArgs& sa, cudaStream_t st, bool pdl) -> cudaError_t {
    // persistent: one CTA per SM at most, each taking a contiguous range of units
    const int units = (sa.c1 - sa.c0) * sa.Hv;
    // pipelined: the SMs that hold a chain CTA take no output CTA (shared memory), so the
    // output kernel's contiguous ranges go to the others only
    const int chain_ctas = a.N * a.Hv * a.nsplit;
    const int sms = plan.nseg > 1 && 2 * chain_ctas < num_sms ? num_sms - chain_ctas : num_sms;
    const int grid = std::max(1, std::min(units, sms));
    trace_begin("gdn_out", st);
    cudaError_t e2 = launch_k(pdl, gdn::gdn_out_persistent_kernel, dim3(grid),
                              dim3(gdn::kOutPThreads), gdn::kOutPSmem, st, sa, mQ, mK, mS, mU);
    trace_end(st);
    return e2;
  };

  const int NCmax = a.T / kC + a.N;
  if (plan.nseg <= 1) {
    a.c0 = 0;
    a.c1 = NCmax;
    a.carry_in = nullptr;
    a.carry_out = nullptr;
    if (a.T > 0 && (e = launch_parallel_front(a, s, true)) != cudaSuccess) return e;
    if ((e = launch_chain_any(a, s, a.T > 0)) != cudaSuccess) return e;
    if (a.T > 0 && (e = launch_out(a, s, true)) != cudaSuccess) return e;
    return cudaSuccess;
  }

  PipeStreams* ps = nullptr;
  if ((e = pipe_streams(&ps)) != cudaSuccess) return e;
  constexpr int W = PipeStreams::kWays;
  cudaStream_t all[2 * W + 1] = {ps->C};
  for (int i = 0; i < W; ++i) {
    all[1 + i] = ps->P[i];
    all[1 + W + i] = ps->O[i];
  }
  // fork: the helper streams start after everything already queued on s (the chunk table)
  if ((e = cudaEventRecord(ps->fork, s)) != cudaSuccess) return e;
  for (cudaStream_t st : all)
    if ((e = cudaStreamWaitEvent(st, ps->fork, 0)) != cudaSuccess) return e;
  for (int k = 0; k < plan.nseg; ++k) {
    gdn::PrefillArgs sa = a;
    sa.c0 = k * plan.seg;
    sa.c1 = std::min(NCmax, (k + 1) * plan.seg);
    sa.carry_in = k > 0 ? carry + (size_t)(k - 1) * carry_stride : nullptr;
    sa.carry_out = k + 1 < plan.nseg ? carry + (size_t)k * carry_stride : nullptr;
    cudaStream_t P = ps->P[k % W], O = ps->O[k % W];
    if ((e = launch_parallel_front(sa, P, false)) != cudaSuccess) return e;
    if ((e = cudaEventRecord(ps->evP, P)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(ps->C, ps->evP, 0)) != cudaSuccess) return e;
    if ((e = launch_chain_any(sa, ps->C, false)) != cudaSuccess) return e;
    if ((e = cudaEventRecord(ps->evC, ps->C)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(O, ps->evC, 0)) != cudaSuccess) return e;
    if ((e = launch_out(sa, O, false)) != cudaSuccess) return e;
  }
  // join: s continues after every helper stream
  for (int i = 0; i < 2 * W + 1; ++i)
    if ((e = cudaEventRecord(ps->join[i], all[i])) != cudaSuccess ||
        (e = cudaStreamWaitEvent(s, ps->join[i], 0)) != cudaSuccess)
      return e;
  return cudaSuccess;
}

}  // namespace gdn_host
