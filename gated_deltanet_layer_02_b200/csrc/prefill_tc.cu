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
// Kernels (one stream, in order):
//   schedule   one CTA: chunk table (sequence, first token, length) from cu_seqlens.
//   prep       per (chunk, key head): conv + SiLU + L2 norms, gates, K K^T on tcgen05, the
//              128x128 inverse (two 64x64 forward substitutions on CUDA cores, joined by two
//              tcgen05 products: T = T_h - T_h N T_h), then W and U~ on tcgen05.
//   chain      per (sequence, value head, d_v block): the sequential part.  S^T lives in TMEM
//              (fp32); per chunk: X = W S_b^T (tcgen05), U = U~ - X, S^T += K^T diag(.) U.
//              W and K tiles arrive by TMA, double-buffered one chunk ahead.
//   out        per (chunk, key head): P from Q K^T (tcgen05), O = e^G Q S^T + P U (tcgen05),
//              z-gated RMSNorm epilogue, bf16 output.
// Workspace tiles are plain row-major [128][128] bf16; TMA loads them with 128-byte swizzle.
#include "args.cuh"
#include "common.cuh"
#include "tc.cuh"

#include <cudaTypedefs.h>

namespace gdn {

constexpr int kC = 128;  // chunk length (tokens)
constexpr int kD = 128;  // head dim
constexpr uint32_t kTile = 16384;  // one [128][64] bf16 row tile



// ------------------------------------------------------------------------------ schedule
__global__ void chunk_schedule_kernel(const int32_t* __restrict__ cu, int N, Workspace ws) {
  // single CTA, sequential prefix over sequences in blocks of blockDim
  __shared__ int carry;
  __shared__ int part[1024];
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < N; base += blockDim.x) {
    const int n = base + threadIdx.x;
    int cnt = 0;
    if (n < N) cnt = (cu[n + 1] - cu[n] + kC - 1) / kC;
    part[threadIdx.x] = cnt;
    __syncthreads();
    for (int off = 1; off < (int)blockDim.x; off <<= 1) {  // inclusive scan
      int v = threadIdx.x >= (unsigned)off ? part[threadIdx.x - off] : 0;
      __syncthreads();
      part[threadIdx.x] += v;
      __syncthreads();
    }
    const int first = carry + part[threadIdx.x] - cnt;
    if (n < N) {
      ws.seq_first[n] = first;
      for (int ci = 0; ci < cnt; ++ci) {
        ChunkInfo info;
        info.n = n;
        info.t0 = cu[n] + ci * kC;
        info.L = min(kC, cu[n + 1] - info.t0);
        info.pad = ci;
        ws.chunks[first + ci] = info;
      }
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry += part[threadIdx.x];
    __syncthreads();
  }
  if (threadIdx.x == 0) ws.seq_first[N] = carry;
}


// ---------------------------------------------------------------------------------- prep
// smem map (bytes from the 1024-aligned base)
constexpr uint32_t kPrepKs = 0;
constexpr uint32_t kPrepV0 = 32768;
constexpr uint32_t kPrepV1 = 65536;
constexpr uint32_t kPrepR1 = 98304;    // A^T blocks (fp32) -> T_h^T (bf16) -> T diag(beta)
constexpr uint32_t kPrepR2 = 131072;   // N (16 KB) + Y' (8 KB) -> K^ = diag(e^G) K
constexpr uint32_t kPrepEnd = 163840;
constexpr uint32_t kPrepSmem = kPrepEnd + 1024 + 4096;
// TMEM columns
constexpr uint32_t kColGram = 0, kColY = 128, kColZ = 192, kColW = 256, kColU = 384;

__device__ __forceinline__ void zero_row_chunk(uint8_t* tile, uint32_t row, uint32_t chunk) {
  *reinterpret_cast<uint4*>(tile + sw128_off(row, chunk)) = make_uint4(0, 0, 0, 0);
}

__global__ void __launch_bounds__(256, 1) gdn_prep_kernel(PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  float* G_s = reinterpret_cast<float*>(sm + kPrepEnd);        // [2][128]
  float* B_s = G_s + 2 * kC;                                    // [2][128]
  float* wt_s = B_s + 2 * kC;                                   // [8] warp totals
  uint64_t* bar = reinterpret_cast<uint64_t*>(wt_s + 8);        // [1]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
  int* abort_s = reinterpret_cast<int*>(tslot + 1);

  const int c = blockIdx.x;
  const int hk = blockIdx.y;
  const int total_chunks = a.ws.seq_first[a.N];
  if (c >= total_chunks) return;
  const ChunkInfo ci = a.ws.chunks[c];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Hk = a.Hk, Hv = a.Hv;
  const int Cc = (2 * Hk + Hv) * kD;
  const int seq_start = __ldg(a.cu + ci.n);

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
    *abort_s = 0;
  }
  if (warp == 0) tmem_alloc(tslot, 512);
  // ---------------- gates: G = inclusive cumsum of g inside the chunk, beta (2 value heads)
  {
    const int r = warp >> 2, i = (warp & 3) * 32 + lane;
    const int h = hk * 2 + r;
    const bool valid = i < ci.L;
    float gv = valid ? __ldg(a.g + (size_t)(ci.t0 + i) * Hv + h) : 0.f;
    const float bv = valid ? __ldg(a.beta + (size_t)(ci.t0 + i) * Hv + h) : 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, gv, o);
      if (lane >= o) gv += y;
    }
    if (lane == 31) wt_s[warp] = gv;
    B_s[r * kC + i] = bv;
    __syncthreads();
    float pre = 0.f;
    for (int w = r * 4; w < warp; ++w) pre += wt_s[w];
    gv += pre;
    G_s[r * kC + i] = gv;
    a.ws.Gw[((size_t)c * Hv + h) * kC + i] = gv;
  }
  // ---------------- conv + SiLU + L2 norms -> Q, K (global), K, V0, V1 (smem operands)
  {
    const int run = tid >> 6, cvec = tid & 63, grp = cvec >> 4, vec = cvec & 15;
    int ch;
    if (grp == 0) ch = hk * kD;
    else if (grp == 1) ch = Hk * kD + hk * kD;
    else ch = 2 * Hk * kD + (hk * 2 + grp - 2) * kD;
    ch += vec * 8;
    float wv[4][8];
    if (a.conv_w) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        uint2 u = *reinterpret_cast<const uint2*>(a.conv_w + (size_t)(ch + e) * 4);
        const __nv_bfloat162* hw = reinterpret_cast<const __nv_bfloat162*>(&u);
        float2 f0 = __bfloat1622float2(hw[0]), f1 = __bfloat1622float2(hw[1]);
        wv[0][e] = f0.x; wv[1][e] = f0.y; wv[2][e] = f1.x; wv[3][e] = f1.y;
      }
    }
    const int i0 = run * 32;
    float hst[3][8];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int t = ci.t0 + i0 - 3 + j;
      if (i0 >= ci.L) {  // the whole run is padding: nothing to read
#pragma unroll
        for (int e = 0; e < 8; ++e) hst[j][e] = 0.f;
      } else if (t >= seq_start) {
        load8(a.x + (size_t)t * Cc + ch, hst[j]);
      } else if (a.conv0) {
        load8(a.conv0 + ((size_t)ci.n * 3 + 3 + (t - seq_start)) * Cc + ch, hst[j]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) hst[j][e] = 0.f;
      }
    }
    uint8_t* vtile = sm + (grp == 2 ? kPrepV0 : kPrepV1);
    const size_t qk_base = ((size_t)c * Hk + hk) * kC * kD;
    for (int ii = 0; ii < 32; ++ii) {
      const int i = i0 + ii;
      const bool valid = i < ci.L;
      float y[8];
      if (valid) {
        float xv[8];
        load8(a.x + (size_t)(ci.t0 + i) * Cc + ch, xv);
        if (a.conv_w) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float acc = wv[0][e] * hst[0][e] + wv[1][e] * hst[1][e] + wv[2][e] * hst[2][e] +
                              wv[3][e] * xv[e];
            y[e] = acc / (1.0f + __expf(-acc));
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) y[e] = xv[e];
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          hst[0][e] = hst[1][e];
          hst[1][e] = hst[2][e];
          hst[2][e] = xv[e];
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = 0.f;
      }
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) ss += y[e] * y[e];
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (grp < 2) {
        const float sc = (grp == 0 ? a.q_scale : 1.0f) * rsqrtf(ss + a.l2_eps);
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = valid ? y[e] * sc : 0.f;
        __nv_bfloat16* dst = (grp == 0 ? a.ws.Qw : a.ws.Kw) + qk_base + (size_t)i * kD + vec * 8;
        store8(dst, y);
        if (grp == 1) st_row8_bf16(sm + kPrepKs, kTile, i, vec, y);
      } else {
        st_row8_bf16(vtile, kTile, i, vec, y);
      }
    }
  }
  fence_proxy_async_smem();
  __syncthreads();
  const uint32_t tmem = *tslot;
  const uint32_t sKs = smem_u32(sm + kPrepKs);
  uint32_t phase = 0;
  // ---------------- gram K K^T
  if (tid == 0) {
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_bf16(tmem + kColGram, desc_kmajor(sKs, kk, kTile), desc_kmajor(sKs, kk, kTile),
               idesc_bf16(128, 128, false, false), kk > 0);
    mma_commit(bar);
  }
  bool ok = mbar_wait(bar, phase);
  phase ^= 1;
  if (__syncthreads_or(!ok)) goto done;
  tc_fence_after();

  for (int r = 0; r < 2; ++r) {
    const int h = hk * 2 + r;
    const float* Gr = G_s + r * kC;
    const float* Br = B_s + r * kC;
    float* AT = reinterpret_cast<float*>(sm + kPrepR1);    // [2][64][64]
    uint8_t* Nt = sm + kPrepR2;                            // [128][64] bf16 tile
    uint8_t* Yt = sm + kPrepR2 + kTile;                    // [64][64] bf16 tile
    // ---- A from the gram: thread row i, columns [half*64, half*64+64)
    {
      const int i = (warp & 3) * 32 + lane, half = warp >> 2;
      const float Gi = Gr[i], bi = Br[i];
      const uint32_t taddr = tmem_at(tmem, (warp & 3) * 32, kColGram + half * 64);
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float v[32];
        tmem_ld32(taddr + cc * 32, v);
        tmem_ld_wait();
        const int j0 = half * 64 + cc * 32;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int j = j0 + e;
          v[e] = (j < i) ? bi * __expf(Gi - Gr[j]) * v[e] : 0.f;
        }
        if ((i >> 6) == half) {
          // diagonal block: store transposed, AT[b][jj][ii]
          float* dst = AT + half * 4096;
#pragma unroll
          for (int e = 0; e < 32; ++e) dst[((j0 + e) & 63) * 64 + (i & 63)] = v[e];
        } else if (half == 0) {
          // lower-left block (i >= 64, j < 64) -> N (bf16, K-major)
#pragma unroll
          for (int q = 0; q < 4; ++q) st_row8_bf16(Nt, kTile, i, (j0 >> 3) + q, v + 8 * q);
        }
      }
      if (i < 64 && half == 0) {
#pragma unroll
        for (int q = 0; q < 8; ++q) zero_row_chunk(Nt, i, q);
      }
    }
    tc_fence_before();
    __syncthreads();
    // ---- two 64x64 unit-lower inverses by forward substitution (column per thread)
    float acc[64];
    const int sb = tid >> 6, sn = tid & 63;
    if (tid < 128) {
#pragma unroll
      for (int rr = 0; rr < 64; ++rr) acc[rr] = (rr == sn) ? 1.f : 0.f;
      const float* ATb = AT + sb * 4096;
#pragma unroll
      for (int ii = 0; ii < 63; ++ii) {
        const float ti = acc[ii];
#pragma unroll
        for (int r4 = (ii + 1) & ~3; r4 < 64; r4 += 4) {
          const float4 av = *reinterpret_cast<const float4*>(ATb + ii * 64 + r4);
          if (r4 + 0 > ii) acc[r4 + 0] -= av.x * ti;
          if (r4 + 1 > ii) acc[r4 + 1] -= av.y * ti;
          if (r4 + 2 > ii) acc[r4 + 2] -= av.z * ti;
          if (r4 + 3 > ii) acc[r4 + 3] -= av.w * ti;
        }
      }
    }
    __syncthreads();
    // ---- T_h^T (bf16) into R1: row n' = column n' of T_h
    uint8_t* TT = sm + kPrepR1;
    if (tid < 128) {
      const int row = sb * 64 + sn;
#pragma unroll
      for (int q = 0; q < 8; ++q) st_row8_bf16(TT, kTile, row, sb * 8 + q, acc + 8 * q);
      if (sb == 1) {
#pragma unroll
        for (int q = 0; q < 8; ++q) zero_row_chunk(TT, row, q);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    // ---- Y = N T_h (M=128, N=64, K=64)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t sN = smem_u32(Nt), sT = smem_u32(TT);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + kColY, desc_kmajor(sN, kk, kTile), desc_kmajor(sT, kk, kTile),
                 idesc_bf16(128, 64, false, false), kk > 0);
      mma_commit(bar);
    }
    ok = mbar_wait(bar, phase);
    phase ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    tc_fence_after();
    // ---- Y' = Y diag(beta) restricted to rows 64..127, cols 0..63 -> bf16 [64][64]
    if ((warp & 3) >= 2) {
      const int j = (warp & 3) * 32 + lane, half = warp >> 2;
      float v[32];
      tmem_ld32(tmem_at(tmem, (warp & 3) * 32, kColY + half * 32), v);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] *= Br[half * 32 + e];
#pragma unroll
      for (int q = 0; q < 4; ++q) st_row8_bf16(Yt, kTile, j - 64, half * 4 + q, v + 8 * q);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- Z' = T_h Y' (M=128, N=64, K=64 over rows 64..127 of T_h)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t sT = smem_u32(TT), sY = smem_u32(Yt);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + kColZ, desc_mnmajor(sT + 8192, kk, kTile), desc_mnmajor(sY, kk, kTile),
                 idesc_bf16(128, 64, true, true), kk > 0);
      mma_commit(bar);
    }
    ok = mbar_wait(bar, phase);
    phase ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    tc_fence_after();
    // ---- T diag(beta) (bf16, K-major [i][j]) into R1; K^ = diag(e^G) K into R2
    uint8_t* TB = sm + kPrepR1;
    uint8_t* Kh = sm + kPrepR2;
    if (tid < 128) {
      // diagonal blocks from the column owners: element (sb*64+rr, sb*64+sn)
      const int col = sb * 64 + sn;
      const float bcol = Br[col];
#pragma unroll
      for (int rr = 0; rr < 64; ++rr) {
        const int row = sb * 64 + rr;
        __nv_bfloat16* p = reinterpret_cast<__nv_bfloat16*>(
            TB + sb * kTile + sw128_off(row, (sn >> 3)) + (sn & 7) * 2);
        *p = __float2bfloat16_rn(acc[rr] * bcol);
      }
    } else if (tid < 192) {
      const int row = tid - 128;  // upper-right block is zero
#pragma unroll
      for (int q = 0; q < 8; ++q) zero_row_chunk(TB + kTile, row, q);
    }
    if ((warp & 3) >= 2) {
      // lower-left block: -Z'
      const int i = (warp & 3) * 32 + lane, half = warp >> 2;
      float v[32];
      tmem_ld32(tmem_at(tmem, (warp & 3) * 32, kColZ + half * 32), v);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = -v[e];
#pragma unroll
      for (int q = 0; q < 4; ++q) st_row8_bf16(TB, kTile, i, half * 4 + q, v + 8 * q);
    }
    {
      // K^ rows: thread pair per row, 8 chunks each; the swizzled position is the same
      const int row = tid >> 1, part = tid & 1;
      const float gam = __expf(Gr[row]);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int chunk16 = part * 8 + q;
        const uint32_t off = (chunk16 >> 3) * kTile + sw128_off(row, chunk16 & 7);
        uint4 u = *reinterpret_cast<const uint4*>(sm + kPrepKs + off);
        __nv_bfloat162* hv = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float2 f = __bfloat1622float2(hv[e]);
          hv[e] = __floats2bfloat162_rn(f.x * gam, f.y * gam);
        }
        *reinterpret_cast<uint4*>(Kh + off) = u;
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- W = T diag(beta) K^,  U~ = T diag(beta) V
    if (tid == 0) {
      tc_fence_after();
      const uint32_t sTB = smem_u32(TB), sK = smem_u32(Kh),
                     sV = smem_u32(sm + (r == 0 ? kPrepV0 : kPrepV1));
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        mma_bf16(tmem + kColW, desc_kmajor(sTB, kk, kTile), desc_mnmajor(sK, kk, kTile),
                 idesc_bf16(128, 128, false, true), kk > 0);
        mma_bf16(tmem + kColU, desc_kmajor(sTB, kk, kTile), desc_mnmajor(sV, kk, kTile),
                 idesc_bf16(128, 128, false, true), kk > 0);
      }
      mma_commit(bar);
    }
    ok = mbar_wait(bar, phase);
    phase ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    tc_fence_after();
    // ---- W, U~ -> workspace (bf16 row-major)
    {
      const int i = (warp & 3) * 32 + lane, half = warp >> 2;
      const size_t base = (((size_t)c * Hv + h) * kC + i) * kD + half * 64;
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        __nv_bfloat16* dst = (m == 0 ? a.ws.Ww : a.ws.Uw) + base;
        const uint32_t col = (m == 0 ? kColW : kColU) + half * 64;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          float v[32];
          tmem_ld32(tmem_at(tmem, (warp & 3) * 32, col + cc * 32), v);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float w8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w8[e] = v[8 * q + e];
            store8(dst + cc * 32 + 8 * q, w8);
          }
        }
      }
    }
    tc_fence_before();
    __syncthreads();
  }
done:
  if (tid == 0 && !ok) report_status(a.status, GDN_ERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(*tslot, 512);
}

// --------------------------------------------------------------------------------- chain
struct ChainMaps {
  CUtensorMap W, K;
};

template <int DV>
struct ChainCfg {
  static constexpr uint32_t kOpTiles = DV > 64 ? 2 : 1;         // 64-col tiles of S_b / U^
  static constexpr uint32_t kStage = 2 * 2 * kTile;             // W + K tiles
  static constexpr uint32_t kSB = 2 * kStage;                   // after two stages
  static constexpr uint32_t kUB = kSB + kOpTiles * kTile;
  static constexpr uint32_t kEnd = kUB + kOpTiles * kTile;
  static constexpr uint32_t kSmem = kEnd + 1024 + 256;
  static constexpr uint32_t kTmemCols = DV < 32 ? 64 : 2 * DV;  // S^T | X
};

template <int DV>
__global__ void __launch_bounds__(128, 1) gdn_chain_kernel(PrefillArgs a,
                                                           const __grid_constant__ CUtensorMap mapW,
                                                           const __grid_constant__ CUtensorMap mapK) {
  using Cfg = ChainCfg<DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + Cfg::kEnd);  // [2]
  uint64_t* bar_mma = bar_tma + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar_mma + 1);

  const int nsplit = a.nsplit;
  const int blk = blockIdx.x % nsplit;
  const int h = (blockIdx.x / nsplit) % a.Hv;
  const int n = blockIdx.x / (nsplit * a.Hv);
  const int hk = h / (a.Hv / a.Hk);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int first = a.ws.seq_first[n];
  const int nch = a.ws.seq_first[n + 1] - first;
  const int v0 = blk * DV;

  if (tid == 0) {
    mbar_init(bar_tma, 1);
    mbar_init(bar_tma + 1, 1);
    mbar_init(bar_mma, 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tslot, Cfg::kTmemCols);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t colS = 0, colX = Cfg::kTmemCols / 2;
  const uint32_t lane_addr = tmem_at(tmem, warp * 32, 0);
  const int k_row = tid;  // TMEM lane = d_k index for S^T, = token index for X

  // ---- S^T initial value: lane k, column v
  {
    const size_t sbase = ((size_t)n * a.Hv + h) * kD * kD;
#pragma unroll
    for (int cc = 0; cc < DV / 32 + (DV < 32 ? 1 : 0); ++cc) {
      float v[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int vv = v0 + cc * 32 + e;
        v[e] = (a.S0 && cc * 32 + e < DV) ? a.S0[sbase + (size_t)vv * kD + k_row] : 0.f;
      }
      tmem_st32(lane_addr + colS + cc * 32, v);
    }
    tmem_st_wait();
  }
  auto issue_tma = [&](int ci, int stage) {
    const int c = first + ci;
    uint8_t* st = sm + stage * Cfg::kStage;
    mbar_arrive_expect_tx(bar_tma + stage, 4 * kTile);
    const int rowW = (c * a.Hv + h) * kC, rowK = (c * a.Hk + hk) * kC;
    tma_load_2d(st, &mapW, bar_tma + stage, 0, rowW);
    tma_load_2d(st + kTile, &mapW, bar_tma + stage, 64, rowW);
    tma_load_2d(st + 2 * kTile, &mapK, bar_tma + stage, 0, rowK);
    tma_load_2d(st + 3 * kTile, &mapK, bar_tma + stage, 64, rowK);
  };
  if (tid == 0 && nch > 0) issue_tma(0, 0);
  uint32_t mma_phase = 0;
  bool ok = true;
  int failed = 0;
  uint8_t* SB = sm + Cfg::kSB;
  uint8_t* UB = sm + Cfg::kUB;
  for (int ci = 0; ci < nch; ++ci) {
    const int c = first + ci, stage = ci & 1;
    if (tid == 0 && ci + 1 < nch) issue_tma(ci + 1, stage ^ 1);
    // per-token inputs of this chunk (row i = tid)
    const float* Gc = a.ws.Gw + ((size_t)c * a.Hv + h) * kC;
    const float Gi = Gc[tid], Glast = Gc[kC - 1];
    __nv_bfloat16* Urow = a.ws.Uw + (((size_t)c * a.Hv + h) * kC + tid) * kD + v0;
    float ut[DV];
#pragma unroll
    for (int q = 0; q < DV / 8; ++q) {
      float t8[8];
      load8(Urow + 8 * q, t8);
#pragma unroll
      for (int e = 0; e < 8; ++e) ut[8 * q + e] = t8[e];
    }
    // ---- S_b (bf16) -> SB operand and workspace; S^T *= e^(G_last)
    {
      const float gam = __expf(Glast);
      __nv_bfloat16* Srow = a.ws.Sw + (((size_t)c * a.Hv + h) * kD + k_row) * kD + v0;
#pragma unroll
      for (int cc = 0; cc < (DV + 31) / 32; ++cc) {
        float v[32];
        tmem_ld32(lane_addr + colS + cc * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (cc * 32 + 8 * q < DV) {
            const int ch = (cc * 32 + 8 * q) >> 3;
            st_row8_bf16(SB, kTile, k_row, ch, v + 8 * q);
            float w8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w8[e] = v[8 * q + e];
            store8(Srow + cc * 32 + 8 * q, w8);
          }
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] *= gam;
        tmem_st32(lane_addr + colS + cc * 32, v);
      }
      tmem_st_wait();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- X = W S_b^T  (M = 128 tokens, N = DV, K = d_k)
    if (tid == 0) {
      ok = mbar_wait(bar_tma + stage, (ci >> 1) & 1);
      tc_fence_after();
      if (ok) {
        const uint32_t sW = smem_u32(sm + stage * Cfg::kStage), sS = smem_u32(SB);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tmem + colX, desc_kmajor(sW, kk, kTile), desc_mnmajor(sS, kk, kTile),
                   idesc_bf16(128, DV, false, true), kk > 0);
        mma_commit(bar_mma);
      }
    }
    if ((failed = __syncthreads_or(!ok))) break;
    ok = mbar_wait(bar_mma, mma_phase);
    mma_phase ^= 1;
    if ((failed = __syncthreads_or(!ok))) break;
    tc_fence_after();
    // ---- U = U~ - X -> workspace; U^ = diag(e^(G_L - G)) U -> UB operand
    {
      const float dec = __expf(Glast - Gi);
#pragma unroll
      for (int cc = 0; cc < (DV + 31) / 32; ++cc) {
        float v[32];
        tmem_ld32(lane_addr + colX + cc * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (cc * 32 + 8 * q < DV) {
            float u8[8], h8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              u8[e] = ut[cc * 32 + 8 * q + e] - v[8 * q + e];
              h8[e] = u8[e] * dec;
            }
            store8(Urow + cc * 32 + 8 * q, u8);
            st_row8_bf16(UB, kTile, tid, (cc * 32 + 8 * q) >> 3, h8);
          }
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- S^T += K^T U^  (M = d_k, N = DV, K = tokens)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t sK = smem_u32(sm + stage * Cfg::kStage + 2 * kTile), sU = smem_u32(UB);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem + colS, desc_mnmajor(sK, kk, kTile), desc_mnmajor(sU, kk, kTile),
                 idesc_bf16(128, DV, true, true), 1);
      mma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, mma_phase);
    mma_phase ^= 1;
    if ((failed = __syncthreads_or(!ok))) break;
    tc_fence_after();
  }
  if (!failed && a.SN) {
    const size_t sbase = ((size_t)n * a.Hv + h) * kD * kD;
#pragma unroll
    for (int cc = 0; cc < (DV + 31) / 32; ++cc) {
      float v[32];
      tmem_ld32(lane_addr + colS + cc * 32, v);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (cc * 32 + e < DV) a.SN[sbase + (size_t)(v0 + cc * 32 + e) * kD + k_row] = v[e];
    }
  }
  if (tid == 0 && failed) report_status(a.status, GDN_ERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, Cfg::kTmemCols);
}

// ----------------------------------------------------------------------------------- out
constexpr uint32_t kOutQ = 0, kOutK = 32768, kOutS = 65536, kOutU = 98304, kOutP = 131072;
constexpr uint32_t kOutEnd = 163840;
constexpr uint32_t kOutSmem = kOutEnd + 1024 + 1024;
constexpr uint32_t kColQK = 0, kColYo = 128, kColPU = 256;

__global__ void __launch_bounds__(128, 1) gdn_out_kernel(PrefillArgs a,
                                                         const __grid_constant__ CUtensorMap mapQ,
                                                         const __grid_constant__ CUtensorMap mapK,
                                                         const __grid_constant__ CUtensorMap mapS,
                                                         const __grid_constant__ CUtensorMap mapU) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint64_t* bar_qk = reinterpret_cast<uint64_t*>(sm + kOutEnd);
  uint64_t* bar_su = bar_qk + 1;
  uint64_t* bar_mma = bar_qk + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar_qk + 3);
  float* G_s = reinterpret_cast<float*>(sm + kOutEnd + 64);   // [128]

  const int c = blockIdx.x, hk = blockIdx.y;
  const int total_chunks = a.ws.seq_first[a.N];
  if (c >= total_chunks) return;
  const ChunkInfo ci = a.ws.chunks[c];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int Hv = a.Hv;
  if (tid == 0) {
    mbar_init(bar_qk, 1);
    mbar_init(bar_su, 1);
    mbar_init(bar_mma, 1);
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tslot, 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t lane_addr = tmem_at(tmem, warp * 32, 0);
  auto load_su = [&](int r) {
    const int row = ((c * Hv) + hk * 2 + r) * kC;
    mbar_arrive_expect_tx(bar_su, 4 * kTile);
    tma_load_2d(sm + kOutS, &mapS, bar_su, 0, row);
    tma_load_2d(sm + kOutS + kTile, &mapS, bar_su, 64, row);
    tma_load_2d(sm + kOutU, &mapU, bar_su, 0, row);
    tma_load_2d(sm + kOutU + kTile, &mapU, bar_su, 64, row);
  };
  if (tid == 0) {
    const int row = (c * a.Hk + hk) * kC;
    mbar_arrive_expect_tx(bar_qk, 4 * kTile);
    tma_load_2d(sm + kOutQ, &mapQ, bar_qk, 0, row);
    tma_load_2d(sm + kOutQ + kTile, &mapQ, bar_qk, 64, row);
    tma_load_2d(sm + kOutK, &mapK, bar_qk, 0, row);
    tma_load_2d(sm + kOutK + kTile, &mapK, bar_qk, 64, row);
    load_su(0);
  }
  const uint32_t sQ = smem_u32(sm + kOutQ), sK = smem_u32(sm + kOutK),
                 sS = smem_u32(sm + kOutS), sU = smem_u32(sm + kOutU), sP = smem_u32(sm + kOutP);
  bool ok = true;
  uint32_t mma_phase = 0;
  if (tid == 0) {
    ok = mbar_wait(bar_qk, 0);
    tc_fence_after();
    if (ok) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tmem + kColQK, desc_kmajor(sQ, kk, kTile), desc_kmajor(sK, kk, kTile),
                 idesc_bf16(128, 128, false, false), kk > 0);
      mma_commit(bar_mma);
    }
  }
  if (__syncthreads_or(!ok)) goto done;
  ok = mbar_wait(bar_mma, mma_phase);
  mma_phase ^= 1;
  if (__syncthreads_or(!ok)) goto done;
  tc_fence_after();
  for (int r = 0; r < 2; ++r) {
    const int h = hk * 2 + r;
    const int i = tid;
    G_s[i] = a.ws.Gw[((size_t)c * Hv + h) * kC + i];
    __syncthreads();
    const float Gi = G_s[i];
    // ---- P (bf16, K-major) from Q K^T
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      float v[32];
      tmem_ld32(lane_addr + kColQK + cc * 32, v);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int j = cc * 32 + e;
        v[e] = (j <= i) ? __expf(Gi - G_s[j]) * v[e] : 0.f;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) st_row8_bf16(sm + kOutP, kTile, i, cc * 4 + q, v + 8 * q);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- Y = Q S^T ; O_intra = P U
    if (tid == 0) {
      ok = mbar_wait(bar_su, r & 1);
      tc_fence_after();
      if (ok) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          mma_bf16(tmem + kColYo, desc_kmajor(sQ, kk, kTile), desc_mnmajor(sS, kk, kTile),
                   idesc_bf16(128, 128, false, true), kk > 0);
          mma_bf16(tmem + kColPU, desc_kmajor(sP, kk, kTile), desc_mnmajor(sU, kk, kTile),
                   idesc_bf16(128, 128, false, true), kk > 0);
        }
        mma_commit(bar_mma);
      }
    }
    if (__syncthreads_or(!ok)) goto done;
    ok = mbar_wait(bar_mma, mma_phase);
    mma_phase ^= 1;
    if (__syncthreads_or(!ok)) goto done;
    tc_fence_after();
    if (tid == 0 && r == 0) load_su(1);  // S and U buffers are free again
    // ---- epilogue: o = e^G Y + P U, gated RMSNorm, bf16 out
    const float eg = __expf(Gi);
    const bool valid = i < ci.L;
    const size_t orow = ((size_t)(ci.t0 + i) * Hv + h) * kD;
    float inv = 1.f;
    if (a.z) {
      float ss = 0.f;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        float y[32], p[32];
        tmem_ld32(lane_addr + kColYo + cc * 32, y);
        tmem_ld32(lane_addr + kColPU + cc * 32, p);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float o = eg * y[e] + p[e];
          ss += o * o;
        }
      }
      inv = rsqrtf(ss / kD + a.norm_eps);
    }
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      float y[32], p[32];
      tmem_ld32(lane_addr + kColYo + cc * 32, y);
      tmem_ld32(lane_addr + kColPU + cc * 32, p);
      tmem_ld_wait();
      if (valid) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float o8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) o8[e] = eg * y[8 * q + e] + p[8 * q + e];
          if (a.z) {
            float z8[8], w8[8];
            load8(a.z + orow + cc * 32 + 8 * q, z8);
            if (a.norm_w) load8(a.norm_w + cc * 32 + 8 * q, w8);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              o8[e] = o8[e] * inv * (a.norm_w ? w8[e] : 1.f) * (z8[e] / (1.f + __expf(-z8[e])));
          }
          store8(a.out + orow + cc * 32 + 8 * q, o8);
        }
      }
    }
    tc_fence_before();
    __syncthreads();
  }
done:
  if (tid == 0 && !ok) report_status(a.status, GDN_ERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace gdn

// =================================================================================== host
namespace gdn_host {

using gdn::kC;
using gdn::kD;

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct WsLayout {
  size_t chunks, seq_first, Qw, Kw, Ww, Uw, Sw, Gw, total;
};

static WsLayout ws_layout(int N, int T, int Hk, int Hv) {
  const size_t NC = (size_t)T / kC + (size_t)N + 1;
  const size_t tile = (size_t)kC * kD * 2;
  WsLayout l;
  size_t o = 0;
  l.chunks = o; o = align_up(o + NC * sizeof(gdn::ChunkInfo), 1024);
  l.seq_first = o; o = align_up(o + (size_t)(N + 1) * 4, 1024);
  l.Qw = o; o = align_up(o + NC * Hk * tile, 1024);
  l.Kw = o; o = align_up(o + NC * Hk * tile, 1024);
  l.Ww = o; o = align_up(o + NC * Hv * tile, 1024);
  l.Uw = o; o = align_up(o + NC * Hv * tile, 1024);
  l.Sw = o; o = align_up(o + NC * Hv * tile, 1024);
  l.Gw = o; o = align_up(o + NC * Hv * kC * 4, 1024);
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

template <int DV>
static cudaError_t launch_chain(const gdn::PrefillArgs& a, const CUtensorMap& mW,
                                const CUtensorMap& mK, cudaStream_t s) {
  using Cfg = gdn::ChainCfg<DV>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(gdn::gdn_chain_kernel<DV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  trace_begin("gdn_chain", s);
  gdn::gdn_chain_kernel<DV><<<a.N * a.Hv * a.nsplit, 128, Cfg::kSmem, s>>>(a, mW, mK);
  trace_end(s);
  return cudaGetLastError();
}

int choose_nsplit(int N, int Hv) {
  const int units = N * Hv;
  if (units >= 148) return 1;
  if (units * 2 >= 148) return 2;
  return 4;
}

cudaError_t launch_prefill_tc(gdn::PrefillArgs a, void* workspace, cudaStream_t s) {
  const WsLayout l = ws_layout(a.N, a.T, a.Hk, a.Hv);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  a.ws.chunks = reinterpret_cast<gdn::ChunkInfo*>(w + l.chunks);
  a.ws.seq_first = reinterpret_cast<int32_t*>(w + l.seq_first);
  a.ws.Qw = reinterpret_cast<__nv_bfloat16*>(w + l.Qw);
  a.ws.Kw = reinterpret_cast<__nv_bfloat16*>(w + l.Kw);
  a.ws.Ww = reinterpret_cast<__nv_bfloat16*>(w + l.Ww);
  a.ws.Uw = reinterpret_cast<__nv_bfloat16*>(w + l.Uw);
  a.ws.Sw = reinterpret_cast<__nv_bfloat16*>(w + l.Sw);
  a.ws.Gw = reinterpret_cast<float*>(w + l.Gw);
  const size_t NC = (size_t)a.T / kC + (size_t)a.N + 1;
  CUtensorMap mQ, mK, mW, mU, mS;
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
      e = cudaFuncSetAttribute(gdn::gdn_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               gdn::kOutSmem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  cudaError_t e;
  trace_begin("chunk_schedule", s);
  gdn::chunk_schedule_kernel<<<1, 1024, 0, s>>>(a.cu, a.N, a.ws);
  trace_end(s);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const dim3 grid_chunks((unsigned)(a.T / kC + a.N), a.Hk);
  if (a.T > 0) {
    trace_begin("gdn_prep", s);
    gdn::gdn_prep_kernel<<<grid_chunks, 256, gdn::kPrepSmem, s>>>(a);
    trace_end(s);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  switch (a.nsplit) {
    case 4: e = launch_chain<32>(a, mW, mK, s); break;
    case 2: e = launch_chain<64>(a, mW, mK, s); break;
    default: a.nsplit = 1; e = launch_chain<128>(a, mW, mK, s); break;
  }
  if (e != cudaSuccess) return e;
  if (a.T > 0) {
    trace_begin("gdn_out", s);
    gdn::gdn_out_kernel<<<grid_chunks, 128, gdn::kOutSmem, s>>>(a, mQ, mK, mS, mU);
    trace_end(s);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace gdn_host
