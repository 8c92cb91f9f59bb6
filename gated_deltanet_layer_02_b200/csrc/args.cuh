// args.cuh -- argument blocks passed by value from the C-ABI layer to the kernels.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

namespace gdn {

// Row of a state pool that holds the states of sequence n: slot[n], or n without a slot map.
__device__ __forceinline__ int state_row(const int32_t* slot, int n) {
  return slot ? __ldg(slot + n) : n;
}

struct DecodeArgs {
  const void* x;
  const void* conv_w;
  const float* beta;
  const float* g;
  const void* z;
  const void* norm_w;
  void* conv_state;
  void* S;  // fp32 or bf16 (see the decode kernel's state type)
  const int32_t* slot_idx;
  void* out;
  int B, Hk, Hv;
  float q_scale, l2_eps, norm_eps;
};

struct RecArgs {
  const float* x;
  const float* conv_w;
  const float* beta;
  const float* g;
  const float* z;
  const float* norm_w;
  const int32_t* cu;
  const float* S0;
  float* SN;
  const float* conv0;
  float* out;
  const int32_t* slot;  // [N] state-pool row of each sequence (S0, SN, conv0), or NULL (= n)
  int N, Hk, Hv;
  float q_scale, l2_eps, norm_eps;
};

struct ChunkInfo {
  int n, t0, L, pad;
};

struct Workspace {
  ChunkInfo* chunks;     // [NCmax]
  int32_t* seq_first;    // [N+1] first chunk of each sequence (prefix sum), [N] = total
  __nv_bfloat16* Qw;     // [NCmax][Hk][128][128]
  __nv_bfloat16* Kw;     // [NCmax][Hk][128][128]
  __nv_bfloat16* Ww;     // [NCmax][Hv][128][128]
  __nv_bfloat16* Uw;     // [NCmax][Hv][128][128]  U~ from prep, overwritten with U by chain
  __nv_bfloat16* Sw;     // [NCmax][Hv][128 (d_k)][128 (d_v)]  S^T entering each chunk
  float* Gw;             // [NCmax][Hv][128]  cumulative log decay inside the chunk
  int* ready;            // [NCmax][Hv]  prep published (chunk, value head); zeroed per call
  int* counter;          // next prep unit of the persistent workers; zeroed per call
};

struct PrefillArgs {
  const __nv_bfloat16* x;
  const __nv_bfloat16* conv_w;
  const float* beta;
  const float* g;
  const __nv_bfloat16* z;
  const __nv_bfloat16* norm_w;
  const int32_t* cu;
  const float* S0;
  float* SN;
  const __nv_bfloat16* conv0;
  __nv_bfloat16* convN;  // written by the q/k/v kernel (and the chunk table for empty sequences)
                         // when set; NULL when the caller wants none or it aliases conv0
  __nv_bfloat16* out;
  float* chunk_states;  // [chunks][Hv][d_v][d_k] fp32: state after each chunk, or NULL
  const int32_t* slot;  // [N] state-pool row of each sequence (S0, SN, conv0, convN), or NULL
  int32_t* status;
  int N, T, Hk, Hv, nsplit;
  float q_scale, l2_eps, norm_eps;
  Workspace ws;
  // chunk range [c0, c1) of this launch (global chunk indices of the chunk table); a sequence
  // that crosses c0 enters with the fp32 state in carry_in, one that crosses c1 leaves it in
  // carry_out ([Hv][d_v][d_k] each: at most one sequence crosses any chunk boundary)
  int c0, c1;
  const float* carry_in;
  float* carry_out;
};

}  // namespace gdn
