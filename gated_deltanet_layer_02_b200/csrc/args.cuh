// args.cuh -- argument blocks passed by value from the C-ABI layer to the kernels.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

namespace gdn {

// Row of a state pool that holds the states of sequence n: slot[n], or n without a slot map.
// A slot outside [0, num_slots) gives -1: the caller then reads that sequence's initial states
// as zero, writes none of its states and reports GDN_ERR_INVALID_ARG.
__device__ __forceinline__ int state_row(const int32_t* slot, int n, int num_slots) {
  if (!slot) return n;
  const int r = __ldg(slot + n);
  return (r >= 0 && r < num_slots) ? r : -1;
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
  int32_t* status;  // device status word (first error wins), or NULL
  int num_slots;    // rows of the state pools (slot_idx entries must lie in [0, num_slots))
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
  int32_t* status;
  int num_slots;
  int N, Hk, Hv;
  float q_scale, l2_eps, norm_eps;
};

struct ChunkInfo {
  int n, t0, L, pad;
};

struct Workspace {
  ChunkInfo* chunks;     // [NCmax]
  int32_t* seq_first;    // [N+1] first chunk of each sequence (prefix sum), [N] = total
  int32_t* page_first;   // [N+1] first 64-token page of each sequence (prefix sum)
  __nv_bfloat16* Qw;     // [NCmax][Hk][128][128]
  __nv_bfloat16* Kw;     // [NCmax][Hk][128][128]
  __nv_bfloat16* Ww;     // [NCmax][Hv][128][128]
  __nv_bfloat16* Uw;     // [NCmax][Hv][128][128]  U~ from prep, overwritten with U by chain
  __nv_bfloat16* Sw;     // [NCmax][Hv][128 (d_k)][128 (d_v)]  S^T entering each chunk
  float* Gw;             // [NCmax][Hv][128]  cumulative log decay inside the chunk
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
  float* chunk_states;  // [entries][Hv][d_v][d_k] fp32: state after each chunk (or each
                        // 64-token page with page64), or NULL
  int page64;           // states every 64 tokens instead of every chunk
  const int32_t* slot;  // [N] state-pool row of each sequence (S0, SN, conv0, convN), or NULL
  int32_t* status;
  uint64_t wait_ns;     // bound of every device wait (ns); a wait that runs out reports
                        // GDN_ERR_TIMEOUT
  int fault_chunk;      // debug fault injection: the first chain CTA skips the W load of this
                        // chunk (-1: none)
  uint64_t* stamps;     // debug: %globaltimer stamps of kernel phases (first CTA), or NULL
  int num_slots;        // rows of the state pools when `slot` is set
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
