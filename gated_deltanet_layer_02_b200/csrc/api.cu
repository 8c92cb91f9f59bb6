// api.cu -- the extern "C" entry points of libgdn.so: argument checks, workspace sizing,
// dispatch to the kernels, launch tracing and the bounded-wait probe.  Declared in gdn.h.
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "common.cuh"
#include "tc.cuh"

#include "args.cuh"

namespace gdn_host {
cudaError_t launch_conv1d(bool bf16, const void* x, void* y, const void* w, const int32_t* cu,
                          int N, int T_total, int Cc, const void* st_in, void* st_out,
                          cudaStream_t s);
cudaError_t launch_conv_state_out(bool bf16, const void* x, const int32_t* cu, int N, int Cc,
                                  const void* st_in, void* st_out, const int32_t* slot,
                                  int num_slots, int32_t* status, cudaStream_t s);
cudaError_t launch_gated_rmsnorm(bool bf16, const void* o, const void* z, const void* w, float eps,
                                 int rows, int dim, void* y, cudaStream_t s);
cudaError_t launch_decode(bool bf16, bool state_bf16, const gdn::DecodeArgs& a, cudaStream_t s);
cudaError_t launch_decode_multi(bool bf16, const gdn::DecodeArgs& a, int k, float* snaps,
                                cudaStream_t s);
cudaError_t launch_recurrent_f32(const gdn::RecArgs& a, cudaStream_t s);
cudaError_t launch_prefill_tc(gdn::PrefillArgs a, void* workspace, cudaStream_t s);
size_t prefill_tc_workspace(int N, int T, int Hk, int Hv);
int choose_nsplit(int N, int T, int Hv);

// ------------------------------------------------------------------------------ tracing
struct TraceRec {
  const char* name;
  cudaEvent_t start, stop;
};
}  // namespace gdn_host

struct gdn_trace {
  std::vector<gdn_host::TraceRec> recs;
  int used = 0;
  static constexpr int kCap = 4096;
};

namespace gdn_host {
static thread_local gdn_trace* t_trace = nullptr;
static thread_local bool t_open = false;

// Records `ev` on `s`.  Inside a stream capture the record becomes an event-record node of the
// graph (cudaEventRecordExternal), so every replay of the graph records the event again and the
// launch times can be read after each replay.
static cudaError_t record_event(cudaEvent_t ev, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    return cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
  return cudaEventRecord(ev, s);
}

void trace_begin(const char* name, cudaStream_t s) {
  gdn_trace* tr = t_trace;
  t_open = false;
  if (!tr || tr->used >= gdn_trace::kCap) return;
  if (tr->used == (int)tr->recs.size()) {
    TraceRec r{};
    if (cudaEventCreate(&r.start) != cudaSuccess) return;
    if (cudaEventCreate(&r.stop) != cudaSuccess) {
      cudaEventDestroy(r.start);
      return;
    }
    tr->recs.push_back(r);
  }
  TraceRec& r = tr->recs[tr->used];
  r.name = name;
  if (record_event(r.start, s) == cudaSuccess) t_open = true;
}

bool trace_attached() { return t_trace != nullptr; }

void trace_end(cudaStream_t s) {
  gdn_trace* tr = t_trace;
  if (!tr || !t_open) return;
  t_open = false;
  if (record_event(tr->recs[tr->used].stop, s) == cudaSuccess) tr->used++;
}
}  // namespace gdn_host

// ---------------------------------------------------------------------- bounded-wait probe
namespace gdn {
__global__ void wait_probe_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    // nothing ever arrives on `bar`: the wait must give up by itself
    const uint64_t t0 = global_timer_ns();
    bool done = false;
    while (!(done = mbar_try_wait(&bar, 0))) {
      if (global_timer_ns() - t0 > limit_ns) break;
      __nanosleep(100);
    }
    if (!done) report_status(status, GDN_ERR_TIMEOUT);
  }
}
}  // namespace gdn

// ============================================================================ entry points
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_dims(const gdn_dims* d) {
  if (!d) return GDN_ERR_INVALID_ARG;
  if (d->num_k_heads <= 0 || d->num_v_heads <= 0 || d->head_dim <= 0 || d->conv_kernel <= 0)
    return GDN_ERR_INVALID_ARG;
  if (d->num_v_heads % d->num_k_heads != 0) return GDN_ERR_INVALID_ARG;
  if (d->head_dim != gdn::kHeadDim || d->conv_kernel != gdn::kConvK) return GDN_ERR_UNSUPPORTED;
  if (!(d->l2_eps >= 0.f) || !(d->norm_eps >= 0.f)) return GDN_ERR_INVALID_ARG;
  return GDN_OK;
}

int64_t channels(const gdn_dims* d) {
  return (int64_t)(2 * d->num_k_heads + d->num_v_heads) * d->head_dim;
}

int map_cuda(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

bool dtype_ok(gdn_dtype t) { return t == GDN_F32 || t == GDN_BF16; }

}  // namespace

namespace gdn_host {
int check_dims_ext(const gdn_dims* d) { return check_dims(d); }

static thread_local gdn_debug_options t_debug = {};
const gdn_debug_options& debug_opts() { return t_debug; }
}  // namespace gdn_host

extern "C" {

int gdn_abi_version(void) { return GDN_ABI_VERSION; }

int64_t gdn_conv_channels(const gdn_dims* dims) {
  return dims ? channels(dims) : -1;
}

const char* gdn_status_string(int status) {
  switch (status) {
    case GDN_OK: return "ok";
    case GDN_ERR_INVALID_ARG: return "invalid argument";
    case GDN_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case GDN_ERR_CUDA: return "CUDA error";
    case GDN_ERR_TIMEOUT: return "device wait timed out";
    case GDN_ERR_WORKSPACE: return "workspace too small";
    case GDN_ERR_BOUNDS: return "index check failed (bounds-check build)";
    default: return "unknown status";
  }
}

int gdn_conv1d_update(const gdn_dims* dims, gdn_dtype dtype, const void* x, void* y,
                      const void* conv_w, const int32_t* cu_seqlens, int32_t num_seqs,
                      int32_t num_tokens, const void* conv_state_in, void* conv_state_out,
                      void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!dtype_ok(dtype)) return GDN_ERR_UNSUPPORTED;
  if (num_seqs < 0 || num_tokens < 0) return GDN_ERR_INVALID_ARG;
  if (!cu_seqlens && num_seqs > 0) return GDN_ERR_INVALID_ARG;
  if (num_tokens > 0 && (!x || !y || !conv_w || num_seqs == 0)) return GDN_ERR_INVALID_ARG;
  if (x == y && x) return GDN_ERR_INVALID_ARG;
  const void* ptrs[] = {x, y, conv_w, conv_state_in, conv_state_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  const int64_t Cc = channels(dims);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return map_cuda(gdn_host::launch_conv1d(dtype == GDN_BF16, x, y, conv_w, cu_seqlens, num_seqs,
                                          num_tokens, (int)Cc, conv_state_in, conv_state_out, s));
}

int gdn_gated_rmsnorm(gdn_dtype dtype, const void* o, const void* z, const void* w, float eps,
                      int32_t rows, int32_t dim, void* y, void* stream) {
  if (!dtype_ok(dtype)) return GDN_ERR_UNSUPPORTED;
  if (rows < 0 || dim <= 0 || dim % 8 != 0) return GDN_ERR_INVALID_ARG;
  if (dim > 1024) return GDN_ERR_UNSUPPORTED;
  if (!(eps >= 0.f)) return GDN_ERR_INVALID_ARG;
  if (rows > 0 && (!o || !z || !y)) return GDN_ERR_INVALID_ARG;
  const void* ptrs[] = {o, z, w, y};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  return map_cuda(gdn_host::launch_gated_rmsnorm(dtype == GDN_BF16, o, z, w, eps, rows, dim, y,
                                                 static_cast<cudaStream_t>(stream)));
}

size_t gdn_chunk_prefill_workspace_size(const gdn_dims* dims, gdn_dtype dtype, int32_t num_seqs,
                                        int32_t num_tokens) {
  if (check_dims(dims) != GDN_OK || num_seqs < 0 || num_tokens < 0) return 0;
  if (dtype != GDN_BF16) return 256;  // the fp32 path keeps everything on chip
  return gdn_host::prefill_tc_workspace(num_seqs, num_tokens, dims->num_k_heads,
                                        dims->num_v_heads);
}

static int prefill_impl(const gdn_dims* dims, gdn_dtype dtype, const void* x,
                        const void* conv_w, const float* beta, const float* g, const void* z,
                        const void* norm_w, const int32_t* cu_seqlens, int32_t num_seqs,
                        int32_t num_tokens, const float* S0, float* SN, const void* conv0,
                        void* convN, void* out, void* workspace, size_t workspace_bytes,
                        int32_t* dev_status, float* chunk_states, const int32_t* slot,
                        int32_t num_slots, void* stream, bool page64 = false) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!dtype_ok(dtype)) return GDN_ERR_UNSUPPORTED;
  if (num_seqs < 0 || num_tokens < 0) return GDN_ERR_INVALID_ARG;
  if (num_seqs == 0 && num_tokens > 0) return GDN_ERR_INVALID_ARG;
  if (num_seqs > 0 && !cu_seqlens) return GDN_ERR_INVALID_ARG;
  if (slot && num_slots <= 0 && num_seqs > 0) return GDN_ERR_INVALID_ARG;
  if (num_tokens > 0 && (!x || !beta || !g || !out)) return GDN_ERR_INVALID_ARG;
  const void* ptrs[] = {x, conv_w, beta, g, z, norm_w, S0, SN, conv0, convN, out, chunk_states};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return GDN_ERR_INVALID_ARG;
  const bool bf16 = dtype == GDN_BF16;
  if (chunk_states && !bf16) return GDN_ERR_UNSUPPORTED;  // the fp32 path has no chunks
  if (bf16 && dims->num_v_heads != 2 * dims->num_k_heads) return GDN_ERR_UNSUPPORTED;
  const size_t need = gdn_chunk_prefill_workspace_size(dims, dtype, num_seqs, num_tokens);
  if (bf16 && (!workspace || workspace_bytes < need)) return GDN_ERR_WORKSPACE;
  if (num_seqs == 0) return GDN_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int Cc = (int)channels(dims);
  if (!bf16) {
    gdn::RecArgs a{};
    a.x = static_cast<const float*>(x);
    a.conv_w = static_cast<const float*>(conv_w);
    a.beta = beta;
    a.g = g;
    a.z = static_cast<const float*>(z);
    a.norm_w = static_cast<const float*>(norm_w);
    a.cu = cu_seqlens;
    a.S0 = S0;
    a.SN = SN;
    a.conv0 = static_cast<const float*>(conv0);
    a.out = static_cast<float*>(out);
    a.slot = slot;
    a.status = dev_status;
    a.num_slots = num_slots;
    a.N = num_seqs;
    a.Hk = dims->num_k_heads;
    a.Hv = dims->num_v_heads;
    a.q_scale = dims->q_scale;
    a.l2_eps = dims->l2_eps;
    a.norm_eps = dims->norm_eps;
    cudaError_t e = gdn_host::launch_recurrent_f32(a, s);
    if (e == cudaSuccess && convN)
      e = gdn_host::launch_conv_state_out(false, x, cu_seqlens, num_seqs, Cc, conv0, convN, slot,
                                          num_slots, dev_status, s);
    return map_cuda(e);
  }
  gdn::PrefillArgs a{};
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.conv_w = static_cast<const __nv_bfloat16*>(conv_w);
  a.beta = beta;
  a.g = g;
  a.z = static_cast<const __nv_bfloat16*>(z);
  a.norm_w = static_cast<const __nv_bfloat16*>(norm_w);
  a.cu = cu_seqlens;
  a.S0 = S0;
  a.SN = SN;
  a.conv0 = static_cast<const __nv_bfloat16*>(conv0);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.chunk_states = chunk_states;
  a.page64 = page64 ? 1 : 0;
  a.slot = slot;
  a.status = dev_status;
  a.num_slots = num_slots;
  {
    const gdn_debug_options& dbg = gdn_host::debug_opts();
    a.wait_ns = dbg.wait_limit_us ? (uint64_t)dbg.wait_limit_us * 1000ull : gdn::kWaitLimitNs;
    a.fault_chunk = dbg.fault == GDN_FAULT_SKIP_CHAIN_LOAD ? dbg.fault_chunk : -1;
    a.stamps = dbg.timestamps;
  }
  a.N = num_seqs;
  a.T = num_tokens;
  a.Hk = dims->num_k_heads;
  a.Hv = dims->num_v_heads;
  a.nsplit = gdn_host::choose_nsplit(num_seqs, num_tokens, dims->num_v_heads);
  a.q_scale = dims->q_scale;
  a.l2_eps = dims->l2_eps;
  a.norm_eps = dims->norm_eps;
  // the final conv history comes out of the q/k/v kernel unless it overwrites conv0 in place
  // (another chunk of the sequence may still read conv0 then)
  const bool separate_conv_state = convN && (convN == conv0 || num_tokens == 0);
  a.convN = separate_conv_state ? nullptr : static_cast<__nv_bfloat16*>(convN);
  cudaError_t e = gdn_host::launch_prefill_tc(a, workspace, s);
  if (e == cudaSuccess && separate_conv_state)
    e = gdn_host::launch_conv_state_out(true, x, cu_seqlens, num_seqs, Cc, conv0, convN, slot,
                                        num_slots, dev_status, s);
  return map_cuda(e);
}

int gdn_chunk_prefill(const gdn_dims* dims, gdn_dtype dtype, const void* x, const void* conv_w,
                      const float* beta, const float* g, const void* z, const void* norm_w,
                      const int32_t* cu_seqlens, int32_t num_seqs, int32_t num_tokens,
                      const float* S0, float* SN, const void* conv0, void* convN, void* out,
                      void* workspace, size_t workspace_bytes, int32_t* dev_status,
                      void* stream) {
  return prefill_impl(dims, dtype, x, conv_w, beta, g, z, norm_w, cu_seqlens, num_seqs,
                      num_tokens, S0, SN, conv0, convN, out, workspace, workspace_bytes,
                      dev_status, nullptr, nullptr, num_seqs, stream);
}

int gdn_chunk_prefill_states(const gdn_dims* dims, gdn_dtype dtype, const void* x,
                             const void* conv_w, const float* beta, const float* g,
                             const void* z, const void* norm_w, const int32_t* cu_seqlens,
                             int32_t num_seqs, int32_t num_tokens, const float* S0, float* SN,
                             const void* conv0, void* convN, void* out, float* chunk_states,
                             void* workspace, size_t workspace_bytes, int32_t* dev_status,
                             void* stream) {
  if (num_tokens > 0 && !chunk_states) return GDN_ERR_INVALID_ARG;
  return prefill_impl(dims, dtype, x, conv_w, beta, g, z, norm_w, cu_seqlens, num_seqs,
                      num_tokens, S0, SN, conv0, convN, out, workspace, workspace_bytes,
                      dev_status, chunk_states, nullptr, num_seqs, stream);
}

int gdn_chunk_prefill_pages(const gdn_dims* dims, gdn_dtype dtype, const void* x,
                            const void* conv_w, const float* beta, const float* g, const void* z,
                            const void* norm_w, const int32_t* cu_seqlens, int32_t num_seqs,
                            int32_t num_tokens, const float* S0, float* SN, const void* conv0,
                            void* convN, void* out, int32_t page_size, float* page_states,
                            void* workspace, size_t workspace_bytes, int32_t* dev_status,
                            void* stream) {
  if (page_size != 64 && page_size != 128) return GDN_ERR_UNSUPPORTED;
  if (num_tokens > 0 && !page_states) return GDN_ERR_INVALID_ARG;
  return prefill_impl(dims, dtype, x, conv_w, beta, g, z, norm_w, cu_seqlens, num_seqs,
                      num_tokens, S0, SN, conv0, convN, out, workspace, workspace_bytes,
                      dev_status, page_states, nullptr, num_seqs, stream, page_size == 64);
}

int gdn_chunk_prefill_slots(const gdn_dims* dims, gdn_dtype dtype, const void* x,
                            const void* conv_w, const float* beta, const float* g, const void* z,
                            const void* norm_w, const int32_t* cu_seqlens, int32_t num_seqs,
                            int32_t num_tokens, const int32_t* slot_idx, int32_t num_slots,
                            float* S_pool, void* conv_pool, void* out, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, void* stream) {
  if (num_seqs > 0 && !S_pool) return GDN_ERR_INVALID_ARG;
  if (num_slots < 0 || (!slot_idx && num_slots < num_seqs)) return GDN_ERR_INVALID_ARG;
  return prefill_impl(dims, dtype, x, conv_w, beta, g, z, norm_w, cu_seqlens, num_seqs,
                      num_tokens, S_pool, S_pool, conv_pool, conv_pool, out, workspace,
                      workspace_bytes, dev_status, nullptr, slot_idx, num_slots, stream);
}

}  // extern "C"

namespace {
int decode_impl(const gdn_dims* dims, gdn_dtype dtype, const void* x, const void* conv_w,
                const float* beta, const float* g, const void* z, const void* norm_w,
                void* conv_state, void* S, bool state_bf16, const int32_t* slot_idx,
                int32_t num_slots, int32_t batch, void* out, int32_t* dev_status, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!dtype_ok(dtype)) return GDN_ERR_UNSUPPORTED;
  if (batch < 0) return GDN_ERR_INVALID_ARG;
  if (num_slots < 0 || (!slot_idx && num_slots < batch)) return GDN_ERR_INVALID_ARG;
  if (batch > 0 && (!x || !conv_w || !beta || !g || !conv_state || !S || !out))
    return GDN_ERR_INVALID_ARG;
  const void* ptrs[] = {x, conv_w, beta, g, z, norm_w, conv_state, S, out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  if (dims->num_v_heads / dims->num_k_heads > 8) return GDN_ERR_UNSUPPORTED;
  gdn::DecodeArgs a{};
  a.x = x;
  a.conv_w = conv_w;
  a.beta = beta;
  a.g = g;
  a.z = z;
  a.norm_w = norm_w;
  a.conv_state = conv_state;
  a.S = S;
  a.slot_idx = slot_idx;
  a.out = out;
  a.status = dev_status;
  a.num_slots = num_slots;
  a.B = batch;
  a.Hk = dims->num_k_heads;
  a.Hv = dims->num_v_heads;
  a.q_scale = dims->q_scale;
  a.l2_eps = dims->l2_eps;
  a.norm_eps = dims->norm_eps;
  return map_cuda(gdn_host::launch_decode(dtype == GDN_BF16, state_bf16, a,
                                          static_cast<cudaStream_t>(stream)));
}
}  // namespace

extern "C" {

int gdn_decode_step(const gdn_dims* dims, gdn_dtype dtype, const void* x, const void* conv_w,
                    const float* beta, const float* g, const void* z, const void* norm_w,
                    void* conv_state, float* S, const int32_t* slot_idx, int32_t num_slots,
                    int32_t batch, void* out, int32_t* dev_status, void* stream) {
  return decode_impl(dims, dtype, x, conv_w, beta, g, z, norm_w, conv_state, S, false, slot_idx,
                     num_slots, batch, out, dev_status, stream);
}

int gdn_decode_multi(const gdn_dims* dims, gdn_dtype dtype, const void* x, const void* conv_w,
                     const float* beta, const float* g, const void* z, const void* norm_w,
                     void* conv_state, float* S, const int32_t* slot_idx, int32_t num_slots,
                     int32_t batch, int32_t tokens, void* out, float* snapshots,
                     int32_t* dev_status, void* stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!dtype_ok(dtype)) return GDN_ERR_UNSUPPORTED;
  if (batch < 0 || tokens < 0) return GDN_ERR_INVALID_ARG;
  if (num_slots < 0 || (!slot_idx && num_slots < batch)) return GDN_ERR_INVALID_ARG;
  if (tokens > 8) return GDN_ERR_UNSUPPORTED;
  if (batch > 0 && tokens > 0 && (!x || !conv_w || !beta || !g || !conv_state || !S || !out))
    return GDN_ERR_INVALID_ARG;
  const void* ptrs[] = {x, conv_w, beta, g, z, norm_w, conv_state, S, out, snapshots};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  if (dims->num_v_heads / dims->num_k_heads > 8) return GDN_ERR_UNSUPPORTED;
  gdn::DecodeArgs a{};
  a.x = x;
  a.conv_w = conv_w;
  a.beta = beta;
  a.g = g;
  a.z = z;
  a.norm_w = norm_w;
  a.conv_state = conv_state;
  a.S = S;
  a.slot_idx = slot_idx;
  a.out = out;
  a.status = dev_status;
  a.num_slots = num_slots;
  a.B = batch;
  a.Hk = dims->num_k_heads;
  a.Hv = dims->num_v_heads;
  a.q_scale = dims->q_scale;
  a.l2_eps = dims->l2_eps;
  a.norm_eps = dims->norm_eps;
  return map_cuda(gdn_host::launch_decode_multi(dtype == GDN_BF16, a, tokens, snapshots,
                                                static_cast<cudaStream_t>(stream)));
}

int gdn_decode_step_bf16_state(const gdn_dims* dims, gdn_dtype dtype, const void* x,
                               const void* conv_w, const float* beta, const float* g,
                               const void* z, const void* norm_w, void* conv_state, void* S,
                               const int32_t* slot_idx, int32_t num_slots, int32_t batch,
                               void* out, int32_t* dev_status, void* stream) {
  return decode_impl(dims, dtype, x, conv_w, beta, g, z, norm_w, conv_state, S, true, slot_idx,
                     num_slots, batch, out, dev_status, stream);
}

int gdn_trace_create(gdn_trace** out) {
  if (!out) return GDN_ERR_INVALID_ARG;
  *out = new (std::nothrow) gdn_trace();
  return *out ? GDN_OK : GDN_ERR_INVALID_ARG;
}

int gdn_trace_destroy(gdn_trace* trace) {
  if (!trace) return GDN_ERR_INVALID_ARG;
  if (gdn_host::t_trace == trace) gdn_host::t_trace = nullptr;
  for (auto& r : trace->recs) {
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
  }
  delete trace;
  return GDN_OK;
}

int gdn_trace_attach(gdn_trace* trace) {
  gdn_host::t_trace = trace;
  return GDN_OK;
}

int gdn_trace_reset(gdn_trace* trace) {
  if (!trace) return GDN_ERR_INVALID_ARG;
  trace->used = 0;
  return GDN_OK;
}

int gdn_trace_count(const gdn_trace* trace) { return trace ? trace->used : 0; }

int gdn_trace_get(gdn_trace* trace, int32_t i, const char** name, float* ms) {
  if (!trace || i < 0 || i >= trace->used) return GDN_ERR_INVALID_ARG;
  auto& r = trace->recs[i];
  if (name) *name = r.name;
  if (ms) {
    if (cudaEventSynchronize(r.stop) != cudaSuccess) return GDN_ERR_CUDA;
    if (cudaEventElapsedTime(ms, r.start, r.stop) != cudaSuccess) return GDN_ERR_CUDA;
  }
  return GDN_OK;
}

int gdn_trace_span(gdn_trace* trace, int32_t i, float* start_ms, float* end_ms) {
  if (!trace || i < 0 || i >= trace->used || !start_ms || !end_ms) return GDN_ERR_INVALID_ARG;
  auto& r0 = trace->recs[0];
  auto& r = trace->recs[i];
  if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventSynchronize(r0.stop) != cudaSuccess)
    return GDN_ERR_CUDA;
  if (cudaEventElapsedTime(start_ms, r0.start, r.start) != cudaSuccess ||
      cudaEventElapsedTime(end_ms, r0.start, r.stop) != cudaSuccess)
    return GDN_ERR_CUDA;
  return GDN_OK;
}

int gdn_debug_set(const gdn_debug_options* opts) {
  if (!opts) {
    gdn_host::t_debug = gdn_debug_options{};
    return GDN_OK;
  }
  const bool split_ok = opts->chain_split == 0 || opts->chain_split == 1 ||
                        opts->chain_split == 2 || opts->chain_split == 4;
  if (opts->wait_limit_us > 10000000u || opts->segment_chunks < 0 || !split_ok ||
      (opts->fault != GDN_FAULT_NONE && opts->fault != GDN_FAULT_SKIP_CHAIN_LOAD) ||
      opts->fault_chunk < 0)
    return GDN_ERR_INVALID_ARG;
  gdn_host::t_debug = *opts;
  return GDN_OK;
}

int gdn_debug_wait_probe(int32_t* dev_status, uint32_t limit_us, void* stream) {
  if (!dev_status || limit_us > 1000000u) return GDN_ERR_INVALID_ARG;
  gdn_host::trace_begin("wait_probe", static_cast<cudaStream_t>(stream));
  gdn::wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      dev_status, (uint64_t)limit_us * 1000ull);
  gdn_host::trace_end(static_cast<cudaStream_t>(stream));
  return map_cuda(cudaGetLastError());
}

}  // extern "C"
