// host_io.cu -- the layer with its per-token tensors in host memory.  The packed batch is cut
// into token segments; the host->device copy of a segment's inputs, the layer on the segment
// before it and the device->host copy of the output before that run at the same time on three
// streams, so the transfers over the host link overlap one another and the kernels.
//
// Source: the layer of gdn_chunk_prefill (the hyper.ai Gated DeltaNet paragraph).  Segments end
// at chunk boundaries of their sequences (multiples of 128 tokens from a sequence's start) or at
// sequence ends, and a sequence cut between two segments enters the second with the fp32 state
// and the conv history that the first one leaves, which is how the layer hands a sequence from
// one chunk to the next: the result is that of one gdn_chunk_prefill call on the whole batch.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <vector>

#include "gdn.h"

namespace gdn_host {
int check_dims_ext(const gdn_dims* d);
}

namespace {

constexpr int kChunk = 128;

struct Segment {
  int n0, nseq, t0, ntok;  // first sequence, sequences, first token, tokens
};

// Cut the batch: whole sequences while they fit, then the longest chunk-aligned part of the next
// one; a segment that cannot take 128 more tokens of the next sequence ends there.  Segments
// with no tokens (runs of empty sequences after the last token) are left out: their states are
// already in the carry buffers.
int plan_segments(const int32_t* cu, int N, int T, int seg_tokens, std::vector<Segment>* segs) {
  segs->clear();
  if (N < 0 || T < 0 || seg_tokens <= 0 || seg_tokens % kChunk != 0) return GDN_ERR_INVALID_ARG;
  if (N == 0) return T == 0 ? GDN_OK : GDN_ERR_INVALID_ARG;
  if (!cu || cu[0] != 0 || cu[N] != T) return GDN_ERR_INVALID_ARG;
  for (int n = 0; n < N; ++n)
    if (cu[n + 1] < cu[n]) return GDN_ERR_INVALID_ARG;
  int n = 0, off = 0;  // next token: sequence n at offset off (a multiple of kChunk)
  while (n < N) {
    Segment sg{n, 0, cu[n] + off, 0};
    while (n < N) {
      const int left = cu[n + 1] - cu[n] - off;
      const int room = seg_tokens - sg.ntok;
      if (left <= room) {
        sg.ntok += left;
        off = 0;
        ++n;
        if (sg.ntok == seg_tokens) break;
        continue;
      }
      const int take = room / kChunk * kChunk;
      if (take == 0) break;  // only when this segment already holds tokens
      sg.ntok += take;
      off += take;
      break;
    }
    sg.nseq = (off > 0 ? n + 1 : n) - sg.n0;
    if (sg.ntok > 0) segs->push_back(sg);
  }
  return GDN_OK;
}

int default_segment_tokens(int T) {
  const int eighth = (T / 8 + kChunk - 1) / kChunk * kChunk;
  return std::max(4 * kChunk, eighth);
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

struct HostWs {
  size_t x, beta, g, z, out, S, conv, cu, layer, layer_bytes, total;
};

HostWs host_ws(const gdn_dims* d, int N, int T, const std::vector<Segment>& segs) {
  const size_t Hv = d->num_v_heads, dh = d->head_dim;
  const size_t Cc = (size_t)(2 * d->num_k_heads + d->num_v_heads) * dh;
  HostWs w{};
  size_t o = 0;
  w.x = o;     o = align256(o + (size_t)T * Cc * 2);
  w.beta = o;  o = align256(o + (size_t)T * Hv * 4);
  w.g = o;     o = align256(o + (size_t)T * Hv * 4);
  w.z = o;     o = align256(o + (size_t)T * Hv * dh * 2);
  w.out = o;   o = align256(o + (size_t)T * Hv * dh * 2);
  w.S = o;     o = align256(o + (size_t)N * Hv * dh * dh * 4);
  w.conv = o;  o = align256(o + (size_t)N * 3 * Cc * 2);
  size_t ncu = 0, layer = 0;
  for (const Segment& sg : segs) {
    ncu += (size_t)sg.nseq + 1;
    layer = std::max(layer, gdn_chunk_prefill_workspace_size(d, GDN_BF16, sg.nseq, sg.ntok));
  }
  w.cu = o;    o = align256(o + ncu * 4);
  w.layer = o;
  w.layer_bytes = layer;
  w.total = o + layer;
  return w;
}

// Copy streams and events of this host thread on one device (created on first use).
struct IoStreams {
  bool ready = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  std::vector<cudaEvent_t> ev;
};

cudaError_t io_streams(size_t nevents, IoStreams** out) {
  constexpr int kMaxDev = 64;
  static thread_local IoStreams t_io[kMaxDev];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  IoStreams& io = t_io[dev];
  if (!io.ready) {
    if ((e = cudaStreamCreateWithFlags(&io.h2d, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithFlags(&io.d2h, cudaStreamNonBlocking)) != cudaSuccess) return e;
    io.ready = true;
  }
  while (io.ev.size() < nevents) {
    cudaEvent_t ev;
    if ((e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming)) != cudaSuccess) return e;
    io.ev.push_back(ev);
  }
  *out = &io;
  return cudaSuccess;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" {

int32_t gdn_chunk_prefill_host_plan(const int32_t* cu_seqlens_host, int32_t num_seqs,
                                    int32_t num_tokens, int32_t segment_tokens,
                                    int32_t* segments, int32_t max_segments) {
  const int seg = segment_tokens ? segment_tokens : default_segment_tokens(num_tokens);
  std::vector<Segment> segs;
  const int rc = plan_segments(cu_seqlens_host, num_seqs, num_tokens, seg, &segs);
  if (rc != GDN_OK) return rc;
  if (segments) {
    if (max_segments < (int)segs.size()) return GDN_ERR_WORKSPACE;
    for (size_t k = 0; k < segs.size(); ++k) {
      segments[4 * k + 0] = segs[k].n0;
      segments[4 * k + 1] = segs[k].nseq;
      segments[4 * k + 2] = segs[k].t0;
      segments[4 * k + 3] = segs[k].ntok;
    }
  }
  return (int32_t)segs.size();
}

size_t gdn_chunk_prefill_host_workspace_size(const gdn_dims* dims, const int32_t* cu_seqlens_host,
                                             int32_t num_seqs, int32_t num_tokens,
                                             int32_t segment_tokens) {
  if (gdn_host::check_dims_ext(dims) != GDN_OK) return 0;
  const int seg = segment_tokens ? segment_tokens : default_segment_tokens(num_tokens);
  std::vector<Segment> segs;
  if (plan_segments(cu_seqlens_host, num_seqs, num_tokens, seg, &segs) != GDN_OK) return 0;
  return host_ws(dims, num_seqs, num_tokens, segs).total;
}

int gdn_chunk_prefill_host(const gdn_dims* dims, const void* x, const void* conv_w,
                           const float* beta, const float* g, const void* z, const void* norm_w,
                           const int32_t* cu_seqlens_host, int32_t num_seqs, int32_t num_tokens,
                           const float* S0, float* SN, const void* conv0, void* convN, void* out,
                           int32_t segment_tokens, void* workspace, size_t workspace_bytes,
                           int32_t* dev_status, void* stream) {
  int rc = gdn_host::check_dims_ext(dims);
  if (rc != GDN_OK) return rc;
  if (dims->num_v_heads != 2 * dims->num_k_heads) return GDN_ERR_UNSUPPORTED;  // the bf16 layer
  // beta and g rows of a segment start at any token: 16-byte alignment needs Hv % 4 == 0
  if (dims->num_v_heads % 4 != 0) return GDN_ERR_UNSUPPORTED;
  if (num_seqs < 0 || num_tokens < 0) return GDN_ERR_INVALID_ARG;
  if (num_tokens > 0 && (!x || !beta || !g || !out)) return GDN_ERR_INVALID_ARG;
  const int seg = segment_tokens ? segment_tokens : default_segment_tokens(num_tokens);
  std::vector<Segment> segs;
  if ((rc = plan_segments(cu_seqlens_host, num_seqs, num_tokens, seg, &segs)) != GDN_OK) return rc;
  const void* dev_ptrs[] = {conv_w, norm_w, S0, SN, conv0, convN};
  for (const void* p : dev_ptrs)
    if (p && !aligned(p, 16)) return GDN_ERR_INVALID_ARG;
  if (workspace && !aligned(workspace, 256)) return GDN_ERR_INVALID_ARG;
  const HostWs l = host_ws(dims, num_seqs, num_tokens, segs);
  if (l.total > 0 && (!workspace || workspace_bytes < l.total)) return GDN_ERR_WORKSPACE;
  if (num_seqs == 0) return GDN_OK;

  const size_t Hv = dims->num_v_heads, dh = dims->head_dim;
  const size_t Cc = (size_t)(2 * dims->num_k_heads + dims->num_v_heads) * dh;
  const size_t sstride = Hv * dh * dh, cstride = 3 * Cc;  // per sequence: floats, bf16 elements
  uint8_t* w = static_cast<uint8_t*>(workspace);
  uint16_t* dx = reinterpret_cast<uint16_t*>(w + l.x);
  float* dbeta = reinterpret_cast<float*>(w + l.beta);
  float* dg = reinterpret_cast<float*>(w + l.g);
  uint16_t* dz = reinterpret_cast<uint16_t*>(w + l.z);
  uint16_t* dout = reinterpret_cast<uint16_t*>(w + l.out);
  float* dS = reinterpret_cast<float*>(w + l.S);
  uint16_t* dconv = reinterpret_cast<uint16_t*>(w + l.conv);
  int32_t* dcu = reinterpret_cast<int32_t*>(w + l.cu);
  const uint16_t* hx = static_cast<const uint16_t*>(x);
  const uint16_t* hz = static_cast<const uint16_t*>(z);
  uint16_t* hout = static_cast<uint16_t*>(out);

  // each segment's cu_seqlens, relative to its first token
  std::vector<int32_t> cu_all;
  std::vector<size_t> cu_off;
  for (const Segment& sg : segs) {
    cu_off.push_back(cu_all.size());
    cu_all.push_back(0);
    for (int i = 0; i < sg.nseq; ++i) {
      const int n = sg.n0 + i;
      const int end = std::min(cu_seqlens_host[n + 1], sg.t0 + sg.ntok);
      cu_all.push_back(end - sg.t0);
    }
  }

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  IoStreams* io = nullptr;
  cudaError_t e = io_streams(2 * segs.size() + 2, &io);
  if (e != cudaSuccess) return GDN_ERR_CUDA;
  cudaEvent_t ev_start = io->ev[0], ev_end = io->ev[1];
  // After a failure with copies already queued, `stream` still joins both copy streams, so that
  // work the caller queues on it afterwards (freeing or reusing the host buffers) waits for
  // every copy in flight (best effort: a failing runtime may refuse these calls as well).
  auto fail = [&](int code) {
    if (cudaEventRecord(ev_start, io->h2d) == cudaSuccess) cudaStreamWaitEvent(s, ev_start, 0);
    if (cudaEventRecord(ev_end, io->d2h) == cudaSuccess) cudaStreamWaitEvent(s, ev_end, 0);
    return code;
  };
#define GDN_TRY(call)                          \
  do {                                         \
    if ((e = (call)) != cudaSuccess) return fail(GDN_ERR_CUDA); \
  } while (0)
  // copies start after the caller's earlier work on `stream` (it may still use this workspace)
  GDN_TRY(cudaEventRecord(ev_start, s));
  GDN_TRY(cudaStreamWaitEvent(io->h2d, ev_start, 0));
  GDN_TRY(cudaStreamWaitEvent(io->d2h, ev_start, 0));
  // carry buffers: the initial states
  if (S0)
    GDN_TRY(cudaMemcpyAsync(dS, S0, num_seqs * sstride * 4, cudaMemcpyDeviceToDevice, s));
  else
    GDN_TRY(cudaMemsetAsync(dS, 0, num_seqs * sstride * 4, s));
  if (conv0)
    GDN_TRY(cudaMemcpyAsync(dconv, conv0, num_seqs * cstride * 2, cudaMemcpyDeviceToDevice, s));
  else
    GDN_TRY(cudaMemsetAsync(dconv, 0, num_seqs * cstride * 2, s));
  if (!cu_all.empty())  // pageable source: staged by the runtime before the call returns
    GDN_TRY(cudaMemcpyAsync(dcu, cu_all.data(), cu_all.size() * 4, cudaMemcpyHostToDevice,
                            io->h2d));
  for (size_t k = 0; k < segs.size(); ++k) {
    const Segment& sg = segs[k];
    const size_t t0 = sg.t0, nt = sg.ntok;
    cudaEvent_t ev_in = io->ev[2 + 2 * k], ev_done = io->ev[3 + 2 * k];
    GDN_TRY(cudaMemcpyAsync(dx + t0 * Cc, hx + t0 * Cc, nt * Cc * 2, cudaMemcpyHostToDevice,
                            io->h2d));
    GDN_TRY(cudaMemcpyAsync(dbeta + t0 * Hv, beta + t0 * Hv, nt * Hv * 4, cudaMemcpyHostToDevice,
                            io->h2d));
    GDN_TRY(cudaMemcpyAsync(dg + t0 * Hv, g + t0 * Hv, nt * Hv * 4, cudaMemcpyHostToDevice,
                            io->h2d));
    if (hz)
      GDN_TRY(cudaMemcpyAsync(dz + t0 * Hv * dh, hz + t0 * Hv * dh, nt * Hv * dh * 2,
                              cudaMemcpyHostToDevice, io->h2d));
    GDN_TRY(cudaEventRecord(ev_in, io->h2d));
    GDN_TRY(cudaStreamWaitEvent(s, ev_in, 0));
    rc = gdn_chunk_prefill(dims, GDN_BF16, dx + t0 * Cc, conv_w, dbeta + t0 * Hv, dg + t0 * Hv,
                           hz ? dz + t0 * Hv * dh : nullptr, norm_w, dcu + cu_off[k], sg.nseq,
                           sg.ntok, dS + sg.n0 * sstride, dS + sg.n0 * sstride,
                           dconv + sg.n0 * cstride, dconv + sg.n0 * cstride, dout + t0 * Hv * dh,
                           w + l.layer, l.layer_bytes, dev_status, s);
    if (rc != GDN_OK) return fail(rc);
    GDN_TRY(cudaEventRecord(ev_done, s));
    GDN_TRY(cudaStreamWaitEvent(io->d2h, ev_done, 0));
    GDN_TRY(cudaMemcpyAsync(hout + t0 * Hv * dh, dout + t0 * Hv * dh, nt * Hv * dh * 2,
                            cudaMemcpyDeviceToHost, io->d2h));
  }
  if (SN)
    GDN_TRY(cudaMemcpyAsync(SN, dS, num_seqs * sstride * 4, cudaMemcpyDeviceToDevice, s));
  if (convN)
    GDN_TRY(cudaMemcpyAsync(convN, dconv, num_seqs * cstride * 2, cudaMemcpyDeviceToDevice, s));
  // the caller's stream completes with the last output copy
  GDN_TRY(cudaEventRecord(ev_end, io->d2h));
  GDN_TRY(cudaStreamWaitEvent(s, ev_end, 0));
#undef GDN_TRY
  return GDN_OK;
}

}  // extern "C"
