// Forward entry points of the C ABI (include/archead.h): argument checks,
// workspace carving, and one of two launch sequences on the caller's stream,
// with no host synchronisation:
//   T < kTcMinTokens (9; any T when g_B is not a multiple of 64):
//     prologue (z_c, z_r, E_t)  ->  decode launches of <= 8 tokens each
//   otherwise:
//     activation operand [h | z_c | z_r]  ->  tensor-core pass  ->  per-token fold
// Vocabulary shards (archead_set_vocab_shard) only shift row ids: the same
// sequences run, and archead_shard_partials / archead_merge_shards carry the
// per-token statistics across shards.
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <new>

#include "device.cuh"
#include "handle.h"

namespace archead {

namespace {
thread_local int g_last_cuda_error = 0;

constexpr int kMaxTokens = 1 << 20;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_device(const archead_handle* h) {
  int dev = -1;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_cuda_error(e);
  return dev == h->device ? ARCHEAD_OK : ARCHEAD_EINVAL;
}

// Tensor-core path: activation operand, the tensor-core kernel, and the
// per-token fold of its partials.
int forward_tc(const archead_handle* h, const uint16_t* hidden, int32_t T, const int32_t* targets, float* logits,
               int32_t* argmax, float* lse, float* ce, float4* shard_out, uint8_t* wb, const WsLayout& w,
               cudaStream_t stream) {
  const Layout& L = h->L;
  const int Kc = tc_kc(L);
  uint32_t* status = reinterpret_cast<uint32_t*>(wb + w.status);
  float* cinv = reinterpret_cast<float*>(wb + w.cinv);
  uint16_t* xop = reinterpret_cast<uint16_t*>(wb + w.xop);
  float4* partials = reinterpret_cast<float4*>(wb + w.tpartials);
  float* tgt = reinterpret_cast<float*>(wb + w.tgt);

  ActParams ap{};
  ap.hidden = hidden;
  ap.R = reinterpret_cast<const int8_t*>(h->arena + L.off_R);
  ap.s_R = reinterpret_cast<const uint16_t*>(h->arena + L.off_sR);
  ap.B = reinterpret_cast<const int8_t*>(h->arena + L.off_B);
  ap.s_B = reinterpret_cast<const uint16_t*>(h->arena + L.off_sB);
  ap.targets = targets;
  ap.status = status;
  ap.xop = xop;
  ap.cinv = cinv;
  ap.T = T;
  ap.d = L.d;
  ap.rcp = L.rcp;
  ap.Kz = L.Kz;
  ap.Kc = Kc;
  ap.g_B = L.g_B;
  ap.V = L.V;
  ap.v_total = h->v_total;
  ap.alpha = h->tc_alpha;
  ap.beta = h->tc_beta;
  ap.gamma = h->tc_gamma;
  ap.mseg = h->tc_mseg;
  // The K-split partials borrow the region of the tensor-core partials: the
  // tensor-core kernel writes there only after this grid has completed.
  const size_t part_bytes = static_cast<size_t>(T) * tc_n_mt128(L) * 16;
  const int splits = act_prep_splits(T, L.d, Kc, h->num_sms, part_bytes);
  ap.zpart = reinterpret_cast<float*>(wb + w.tpartials);
  ap.zticket = reinterpret_cast<uint32_t*>(wb + kActTicketOff);
  cudaError_t e = launch_act_prep(ap, splits, stream);
  if (e != cudaSuccess) return set_cuda_error(e);

  TcParams tp{};
  tp.mtiles = h->arena;
  tp.targets = targets;
  tp.cinv = cinv;
  tp.logits = logits;
  tp.partials = partials;
  tp.tgt = tgt;
  tp.status = status;
  tp.T = T;
  tp.V = L.V;
  tp.row0 = h->row0;
  tp.n_nt = (T + kTcMaxBN - 1) / kTcMaxBN;
  const int per = (T + tp.n_nt - 1) / tp.n_nt;
  tp.BN = (per + 15) / 16 * 16;
  tp.n_mt128 = tc_n_mt128(L);
  tp.n_units = tp.n_mt128 * tp.n_nt;
  tp.n_res = L.n_res;
  tp.n_L = L.n_L;
  tp.n_A = L.n_A;
  tp.n_mtiles = L.n_mtiles;
  int lg = 0;
  while ((1 << lg) < L.g) ++lg;
  tp.g_log2 = lg;
  tp.ks_core = L.n_res;
  tp.ks_corr = L.n_res + L.n_L;
  tp.n_ks = Kc / kTcBK;
  tp.n_st = (tp.n_ks + kTcStepsPerStage - 1) / kTcStepsPerStage;
  tp.off_res = L.off_res;
  tp.off_Lnib = L.off_Lnib;
  tp.off_Lhi = L.off_Lhi;
  tp.off_A = L.off_A;
  tp.off_sres = L.off_sres;
  tp.off_sL = L.off_sL;
  tp.off_sA = L.off_sA;
  tp.mblk_bytes = L.mblk_bytes;
  tp.sc_res = std::ldexp(1.f, h->tc_alpha);
  tp.sc_L = std::ldexp(1.f, h->tc_beta);
  tp.sc_A = std::ldexp(1.f, h->tc_gamma);
  tc_smem_plan(tp);
  CUtensorMap map;
  e = tc_encode_xmap(&map, xop, T, Kc, tp.BN);
  if (e != cudaSuccess) return set_cuda_error(e);
  const int grid = tp.n_units < h->num_sms ? tp.n_units : h->num_sms;
  if (h->ev_before != nullptr) {
    e = cudaEventRecord(h->ev_before, stream);
    if (e != cudaSuccess) return set_cuda_error(e);
  }
  e = launch_tc(tp, map, grid, stream);
  if (e != cudaSuccess) return set_cuda_error(e);
  if (h->ev_after != nullptr) {
    e = cudaEventRecord(h->ev_after, stream);
    if (e != cudaSuccess) return set_cuda_error(e);
  }
  if (argmax != nullptr || lse != nullptr || ce != nullptr || shard_out != nullptr) {
    e = launch_tc_merge(partials, tp.n_mt128, T, targets, tgt, L.V, h->row0, lse, argmax, ce, shard_out, stream);
    if (e != cudaSuccess) return set_cuda_error(e);
  }
  return ARCHEAD_OK;
}

// Sampling request of one call (decode kernel only).
struct SampleArgs {
  int32_t* sampled;
  float inv_temp;
  uint64_t seed, offset;
};

int forward(const archead_handle* h, const uint16_t* hidden, int32_t T, const int32_t* targets, float* logits,
            int32_t* argmax, float* lse, float* ce, void* ws, size_t ws_bytes, cudaStream_t stream,
            float4* shard_out = nullptr, const SampleArgs* sample = nullptr) {
  if (h == nullptr || hidden == nullptr || ws == nullptr) return ARCHEAD_EINVAL;
  if (T <= 0 || T > kMaxTokens) return ARCHEAD_EINVAL;
  if (logits == nullptr && argmax == nullptr && lse == nullptr && shard_out == nullptr && sample == nullptr)
    return ARCHEAD_EINVAL;
  if (ce != nullptr && targets == nullptr) return ARCHEAD_EINVAL;
  if (!aligned(hidden, 16) || !aligned(ws, 256)) return ARCHEAD_EALIGN;
  if (!aligned(logits, 4) || !aligned(argmax, 4) || !aligned(lse, 4) || !aligned(ce, 4) || !aligned(targets, 4))
    return ARCHEAD_EALIGN;
  const WsLayout w = ws_layout(*h, T);
  if (ws_bytes < w.total) return ARCHEAD_ENOMEM;
  const int dc = check_device(h);
  if (dc != ARCHEAD_OK) return dc;

  uint8_t* wb = static_cast<uint8_t*>(ws);
  if (sample == nullptr && use_tc(*h, T))
    return forward_tc(h, hidden, T, targets, logits, argmax, lse, ce, shard_out, wb, w, stream);
  const Layout& L = h->L;
  uint32_t* counter = reinterpret_cast<uint32_t*>(wb + w.counter);
  uint32_t* status = reinterpret_cast<uint32_t*>(wb + w.status);
  int32_t* escale = reinterpret_cast<int32_t*>(wb + w.escale);
  uint16_t* zhi = reinterpret_cast<uint16_t*>(wb + w.zhi);
  uint16_t* zlo = reinterpret_cast<uint16_t*>(wb + w.zlo);

  PrologueParams pp{};
  pp.hidden = hidden;
  pp.R = reinterpret_cast<const int8_t*>(h->arena + L.off_R);
  pp.s_R = reinterpret_cast<const uint16_t*>(h->arena + L.off_sR);
  pp.B = reinterpret_cast<const int8_t*>(h->arena + L.off_B);
  pp.s_B = reinterpret_cast<const uint16_t*>(h->arena + L.off_sB);
  pp.targets = targets;
  pp.zhi = zhi;
  pp.zlo = zlo;
  pp.escale = escale;
  pp.counter = counter;
  pp.status = status;
  pp.e_B = h->e_B;
  pp.T = T;
  pp.d = L.d;
  pp.rcp = L.rcp;
  pp.rrp = L.rrp;
  pp.Kz = L.Kz;
  pp.g_B = L.g_B;
  pp.V = L.V;
  pp.v_total = h->v_total;
  cudaError_t e = launch_prologue(pp, stream);
  if (e != cudaSuccess) return set_cuda_error(e);

  DecodeParams dp{};
  dp.mtiles = h->arena;
  dp.hidden = hidden;
  dp.zhi = zhi;
  dp.zlo = zlo;
  dp.escale = escale;
  dp.targets = targets;
  dp.logits = logits;
  dp.argmax = argmax;
  dp.lse = lse;
  dp.ce = ce;
  dp.partials = reinterpret_cast<float4*>(wb + w.partials);
  dp.tgt = reinterpret_cast<float*>(wb + w.tgt);
  dp.counter = counter;
  dp.status = status;
  dp.T = T;
  dp.V = L.V;
  dp.row0 = h->row0;
  dp.shard_out = shard_out;
  if (sample != nullptr) {
    dp.sampled = sample->sampled;
    dp.spart = reinterpret_cast<float2*>(wb + w.spart);
    dp.inv_temp = sample->inv_temp;
    dp.seed = sample->seed;
    dp.ctr0 = sample->offset;
  }
  dp.d = L.d;
  dp.Kz = L.Kz;
  dp.rcp = L.rcp;
  dp.e_B = h->e_B;
  dp.n_res = L.n_res;
  dp.n_L = L.n_L;
  dp.n_A = L.n_A;
  dp.n_mtiles = L.n_mtiles;
  int lg = 0;
  while ((1 << lg) < L.g_steps) ++lg;
  dp.g_steps_log2 = lg;
  dp.off_res = L.off_res;
  dp.off_Lnib = L.off_Lnib;
  dp.off_Lhi = L.off_Lhi;
  dp.off_A = L.off_A;
  dp.off_sres = L.off_sres;
  dp.off_sL = L.off_sL;
  dp.off_sA = L.off_sA;
  dp.mblk_bytes = L.mblk_bytes;
  dp.nw_res = h->nw_res;
  dp.nw_L = h->nw_L;
  dp.nw_A = h->nw_A;
  dp.nw_work = h->nw_work;
  dp.wait_limit_ns = h->wait_limit_ns;
  dp.test_stall = h->test_stall;
  if (h->ev_before != nullptr) {
    e = cudaEventRecord(h->ev_before, stream);
    if (e != cudaSuccess) return set_cuda_error(e);
  }
  for (int t0 = 0; t0 < T; t0 += kDecodeTokens) {
    dp.t0 = t0;
    dp.nt = (T - t0 < kDecodeTokens) ? (T - t0) : kDecodeTokens;
    // Partial logits move in groups of mg m-tiles with mg * nt <= 8; four slots.
    dp.mg_log2 = dp.nt <= 1 ? 3 : dp.nt <= 2 ? 2 : dp.nt <= 4 ? 1 : 0;
    dp.mg = 1 << dp.mg_log2;
    dp.slots = 4;
    dp.slots_log2 = 2;
    decode_smem_plan(dp, L.g_steps);
    e = launch_decode(L.g_steps, dp, h->grid, decode_smem_bytes(dp), stream);
    if (e != cudaSuccess) return set_cuda_error(e);
  }
  if (h->ev_after != nullptr) {
    e = cudaEventRecord(h->ev_after, stream);
    if (e != cudaSuccess) return set_cuda_error(e);
  }
  return ARCHEAD_OK;
}

}  // namespace

int set_cuda_error(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  return ARCHEAD_ECUDA;
}

// ---------------------------------------------------- host-buffer sequences
// A host-buffer call is a fixed sequence (copies in, the forward launches,
// copies out).  When every host buffer is pinned, the sequence is captured
// once per distinct argument set on a private stream and replayed with one
// graph launch on the caller's stream: one driver call instead of five to
// seven, so the GPU runs the steps back to back.  Any capture failure falls
// back to the direct sequence (and is remembered for that argument set).
struct HostGraphKey {
  int kind, T;
  const void* in[2];
  void* out[3];
  void* ws;
  size_t ws_bytes;
  bool operator==(const HostGraphKey& o) const { return std::memcmp(this, &o, sizeof(*this)) == 0; }
};

struct HostGraphCache {
  static constexpr int kEntries = 4;
  std::mutex mu;
  cudaStream_t cap = nullptr;   // capture stream (non-blocking), created on first use
  struct Entry {
    bool used = false, failed = false;
    HostGraphKey key{};
    cudaGraphExec_t exec = nullptr;
  } e[kEntries];
  int next = 0;
};

HostGraphCache* host_graph_cache_new() { return new (std::nothrow) HostGraphCache(); }

void host_graph_cache_free(HostGraphCache* c) {
  if (c == nullptr) return;
  for (auto& en : c->e)
    if (en.exec != nullptr) cudaGraphExecDestroy(en.exec);
  if (c->cap != nullptr) cudaStreamDestroy(c->cap);
  delete c;
}

namespace {

bool pinned(const void* p) {
  if (p == nullptr) return true;
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

// The device address of a pinned host buffer, or null: the kernels write such
// an output straight into host memory (no copy after them).
template <class P>
P* mapped(P* p) {
  if (p == nullptr) return nullptr;
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return a.type == cudaMemoryTypeHost ? static_cast<P*>(a.devicePointer) : nullptr;
}

// Runs `enqueue` through the cache: a replay, or a capture then a replay.
// Returns ARCHEAD_OK with the sequence launched on `s`, kNoGraph when the
// caller should run the direct sequence, or an error.
constexpr int kNoGraph = 1;
template <class F>
int via_graph(const archead_handle* h, const HostGraphKey& key, cudaStream_t s, F enqueue) {
  HostGraphCache* c = h->graphs;
  if (c == nullptr || h->ev_before != nullptr) return kNoGraph;   // profiling events are per call
  std::lock_guard<std::mutex> lock(c->mu);
  for (auto& en : c->e) {
    if (en.used && en.key == key) {
      if (en.failed) return kNoGraph;
      const cudaError_t e = cudaGraphLaunch(en.exec, s);
      return e == cudaSuccess ? ARCHEAD_OK : set_cuda_error(e);
    }
  }
  HostGraphCache::Entry& en = c->e[c->next];
  c->next = (c->next + 1) % HostGraphCache::kEntries;
  if (en.exec != nullptr) cudaGraphExecDestroy(en.exec);
  en = HostGraphCache::Entry{};
  en.used = true;
  en.key = key;
  en.failed = true;
  if (c->cap == nullptr && cudaStreamCreateWithFlags(&c->cap, cudaStreamNonBlocking) != cudaSuccess) {
    c->cap = nullptr;
    cudaGetLastError();
    return kNoGraph;
  }
  cudaGraph_t g = nullptr;
  if (cudaStreamBeginCapture(c->cap, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    cudaGetLastError();
    return kNoGraph;
  }
  const int rc = enqueue(c->cap);
  const cudaError_t ee = cudaStreamEndCapture(c->cap, &g);
  cudaGetLastError();   // a capture that failed leaves no sticky error; clear the record
  if (rc == ARCHEAD_OK && ee == cudaSuccess && g != nullptr &&
      cudaGraphInstantiate(&en.exec, g, 0) == cudaSuccess) {
    en.failed = false;
  } else {
    en.exec = nullptr;
    cudaGetLastError();
  }
  if (g != nullptr) cudaGraphDestroy(g);
  if (en.failed) return kNoGraph;
  const cudaError_t e = cudaGraphLaunch(en.exec, s);
  return e == cudaSuccess ? ARCHEAD_OK : set_cuda_error(e);
}

}  // namespace

}  // namespace archead

using namespace archead;

extern "C" ARCHEAD_API int archead_forward_kernel(const archead_handle* handle, int32_t T) {
  if (handle == nullptr || T <= 0 || T > kMaxTokens) return -1;
  return use_tc(*handle, T) ? ARCHEAD_KERNEL_TENSOR_CORE : ARCHEAD_KERNEL_DECODE;
}

extern "C" ARCHEAD_API size_t archead_workspace_bytes(const archead_handle* handle, int32_t T) {
  if (handle == nullptr || T <= 0 || T > kMaxTokens) return 0;
  return ws_layout(*handle, T).total;
}

extern "C" ARCHEAD_API size_t archead_host_workspace_bytes(const archead_handle* handle, int32_t T) {
  if (handle == nullptr || T <= 0 || T > kMaxTokens) return 0;
  return ws_layout(*handle, T).host_total;
}

extern "C" ARCHEAD_API int archead_logits(const archead_handle* handle, const uint16_t* hidden, int32_t T,
                                          float* logits, int32_t* argmax, void* workspace, size_t workspace_bytes,
                                          archead_stream_t stream) {
  if (logits == nullptr && argmax == nullptr) return ARCHEAD_EINVAL;
  return forward(handle, hidden, T, nullptr, logits, argmax, nullptr, nullptr, workspace, workspace_bytes,
                 reinterpret_cast<cudaStream_t>(stream));
}

extern "C" ARCHEAD_API int archead_logits_lse_argmax(const archead_handle* handle, const uint16_t* hidden,
                                                     int32_t T, const int32_t* targets, float* lse,
                                                     int32_t* argmax, float* ce, void* workspace,
                                                     size_t workspace_bytes, archead_stream_t stream) {
  if (lse == nullptr || argmax == nullptr) return ARCHEAD_EINVAL;
  return forward(handle, hidden, T, targets, nullptr, argmax, lse, ce, workspace, workspace_bytes,
                 reinterpret_cast<cudaStream_t>(stream));
}

extern "C" ARCHEAD_API int archead_lse_argmax_host(const archead_handle* handle, const uint16_t* hidden_host,
                                                   int32_t T, const int32_t* targets_host, float* lse_host,
                                                   int32_t* argmax_host, float* ce_host, void* workspace,
                                                   size_t workspace_bytes, archead_stream_t stream) {
  if (handle == nullptr || hidden_host == nullptr || lse_host == nullptr || argmax_host == nullptr ||
      workspace == nullptr)
    return ARCHEAD_EINVAL;
  if (T <= 0 || T > kMaxTokens) return ARCHEAD_EINVAL;
  if (ce_host != nullptr && targets_host == nullptr) return ARCHEAD_EINVAL;
  if (!aligned(workspace, 256)) return ARCHEAD_EALIGN;
  const WsLayout w = ws_layout(*handle, T);
  if (workspace_bytes < w.host_total) return ARCHEAD_ENOMEM;
  const int dc = check_device(handle);
  if (dc != ARCHEAD_OK) return dc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* wb = static_cast<uint8_t*>(workspace);
  uint16_t* d_hidden = reinterpret_cast<uint16_t*>(wb + w.h_hidden);
  int32_t* d_targets = targets_host ? reinterpret_cast<int32_t*>(wb + w.h_targets) : nullptr;
  // Per-token outputs in pinned host memory are written there by the kernels
  // (no copies after them); the others go through the workspace and a copy.
  float* m_lse = mapped(lse_host);
  int32_t* m_argmax = mapped(argmax_host);
  float* m_ce = mapped(ce_host);
  float* d_lse = m_lse ? m_lse : reinterpret_cast<float*>(wb + w.h_lse);
  int32_t* d_argmax = m_argmax ? m_argmax : reinterpret_cast<int32_t*>(wb + w.h_argmax);
  float* d_ce = !ce_host ? nullptr : m_ce ? m_ce : reinterpret_cast<float*>(wb + w.h_ce);
  const size_t t = static_cast<size_t>(T);
  auto enqueue = [&](cudaStream_t q) -> int {
    cudaError_t e = cudaMemcpyAsync(d_hidden, hidden_host, t * handle->L.d * 2, cudaMemcpyHostToDevice, q);
    if (e == cudaSuccess && d_targets) e = cudaMemcpyAsync(d_targets, targets_host, t * 4, cudaMemcpyHostToDevice, q);
    if (e != cudaSuccess) return set_cuda_error(e);
    const int rc = forward(handle, d_hidden, T, d_targets, nullptr, d_argmax, d_lse, d_ce, workspace, w.total, q);
    if (rc != ARCHEAD_OK) return rc;
    if (!m_lse) e = cudaMemcpyAsync(lse_host, d_lse, t * 4, cudaMemcpyDeviceToHost, q);
    if (e == cudaSuccess && !m_argmax) e = cudaMemcpyAsync(argmax_host, d_argmax, t * 4, cudaMemcpyDeviceToHost, q);
    if (e == cudaSuccess && ce_host && !m_ce) e = cudaMemcpyAsync(ce_host, d_ce, t * 4, cudaMemcpyDeviceToHost, q);
    return e == cudaSuccess ? ARCHEAD_OK : set_cuda_error(e);
  };
  int rc = kNoGraph;
  if (pinned(hidden_host) && pinned(targets_host) && pinned(lse_host) && pinned(argmax_host) && pinned(ce_host)) {
    const HostGraphKey key{0, T, {hidden_host, targets_host}, {lse_host, argmax_host, ce_host}, workspace,
                           workspace_bytes};
    rc = via_graph(handle, key, s, enqueue);
  }
  if (rc == kNoGraph) rc = enqueue(s);
  if (rc != ARCHEAD_OK) return rc;
  const cudaError_t e = cudaStreamSynchronize(s);
  return e == cudaSuccess ? ARCHEAD_OK : set_cuda_error(e);
}

extern "C" ARCHEAD_API size_t archead_host_logits_workspace_bytes(const archead_handle* handle, int32_t T) {
  if (handle == nullptr || T <= 0 || T > kMaxTokens) return 0;
  return ws_layout(*handle, T).host_logits_total;
}

extern "C" ARCHEAD_API int archead_logits_host(const archead_handle* handle, const uint16_t* hidden_host, int32_t T,
                                               float* logits_host, int32_t* argmax_host, void* workspace,
                                               size_t workspace_bytes, archead_stream_t stream) {
  if (handle == nullptr || hidden_host == nullptr || workspace == nullptr) return ARCHEAD_EINVAL;
  if (logits_host == nullptr && argmax_host == nullptr) return ARCHEAD_EINVAL;
  if (T <= 0 || T > kMaxTokens) return ARCHEAD_EINVAL;
  if (!aligned(workspace, 256)) return ARCHEAD_EALIGN;
  const WsLayout w = ws_layout(*handle, T);
  if (workspace_bytes < w.host_logits_total) return ARCHEAD_ENOMEM;
  const int dc = check_device(handle);
  if (dc != ARCHEAD_OK) return dc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* wb = static_cast<uint8_t*>(workspace);
  uint16_t* d_hidden = reinterpret_cast<uint16_t*>(wb + w.h_hidden);
  // Outputs in pinned host memory are written there by the kernels (the
  // logits stream over the host link while the head streams from HBM); the
  // others go through the workspace and a copy.
  float* m_logits = mapped(logits_host);
  int32_t* m_argmax = mapped(argmax_host);
  float* d_logits = !logits_host ? nullptr : m_logits ? m_logits : reinterpret_cast<float*>(wb + w.h_logits);
  int32_t* d_argmax = !argmax_host ? nullptr : m_argmax ? m_argmax : reinterpret_cast<int32_t*>(wb + w.h_argmax);
  const size_t t = static_cast<size_t>(T);
  auto enqueue = [&](cudaStream_t q) -> int {
    cudaError_t e = cudaMemcpyAsync(d_hidden, hidden_host, t * handle->L.d * 2, cudaMemcpyHostToDevice, q);
    if (e != cudaSuccess) return set_cuda_error(e);
    const int rc = forward(handle, d_hidden, T, nullptr, d_logits, d_argmax, nullptr, nullptr, workspace, w.total, q);
    if (rc != ARCHEAD_OK) return rc;
    if (logits_host && !m_logits)
      e = cudaMemcpyAsync(logits_host, d_logits, t * handle->L.V * 4, cudaMemcpyDeviceToHost, q);
    if (e == cudaSuccess && argmax_host && !m_argmax)
      e = cudaMemcpyAsync(argmax_host, d_argmax, t * 4, cudaMemcpyDeviceToHost, q);
    return e == cudaSuccess ? ARCHEAD_OK : set_cuda_error(e);
  };
  int rc = kNoGraph;
  if (pinned(hidden_host) && pinned(logits_host) && pinned(argmax_host)) {
    const HostGraphKey key{1, T, {hidden_host, nullptr}, {logits_host, argmax_host, nullptr}, workspace,
                           workspace_bytes};
    rc = via_graph(handle, key, s, enqueue);
  }
  if (rc == kNoGraph) rc = enqueue(s);
  if (rc != ARCHEAD_OK) return rc;
  const cudaError_t e = cudaStreamSynchronize(s);
  return e == cudaSuccess ? ARCHEAD_OK : set_cuda_error(e);
}

extern "C" ARCHEAD_API int archead_sample(const archead_handle* handle, const uint16_t* hidden, int32_t T,
                                          float temperature, uint64_t seed, uint64_t offset, int32_t* sampled,
                                          float* lse, int32_t* argmax, void* workspace, size_t workspace_bytes,
                                          archead_stream_t stream) {
  if (sampled == nullptr || !(temperature > 0.f) || !(temperature < INFINITY)) return ARCHEAD_EINVAL;
  if (!aligned(sampled, 4)) return ARCHEAD_EALIGN;
  const SampleArgs sa{sampled, 1.f / temperature, seed, offset};
  return forward(handle, hidden, T, nullptr, nullptr, argmax, lse, nullptr, workspace, workspace_bytes,
                 reinterpret_cast<cudaStream_t>(stream), nullptr, &sa);
}

namespace archead {

// Sampling across vocabulary shards.  The decode kernel leaves each block's
// pick in the workspace (spart [T][grid]: the largest y / tau + G of the
// block's rows, its global row); one warp per token folds them into this
// shard's pair.  First maximum: pick_merge keeps the lower row on ties.
__global__ void sample_partials_kernel(const float2* __restrict__ spart, int grid, int T, float2* __restrict__ out) {
  const int t = static_cast<int>(blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32), lane = threadIdx.x & 31;
  if (t >= T) return;
  PickState b = pick_init();
  for (int k = lane; k < grid; k += 32) {
    const float2 q = spart[static_cast<size_t>(t) * grid + k];
    b = pick_merge(b, PickState{q.x, __float_as_int(q.y)});
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) b = pick_merge(b, pick_shfl_xor(b, o));
  if (lane == 0) out[t] = make_float2(b.z, __int_as_float(b.idx));
}

// Per token, the first maximum over n shards' pairs stacked in increasing row
// order: the pick over all rows.
__global__ void merge_sample_shards_kernel(const float2* __restrict__ parts, int n, int T,
                                           int32_t* __restrict__ sampled) {
  const int t = static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x);
  if (t >= T) return;
  PickState b = pick_init();
  for (int r = 0; r < n; ++r) {
    const float2 q = parts[static_cast<size_t>(r) * T + t];
    b = pick_merge(b, PickState{q.x, __float_as_int(q.y)});
  }
  sampled[t] = b.idx;
}

}  // namespace archead

extern "C" ARCHEAD_API int archead_sample_partials(const archead_handle* handle, const uint16_t* hidden,
                                                   int32_t T, float temperature, uint64_t seed, uint64_t offset,
                                                   float* sample_partials, void* workspace, size_t workspace_bytes,
                                                   archead_stream_t stream) {
  if (handle == nullptr || sample_partials == nullptr || !(temperature > 0.f) || !(temperature < INFINITY))
    return ARCHEAD_EINVAL;
  if (!aligned(sample_partials, 8)) return ARCHEAD_EALIGN;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The kernel's own picks land in the first half of the output buffer, which
  // the fold below then overwrites with the (value, row) pairs.
  const SampleArgs sa{reinterpret_cast<int32_t*>(sample_partials), 1.f / temperature, seed, offset};
  const int rc = forward(handle, hidden, T, nullptr, nullptr, nullptr, nullptr, nullptr, workspace, workspace_bytes,
                         s, nullptr, &sa);
  if (rc != ARCHEAD_OK) return rc;
  const WsLayout w = ws_layout(*handle, T);
  archead::sample_partials_kernel<<<(T + 7) / 8, 256, 0, s>>>(
      reinterpret_cast<const float2*>(static_cast<const uint8_t*>(workspace) + w.spart), handle->grid, T,
      reinterpret_cast<float2*>(sample_partials));
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ARCHEAD_OK : set_cuda_error(e);
}

extern "C" ARCHEAD_API int archead_merge_sample_shards(const float* sample_partials, int32_t n_shards, int32_t T,
                                                       int32_t* sampled, archead_stream_t stream) {
  if (sample_partials == nullptr || sampled == nullptr || n_shards <= 0 || T <= 0 || T > kMaxTokens)
    return ARCHEAD_EINVAL;
  if (!aligned(sample_partials, 8) || !aligned(sampled, 4)) return ARCHEAD_EALIGN;
  archead::merge_sample_shards_kernel<<<(T + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const float2*>(sample_partials), n_shards, T, sampled);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ARCHEAD_OK : set_cuda_error(e);
}

extern "C" ARCHEAD_API int archead_set_vocab_shard(archead_handle* handle, int32_t row_offset, int32_t vocab_total) {
  if (handle == nullptr || row_offset < 0 || vocab_total <= 0) return ARCHEAD_EINVAL;
  if (row_offset % 16 != 0) return ARCHEAD_EINVAL;   // shards start on m-tile (16-row) boundaries
  if (static_cast<int64_t>(row_offset) + handle->L.V > vocab_total) return ARCHEAD_EINVAL;
  handle->row0 = row_offset;
  handle->v_total = vocab_total;
  return ARCHEAD_OK;
}

extern "C" ARCHEAD_API int archead_shard_partials(const archead_handle* handle, const uint16_t* hidden, int32_t T,
                                                  const int32_t* targets, float* partials, void* workspace,
                                                  size_t workspace_bytes, archead_stream_t stream) {
  if (partials == nullptr) return ARCHEAD_EINVAL;
  if (!aligned(partials, 16)) return ARCHEAD_EALIGN;
  return forward(handle, hidden, T, targets, nullptr, nullptr, nullptr, nullptr, workspace, workspace_bytes,
                 reinterpret_cast<cudaStream_t>(stream), reinterpret_cast<float4*>(partials));
}

extern "C" ARCHEAD_API int archead_merge_shards(const float* partials, int32_t n_shards, int32_t T, float* lse,
                                                int32_t* argmax, float* ce, archead_stream_t stream) {
  if (partials == nullptr || n_shards <= 0 || T <= 0 || T > kMaxTokens) return ARCHEAD_EINVAL;
  if (lse == nullptr && argmax == nullptr && ce == nullptr) return ARCHEAD_EINVAL;
  if (!aligned(partials, 16) || !aligned(lse, 4) || !aligned(argmax, 4) || !aligned(ce, 4)) return ARCHEAD_EALIGN;
  const cudaError_t e = launch_shard_merge(reinterpret_cast<const float4*>(partials), n_shards, T, lse, argmax, ce,
                                           reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ARCHEAD_OK : set_cuda_error(e);
}

extern "C" ARCHEAD_API int archead_workspace_status(void* workspace, int clear, archead_stream_t stream,
                                                    uint32_t* status_out) {
  if (workspace == nullptr || status_out == nullptr) return ARCHEAD_EINVAL;
  if (!aligned(workspace, 256)) return ARCHEAD_EALIGN;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* st = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + 4);
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, st, 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && clear) e = cudaMemsetAsync(st, 0, 4, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return set_cuda_error(e);
  *status_out = v;
  return (v & ARCHEAD_STATUS_WAIT_TIMEOUT) ? ARCHEAD_ETIMEOUT : ARCHEAD_OK;
}

extern "C" ARCHEAD_API int archead_set_profile_events(archead_handle* handle, void* before, void* after) {
  if (handle == nullptr || ((before == nullptr) != (after == nullptr))) return ARCHEAD_EINVAL;
  handle->ev_before = static_cast<cudaEvent_t>(before);
  handle->ev_after = static_cast<cudaEvent_t>(after);
  return ARCHEAD_OK;
}

extern "C" ARCHEAD_API int archead_test_decode_waits(archead_handle* handle, uint64_t wait_limit_ns, int stall) {
  if (handle == nullptr || wait_limit_ns == 0) return ARCHEAD_EINVAL;
  handle->wait_limit_ns = wait_limit_ns;
  handle->test_stall = stall != 0 ? 1 : 0;
  return ARCHEAD_OK;
}

extern "C" ARCHEAD_API int archead_last_cuda_error(void) { return g_last_cuda_error; }

extern "C" ARCHEAD_API const char* archead_status_string(int status) {
  switch (status) {
    case ARCHEAD_OK: return "ok";
    case ARCHEAD_EINVAL: return "invalid argument";
    case ARCHEAD_EALIGN: return "misaligned pointer";
    case ARCHEAD_EUNSUP: return "unsupported shape or device";
    case ARCHEAD_ECUDA: return "CUDA runtime error";
    case ARCHEAD_ENOMEM: return "out of memory or buffer too small";
    case ARCHEAD_ETIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}
