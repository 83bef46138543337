// Host-side handle of a packed head loaded into a caller-owned device arena.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>

#include "layout.h"
#include "params.h"
#include "tc_params.h"

namespace archead {
struct HostGraphCache;
}  // namespace archead
using archead::HostGraphCache;

struct archead_handle {
  archead::Layout L;
  const uint8_t* arena;     // device, not owned
  int device;
  int num_sms;
  int grid;                 // decode blocks (one per SM, at most one per m-tile)
  int nw_res, nw_L, nw_A, nw_work;   // decode compute warps by role
  int smem_optin;           // shared memory a block may use on this device
  int e_B;                  // 2^e_B bounds the L1 norm of every dequantised R / B row
  // Tensor-core path (tc_params.h): per-segment weight exponents and whether
  // the shape can take it.
  bool tc_ok;
  int tc_alpha, tc_beta, tc_gamma, tc_mseg;
  int row0;                 // vocabulary shard: global id of row 0, and the global vocabulary size
  int v_total;
  cudaEvent_t ev_before;    // optional profiling events (not owned)
  cudaEvent_t ev_after;
  uint64_t wait_limit_ns;   // decode kernel: limit of every bounded wait (test hook; default kWaitLimitNs)
  int test_stall;           // decode kernel: test hook, a wait that nothing completes
  struct HostGraphCache* graphs;   // host-buffer entry points: captured sequences (api.cu), owned
};

namespace archead {

// Calls with at least kTcMinTokens tokens take the tensor-core path when the
// shape allows it; smaller ones the decode kernel, which streams the whole
// head once per 8 tokens.  At the Qwen shape one decode launch (8 tokens)
// takes ~125 us and the tensor-core pass ~177 us for any count up to 128, so
// a second decode launch (9-16 tokens: 214-286 us) loses to it.
inline bool use_tc(const archead_handle& h, int T) { return h.tc_ok && T >= kTcMinTokens; }

// K columns of the tensor-core path: d + r_c' + r_r' rounded up to 64.
inline int tc_kc(const Layout& L) { return L.d + L.rcp + static_cast<int>(round_up(L.rrp, 64)); }
inline int tc_n_mt128(const Layout& L) { return (L.n_mtiles + 7) / 8; }

// Workspace regions of one forward call with T tokens.  Both kernels' regions
// start after the shared header and target logits, so one workspace of the
// larger size serves whichever kernel a call takes.
struct WsLayout {
  size_t counter, status, tgt;
  size_t escale, zhi, zlo, partials, spart;   // decode path
  size_t cinv, xop, tpartials;                // tensor-core path
  size_t total;
  // host-buffer forms only
  size_t h_hidden, h_targets, h_lse, h_argmax, h_ce, host_total;
  size_t h_logits, host_logits_total;   // logits form: [T, V] fp32 staging after host_total
};

// The K-split tickets of the activation kernel sit in the zero-filled head of
// the workspace, between the status word and the target logits.
static_assert(kActTicketOff >= 8 && kActTicketOff + 4 * kActTickets <= 256, "ticket block of the workspace head");

inline WsLayout ws_layout(const archead_handle& h, int T) {
  WsLayout w{};
  const size_t t = static_cast<size_t>(T);
  w.counter = 0;
  w.status = 4;
  w.tgt = 256;
  const size_t base = w.tgt + round_up(t * 4, 256);
  size_t o = base;
  w.escale = o;   o += round_up(t * 4, 256);
  w.zhi = o;      o += round_up(t * h.L.Kz * 2, 256);
  w.zlo = o;      o += round_up(t * h.L.Kz * 2, 256);
  w.partials = o; o += round_up(t * h.grid * 16, 256);
  w.spart = o;    o += round_up(t * h.grid * 8, 256);
  const size_t dec_end = o;
  o = base;
  if (use_tc(h, T)) {
    w.cinv = o;      o += round_up(t * 4, 256);
    w.xop = o;       o += round_up(t * tc_kc(h.L) * 2, 256);
    w.tpartials = o; o += round_up(t * tc_n_mt128(h.L) * 16, 256);
  }
  w.total = o > dec_end ? o : dec_end;
  o = w.total;
  w.h_hidden = o;  o += round_up(t * h.L.d * 2, 256);
  w.h_targets = o; o += round_up(t * 4, 256);
  w.h_lse = o;     o += round_up(t * 4, 256);
  w.h_argmax = o;  o += round_up(t * 4, 256);
  w.h_ce = o;      o += round_up(t * 4, 256);
  w.host_total = o;
  w.h_logits = o;  o += round_up(t * static_cast<size_t>(h.L.V) * 4, 256);
  w.host_logits_total = o;
  return w;
}

// Kernel launchers and attributes (decode.cu, prologue.cu).
void decode_smem_plan(DecodeParams& p, int g_steps);
size_t decode_smem_bytes(const DecodeParams& p);
cudaError_t decode_set_attributes(int g_steps, size_t smem);
cudaError_t launch_decode(int g_steps, const DecodeParams& p, int grid, size_t smem, cudaStream_t stream);
cudaError_t launch_prologue(const PrologueParams& p, cudaStream_t stream);

// Tensor-core path (actprep.cu, tcgemm.cu).
cudaError_t launch_act_prep(const ActParams& p, int splits, cudaStream_t stream);
// K splits of the activation kernel for T tokens; their partials need
// splits x tiles x z blocks x kActPartFloats floats of scratch_bytes.
int act_prep_splits(int T, int d, int Kc, int num_sms, size_t scratch_bytes);
void tc_smem_plan(TcParams& p);
size_t tc_smem_bytes(const TcParams& p);
size_t tc_smem_max();
cudaError_t tc_set_attributes();
cudaError_t tc_encode_xmap(CUtensorMap* map, const uint16_t* xop, int T, int Kc, int BN);
cudaError_t launch_tc(const TcParams& p, const CUtensorMap& map, int grid, cudaStream_t stream);
cudaError_t launch_tc_merge(const float4* partials, int n_mt128, int T, const int32_t* targets, const float* tgt,
                            int V, int row0, float* lse, int32_t* argmax, float* ce, float4* shard_out,
                            cudaStream_t stream);
cudaError_t launch_shard_merge(const float4* parts, int n, int T, float* lse, int32_t* argmax, float* ce,
                               cudaStream_t stream);

// Thread-local record of the last CUDA error (api.cu).
int set_cuda_error(cudaError_t e);

// Cache of captured host-buffer call sequences of a handle (api.cu).
HostGraphCache* host_graph_cache_new();
void host_graph_cache_free(HostGraphCache* c);

}  // namespace archead
