// Launch parameters shared by the host launcher and the kernels.
#pragma once
#include <stdint.h>

namespace archead {

// A bounded device-side wait gives up after this long (a legitimate wait is
// microseconds).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Work split of the decode kernel: each residual warp owns kCRes 64-column
// chunks of d (16 k16 steps), each core warp kCL 64-column chunks of r_c',
// each correction warp kCA 32-column chunks of r_r'.
constexpr int kCRes = 4;
constexpr int kCL = 2;
constexpr int kCA = 2;
constexpr int kMaxDecodeWarps = 24;      // launch bound of the decode kernel
constexpr int kEpiWarps = 2;             // decode epilogue warps (share each group of partial logits)
constexpr int kDecodeTokens = 8;         // N of one m16n8k16 fragment
constexpr int kRing = 4;                 // m-tiles in flight per compute warp
// fp16 copies of h are scaled by 2^(kScaleExp - E), E the binary exponent of
// the maximum of |h_t| over the columns they cover (the whole row for the
// prologue's E_t, a residual warp's own columns in the decode kernel), so
// they stay below 2^kScaleExp.
constexpr int kScaleExp = 14;

struct DecodeParams {
  const uint8_t* mtiles;       // arena: m-tile blocks
  const uint16_t* hidden;      // [T, d] bf16
  const uint16_t* zhi;         // [T, Kz] fp16: high part of (z_c | z_r) * 2^(kScaleExp - E_t - e_B)
  const uint16_t* zlo;         // [T, Kz] fp16: remainder
  const int32_t* escale;       // [T] E_t
  const int32_t* targets;      // [T] or null
  float* logits;               // [T, V] or null
  int32_t* argmax;             // [T] or null
  float* lse;                  // [T] or null
  float* ce;                   // [T] or null
  float4* partials;            // [T, gridDim.x]: (m, s, idx bits, unused)
  float* tgt;                  // [T] target logits
  uint32_t* counter;           // completion ticket
  uint32_t* status;            // ARCHEAD_STATUS_* bits
  int32_t T, t0, nt;           // this launch covers tokens [t0, t0 + nt), nt <= 8
  int32_t V, d, Kz, rcp, e_B;
  int32_t row0;                // global id of local row 0 (vocabulary shard); targets and argmax are global
  float4* shard_out;           // [T] (lse, max, argmax bits, target logit or NaN) of this shard, or null
  // Sampling (sampled != null): per token the first maximum of y / tau + G,
  // G Gumbel draws from Philox4x64-10 keyed by seed at counter (ctr0 + t, row / 4).
  int32_t* sampled;            // [T] or null
  float2* spart;               // [T, gridDim.x]: (max of y / tau + G, row bits) per block
  float inv_temp;
  uint64_t seed, ctr0;
  int32_t n_res, n_L, n_A, n_mtiles, g_steps_log2;
  uint32_t off_res, off_Lnib, off_Lhi, off_A, off_sres, off_sL, off_sA, mblk_bytes;
  int32_t nw_res, nw_L, nw_A, nw_work;   // compute warps by role
  int32_t slots, slots_log2;   // partial-logit slots between compute and epilogue warps (power of two)
  int32_t mg, mg_log2;         // m-tiles per partial-logit group (mg * nt <= 8, power of two)
  // Shared-memory rings: one per compute warp, kRing slices each.
  uint32_t res_slice_bytes, core_slice_bytes, corr_slice_bytes;
  uint32_t core_ring_off, corr_ring_off, ring_bytes;
  // Bounded waits: limit per wait, and (test hook only) a stall that makes the
  // epilogue wait on a barrier no one arrives on, so that the limit expires.
  uint64_t wait_limit_ns;
  int32_t test_stall;
};

struct PrologueParams {
  const uint16_t* hidden;      // [T, d] bf16
  const int8_t* R;             // [rcp, d]
  const uint16_t* s_R;         // [rcp]
  const int8_t* B;             // [rrp, d]
  const uint16_t* s_B;         // [rrp, d / g_B]
  const int32_t* targets;      // [T] or null
  uint16_t* zhi;               // [T, Kz] fp16
  uint16_t* zlo;               // [T, Kz] fp16
  int32_t* escale;             // [T]
  uint32_t* counter;
  uint32_t* status;
  int32_t T, d, rcp, rrp, Kz, g_B, V, e_B;
  int32_t v_total;             // target ids are checked against [0, v_total)
};

}  // namespace archead
