// Launch parameters of the tensor-core forward (many tokens per call).
//
// The head is applied as one contraction over a concatenated K axis:
//   y[t, v] = sum_k W~[v, k] X[t, k] * 2^-c_t,
//   W~ = [ s_res q | s_L L | s_A A ] (per segment times a power of two),
//   X  = [ h       | z_c    | z_r  ] (per segment times a power of two),
// with z_c = s_R R h and z_r = (s_B B) h from the activation kernel.  The
// weight side is dequantised tile by tile into tensor memory; the activation
// side is an fp16 matrix in HBM read by TMA.
#pragma once
#include <stdint.h>

namespace archead {

constexpr int kTcBM = 128;            // vocabulary rows per unit (8 m-tile blocks of 16)
constexpr int kTcBK = 64;             // K columns per k-step (one 128-byte row of fp16)
constexpr int kTcStepsPerStage = 2;   // k-steps per pipeline stage
constexpr int kTcMaxBN = 128;         // tokens per unit
constexpr int kTcMaxStages = 8;       // stages in flight between the producers and the MMA (even)
constexpr int kTcMinRing = 2;         // ring slots (stages of packed bytes) per dequantising warp:
constexpr int kTcMaxRing = 5;         //   as many as shared memory holds next to the stage buffers
constexpr int kTcSmemBudget = 232448; // dynamic shared memory a block may use on sm_100a (227 KB)
constexpr int kTcSlotBytes = 1056;    // one packed k-step of one m-tile block (codes + scales)
constexpr int kTcDeqWarps = 16;       // two per m-tile block of a unit (even / odd k-steps)
constexpr int kTcWarps = 22;          // 16 dequantising, 1 TMA, 1 MMA, 4 epilogue
constexpr int kTcMinTokens = 9;       // calls with fewer tokens take the decode kernel (one launch)
constexpr int kActMaxSplits = 8;      // K splits of one block of z in the activation kernel
constexpr int kActPartFloats = 16 * 64 + 16;   // one split's partial sums and token exponents
constexpr int kActTicketOff = 64;     // workspace byte offset of the K-split tickets (inside the zeroed head)
constexpr int kActTickets = 48;       // tickets available there: K splits need tiles x z blocks <= this

struct TcParams {
  const uint8_t* mtiles;      // arena: m-tile blocks
  const int32_t* targets;     // [T] or null
  const float* cinv;          // [T] 2^-c_t
  float* logits;              // [T, V] or null
  float4* partials;           // [T, n_mt128]: (max, sum, argmax bits, unused) per 128-row tile
  float* tgt;                 // [T] target logits
  uint32_t* status;
  int32_t T, V, BN, n_nt, n_mt128, n_units;
  int32_t row0;                                // global id of local row 0 (vocabulary shard)
  int32_t n_res, n_L, n_A, n_mtiles, g_log2;   // chunks per segment; log2 of the residual group
  int32_t n_ks, ks_core, ks_corr;              // k-steps: total, first core, first correction
  int32_t n_st;                                // stages per unit: ceil(n_ks / 2)
  uint32_t off_res, off_Lnib, off_Lhi, off_A, off_sres, off_sL, off_sA, mblk_bytes;
  float sc_res, sc_L, sc_A;                    // 2^alpha, 2^beta, 2^gamma
  int32_t stages, ring;                        // stage buffers (even, <= kTcMaxStages); ring slots per warp
  uint32_t acc_stride, acol0;                  // TMEM columns: accumulator stride, first A stage
  uint32_t bstage_bytes, ring_off, epi_off, bar_off;   // shared-memory plan
};

struct ActParams {
  const uint16_t* hidden;     // [T, d] bf16
  const int8_t* R;            // [rcp, d]
  const uint16_t* s_R;        // [rcp]
  const int8_t* B;            // [rrp, d]
  const uint16_t* s_B;        // [rrp, d / g_B]
  const int32_t* targets;     // [T] or null
  uint32_t* status;
  uint16_t* xop;              // [T, Kc] fp16 activation operand
  float* cinv;                // [T] 2^-c_t
  float* zpart;               // K-split partials: [tile][z block][split] x (16 x 64 sums, 16 exponents)
  uint32_t* zticket;          // [tile][z block] completion tickets of the K splits (zero between calls)
  int32_t T, d, rcp, Kz, Kc, g_B, V;
  int32_t v_total;                             // target ids are checked against [0, v_total)
  int32_t alpha, beta, gamma, mseg;
};

}  // namespace archead
