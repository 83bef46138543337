// Decode kernel: the packed-head forward (ARCHead paper, §3.2 Eq. 7) for up
// to 8 tokens per launch, streaming the packed head once from HBM.
//
// Per vocabulary row v and token t it forms
//   y[t,v] = sum_g s_res[v,g] (sum_{j in g} q[v,j] h[t,j])          residual (SC4)
//          + s_L[v] sum_k L[v,k] z_c[t,k]                         core (Eq. 3)
//          + s_A[v] sum_k A[v,k] z_r[t,k]                         correction (Eq. 4-6)
// with z_c, z_r from the prologue kernel.  Codes are unpacked in registers to
// exact fp16 integers (offset code, plus 64 in half of the columns) and
// multiplied on the tensor cores (m16n8k16: vocabulary rows as M, tokens as
// N, fp32 accumulation).  The constant part is removed once per scale group in
// fp32 with a per-token sum of the same fp16 operands, and the fp16 group /
// row scales multiply fp32 partial sums, so no scaled weight is ever rounded.
// h enters as fp16 scaled by a per-token power of two (exact for bf16 inputs);
// z as an fp16 pair (high part + remainder) under its own power of two.
//
// Work split (one block per SM, persistent over the m-tiles m = block,
// block + grid, ...): every compute warp owns a fixed slice of every m-tile
// block, so it streams its own bytes:
//   residual warps    16 k16 steps of d each; their fp16 h fragments stay in
//                     registers for the whole launch, each warp's columns
//                     under a power of two of their own (from their own
//                     maximum), so a warp starts as soon as its h and first
//                     m-tile have landed, waiting for no other warp and not
//                     for the prologue
//   core warps        kCL 64-column chunks of r_c' each
//   correction warps  kCA 32-column chunks of r_r' each (these and the core
//                     warps wait for the prologue's z)
// Residual and core warps take m-tiles in interleaved pairs (two independent
// MMA chains).  Each compute warp prefetches its slice of the next kRing
// m-tiles into a private shared-memory ring with cp.async (16 B per lane, L2
// only, evict-first: the head is read once) and waits only on its own copies:
// no producer warp and no block-wide synchronisation.  After an m-tile the warp stores its 16 x nt partial logits
// in its own region of a slot and arrives on reduced[r].  Warps 0-1, the
// epilogue, each take half of a slot's elements (two adjacent per lane), sum
// the warps' regions in warp order (deterministic), push the logits into
// running log-sum-exp / argmax states, write logits when asked, and free the
// slot (redfree[r]).  At the end every block writes one partial per token; the
// last block to finish (atomic ticket, no spinning) merges them into LSE,
// argmax and CE.  Every mbarrier wait is bounded (kWaitLimitNs); on expiry the
// block raises ARCHEAD_STATUS_WAIT_TIMEOUT and skips the remaining work.
#include <cuda_runtime.h>

#include "device.cuh"
#include "params.h"

namespace archead {

namespace {

constexpr int kGroupTile = 8;    // m-tiles x tokens per partial-logit group (mg * nt)
constexpr int kMergeLoads = 5;   // partials per token a lane of the last block loads at once (grids up to 160 blocks in one round)
constexpr int kMergeLoadsOne = 8;   // the same when one warp merges one token at a time

struct SmemView {
  uint8_t* rings;                // per compute warp: kRing slices
  float* part;                   // [slots][nw_work][mg][nt][16 rows] per-warp partial logits
  uint64_t* reduced;             // [slots] compute warps -> epilogue warps
  uint64_t* redfree;             // [slots] epilogue warps -> compute warps
  float4* tokstate;              // [4 kEpiWarps] LSE state of each epilogue octet (q = 4 ew + lane / 8)
  float2* pickstate;             // [4 kEpiWarps] sampling state of each epilogue octet
  uint64_t* stall;               // test hook: a barrier nothing arrives on
  int* flags;                    // [0] abort, [1] this block merges the partials
};

__device__ __forceinline__ SmemView smem_view(uint8_t* smem, const DecodeParams& p) {
  SmemView v;
  v.rings = smem;
  v.part = reinterpret_cast<float*>(smem + p.ring_bytes);
  v.reduced = reinterpret_cast<uint64_t*>(v.part + static_cast<size_t>(p.slots) * p.nw_work * kGroupTile * 16);
  v.redfree = v.reduced + p.slots;
  v.tokstate = reinterpret_cast<float4*>(v.redfree + p.slots);
  v.pickstate = reinterpret_cast<float2*>(v.tokstate + kEpiWarps * kDecodeTokens);
  v.stall = reinterpret_cast<uint64_t*>(v.pickstate + kEpiWarps * kDecodeTokens);
  v.flags = reinterpret_cast<int*>(v.stall + 1);
  return v;
}

__device__ __forceinline__ bool aborted(const SmemView& sv) {
  return *reinterpret_cast<volatile int*>(sv.flags) != 0;
}

__device__ __forceinline__ void raise_timeout(const SmemView& sv, uint32_t* status) {
  *reinterpret_cast<volatile int*>(sv.flags) = 1;
  atomicOr(status, static_cast<uint32_t>(ARCHEAD_STATUS_WAIT_TIMEOUT));
}

// Warp-uniform bounded wait; false if the block has aborted or the wait expired.
__device__ __forceinline__ bool warp_wait(const SmemView& sv, uint64_t* bar, uint32_t parity, uint32_t* status,
                                          int lane, uint64_t limit_ns) {
  bool ok = !aborted(sv) && mbar_wait(smem_addr(bar), parity, limit_ns);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && lane == 0 && !aborted(sv)) raise_timeout(sv, status);
  return ok;
}

__device__ __forceinline__ int mtile_of(int i) {
  return static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
}

// B-operand fragment (16 x 8, column = token) from the fp16 row of token gr:
// lane (gr, cc) holds rows k0 + 2cc, +1 and k0 + 2cc + 8, +9.
__device__ __forceinline__ void load_b_frag_f16(const uint16_t* base, int k0, int lane, bool valid,
                                                uint32_t& b0, uint32_t& b1) {
  const int cc = lane & 3;
  if (valid) {
    const uint16_t* r = base + k0 + 2 * cc;
    b0 = *reinterpret_cast<const uint32_t*>(r);
    b1 = *reinterpret_cast<const uint32_t*>(r + 8);
  } else {
    b0 = 0u;
    b1 = 0u;
  }
}

// bias_lo * (x + y) over the pair b0 plus bias_hi * (x + y) over the pair b1.
__device__ __forceinline__ float bias_dot(uint32_t b0, uint32_t b1, float bias_lo, float bias_hi) {
  const float2 f0 = half2_bits_to_float2(b0);
  const float2 f1 = half2_bits_to_float2(b1);
  return bias_lo * (f0.x + f0.y) + bias_hi * (f1.x + f1.y);
}

// Per-token constants of this lane's accumulator columns (tokens 2cc, 2cc+1)
// from a per-token value held by the lanes of token gr (after a quad reduce).
__device__ __forceinline__ float2 column_pair(float v_of_gr, int lane) {
  const int cc = lane & 3;
  return make_float2(__shfl_sync(0xffffffffu, v_of_gr, 8 * cc), __shfl_sync(0xffffffffu, v_of_gr, 8 * cc + 4));
}

__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  return v;
}

// Partial logits travel in groups of p.mg consecutive m-tiles of this block
// (p.mg * p.nt = 8): slot r = group & (slots - 1) holds, per compute warp, a
// [mg][nt][16] tile.  A compute warp checks once per group that the epilogue
// has drained the slot's previous group, stores each m-tile's partial tile
// with plain stores, and arrives on reduced[r] once per group.  The epilogue
// sums the warps' tiles in warp order, so results do not depend on timing.
__device__ __forceinline__ float* group_begin(const SmemView& sv, const DecodeParams& p, int i, int cw, int lane) {
  const int grp = i >> p.mg_log2;
  const int r = grp & (p.slots - 1);
  if (grp >= p.slots) warp_wait(sv, &sv.redfree[r], ((grp >> p.slots_log2) - 1) & 1, p.status, lane, p.wait_limit_ns);
  return sv.part + (r * p.nw_work + cw) * (kGroupTile * 16);
}

__device__ __forceinline__ void store_partial(float* tile, const DecodeParams& p, int i, int lane,
                                              const float (&acc)[4]) {
  const int gr = lane >> 2, cc = lane & 3;
  float* t = tile + (i & (p.mg - 1)) * p.nt * 16;
  const int t0 = 2 * cc, t1 = 2 * cc + 1;
  if (t0 < p.nt) {
    t[t0 * 16 + gr] = acc[0];
    t[t0 * 16 + gr + 8] = acc[2];
  }
  if (t1 < p.nt) {
    t[t1 * 16 + gr] = acc[1];
    t[t1 * 16 + gr + 8] = acc[3];
  }
}

__device__ __forceinline__ void group_end(const SmemView& sv, const DecodeParams& p, int i, int n_my, int lane) {
  if ((i & (p.mg - 1)) == p.mg - 1 || i == n_my - 1) {
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&sv.reduced[(i >> p.mg_log2) & (p.slots - 1)]));
  }
}

// ------------------------------------------------------------ residual warps
// Ring slice: [kCRes chunks x 512 B of codes][groups x 32 B of scales].
struct ResSlice {
  int chunk0, nchunks;     // residual chunks of this warp
  int grp0, ng;            // scale groups its columns touch
};

__device__ __forceinline__ ResSlice res_slice(const DecodeParams& p, int wres) {
  ResSlice r;
  r.chunk0 = wres * kCRes;
  r.nchunks = min(kCRes, p.n_res - r.chunk0);
  const int col0 = r.chunk0 * kResChunkK, col1 = col0 + r.nchunks * kResChunkK - 1;
  r.grp0 = col0 >> (p.g_steps_log2 + 4);
  r.ng = (col1 >> (p.g_steps_log2 + 4)) - r.grp0 + 1;
  return r;
}

// Copy this lane's 16-byte pieces of one m-tile's residual slice: codes at
// `codes` (already offset to the lane), scales at `scales` (lanes that own a
// piece only).  kFull: all kCRes chunks present.
template <bool kFull>
__device__ __forceinline__ void issue_res(uint32_t dst, const uint8_t* codes, const uint8_t* scales, int nchunks,
                                          bool scale_lane) {
#pragma unroll
  for (int c = 0; c < kCRes; ++c)
    if (kFull || c < nchunks) cp_async16_hint(dst + c * kResChunkBytes, codes + c * kResChunkBytes, l2_evict_first_policy());
  if (scale_lane) cp_async16_hint(dst + kCRes * kResChunkBytes, scales, l2_evict_first_policy());
}

// One m-tile of a residual warp: 16 k16 steps over its 4 chunks, flushing
// each scale group into acc.  kFull: all 4 chunks present (no guards).
template <int G, bool kFull>
__device__ __forceinline__ void residual_tile(const uint8_t* slot, const ResSlice& rs,
                                              const uint32_t (&hf)[kCRes][4][2], const float2 (&cgc)[16 / G],
                                              int step0, int last_step, int g_log2, int lane, float (&acc)[4]) {
  const int gr = lane >> 2;
  float t0[4] = {0.f, 0.f, 0.f, 0.f};
  float t1[4] = {0.f, 0.f, 0.f, 0.f};
  const uint8_t* sres = slot + kCRes * kResChunkBytes + gr * 4;
#pragma unroll
  for (int c = 0; c < kCRes; ++c) {
    if (kFull || c < rs.nchunks) {
      const uint4 nib = *reinterpret_cast<const uint4*>(slot + c * kResChunkBytes + lane * 16);
      const uint32_t wv[4] = {nib.x, nib.y, nib.z, nib.w};
#pragma unroll
      for (int st = 0; st < 4; ++st) {
        const int step = 4 * c + st;
        const int lg = step / G;
        float(&tmp)[4] = (lg & 1) ? t1 : t0;
        uint32_t a[4];
        unpack_int4_biased(wv[st], a);
        mma_f16_16816(tmp, a, hf[c][st][0], hf[c][st][1]);
        if ((step + 1) % G == 0 || (G == 16 && step == last_step)) {
          const int grp = ((step0 + step) >> g_log2) - rs.grp0;
          const float2 sc = half2_bits_to_float2(*reinterpret_cast<const uint32_t*>(sres + grp * kSresGroupBytes));
          acc[0] = fmaf(sc.x, tmp[0] - cgc[lg].x, acc[0]);
          acc[1] = fmaf(sc.x, tmp[1] - cgc[lg].y, acc[1]);
          acc[2] = fmaf(sc.y, tmp[2] - cgc[lg].x, acc[2]);
          acc[3] = fmaf(sc.y, tmp[3] - cgc[lg].y, acc[3]);
          tmp[0] = tmp[1] = tmp[2] = tmp[3] = 0.f;
        }
      }
    }
  }
}

// Two m-tiles of a residual warp at once (all 4 chunks present): the two
// independent MMA chains interleave, so the warp has work while one waits.
template <int G>
__device__ __forceinline__ void residual_tile_pair(const uint8_t* slot_a, const uint8_t* slot_b, const ResSlice& rs,
                                                   const uint32_t (&hf)[kCRes][4][2], const float2 (&cgc)[16 / G],
                                                   int step0, int g_log2, int lane, float (&acc_a)[4],
                                                   float (&acc_b)[4]) {
  const int gr = lane >> 2;
  float ta[4] = {0.f, 0.f, 0.f, 0.f};
  float tb[4] = {0.f, 0.f, 0.f, 0.f};
  const uint8_t* sres_a = slot_a + kCRes * kResChunkBytes + gr * 4;
  const uint8_t* sres_b = slot_b + kCRes * kResChunkBytes + gr * 4;
#pragma unroll
  for (int c = 0; c < kCRes; ++c) {
    const uint4 na = *reinterpret_cast<const uint4*>(slot_a + c * kResChunkBytes + lane * 16);
    const uint4 nb = *reinterpret_cast<const uint4*>(slot_b + c * kResChunkBytes + lane * 16);
    const uint32_t wa[4] = {na.x, na.y, na.z, na.w};
    const uint32_t wb[4] = {nb.x, nb.y, nb.z, nb.w};
#pragma unroll
    for (int st = 0; st < 4; ++st) {
      const int step = 4 * c + st;
      uint32_t a[4];
      unpack_int4_biased(wa[st], a);
      mma_f16_16816(ta, a, hf[c][st][0], hf[c][st][1]);
      unpack_int4_biased(wb[st], a);
      mma_f16_16816(tb, a, hf[c][st][0], hf[c][st][1]);
      if ((step + 1) % G == 0) {
        const int lg = step / G;
        const int grp = ((step0 + step) >> g_log2) - rs.grp0;
        const float2 sa = half2_bits_to_float2(*reinterpret_cast<const uint32_t*>(sres_a + grp * kSresGroupBytes));
        const float2 sb = half2_bits_to_float2(*reinterpret_cast<const uint32_t*>(sres_b + grp * kSresGroupBytes));
        acc_a[0] = fmaf(sa.x, ta[0] - cgc[lg].x, acc_a[0]);
        acc_a[1] = fmaf(sa.x, ta[1] - cgc[lg].y, acc_a[1]);
        acc_a[2] = fmaf(sa.y, ta[2] - cgc[lg].x, acc_a[2]);
        acc_a[3] = fmaf(sa.y, ta[3] - cgc[lg].y, acc_a[3]);
        acc_b[0] = fmaf(sb.x, tb[0] - cgc[lg].x, acc_b[0]);
        acc_b[1] = fmaf(sb.x, tb[1] - cgc[lg].y, acc_b[1]);
        acc_b[2] = fmaf(sb.y, tb[2] - cgc[lg].x, acc_b[2]);
        acc_b[3] = fmaf(sb.y, tb[3] - cgc[lg].y, acc_b[3]);
        ta[0] = ta[1] = ta[2] = ta[3] = 0.f;
        tb[0] = tb[1] = tb[2] = tb[3] = 0.f;
      }
    }
  }
}

// G = k16 steps per scale group within the warp's 16 steps (16 when a group
// spans the whole warp range or more).
template <int G>
__device__ void residual_warp(const DecodeParams& p, const SmemView& sv, int n_my, int wres, int cw, int lane) {
  constexpr int kNG = 16 / G;    // local scale groups
  const int gr = lane >> 2;
  const ResSlice rs = res_slice(p, wres);
  const uint32_t sbytes = p.res_slice_bytes;
  uint8_t* ring = sv.rings + static_cast<size_t>(wres) * kRing * sbytes;
  const uint32_t ring_s = smem_addr(ring) + lane * 16;
  // Global pieces of m-tile 0 of this block; m-tile i is `stride` bytes further per step.
  const size_t stride = static_cast<size_t>(gridDim.x) * p.mblk_bytes;
  const uint8_t* base = p.mtiles + static_cast<size_t>(blockIdx.x) * p.mblk_bytes;
  const uint8_t* g_codes = base + p.off_res + rs.chunk0 * kResChunkBytes + lane * 16;
  const uint8_t* g_scales = base + p.off_sres + rs.grp0 * kSresGroupBytes + lane * 16;
  const bool scale_lane = lane * 16 < rs.ng * kSresGroupBytes;
  const bool full = rs.nchunks == kCRes;
  // Each warp scales its own columns of h_t by 2^(kScaleExp - E), with
  // max|h_t| < 2^E over those columns: exact for bf16 inputs, and undone on
  // the warp's fp32 partial sums (a power of two), so warps need not agree on
  // E.  The h loads go out first, ahead of the ring's copies, so E is known
  // by the time the first m-tile has landed.
  const bool tok = gr < p.nt;
  const uint16_t* hrow = p.hidden + static_cast<size_t>(p.t0 + (tok ? gr : 0)) * p.d;
  uint32_t hf[kCRes][4][2];   // bf16 pairs of this warp's columns, then fp16 fragments
#pragma unroll
  for (int c = 0; c < kCRes; ++c) {
#pragma unroll
    for (int s = 0; s < 4; ++s) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        uint32_t bits = 0u;
        if (tok && c < rs.nchunks)
          bits = *reinterpret_cast<const uint32_t*>(hrow + (rs.chunk0 + c) * kResChunkK + s * 16 + 2 * (lane & 3) + 8 * j);
        hf[c][s][j] = bits;
      }
    }
  }
  // Start streaming before the prologue's results are needed.
#pragma unroll
  for (int k = 0; k < kRing; ++k) {
    if (k < n_my) {
      if (full) issue_res<true>(ring_s + k * sbytes, g_codes + k * stride, g_scales + k * stride, rs.nchunks, scale_lane);
      else issue_res<false>(ring_s + k * sbytes, g_codes + k * stride, g_scales + k * stride, rs.nchunks, scale_lane);
    }
    cp_async_commit();
  }
  g_codes += kRing * stride;
  g_scales += kRing * stride;
  float mx = 0.f;
#pragma unroll
  for (int c = 0; c < kCRes; ++c)
#pragma unroll
    for (int s = 0; s < 4; ++s)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const uint32_t bits = hf[c][s][j];
        mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(bits << 16)), fabsf(__uint_as_float(bits & 0xFFFF0000u))));
      }
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  float hs = 0.f;
  if (tok) {
    int E = 0;
    frexpf(mx, &E);
    hs = ldexpf(1.f, kScaleExp - E);
  }
  // fp16 h fragments of this warp's columns, and the constant-part sum of each
  // local group for token gr.
  float cg[kNG];
#pragma unroll
  for (int g = 0; g < kNG; ++g) cg[g] = 0.f;
#pragma unroll
  for (int c = 0; c < kCRes; ++c) {
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      uint32_t b[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const uint32_t bits = hf[c][s][j];
        b[j] = pack_half2(__uint_as_float(bits << 16) * hs, __uint_as_float(bits & 0xFFFF0000u) * hs);
      }
      hf[c][s][0] = b[0];
      hf[c][s][1] = b[1];
      cg[(4 * c + s) / G] += bias_dot(b[0], b[1], kBiasLo + 8.f, kBiasHi + 8.f);
    }
  }
  float2 cgc[kNG];
#pragma unroll
  for (int g = 0; g < kNG; ++g) cgc[g] = column_pair(quad_sum(cg[g]), lane);
  const float2 unscale = column_pair(tok ? 1.f / hs : 0.f, lane);
  const int last_step = rs.nchunks * 4 - 1;
  const int step0 = wres * 16;

  float* tile = nullptr;
  int i = 0;
  if (full && G == 8) {
    // Pairs of m-tiles (two scale groups per warp range; smaller groups keep
    // too many per-group sums live for two tiles).
    for (; i + 1 < n_my; i += 2) {
      const uint32_t k = static_cast<uint32_t>(i) & (kRing - 1);   // even: k, k + 1 < kRing
      const uint8_t* slot = ring + k * sbytes;
      cp_async_wait<kRing - 2>();
      __syncwarp();
      float acc_a[4] = {0.f, 0.f, 0.f, 0.f};
      float acc_b[4] = {0.f, 0.f, 0.f, 0.f};
      residual_tile_pair<G>(slot, slot + sbytes, rs, hf, cgc, step0, p.g_steps_log2, lane, acc_a, acc_b);
      acc_a[0] *= unscale.x;
      acc_a[1] *= unscale.y;
      acc_a[2] *= unscale.x;
      acc_a[3] *= unscale.y;
      acc_b[0] *= unscale.x;
      acc_b[1] *= unscale.y;
      acc_b[2] *= unscale.x;
      acc_b[3] *= unscale.y;
      __syncwarp();   // every lane is done reading both slots
      if (i + kRing < n_my) issue_res<true>(ring_s + k * sbytes, g_codes, g_scales, kCRes, scale_lane);
      cp_async_commit();
      if (i + 1 + kRing < n_my)
        issue_res<true>(ring_s + (k + 1) * sbytes, g_codes + stride, g_scales + stride, kCRes, scale_lane);
      cp_async_commit();
      g_codes += 2 * stride;
      g_scales += 2 * stride;
      if ((i & (p.mg - 1)) == 0) tile = group_begin(sv, p, i, cw, lane);
      store_partial(tile, p, i, lane, acc_a);
      group_end(sv, p, i, n_my, lane);
      if (((i + 1) & (p.mg - 1)) == 0) tile = group_begin(sv, p, i + 1, cw, lane);
      store_partial(tile, p, i + 1, lane, acc_b);
      group_end(sv, p, i + 1, n_my, lane);
    }
  }
  for (; i < n_my; ++i) {
    if ((i & (p.mg - 1)) == 0) tile = group_begin(sv, p, i, cw, lane);
    const uint32_t k = static_cast<uint32_t>(i) & (kRing - 1);
    const uint8_t* slot = ring + k * sbytes;
    cp_async_wait<kRing - 1>();
    __syncwarp();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (full)
      residual_tile<G, true>(slot, rs, hf, cgc, step0, kCRes * 4 - 1, p.g_steps_log2, lane, acc);
    else
      residual_tile<G, false>(slot, rs, hf, cgc, step0, last_step, p.g_steps_log2, lane, acc);
    acc[0] *= unscale.x;
    acc[1] *= unscale.y;
    acc[2] *= unscale.x;
    acc[3] *= unscale.y;
    __syncwarp();   // every lane is done reading the slot
    if (i + kRing < n_my) {
      if (full) issue_res<true>(ring_s + k * sbytes, g_codes, g_scales, rs.nchunks, scale_lane);
      else issue_res<false>(ring_s + k * sbytes, g_codes, g_scales, rs.nchunks, scale_lane);
    }
    g_codes += stride;
    g_scales += stride;
    cp_async_commit();
    store_partial(tile, p, i, lane, acc);
    group_end(sv, p, i, n_my, lane);
  }
  cp_async_wait_all();
}

// ---------------------------------------------------------------- core warps
// Ring slice: [kCL x 512 B nibbles][kCL x 128 B fifth bits][32 B s_L].
// One m-tile's core slice for this lane: nibble planes, fifth-bit planes
// (lanes below nch * 8) and row scales (lanes 0, 1).  Global pointers are
// already offset to the lane.
__device__ __forceinline__ void issue_core(uint32_t dst, const uint8_t* g_nib, const uint8_t* g_hi,
                                           const uint8_t* g_sl, int nch, bool hi_lane, bool sl_lane) {
#pragma unroll
  for (int c = 0; c < kCL; ++c)
    if (c < nch) cp_async16_hint(dst + c * kLNibChunkBytes, g_nib + c * kLNibChunkBytes, l2_evict_first_policy());
  if (hi_lane) cp_async16_hint(dst + kCL * kLNibChunkBytes, g_hi, l2_evict_first_policy());
  if (sl_lane) cp_async16_hint(dst + kCL * (kLNibChunkBytes + kLHiChunkBytes), g_sl, l2_evict_first_policy());
}

// One core chunk (4 k16 steps, fp16 pair hi + lo of z) of one m-tile slot into acc.
__device__ __forceinline__ void core_chunk(const uint8_t* slot, int c, int lane, const uint32_t (&zf)[kCL][4][2][2],
                                           float (&acc)[4]) {
  const uint4 nib = *reinterpret_cast<const uint4*>(slot + c * kLNibChunkBytes + lane * 16);
  const uint32_t hb = *reinterpret_cast<const uint32_t*>(slot + kCL * kLNibChunkBytes + c * kLHiChunkBytes + lane * 4);
  uint32_t a[4];
  unpack_int5_biased<0>(nib.x, hb, a);
  mma_f16_16816(acc, a, zf[c][0][0][0], zf[c][0][0][1]);
  mma_f16_16816(acc, a, zf[c][0][1][0], zf[c][0][1][1]);
  unpack_int5_biased<1>(nib.y, hb, a);
  mma_f16_16816(acc, a, zf[c][1][0][0], zf[c][1][0][1]);
  mma_f16_16816(acc, a, zf[c][1][1][0], zf[c][1][1][1]);
  unpack_int5_biased<2>(nib.z, hb, a);
  mma_f16_16816(acc, a, zf[c][2][0][0], zf[c][2][0][1]);
  mma_f16_16816(acc, a, zf[c][2][1][0], zf[c][2][1][1]);
  unpack_int5_biased<3>(nib.w, hb, a);
  mma_f16_16816(acc, a, zf[c][3][0][0], zf[c][3][0][1]);
  mma_f16_16816(acc, a, zf[c][3][1][0], zf[c][3][1][1]);
}

// Row scale, constant part and token scale of a finished core tile.
__device__ __forceinline__ void core_finish(const uint8_t* slot, int gr, float2 cbc, float2 unscale, float (&acc)[4]) {
  const float2 sc = half2_bits_to_float2(
      *reinterpret_cast<const uint32_t*>(slot + kCL * (kLNibChunkBytes + kLHiChunkBytes) + gr * 4));
  acc[0] = (acc[0] - cbc.x) * (sc.x * unscale.x);
  acc[1] = (acc[1] - cbc.y) * (sc.x * unscale.y);
  acc[2] = (acc[2] - cbc.x) * (sc.y * unscale.x);
  acc[3] = (acc[3] - cbc.y) * (sc.y * unscale.y);
}

__device__ void core_warp(const DecodeParams& p, const SmemView& sv, int n_my, int wl, int cw, int lane) {
  const int gr = lane >> 2;
  const int chunk0 = wl * kCL;
  const int nch = min(kCL, p.n_L - chunk0);
  const uint32_t sbytes = p.core_slice_bytes;
  uint8_t* ring = sv.rings + p.core_ring_off + static_cast<size_t>(wl) * kRing * sbytes;
  const uint32_t ring_s = smem_addr(ring) + lane * 16;
  const size_t stride = static_cast<size_t>(gridDim.x) * p.mblk_bytes;
  const uint8_t* base = p.mtiles + static_cast<size_t>(blockIdx.x) * p.mblk_bytes;
  const uint8_t* g_nib = base + p.off_Lnib + chunk0 * kLNibChunkBytes + lane * 16;
  const uint8_t* g_hi = base + p.off_Lhi + chunk0 * kLHiChunkBytes + lane * 16;
  const uint8_t* g_sl = base + p.off_sL + lane * 16;
  const bool hi_lane = lane * 16 < nch * kLHiChunkBytes, sl_lane = lane < 2;
#pragma unroll
  for (int k = 0; k < kRing; ++k) {
    if (k < n_my) issue_core(ring_s + k * sbytes, g_nib + k * stride, g_hi + k * stride, g_sl + k * stride, nch,
                             hi_lane, sl_lane);
    cp_async_commit();
  }
  g_nib += kRing * stride;
  g_hi += kRing * stride;
  g_sl += kRing * stride;
  grid_dependency_wait();
  const bool tok = gr < p.nt;
  uint32_t zf[kCL][4][2][2];
  float cb = 0.f;
  const uint16_t* zh = p.zhi + static_cast<size_t>(p.t0 + (tok ? gr : 0)) * p.Kz;
  const uint16_t* zl = p.zlo + static_cast<size_t>(p.t0 + (tok ? gr : 0)) * p.Kz;
#pragma unroll
  for (int c = 0; c < kCL; ++c) {
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int k0 = (chunk0 + c) * kLChunkK + s * 16;
      const bool ok = tok && c < nch;
      load_b_frag_f16(zh, k0, lane, ok, zf[c][s][0][0], zf[c][s][0][1]);
      load_b_frag_f16(zl, k0, lane, ok, zf[c][s][1][0], zf[c][s][1][1]);
      cb += bias_dot(zf[c][s][0][0], zf[c][s][0][1], kBiasLo + 16.f, kBiasHi + 16.f);
      cb += bias_dot(zf[c][s][1][0], zf[c][s][1][1], kBiasLo + 16.f, kBiasHi + 16.f);
    }
  }
  const float2 cbc = column_pair(quad_sum(cb), lane);
  const float zs = tok ? ldexpf(1.f, p.escale[p.t0 + gr] + p.e_B - kScaleExp) : 0.f;
  const float2 unscale = column_pair(zs, lane);

  float* tile = nullptr;
  int i = 0;
  if (nch == kCL) {
    // Pairs of m-tiles: two independent MMA chains interleave.
    for (; i + 1 < n_my; i += 2) {
      const uint32_t k = static_cast<uint32_t>(i) & (kRing - 1);   // even: k, k + 1 < kRing
      const uint8_t* slot = ring + k * sbytes;
      cp_async_wait<kRing - 2>();
      __syncwarp();
      float acc_a[4] = {0.f, 0.f, 0.f, 0.f};
      float acc_b[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < kCL; ++c) {
        core_chunk(slot, c, lane, zf, acc_a);
        core_chunk(slot + sbytes, c, lane, zf, acc_b);
      }
      core_finish(slot, gr, cbc, unscale, acc_a);
      core_finish(slot + sbytes, gr, cbc, unscale, acc_b);
      __syncwarp();   // every lane is done reading both slots
      if (i + kRing < n_my) issue_core(ring_s + k * sbytes, g_nib, g_hi, g_sl, nch, hi_lane, sl_lane);
      cp_async_commit();
      if (i + 1 + kRing < n_my)
        issue_core(ring_s + (k + 1) * sbytes, g_nib + stride, g_hi + stride, g_sl + stride, nch, hi_lane, sl_lane);
      cp_async_commit();
      g_nib += 2 * stride;
      g_hi += 2 * stride;
      g_sl += 2 * stride;
      if ((i & (p.mg - 1)) == 0) tile = group_begin(sv, p, i, cw, lane);
      store_partial(tile, p, i, lane, acc_a);
      group_end(sv, p, i, n_my, lane);
      if (((i + 1) & (p.mg - 1)) == 0) tile = group_begin(sv, p, i + 1, cw, lane);
      store_partial(tile, p, i + 1, lane, acc_b);
      group_end(sv, p, i + 1, n_my, lane);
    }
  }
  for (; i < n_my; ++i) {
    if ((i & (p.mg - 1)) == 0) tile = group_begin(sv, p, i, cw, lane);
    const uint32_t k = static_cast<uint32_t>(i) & (kRing - 1);
    const uint8_t* slot = ring + k * sbytes;
    cp_async_wait<kRing - 1>();
    __syncwarp();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < kCL; ++c)
      if (c < nch) core_chunk(slot, c, lane, zf, acc);
    core_finish(slot, gr, cbc, unscale, acc);
    __syncwarp();
    if (i + kRing < n_my) issue_core(ring_s + k * sbytes, g_nib, g_hi, g_sl, nch, hi_lane, sl_lane);
    g_nib += stride;
    g_hi += stride;
    g_sl += stride;
    cp_async_commit();
    store_partial(tile, p, i, lane, acc);
    group_end(sv, p, i, n_my, lane);
  }
  cp_async_wait_all();
}

// ---------------------------------------------------------- correction warps
// Ring slice: [kCA x 512 B codes][32 B s_A].
// One m-tile's correction slice for this lane: codes and row scales (lanes 0, 1).
__device__ __forceinline__ void issue_corr(uint32_t dst, const uint8_t* g_codes, const uint8_t* g_sa, int nch,
                                           bool sa_lane) {
#pragma unroll
  for (int c = 0; c < kCA; ++c)
    if (c < nch) cp_async16_hint(dst + c * kAChunkBytes, g_codes + c * kAChunkBytes, l2_evict_first_policy());
  if (sa_lane) cp_async16_hint(dst + kCA * kAChunkBytes, g_sa, l2_evict_first_policy());
}

__device__ void correction_warp(const DecodeParams& p, const SmemView& sv, int n_my, int wa, int cw, int lane) {
  const int gr = lane >> 2;
  const int chunk0 = wa * kCA;
  const int nch = min(kCA, p.n_A - chunk0);
  const uint32_t sbytes = p.corr_slice_bytes;
  uint8_t* ring = sv.rings + p.corr_ring_off + static_cast<size_t>(wa) * kRing * sbytes;
  const uint32_t ring_s = smem_addr(ring) + lane * 16;
  const size_t stride = static_cast<size_t>(gridDim.x) * p.mblk_bytes;
  const uint8_t* base = p.mtiles + static_cast<size_t>(blockIdx.x) * p.mblk_bytes;
  const uint8_t* g_codes = base + p.off_A + chunk0 * kAChunkBytes + lane * 16;
  const uint8_t* g_sa = base + p.off_sA + lane * 16;
  const bool sa_lane = lane < 2;
#pragma unroll
  for (int k = 0; k < kRing; ++k) {
    if (k < n_my) issue_corr(ring_s + k * sbytes, g_codes + k * stride, g_sa + k * stride, nch, sa_lane);
    cp_async_commit();
  }
  g_codes += kRing * stride;
  g_sa += kRing * stride;
  grid_dependency_wait();
  const bool tok = gr < p.nt;
  uint32_t zf[kCA][2][2][2];
  float cb = 0.f;
  const uint16_t* zh = p.zhi + static_cast<size_t>(p.t0 + (tok ? gr : 0)) * p.Kz;
  const uint16_t* zl = p.zlo + static_cast<size_t>(p.t0 + (tok ? gr : 0)) * p.Kz;
#pragma unroll
  for (int c = 0; c < kCA; ++c) {
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int k0 = p.rcp + (chunk0 + c) * kAChunkK + s * 16;
      const bool ok = tok && c < nch;
      load_b_frag_f16(zh, k0, lane, ok, zf[c][s][0][0], zf[c][s][0][1]);
      load_b_frag_f16(zl, k0, lane, ok, zf[c][s][1][0], zf[c][s][1][1]);
      cb += bias_dot(zf[c][s][0][0], zf[c][s][0][1], kInt8Offset, kInt8Offset);
      cb += bias_dot(zf[c][s][1][0], zf[c][s][1][1], kInt8Offset, kInt8Offset);
    }
  }
  const float2 cbc = column_pair(quad_sum(cb), lane);
  const float zs = tok ? ldexpf(1.f, p.escale[p.t0 + gr] + p.e_B - kScaleExp) : 0.f;
  const float2 unscale = column_pair(zs, lane);

  float* tile = nullptr;
  for (int i = 0; i < n_my; ++i) {
    if ((i & (p.mg - 1)) == 0) tile = group_begin(sv, p, i, cw, lane);
    const uint32_t k = static_cast<uint32_t>(i) & (kRing - 1);
    const uint8_t* slot = ring + k * sbytes;
    cp_async_wait<kRing - 1>();
    __syncwarp();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < kCA; ++c) {
      if (c < nch) {
        const uint4 w = *reinterpret_cast<const uint4*>(slot + c * kAChunkBytes + lane * 16);
        uint32_t a[4];
        unpack_int8_biased(w.x, w.y, a);
        mma_f16_16816(acc, a, zf[c][0][0][0], zf[c][0][0][1]);
        mma_f16_16816(acc, a, zf[c][0][1][0], zf[c][0][1][1]);
        unpack_int8_biased(w.z, w.w, a);
        mma_f16_16816(acc, a, zf[c][1][0][0], zf[c][1][0][1]);
        mma_f16_16816(acc, a, zf[c][1][1][0], zf[c][1][1][1]);
      }
    }
    const float2 sc =
        half2_bits_to_float2(*reinterpret_cast<const uint32_t*>(slot + kCA * kAChunkBytes + gr * 4));
    acc[0] = (acc[0] - cbc.x) * (sc.x * unscale.x);
    acc[1] = (acc[1] - cbc.y) * (sc.x * unscale.y);
    acc[2] = (acc[2] - cbc.x) * (sc.y * unscale.x);
    acc[3] = (acc[3] - cbc.y) * (sc.y * unscale.y);
    __syncwarp();
    if (i + kRing < n_my) issue_corr(ring_s + k * sbytes, g_codes, g_sa, nch, sa_lane);
    g_codes += stride;
    g_sa += stride;
    cp_async_commit();
    store_partial(tile, p, i, lane, acc);
    group_end(sv, p, i, n_my, lane);
  }
  cp_async_wait_all();
}

// ----------------------------------------------------------- epilogue warps
// kEpiWarps warps share each group tile: lane l of epilogue warp ew holds the
// two adjacent elements e, e + 1 with e = 2 (32 ew + l) of every group (same
// token, rows r and r + 1), so a lane keeps one running state and reads each
// warp's region with one 8-byte load.
static_assert(kGroupTile * 16 == 64 * kEpiWarps, "two elements per epilogue lane");
static_assert(4 * kEpiWarps >= kDecodeTokens, "every token of a launch has an epilogue octet");
// kShared: the last block merges on both epilogue warps (launches of three or
// more tokens); otherwise on one.  Two instances, so that the code of one
// path does not change the other's (the one-token kernel measured ~6 us slower
// with both paths compiled into it).
// The prologue resets the completion ticket (after the previous launch on the
// workspace is done with it), so the ticket may be taken only once the
// prologue grid is complete.  The core and correction warps wait for that
// grid (griddepcontrol.wait) before they produce a partial, and the epilogue
// takes the ticket after it has consumed every partial of the block, so a
// second wait is needed only when the block has no such warp or no m-tile.
__device__ __forceinline__ bool ticket_needs_wait(const DecodeParams& p, int n_my) {
  return p.nw_work == p.nw_res || n_my == 0;
}

// The block's partial of token t, from the octets q = t, t + nt, ... < 8
// merged in increasing q (deterministic), written by lane t of the calling
// warp; the warp barrier orders the stores before lane 0's ticket.
__device__ __forceinline__ void write_block_partials(const DecodeParams& p, const SmemView& sv, int lane) {
  if (lane < p.nt) {
    LseState a = lse_init();
    PickState b = pick_init();
#pragma unroll 1
    for (int q = lane; q < 4 * kEpiWarps; q += p.nt) {
      const float4 s = sv.tokstate[q];
      a = lse_merge(a, LseState{s.x, s.y, __float_as_int(s.z)});
      const float2 r = sv.pickstate[q];
      b = pick_merge(b, PickState{r.x, __float_as_int(r.y)});
    }
    const size_t at = static_cast<size_t>(p.t0 + lane) * gridDim.x + blockIdx.x;
    p.partials[at] = make_float4(a.m, a.s, __int_as_float(a.idx), 0.f);
    if (p.sampled != nullptr) p.spart[at] = make_float2(b.z, __int_as_float(b.idx));
  }
  __syncwarp();
}

template <bool kShared>
__device__ void epilogue_warp(const DecodeParams& p, const SmemView& sv, int n_my, int ew, int lane) {
  const int e = 2 * (32 * ew + lane);
  LseState st = lse_init();
  PickState pk = pick_init();   // sampling: first maximum of y / tau + G
  // target as a local row (a target in another vocabulary shard never matches)
  const int target = p.targets != nullptr ? p.targets[p.t0 + (e >> 4) % p.nt] - p.row0 : -1;
  const int m = e / (16 * p.nt);            // m-tile of the group, token t, rows r, r + 1
  const int t = (e >> 4) - m * p.nt, row = e & 15;
  const int ngroups = (n_my + p.mg - 1) >> p.mg_log2;
  // Test hook: a wait on a barrier that nothing completes runs out its limit,
  // raises the timeout status and aborts the block.
  if (p.test_stall) warp_wait(sv, sv.stall, 0, p.status, lane, p.wait_limit_ns);
  for (int grp = 0; grp < ngroups; ++grp) {
    const int r = grp & (p.slots - 1);
    const bool ok = warp_wait(sv, &sv.reduced[r], (grp >> p.slots_log2) & 1, p.status, lane, p.wait_limit_ns);
    const float* part = sv.part + r * p.nw_work * (kGroupTile * 16) + e;
    const int i0 = grp << p.mg_log2;
    if (ok && m < p.mg && i0 + m < n_my) {
      // warp-order sums, two independent chains per element
      float2 ya = make_float2(0.f, 0.f), yb = make_float2(0.f, 0.f);
      int w = 0;
      for (; w + 2 <= p.nw_work; w += 2) {
        const float2 qa = *reinterpret_cast<const float2*>(part + (w + 0) * (kGroupTile * 16));
        const float2 qb = *reinterpret_cast<const float2*>(part + (w + 1) * (kGroupTile * 16));
        ya.x += qa.x;
        ya.y += qa.y;
        yb.x += qb.x;
        yb.y += qb.y;
      }
      if (w < p.nw_work) {
        const float2 qa = *reinterpret_cast<const float2*>(part + w * (kGroupTile * 16));
        ya.x += qa.x;
        ya.y += qa.y;
      }
      const float y0 = ya.x + yb.x, y1 = ya.y + yb.y;
      const int v = mtile_of(i0 + m) * kMT + row;
      if (p.sampled != nullptr) {
        // Rows v, v + 1 (global row even: shards start on 16-row boundaries)
        // share one Philox block of four words.
        const uint64_t vg = static_cast<uint64_t>(p.row0 + v);
        uint64_t w[4];
        philox4x64_10(p.ctr0 + static_cast<uint64_t>(p.t0 + t), vg >> 2, p.seed, w);
        const bool upper = (vg & 2u) != 0;
        if (v < p.V) pick_push(pk, fmaf(y0, p.inv_temp, gumbel_of(upper ? w[2] : w[0])), p.row0 + v);
        if (v + 1 < p.V) pick_push(pk, fmaf(y1, p.inv_temp, gumbel_of(upper ? w[3] : w[1])), p.row0 + v + 1);
      }
      if (v < p.V) {
        lse_push(st, y0, v);
        if (v == target) p.tgt[p.t0 + t] = y0;
      }
      if (v + 1 < p.V) {
        lse_push(st, y1, v + 1);
        if (v + 1 == target) p.tgt[p.t0 + t] = y1;
      }
      if (p.logits != nullptr && v < p.V) {
        // The row pair in one 8-byte store where it is aligned (a warp then
        // writes 256 contiguous bytes, also when the logits live in host memory).
        float* dst = p.logits + static_cast<size_t>(p.t0 + t) * p.V + v;
        if (v + 1 < p.V && (reinterpret_cast<uintptr_t>(dst) & 7u) == 0) {
          *reinterpret_cast<float2*>(dst) = make_float2(y0, y1);
        } else {
          dst[0] = y0;
          if (v + 1 < p.V) dst[1] = y1;
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&sv.redfree[r]));
  }
  // Merge each octet of lanes (16 rows of one token; octet q = 4 ew + lane / 8
  // carries token q mod nt) and leave its state in shared memory.  The code
  // from here on runs once per launch, after the packed head has streamed
  // through L2, so its instructions are fetched cold: its loops stay rolled.
#pragma unroll 1
  for (int o = 4; o >= 1; o >>= 1) {
    st = lse_merge(st, lse_shfl_xor(st, o));
    pk = pick_merge(pk, pick_shfl_xor(pk, o));
  }
  if ((lane & 7) == 0) {
    sv.tokstate[4 * ew + (lane >> 3)] = make_float4(st.m, st.s, __int_as_float(st.idx), 0.f);
    sv.pickstate[4 * ew + (lane >> 3)] = make_float2(pk.z, __int_as_float(pk.idx));
  }
  named_bar_sync(1, kEpiWarps * 32);
  if constexpr (!kShared) {
    // One warp writes the block's partials, takes the ticket and, in the last
    // block, merges.
    if (ew != 0) return;
    if (ticket_needs_wait(p, n_my)) grid_dependency_wait();
    write_block_partials(p, sv, lane);
    unsigned prev = 0;
    if (lane == 0) prev = ticket_acq_rel(p.counter);
    prev = __shfl_sync(0xffffffffu, prev, 0);
    if (prev != gridDim.x - 1) return;
    __syncwarp();   // the lanes' loads below come after lane 0's acquire

    // Last block: merge the per-block partials of every token of this launch.
    // A lane issues all of its loads of a round (kMergeLoadsOne partials) before
    // merging any, so a 148-block grid costs one L2 round trip, not five.
    const int nblk = static_cast<int>(gridDim.x);
    for (int t = 0; t < p.nt; ++t) {
      const float4* part = p.partials + static_cast<size_t>(p.t0 + t) * gridDim.x;
      LseState a = lse_init();
      for (int b0 = 0; b0 < nblk; b0 += 32 * kMergeLoadsOne) {
        float4 q[kMergeLoadsOne];
#pragma unroll
        for (int u = 0; u < kMergeLoadsOne; ++u) {
          const int b = b0 + lane + 32 * u;
          q[u] = b < nblk ? __ldcg(part + b) : make_float4(-INFINITY, 0.f, __int_as_float(0x7fffffff), 0.f);
        }
#pragma unroll
        for (int u = 0; u < kMergeLoadsOne; ++u) a = lse_merge(a, LseState{q[u].x, q[u].y, __float_as_int(q[u].z)});
      }
#pragma unroll 1
      for (int m = 16; m >= 1; m >>= 1) a = lse_merge(a, lse_shfl_xor(a, m));
      if (p.sampled != nullptr) {
        const float2* sp = p.spart + static_cast<size_t>(p.t0 + t) * gridDim.x;
        PickState b = pick_init();
        for (int b0 = 0; b0 < nblk; b0 += 32 * kMergeLoadsOne) {
          float2 q[kMergeLoadsOne];
#pragma unroll
          for (int u = 0; u < kMergeLoadsOne; ++u) {
            const int blk = b0 + lane + 32 * u;
            q[u] = blk < nblk ? __ldcg(sp + blk) : make_float2(-INFINITY, __int_as_float(0x7fffffff));
          }
#pragma unroll
          for (int u = 0; u < kMergeLoadsOne; ++u) b = pick_merge(b, PickState{q[u].x, __float_as_int(q[u].y)});
        }
#pragma unroll 1
        for (int m = 16; m >= 1; m >>= 1) b = pick_merge(b, pick_shfl_xor(b, m));
        if (lane == 0) p.sampled[p.t0 + t] = b.idx;
      }
      if (lane == 0) {
        const int tg = p.t0 + t;
        const float lse = a.m + logf(a.s);
        const int gidx = a.idx + p.row0;
        // target logit when the target row is one of this head's rows
        const int tl = p.targets != nullptr ? p.targets[tg] - p.row0 : -1;
        const float tgt = (tl >= 0 && tl < p.V) ? __ldcg(p.tgt + tg) : __int_as_float(0x7fc00000);
        if (p.lse != nullptr) p.lse[tg] = lse;
        if (p.argmax != nullptr) p.argmax[tg] = gidx;
        if (p.ce != nullptr) p.ce[tg] = lse - tgt;
        if (p.shard_out != nullptr) p.shard_out[tg] = make_float4(lse, a.m, __int_as_float(gidx), tgt);
      }
    }
    if (lane == 0) *p.counter = 0u;
    return;
  }
  if (ew == 0) {
    if (ticket_needs_wait(p, n_my)) grid_dependency_wait();
    write_block_partials(p, sv, lane);
    if (lane == 0) sv.flags[1] = ticket_acq_rel(p.counter) == gridDim.x - 1 ? 1 : 0;
  }
  named_bar_sync(1, kEpiWarps * 32);   // also orders both warps' loads below after the acquire
  if (*reinterpret_cast<volatile int*>(&sv.flags[1]) == 0) return;

  // Last block: merge the per-block partials of every token of this launch.
  // The tokens are split over the epilogue warps, two per warp per round, and
  // a lane issues all of its loads of a round before merging any, so a
  // 148-block grid costs one L2 round trip per round (not one per partial).
  const int nblk = static_cast<int>(gridDim.x);
  for (int tp = ew; tp < p.nt; tp += 2 * kEpiWarps) {
    const int tq = tp + kEpiWarps;   // the round's second token (may be past nt)
    const bool two = tq < p.nt;
    const float4* part0 = p.partials + static_cast<size_t>(p.t0 + tp) * gridDim.x;
    const float4* part1 = p.partials + static_cast<size_t>(p.t0 + (two ? tq : tp)) * gridDim.x;
    LseState a0 = lse_init(), a1 = lse_init();
    for (int b0 = 0; b0 < nblk; b0 += 32 * kMergeLoads) {
      float4 q0[kMergeLoads], q1[kMergeLoads];
#pragma unroll
      for (int u = 0; u < kMergeLoads; ++u) {
        const int b = b0 + lane + 32 * u;
        const float4 none = make_float4(-INFINITY, 0.f, __int_as_float(0x7fffffff), 0.f);
        q0[u] = b < nblk ? __ldcg(part0 + b) : none;
        q1[u] = (two && b < nblk) ? __ldcg(part1 + b) : none;
      }
#pragma unroll
      for (int u = 0; u < kMergeLoads; ++u) {
        a0 = lse_merge(a0, LseState{q0[u].x, q0[u].y, __float_as_int(q0[u].z)});
        a1 = lse_merge(a1, LseState{q1[u].x, q1[u].y, __float_as_int(q1[u].z)});
      }
    }
#pragma unroll 1
    for (int m = 16; m >= 1; m >>= 1) {
      a0 = lse_merge(a0, lse_shfl_xor(a0, m));
      a1 = lse_merge(a1, lse_shfl_xor(a1, m));
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int t = k == 0 ? tp : tq;
      if (k == 1 && !two) break;
      const LseState a = k == 0 ? a0 : a1;
      if (p.sampled != nullptr) {
        const float2* sp = p.spart + static_cast<size_t>(p.t0 + t) * gridDim.x;
        PickState b = pick_init();
        for (int b0 = 0; b0 < nblk; b0 += 32 * kMergeLoads) {
          float2 q[kMergeLoads];
#pragma unroll
          for (int u = 0; u < kMergeLoads; ++u) {
            const int blk = b0 + lane + 32 * u;
            q[u] = blk < nblk ? __ldcg(sp + blk) : make_float2(-INFINITY, __int_as_float(0x7fffffff));
          }
#pragma unroll
          for (int u = 0; u < kMergeLoads; ++u) b = pick_merge(b, PickState{q[u].x, __float_as_int(q[u].y)});
        }
#pragma unroll 1
        for (int m = 16; m >= 1; m >>= 1) b = pick_merge(b, pick_shfl_xor(b, m));
        if (lane == 0) p.sampled[p.t0 + t] = b.idx;
      }
      if (lane == 0) {
        const int tg = p.t0 + t;
        const float lse = a.m + logf(a.s);
        const int gidx = a.idx + p.row0;
        // target logit when the target row is one of this head's rows
        const int tl = p.targets != nullptr ? p.targets[tg] - p.row0 : -1;
        const float tgt = (tl >= 0 && tl < p.V) ? __ldcg(p.tgt + tg) : __int_as_float(0x7fc00000);
        if (p.lse != nullptr) p.lse[tg] = lse;
        if (p.argmax != nullptr) p.argmax[tg] = gidx;
        if (p.ce != nullptr) p.ce[tg] = lse - tgt;
        if (p.shard_out != nullptr) p.shard_out[tg] = make_float4(lse, a.m, __int_as_float(gidx), tgt);
      }
    }
  }
  if (lane == 0) *p.counter = 0u;
}

}  // namespace

template <int G, bool kShared>
__global__ void __launch_bounds__(kMaxDecodeWarps * 32, 1) decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const SmemView sv = smem_view(smem, p);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_my = (p.n_mtiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                   static_cast<int>(gridDim.x);
  if (threadIdx.x == 0) {
    for (int r = 0; r < p.slots; ++r) {
      mbar_init(smem_addr(&sv.reduced[r]), p.nw_work);
      mbar_init(smem_addr(&sv.redfree[r]), kEpiWarps);
    }
    mbar_init(smem_addr(sv.stall), 1);
    sv.flags[0] = 0;
    mbar_fence_init();
  }
  __syncthreads();

  if (warp < kEpiWarps) {
    epilogue_warp<kShared>(p, sv, n_my, warp, lane);
    return;
  }
  const int cw = warp - kEpiWarps;
  if (cw < p.nw_res) {
    residual_warp<G>(p, sv, n_my, cw, cw, lane);
  } else if (cw < p.nw_res + p.nw_L) {
    core_warp(p, sv, n_my, cw - p.nw_res, cw, lane);
  } else if (cw < p.nw_work) {
    correction_warp(p, sv, n_my, cw - p.nw_res - p.nw_L, cw, lane);
  }
}

// Shared-memory plan of one launch (host side): ring slices per role.
void decode_smem_plan(DecodeParams& p, int g_steps) {
  const int g = g_steps * 16;
  const int span = kCRes * kResChunkK;                       // columns of one residual warp
  const int ng = (g >= span) ? 2 : span / g;                 // groups a warp's columns can touch
  p.res_slice_bytes = kCRes * kResChunkBytes + ng * kSresGroupBytes;
  p.core_slice_bytes = kCL * (kLNibChunkBytes + kLHiChunkBytes) + 32;
  p.corr_slice_bytes = kCA * kAChunkBytes + 32;
  p.core_ring_off = static_cast<uint32_t>(p.nw_res) * kRing * p.res_slice_bytes;
  p.corr_ring_off = p.core_ring_off + static_cast<uint32_t>(p.nw_L) * kRing * p.core_slice_bytes;
  p.ring_bytes = p.corr_ring_off + static_cast<uint32_t>(p.nw_A) * kRing * p.corr_slice_bytes;
}

size_t decode_smem_bytes(const DecodeParams& p) {
  return static_cast<size_t>(p.ring_bytes) + static_cast<size_t>(p.slots) * p.nw_work * kGroupTile * 16 * 4 +
         static_cast<size_t>(2) * p.slots * 8 + kEpiWarps * kDecodeTokens * (16 + 8) + 8 + 16;
}

namespace {
template <int G>
const void* kernel_ptr(bool shared) {
  return shared ? reinterpret_cast<const void*>(&decode_kernel<G, true>)
                : reinterpret_cast<const void*>(&decode_kernel<G, false>);
}
const void* kernel_for(int g_steps, bool shared) {
  switch (g_steps) {
    case 1: return kernel_ptr<1>(shared);
    case 2: return kernel_ptr<2>(shared);
    case 4: return kernel_ptr<4>(shared);
    case 8: return kernel_ptr<8>(shared);
    default: return kernel_ptr<16>(shared);
  }
}
}  // namespace

cudaError_t decode_set_attributes(int g_steps, size_t smem) {
  cudaError_t e = cudaFuncSetAttribute(kernel_for(g_steps, false), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kernel_for(g_steps, true), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
  return e;
}

cudaError_t launch_decode(int g_steps, const DecodeParams& p, int grid, size_t smem, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3((kEpiWarps + p.nw_work) * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[] = {const_cast<DecodeParams*>(&p)};
  return cudaLaunchKernelExC(&cfg, kernel_for(g_steps, p.nt > 2), args);
}

}  // namespace archead
