// Decode kernel: the packed-head forward (ARCHead paper, §3.2 Eq. 7) for up
// to 8 tokens per launch, streaming the packed head once from HBM.
//
// Per vocabulary row v and token t it forms
//   y[t,v] = sum_g s_res[v,g] (sum_{j in g} q[v,j] h[t,j])          residual (SC4)
//          + s_L[v] sum_k L[v,k] z_c[t,k]                         core (Eq. 3)
//          + s_A[v] sum_k A[v,k] z_r[t,k]                         correction (Eq. 4-6)
// with z_c, z_r from the prologue kernel.  Codes are unpacked in registers to
// exact fp16 values (bias + offset code) and multiplied on the tensor cores
// (m16n8k16: vocabulary rows as M, tokens as N, fp32 accumulation).  The bias
// is removed once per scale group in fp32 with a per-token constant computed
// from the same fp16 operands, and the fp16 group / row scales multiply fp32
// partial sums, so no scaled weight is ever rounded.  h enters as fp16 scaled
// by a per-token power of two (exact for bf16 inputs); z as an fp16 pair
// (high part + remainder) under its own power of two.
//
// Block organisation (one block per SM, persistent over m-tiles; no block-wide
// barrier after setup):
//   warp 0            producer: bulk-copies whole m-tile blocks HBM -> SMEM
//                     into a ring of `stages` buffers (full[s]); a buffer is
//                     refilled as soon as every compute warp has read it
//                     (empty[s]), independent of the epilogue
//   warp 1            epilogue: takes the summed 16 x nt logit tile of a slot
//                     (reduced[r]), pushes each logit into a running
//                     log-sum-exp / argmax state, writes logits when asked,
//                     clears the slot and frees it                (redfree[r])
//   residual warps    each owns 16 k16 steps of d for every m-tile; the fp16
//                     h fragments of its columns stay in registers
//   core warps        each owns kCL 64-column chunks of r_c'
//   correction warps  each owns kCA 32-column chunks of r_r'
// Each compute warp adds its 16 x nt partial logits into a fixed-point slot
// tile (integer adds: same bits in any order) and signals the epilogue warp;
// no warp ever waits for another to finish an m-tile.  At the end every block writes one partial per token; the last block to
// finish (atomic ticket, no spinning) merges them into LSE, argmax and CE.
// Every wait on an mbarrier is bounded (kWaitLimitNs); on expiry the block
// raises ARCHEAD_STATUS_WAIT_TIMEOUT, skips the remaining work and drains its
// copies before exiting.
#include <cuda_runtime.h>

#include "device.cuh"
#include "params.h"

namespace archead {

namespace {

constexpr int kEpiSlots = 4;     // 16 rows x 8 tokens / 32 lanes

struct SmemView {
  uint8_t* stages;
  unsigned long long* tsum;  // [slots][nt][16 rows] fixed-point logit sums
  uint64_t* full;      // [stages] producer -> compute warps (bytes landed)
  uint64_t* empty;     // [stages] compute warps -> producer (stage read)
  uint64_t* reduced;   // [slots]  compute warps -> epilogue warp
  uint64_t* redfree;   // [slots]  epilogue warp -> compute warps
  int* flags;          // [0] abort
};

__device__ __forceinline__ SmemView smem_view(uint8_t* smem, const DecodeParams& p) {
  SmemView v;
  const size_t tile = static_cast<size_t>(p.nt) * 16;
  v.stages = smem;
  v.tsum = reinterpret_cast<unsigned long long*>(smem + static_cast<size_t>(p.stages) * p.mblk_bytes);
  v.full = reinterpret_cast<uint64_t*>(v.tsum + static_cast<size_t>(p.slots) * tile);
  v.empty = v.full + p.stages;
  v.reduced = v.empty + p.stages;
  v.redfree = v.reduced + p.slots;
  v.flags = reinterpret_cast<int*>(v.redfree + p.slots);
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
                                          int lane) {
  bool ok = !aborted(sv) && mbar_wait(smem_addr(bar), parity);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && lane == 0 && !aborted(sv)) raise_timeout(sv, status);
  return ok;
}

__device__ __forceinline__ int mtile_of(int i) { return static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x); }

// ----------------------------------------------------------------- producer
__device__ void producer(const DecodeParams& p, const SmemView& sv, int n_my) {
  const int S = p.stages;
  int issued = 0;
  for (int i = 0; i < n_my; ++i) {
    const int s = i % S;
    const int u = i / S;
    if (aborted(sv)) break;
    if (u > 0 && !mbar_wait(smem_addr(&sv.empty[s]), (u - 1) & 1)) {
      raise_timeout(sv, p.status);
      break;
    }
    const uint32_t full = smem_addr(&sv.full[s]);
    mbar_arrive_expect_tx(full, p.mblk_bytes);
    const uint8_t* src = p.mtiles + static_cast<size_t>(mtile_of(i)) * p.mblk_bytes;
    const uint32_t dst = smem_addr(sv.stages + static_cast<size_t>(s) * p.mblk_bytes);
    for (uint32_t off = 0; off < p.mblk_bytes; off += 16384u) {
      const uint32_t n = min(16384u, p.mblk_bytes - off);
      bulk_copy_g2s(dst + off, src + off, n, full);
    }
    ++issued;
  }
  // Every issued copy must have landed before this block may exit.
  for (int i = max(0, issued - S); i < issued; ++i) {
    if (!mbar_wait(smem_addr(&sv.full[i % S]), (i / S) & 1)) raise_timeout(sv, p.status);
  }
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

// sum over the fp16 pair of bias_lo * (x + y) for b0 and bias_hi * (x + y) for b1.
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

// Logit partial sums of the compute warps meet in a fixed-point tile: each
// value is rounded to a multiple of 2^-32 (error <= 2^-33, far below the
// logit tolerance) and added as a 64-bit integer.  Integer addition is
// associative, so the tile holds the same bits whatever the order in which the
// warps arrive.  |partial| < 2^31 is assumed (the conversion saturates).
constexpr float kFixScale = 4294967296.0f;   // 2^32

__device__ __forceinline__ void add_partial(const SmemView& sv, const DecodeParams& p, int r, int lane,
                                            const float (&acc)[4]) {
  const int gr = lane >> 2, cc = lane & 3;
  unsigned long long* tile = sv.tsum + static_cast<size_t>(r) * p.nt * 16;
  const int t0 = 2 * cc;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int t = t0 + j;
    if (t < p.nt) {
      const long long lo = __float2ll_rn(acc[j] * kFixScale);
      const long long hi = __float2ll_rn(acc[2 + j] * kFixScale);
      atomicAdd(tile + t * 16 + gr, static_cast<unsigned long long>(lo));
      atomicAdd(tile + t * 16 + gr + 8, static_cast<unsigned long long>(hi));
    }
  }
}

// End of one m-tile for a compute warp: release the stage buffer, add the
// partial logits into slot r (after the epilogue has drained the slot's
// previous use) and report to the epilogue warp.
__device__ __forceinline__ void finish_mtile(const SmemView& sv, const DecodeParams& p, int i, int s, int lane,
                                             const float (&acc)[4]) {
  __syncwarp();
  if (lane == 0) mbar_arrive(smem_addr(&sv.empty[s]));
  const int r = i % p.slots;
  if (i >= p.slots) warp_wait(sv, &sv.redfree[r], ((i / p.slots) - 1) & 1, p.status, lane);
  add_partial(sv, p, r, lane, acc);
  __syncwarp();
  if (lane == 0) mbar_arrive(smem_addr(&sv.reduced[r]));
}

// ------------------------------------------------------------ residual warps
// G = k16 steps per scale group within the warp's 16 steps (16 when a group
// spans the whole warp range or more).
template <int G>
__device__ void residual_warp(const DecodeParams& p, const SmemView& sv, int n_my, int wres, int cw, int lane) {
  constexpr int kNG = 16 / G;    // local scale groups
  const int gr = lane >> 2;
  const int S = p.stages;
  const bool tok = gr < p.nt;
  float hs = 0.f;
  if (tok) hs = ldexpf(1.f, kScaleExp - p.escale[p.t0 + gr]);
  // fp16 h fragments of this warp's columns, and the bias constant of each
  // local group for token gr.
  uint32_t hf[kCRes][4][2];
  float cg[kNG];
#pragma unroll
  for (int g = 0; g < kNG; ++g) cg[g] = 0.f;
  const uint16_t* hrow = p.hidden + static_cast<size_t>(p.t0 + (tok ? gr : 0)) * p.d;
#pragma unroll
  for (int c = 0; c < kCRes; ++c) {
    const int chunk = wres * kCRes + c;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      uint32_t b[2] = {0u, 0u};
      if (tok && chunk < p.n_res) {
        const uint16_t* r = hrow + chunk * kResChunkK + s * 16 + 2 * (lane & 3);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint32_t bits = *reinterpret_cast<const uint32_t*>(r + 8 * j);
          const float lo = __uint_as_float(bits << 16) * hs;
          const float hi = __uint_as_float(bits & 0xFFFF0000u) * hs;
          b[j] = pack_half2(lo, hi);
        }
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
  const int last_step = min(16, (p.n_res - wres * kCRes) * 4) - 1;
  const int step0 = wres * 16;

  for (int i = 0; i < n_my; ++i) {
    const int s = i % S;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (warp_wait(sv, &sv.full[s], (i / S) & 1, p.status, lane)) {
      const uint8_t* stg = sv.stages + static_cast<size_t>(s) * p.mblk_bytes;
      float t0[4] = {0.f, 0.f, 0.f, 0.f};
      float t1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < kCRes; ++c) {
        const int chunk = wres * kCRes + c;
        if (chunk < p.n_res) {
          const uint4 nib = *reinterpret_cast<const uint4*>(stg + p.off_res + chunk * kResChunkBytes + lane * 16);
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
              const int grp = (step0 + step) >> p.g_steps_log2;
              const float2 sc = half2_bits_to_float2(
                  *reinterpret_cast<const uint32_t*>(stg + p.off_sres + grp * kSresGroupBytes + gr * 4));
              acc[0] = fmaf(sc.x, tmp[0] - cgc[lg].x, acc[0]);
              acc[1] = fmaf(sc.x, tmp[1] - cgc[lg].y, acc[1]);
              acc[2] = fmaf(sc.y, tmp[2] - cgc[lg].x, acc[2]);
              acc[3] = fmaf(sc.y, tmp[3] - cgc[lg].y, acc[3]);
              tmp[0] = tmp[1] = tmp[2] = tmp[3] = 0.f;
            }
          }
        }
      }
      acc[0] *= unscale.x;
      acc[1] *= unscale.y;
      acc[2] *= unscale.x;
      acc[3] *= unscale.y;
    }
    finish_mtile(sv, p, i, s, lane, acc);
  }
}

// ---------------------------------------------------------------- core warps
__device__ void core_warp(const DecodeParams& p, const SmemView& sv, int n_my, int wl, int cw, int lane) {
  const int gr = lane >> 2;
  const int S = p.stages;
  const bool tok = gr < p.nt;
  uint32_t zf[kCL][4][2][2];
  float cb = 0.f;
  const uint16_t* zh = p.zhi + static_cast<size_t>(p.t0 + (tok ? gr : 0)) * p.Kz;
  const uint16_t* zl = p.zlo + static_cast<size_t>(p.t0 + (tok ? gr : 0)) * p.Kz;
#pragma unroll
  for (int c = 0; c < kCL; ++c) {
    const int chunk = wl * kCL + c;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int k0 = chunk * kLChunkK + s * 16;
      const bool ok = tok && chunk < p.n_L;
      load_b_frag_f16(zh, k0, lane, ok, zf[c][s][0][0], zf[c][s][0][1]);
      load_b_frag_f16(zl, k0, lane, ok, zf[c][s][1][0], zf[c][s][1][1]);
      cb += bias_dot(zf[c][s][0][0], zf[c][s][0][1], kBiasLo + 16.f, kBiasHi + 16.f);
      cb += bias_dot(zf[c][s][1][0], zf[c][s][1][1], kBiasLo + 16.f, kBiasHi + 16.f);
    }
  }
  const float2 cbc = column_pair(quad_sum(cb), lane);
  const float zs = tok ? ldexpf(1.f, p.escale[p.t0 + gr] + p.e_B - kScaleExp) : 0.f;
  const float2 unscale = column_pair(zs, lane);

  for (int i = 0; i < n_my; ++i) {
    const int s = i % S;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (warp_wait(sv, &sv.full[s], (i / S) & 1, p.status, lane)) {
      const uint8_t* stg = sv.stages + static_cast<size_t>(s) * p.mblk_bytes;
      bool any = false;
#pragma unroll
      for (int c = 0; c < kCL; ++c) {
        const int chunk = wl * kCL + c;
        if (chunk < p.n_L) {
          any = true;
          const uint4 nib = *reinterpret_cast<const uint4*>(stg + p.off_Lnib + chunk * kLNibChunkBytes + lane * 16);
          const uint32_t hb = *reinterpret_cast<const uint32_t*>(stg + p.off_Lhi + chunk * kLHiChunkBytes + lane * 4);
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
      }
      if (any) {
        const float2 sc = half2_bits_to_float2(*reinterpret_cast<const uint32_t*>(stg + p.off_sL + gr * 4));
        acc[0] = (acc[0] - cbc.x) * (sc.x * unscale.x);
        acc[1] = (acc[1] - cbc.y) * (sc.x * unscale.y);
        acc[2] = (acc[2] - cbc.x) * (sc.y * unscale.x);
        acc[3] = (acc[3] - cbc.y) * (sc.y * unscale.y);
      }
    }
    finish_mtile(sv, p, i, s, lane, acc);
  }
}

// ---------------------------------------------------------- correction warps
__device__ void correction_warp(const DecodeParams& p, const SmemView& sv, int n_my, int wa, int cw, int lane) {
  const int gr = lane >> 2;
  const int S = p.stages;
  const bool tok = gr < p.nt;
  uint32_t zf[kCA][2][2][2];
  float cb = 0.f;
  const uint16_t* zh = p.zhi + static_cast<size_t>(p.t0 + (tok ? gr : 0)) * p.Kz;
  const uint16_t* zl = p.zlo + static_cast<size_t>(p.t0 + (tok ? gr : 0)) * p.Kz;
#pragma unroll
  for (int c = 0; c < kCA; ++c) {
    const int chunk = wa * kCA + c;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int k0 = p.rcp + chunk * kAChunkK + s * 16;
      const bool ok = tok && chunk < p.n_A;
      load_b_frag_f16(zh, k0, lane, ok, zf[c][s][0][0], zf[c][s][0][1]);
      load_b_frag_f16(zl, k0, lane, ok, zf[c][s][1][0], zf[c][s][1][1]);
      cb += bias_dot(zf[c][s][0][0], zf[c][s][0][1], kBiasLo + 128.f, kBiasLo + 128.f);
      cb += bias_dot(zf[c][s][1][0], zf[c][s][1][1], kBiasLo + 128.f, kBiasLo + 128.f);
    }
  }
  const float2 cbc = column_pair(quad_sum(cb), lane);
  const float zs = tok ? ldexpf(1.f, p.escale[p.t0 + gr] + p.e_B - kScaleExp) : 0.f;
  const float2 unscale = column_pair(zs, lane);

  for (int i = 0; i < n_my; ++i) {
    const int s = i % S;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (warp_wait(sv, &sv.full[s], (i / S) & 1, p.status, lane)) {
      const uint8_t* stg = sv.stages + static_cast<size_t>(s) * p.mblk_bytes;
      bool any = false;
#pragma unroll
      for (int c = 0; c < kCA; ++c) {
        const int chunk = wa * kCA + c;
        if (chunk < p.n_A) {
          any = true;
          const uint4 w = *reinterpret_cast<const uint4*>(stg + p.off_A + chunk * kAChunkBytes + lane * 16);
          uint32_t a[4];
          unpack_int8_biased(w.x, w.y, a);
          mma_f16_16816(acc, a, zf[c][0][0][0], zf[c][0][0][1]);
          mma_f16_16816(acc, a, zf[c][0][1][0], zf[c][0][1][1]);
          unpack_int8_biased(w.z, w.w, a);
          mma_f16_16816(acc, a, zf[c][1][0][0], zf[c][1][0][1]);
          mma_f16_16816(acc, a, zf[c][1][1][0], zf[c][1][1][1]);
        }
      }
      if (any) {
        const float2 sc = half2_bits_to_float2(*reinterpret_cast<const uint32_t*>(stg + p.off_sA + gr * 4));
        acc[0] = (acc[0] - cbc.x) * (sc.x * unscale.x);
        acc[1] = (acc[1] - cbc.y) * (sc.x * unscale.y);
        acc[2] = (acc[2] - cbc.x) * (sc.y * unscale.x);
        acc[3] = (acc[3] - cbc.y) * (sc.y * unscale.y);
      }
    }
    finish_mtile(sv, p, i, s, lane, acc);
  }
}

// ------------------------------------------------------------ epilogue warp
__device__ void epilogue_warp(const DecodeParams& p, const SmemView& sv, int n_my, int lane) {
  const int nel = 16 * p.nt;
  LseState st[kEpiSlots];
  int target[kEpiSlots];
#pragma unroll
  for (int k = 0; k < kEpiSlots; ++k) {
    st[k] = lse_init();
    const int e = lane + 32 * k;
    target[k] = (e < nel && p.targets != nullptr) ? p.targets[p.t0 + (e >> 4)] : -1;
  }
  for (int i = 0; i < n_my; ++i) {
    const int r = i % p.slots;
    const bool ok = warp_wait(sv, &sv.reduced[r], (i / p.slots) & 1, p.status, lane);
    unsigned long long* tsum = sv.tsum + static_cast<size_t>(r) * nel;
    const int vbase = mtile_of(i) * kMT;
#pragma unroll
    for (int k = 0; k < kEpiSlots; ++k) {
      const int e = lane + 32 * k;
      if (e < nel) {
        const long long fx = static_cast<long long>(tsum[e]);
        tsum[e] = 0ull;   // ready for the slot's next use
        if (!ok) continue;
        const float y = __ll2float_rn(fx) * (1.0f / kFixScale);
        const int row = e & 15, t = e >> 4;
        const int v = vbase + row;
        if (v < p.V) {
          lse_push(st[k], y, v);
          if (p.logits != nullptr) p.logits[static_cast<size_t>(p.t0 + t) * p.V + v] = y;
          if (v == target[k]) p.tgt[p.t0 + t] = y;
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&sv.redfree[r]));
  }
  // Block partial per token: slot k of lanes 16h..16h+15 holds token 2k + h.
#pragma unroll
  for (int k = 0; k < kEpiSlots; ++k) {
#pragma unroll
    for (int m = 8; m >= 1; m >>= 1) st[k] = lse_merge(st[k], lse_shfl_xor(st[k], m));
    const int t = 2 * k + (lane >> 4);
    if ((lane & 15) == 0 && t < p.nt)
      p.partials[static_cast<size_t>(p.t0 + t) * gridDim.x + blockIdx.x] =
          make_float4(st[k].m, st[k].s, __int_as_float(st[k].idx), 0.f);
  }
  __threadfence();
  __syncwarp();
  unsigned prev = 0;
  if (lane == 0) prev = atomicAdd(p.counter, 1u);
  prev = __shfl_sync(0xffffffffu, prev, 0);
  if (prev != gridDim.x - 1) return;

  // Last block: merge the per-block partials of every token of this launch.
  __threadfence();
  for (int t = 0; t < p.nt; ++t) {
    const float4* part = p.partials + static_cast<size_t>(p.t0 + t) * gridDim.x;
    LseState a = lse_init();
    for (int b = lane; b < static_cast<int>(gridDim.x); b += 32) {
      const float4 q = __ldcg(part + b);
      a = lse_merge(a, LseState{q.x, q.y, __float_as_int(q.z)});
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) a = lse_merge(a, lse_shfl_xor(a, m));
    if (lane == 0) {
      const int tg = p.t0 + t;
      const float lse = a.m + logf(a.s);
      if (p.lse != nullptr) p.lse[tg] = lse;
      if (p.argmax != nullptr) p.argmax[tg] = a.idx;
      if (p.ce != nullptr) {
        const int target_id = p.targets[tg];
        p.ce[tg] = (target_id >= 0 && target_id < p.V) ? lse - __ldcg(p.tgt + tg) : __int_as_float(0x7fc00000);
      }
    }
  }
  if (lane == 0) *p.counter = 0u;
}

}  // namespace

template <int G>
__global__ void __launch_bounds__(kMaxDecodeWarps * 32, 1) decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const SmemView sv = smem_view(smem, p);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_my = (p.n_mtiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                   static_cast<int>(gridDim.x);
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(smem_addr(&sv.full[s]), 1);
      mbar_init(smem_addr(&sv.empty[s]), p.nw_work);
    }
    for (int r = 0; r < p.slots; ++r) {
      mbar_init(smem_addr(&sv.reduced[r]), p.nw_work);
      mbar_init(smem_addr(&sv.redfree[r]), 1);
    }
    for (int e = 0; e < p.slots * p.nt * 16; ++e) sv.tsum[e] = 0ull;
    sv.flags[0] = 0;
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) producer(p, sv, n_my);
    return;
  }
  // Everything below reads the prologue's output or the workspace.
  grid_dependency_wait();
  if (warp == 1) {
    epilogue_warp(p, sv, n_my, lane);
    return;
  }
  const int cw = warp - 2;
  if (cw < p.nw_res) {
    residual_warp<G>(p, sv, n_my, cw, cw, lane);
  } else if (cw < p.nw_res + p.nw_L) {
    core_warp(p, sv, n_my, cw - p.nw_res, cw, lane);
  } else if (cw < p.nw_work) {
    correction_warp(p, sv, n_my, cw - p.nw_res - p.nw_L, cw, lane);
  }
}

size_t decode_smem_bytes(int stages, int slots, uint32_t mblk_bytes, int nw_work, int nt) {
  (void)nw_work;
  return static_cast<size_t>(stages) * mblk_bytes + static_cast<size_t>(slots) * nt * 16 * 8 +
         static_cast<size_t>(2) * stages * 8 + static_cast<size_t>(2) * slots * 8 + 16;
}

namespace {
template <int G>
const void* kernel_ptr() {
  return reinterpret_cast<const void*>(&decode_kernel<G>);
}
const void* kernel_for(int g_steps) {
  switch (g_steps) {
    case 1: return kernel_ptr<1>();
    case 2: return kernel_ptr<2>();
    case 4: return kernel_ptr<4>();
    case 8: return kernel_ptr<8>();
    default: return kernel_ptr<16>();
  }
}
}  // namespace

cudaError_t decode_set_attributes(int g_steps, size_t smem) {
  return cudaFuncSetAttribute(kernel_for(g_steps), cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(smem));
}

cudaError_t launch_decode(int g_steps, const DecodeParams& p, int grid, size_t smem, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3((2 + p.nw_work) * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[] = {const_cast<DecodeParams*>(&p)};
  return cudaLaunchKernelExC(&cfg, kernel_for(g_steps), args);
}

}  // namespace archead
