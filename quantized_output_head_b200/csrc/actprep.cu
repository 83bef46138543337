// Activation operand of the tensor-core forward (ARCHead paper, §3.2 Eq. 7:
// the factored form h·R^T then L, and the correction h·B^T then A).
//
// For a tile of 16 tokens the kernel computes, per token t,
//   E_t with max_j |h[t,j]| < 2^E_t and c_t = kScaleExp - E_t + mseg,
// and writes one fp16 row of the concatenated activation matrix
//   X[t] = [ h[t]·2^(c_t-alpha) | z_c[t]·2^(c_t-beta) | z_r[t]·2^(c_t-gamma) ],
//   z_c[t,k] = s_R[k] sum_j R[k,j] h[t,j],   z_r[t,k] = sum_j s_B[k,j/g_B] B[k,j] h[t,j].
// alpha, beta, gamma put the largest dequantised weight of each segment just
// below 2^kScaleExp; mseg = min(alpha, beta - e_B, gamma - e_B) keeps every
// entry of X below 2^kScaleExp as well (2^e_B bounds the L1 norm of each
// dequantised R and B row), so the product of the two sides is
// y[t,v]·2^c_t with no fp16 overflow.
//
// grid.y = Kz'/64 + 1: blocks y < Kz'/64 compute 64 entries of z for the 16
// tokens with m16n8k16 MMAs (tokens as M, z rows as N, fp16 h scaled by a
// power of two, exact int8 codes as fp16, fp32 accumulation; the group
// scales of B are applied in fp32 at each group end); block y = last
// converts h.  Within every 16-column block X is stored in the column order
// of the dequantised weights in tensor memory (tc_kpos).
//
// grid.z splits the columns of d when there are few tokens, so that the
// short z computation spreads over the SMs: split s scales h by
// 2^(kScaleExp - E_s) with E_s from its own columns, writes its fp32 sums
// and E_s, and the last split to arrive (acquire-release ticket) adds the
// splits in order, each times 2^(E_s - E_t) (E_t = max_s E_s), and writes X.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "device.cuh"
#include "params.h"
#include "tc_params.h"
#include "tcgen05.cuh"

namespace archead {

namespace {

constexpr int kNoExp = -(1 << 20);   // exponent of a split whose columns are all zero

// bf16 pair -> fp16 pair times 2^e (exact while the result is a normal fp16).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t bits, float scale) {
  const float lo = __uint_as_float(bits << 16) * scale;
  const float hi = __uint_as_float(bits & 0xFFFF0000u) * scale;
  return pack_half2(lo, hi);
}

// int8 quadruple (columns c..c+3) -> exact fp16 pairs (c, c+1) and (c+2, c+3).
__device__ __forceinline__ void int8x4_to_f16(uint32_t w, uint32_t& b0, uint32_t& b1) {
  const uint32_t u = w ^ 0x80808080u;   // offset binary: code + 128
  b0 = hsub2_bits(__byte_perm(u, 0x64646464u, 0x4140u), kH2_1152);
  b1 = hsub2_bits(__byte_perm(u, 0x64646464u, 0x4342u), kH2_1152);
}

// One warp's share of the 16-token x 64-row block of z, over 64-column blocks
// [b0, b1) of d.  kCorr: rows of B with group scales (flushed in fp32 at every
// group end); otherwise rows of R (row scale applied by the caller).
// The k order inside an MMA is a permutation of the columns that A and B
// share: lane cc covers columns 16cc..16cc+15 of each 64-column block, step st
// columns 16cc + 4st + 0..3.
template <bool kCorr>
__device__ __forceinline__ void z_block(const ActParams& p, int n0, int b0, int b1, const float (&hs)[2],
                                        const uint16_t* hrow_a, const uint16_t* hrow_b, int lane,
                                        float (&acc)[8][4]) {
  const int gr = lane >> 2, cc = lane & 3;
  const int ngB = p.d / p.g_B;
  float tmp[8][4];
#pragma unroll
  for (int n = 0; n < 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) tmp[n][e] = 0.f;
  const int8_t* rows[8];
#pragma unroll
  for (int n = 0; n < 8; ++n) {
    const int zr = n0 + 8 * n + gr;
    rows[n] = nullptr;
    if (zr < p.Kz) rows[n] = kCorr ? p.B + static_cast<size_t>(zr - p.rcp) * p.d : p.R + static_cast<size_t>(zr) * p.d;
  }
  for (int blk = b0; blk < b1; ++blk) {
    const int c0 = blk * 64 + 16 * cc;
    uint32_t ha[4][4];
    {
      uint4 a0 = make_uint4(0, 0, 0, 0), a1 = a0, b0v = a0, b1v = a0;
      if (hrow_a != nullptr) {
        a0 = *reinterpret_cast<const uint4*>(hrow_a + c0);
        a1 = *reinterpret_cast<const uint4*>(hrow_a + c0 + 8);
      }
      if (hrow_b != nullptr) {
        b0v = *reinterpret_cast<const uint4*>(hrow_b + c0);
        b1v = *reinterpret_cast<const uint4*>(hrow_b + c0 + 8);
      }
      const uint32_t pa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const uint32_t pb[8] = {b0v.x, b0v.y, b0v.z, b0v.w, b1v.x, b1v.y, b1v.z, b1v.w};
#pragma unroll
      for (int st = 0; st < 4; ++st) {
        ha[st][0] = bf16x2_to_f16x2(pa[2 * st], hs[0]);
        ha[st][2] = bf16x2_to_f16x2(pa[2 * st + 1], hs[0]);
        ha[st][1] = bf16x2_to_f16x2(pb[2 * st], hs[1]);
        ha[st][3] = bf16x2_to_f16x2(pb[2 * st + 1], hs[1]);
      }
    }
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      uint4 rv = make_uint4(0, 0, 0, 0);
      if (rows[n] != nullptr) rv = *reinterpret_cast<const uint4*>(rows[n] + c0);
      const uint32_t wv[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
      for (int st = 0; st < 4; ++st) {
        uint32_t bb0, bb1;
        int8x4_to_f16(wv[st], bb0, bb1);
        if constexpr (kCorr) mma_f16_16816(tmp[n], ha[st], bb0, bb1);
        else mma_f16_16816(acc[n], ha[st], bb0, bb1);
      }
    }
    if (kCorr && (((blk + 1) * 64) % p.g_B == 0 || blk + 1 == b1)) {
      const int grp = (blk * 64) / p.g_B;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const int zc = n0 + 8 * n + 2 * cc;
        const float s0 = zc < p.Kz ? __half2float(__ushort_as_half(p.s_B[static_cast<size_t>(zc - p.rcp) * ngB + grp])) : 0.f;
        const float s1 =
            zc + 1 < p.Kz ? __half2float(__ushort_as_half(p.s_B[static_cast<size_t>(zc + 1 - p.rcp) * ngB + grp])) : 0.f;
        acc[n][0] = fmaf(s0, tmp[n][0], acc[n][0]);
        acc[n][1] = fmaf(s1, tmp[n][1], acc[n][1]);
        acc[n][2] = fmaf(s0, tmp[n][2], acc[n][2]);
        acc[n][3] = fmaf(s1, tmp[n][3], acc[n][3]);
        tmp[n][0] = tmp[n][1] = tmp[n][2] = tmp[n][3] = 0.f;
      }
    }
  }
}

}  // namespace

__global__ void __launch_bounds__(256, 1) act_prep_kernel(const ActParams p) {
  __shared__ float red[8][16][64];
  __shared__ int s_E[16];
  __shared__ bool s_nz[16];
  __shared__ int s_Ez[kActMaxSplits][16];
  __shared__ int s_last;
  // The tensor-core kernel may start streaming the packed head right away; it
  // waits (griddepcontrol.wait) before it reads anything written here.
  grid_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * 16;
  const bool conv = blockIdx.y == gridDim.y - 1;
  // 64-column blocks [kb0, kb1) of d: this split's (its share of the h
  // segment for the converting blocks, whose exponents cover all of d)
  const int nb = p.d / 64;
  const int kb0 = static_cast<int>(blockIdx.z) * nb / static_cast<int>(gridDim.z);
  const int kb1 = (static_cast<int>(blockIdx.z) + 1) * nb / static_cast<int>(gridDim.z);
  const int eb0 = conv ? 0 : kb0, eb1 = conv ? nb : kb1;
  if (p.targets != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) {
    for (int t = threadIdx.x; t < p.T; t += blockDim.x) {
      const int v = p.targets[t];
      if (v < 0 || v >= p.v_total) atomicOr(p.status, static_cast<uint32_t>(ARCHEAD_STATUS_BAD_TARGET));
    }
  }
  // E of the tile's tokens over columns [64 eb0, 64 eb1) (E_t for the whole
  // row): |bf16| orders like its bit pattern without the sign.  Warp w takes
  // tokens 2w and 2w + 1, a lane kEU 16-byte pieces of each per round, all
  // loads of a round in flight together.
  constexpr int kEU = 4;
  uint32_t mx[2] = {0u, 0u};
  {
    const uint4* rows[2];
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      const int t = t0 + 2 * warp + tt;
      rows[tt] = t < p.T ? reinterpret_cast<const uint4*>(p.hidden + static_cast<size_t>(t) * p.d) : nullptr;
    }
    for (int i0 = 8 * eb0 + lane; i0 < 8 * eb1; i0 += 32 * kEU) {
      uint4 v[2][kEU];
#pragma unroll
      for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int u = 0; u < kEU; ++u) {
          const int i = i0 + 32 * u;
          v[tt][u] = (rows[tt] != nullptr && i < 8 * eb1) ? rows[tt][i] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
      for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int u = 0; u < kEU; ++u) {
          mx[tt] = __vmaxu2(mx[tt], v[tt][u].x & 0x7FFF7FFFu);
          mx[tt] = __vmaxu2(mx[tt], v[tt][u].y & 0x7FFF7FFFu);
          mx[tt] = __vmaxu2(mx[tt], v[tt][u].z & 0x7FFF7FFFu);
          mx[tt] = __vmaxu2(mx[tt], v[tt][u].w & 0x7FFF7FFFu);
        }
    }
  }
  for (int tt = 0; tt < 2; ++tt) {
    const int tl = 2 * warp + tt;
    const uint32_t m16 = __reduce_max_sync(0xffffffffu, max(mx[tt] & 0xFFFFu, mx[tt] >> 16));
    if (lane == 0) {
      int E = 0;
      if (m16 != 0) frexpf(__uint_as_float(m16 << 16), &E);   // max|h_t| < 2^E
      s_E[tl] = E;
      s_nz[tl] = m16 != 0;
    }
  }
  __syncthreads();

  if (conv) {
    // h segment, 16-column blocks [4 kb0, 4 kb1) of this split:
    // X[t, j] = h[t, j]·2^(c_t - alpha), c_t = kScaleExp - E_t + mseg.
    if (blockIdx.z == 0 && threadIdx.x < 16 && t0 + static_cast<int>(threadIdx.x) < p.T)
      p.cinv[t0 + threadIdx.x] = ldexpf(1.f, s_E[threadIdx.x] - kScaleExp - p.mseg);
    const int nbr = 4 * (kb1 - kb0), n_items = 16 * nbr;
    constexpr int kCU = 2;   // items of a thread in flight together
    for (int item0 = threadIdx.x; item0 < n_items; item0 += kCU * blockDim.x) {
      uint4 lo[kCU], hi[kCU];
#pragma unroll
      for (int u = 0; u < kCU; ++u) {
        const int item = item0 + u * static_cast<int>(blockDim.x);
        const int tl = item / nbr, t = t0 + tl;
        lo[u] = hi[u] = make_uint4(0u, 0u, 0u, 0u);
        if (item < n_items && t < p.T) {
          const uint4* src =
              reinterpret_cast<const uint4*>(p.hidden + static_cast<size_t>(t) * p.d + (4 * kb0 + item - tl * nbr) * 16);
          lo[u] = src[0];
          hi[u] = src[1];
        }
      }
#pragma unroll
      for (int u = 0; u < kCU; ++u) {
        const int item = item0 + u * static_cast<int>(blockDim.x);
        const int tl = item / nbr, t = t0 + tl;
        if (item >= n_items || t >= p.T) continue;
        const float sc = ldexpf(1.f, kScaleExp - s_E[tl] + p.mseg - p.alpha);
        const uint32_t in[8] = {lo[u].x, lo[u].y, lo[u].z, lo[u].w, hi[u].x, hi[u].y, hi[u].z, hi[u].w};   // column pairs 2i, 2i+1
        uint32_t out[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) out[jj] = bf16x2_to_f16x2(in[(jj >> 1) + 4 * (jj & 1)], sc);
        uint4* dst = reinterpret_cast<uint4*>(p.xop + static_cast<size_t>(t) * p.Kc + (4 * kb0 + item - tl * nbr) * 16);
        dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
        dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
      }
    }
    return;
  }

  // z segment: rows n0 .. n0 + 63 of (R | B), all of one kind (r_c' is a multiple of 64).
  const int n0 = blockIdx.y * 64;
  const int gr = lane >> 2;
  const int b0 = kb0 + warp * (kb1 - kb0) / 8, b1 = kb0 + (warp + 1) * (kb1 - kb0) / 8;
  const int ta = t0 + gr, tb = t0 + gr + 8;
  const float hs[2] = {ta < p.T ? ldexpf(1.f, kScaleExp - s_E[gr]) : 0.f,
                       tb < p.T ? ldexpf(1.f, kScaleExp - s_E[gr + 8]) : 0.f};
  const uint16_t* hrow_a = ta < p.T ? p.hidden + static_cast<size_t>(ta) * p.d : nullptr;
  const uint16_t* hrow_b = tb < p.T ? p.hidden + static_cast<size_t>(tb) * p.d : nullptr;
  float acc[8][4];
#pragma unroll
  for (int n = 0; n < 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
  const bool corr = n0 >= p.rcp;
  if (corr) z_block<true>(p, n0, b0, b1, hs, hrow_a, hrow_b, lane, acc);
  else z_block<false>(p, n0, b0, b1, hs, hrow_a, hrow_b, lane, acc);
  const int cc = lane & 3;
#pragma unroll
  for (int n = 0; n < 8; ++n) {
    red[warp][gr][8 * n + 2 * cc] = acc[n][0];
    red[warp][gr][8 * n + 2 * cc + 1] = acc[n][1];
    red[warp][gr + 8][8 * n + 2 * cc] = acc[n][2];
    red[warp][gr + 8][8 * n + 2 * cc + 1] = acc[n][3];
  }
  __syncthreads();
  const int zb = static_cast<int>(blockIdx.x * (gridDim.y - 1) + blockIdx.y);   // tile x z block
  if (gridDim.z > 1) {
    // This split's sums (in the 2^(kScaleExp - E_s) domain) and exponents.
    float* mine = p.zpart + (static_cast<size_t>(zb) * gridDim.z + blockIdx.z) * kActPartFloats;
    for (int idx = threadIdx.x; idx < 16 * 64; idx += blockDim.x) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) s += red[w][idx >> 6][idx & 63];
      mine[idx] = s;
    }
    // (a split whose columns are all zero carries no exponent)
    if (threadIdx.x < 16) mine[16 * 64 + threadIdx.x] = __int_as_float(s_nz[threadIdx.x] ? s_E[threadIdx.x] : kNoExp);
    __syncthreads();   // the block's stores come before thread 0's release
    if (threadIdx.x == 0) s_last = ticket_acq_rel(p.zticket + zb) == gridDim.z - 1 ? 1 : 0;
    __syncthreads();   // and every thread's loads below after its acquire
    if (!s_last) return;
    const int nz = static_cast<int>(gridDim.z);
    const float* all = p.zpart + static_cast<size_t>(zb) * nz * kActPartFloats;
    if (static_cast<int>(threadIdx.x) < 16 * nz)
      s_Ez[threadIdx.x >> 4][threadIdx.x & 15] =
          __float_as_int(__ldcg(all + static_cast<size_t>(threadIdx.x >> 4) * kActPartFloats + 16 * 64 + (threadIdx.x & 15)));
    __syncthreads();
    if (threadIdx.x < 16) {
      int E = kNoExp;
      for (int z = 0; z < nz; ++z) E = max(E, s_Ez[z][threadIdx.x]);
      s_E[threadIdx.x] = E == kNoExp ? 0 : E;   // E_t (0 for an all-zero token, as for a whole row)
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < 16 * 64; idx += blockDim.x) {
      const int tl = idx >> 6;
      float v[kActMaxSplits];
#pragma unroll
      for (int z = 0; z < kActMaxSplits; ++z)
        v[z] = z < nz ? __ldcg(all + static_cast<size_t>(z) * kActPartFloats + idx) : 0.f;
      float s = 0.f;
#pragma unroll
      for (int z = 0; z < kActMaxSplits; ++z)
        if (z < nz) s += ldexpf(v[z], s_Ez[z][tl] - s_E[tl]);
      red[0][tl][idx & 63] = s;
    }
    if (threadIdx.x == 0) p.zticket[zb] = 0u;   // every split has arrived: ready for the next call
    __syncthreads();
  }
  // X[t, d + n] = z·2^(c_t - beta|gamma): with c_t = kScaleExp - E_t + mseg the
  // token exponent cancels against the 2^(kScaleExp - E_t) of h.
  const float sc_core = ldexpf(1.f, p.mseg - p.beta);
  const float sc_corr = ldexpf(1.f, p.mseg - p.gamma);
  const int nw = gridDim.z > 1 ? 1 : 8;   // warp partials still to add
  for (int idx = threadIdx.x; idx < 16 * 64; idx += blockDim.x) {
    const int tl = idx >> 6, c = idx & 63, t = t0 + tl, n = n0 + c;
    if (t >= p.T) continue;
    float s = 0.f;
    for (int w = 0; w < nw; ++w) s += red[w][tl][c];
    float val = 0.f;
    if (n < p.rcp) val = s * __half2float(__ushort_as_half(p.s_R[n])) * sc_core;
    else if (n < p.Kz) val = s * sc_corr;
    const int col = p.d + (n & ~15) + tc_kpos(n & 15);
    p.xop[static_cast<size_t>(t) * p.Kc + col] = __half_as_ushort(__float2half_rn(val));
  }
}

cudaError_t launch_act_prep(const ActParams& p, int splits, cudaStream_t stream) {
  const dim3 grid((p.T + 15) / 16, (p.Kc - p.d) / 64 + 1, splits);
  act_prep_kernel<<<grid, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

int act_prep_splits(int T, int d, int Kc, int num_sms, size_t scratch_bytes) {
  const int tiles = ((T + 15) / 16) * ((Kc - d) / 64);
  if (tiles == 0 || tiles > kActTickets) return 1;
  int s = std::min(std::min(kActMaxSplits, d / 64), std::max(1, num_sms / tiles));
  while (s > 1 && static_cast<size_t>(s) * tiles * kActPartFloats * 4 > scratch_bytes) --s;
  return s;
}

}  // namespace archead
