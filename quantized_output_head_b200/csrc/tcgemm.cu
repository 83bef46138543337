// Tensor-core forward for many tokens (ARCHead paper, §3.2 Eq. 7 with the
// residual of §3.1 and the correction of Eq. 4-6), on the 5th-generation
// tensor cores of sm_100a.
//
// Work unit: 128 vocabulary rows (8 m-tile blocks) x BN tokens.  One CTA per
// SM walks its units; per unit the K axis is the concatenation
//   [ residual: d columns | core: r_c' columns | correction: r_r' columns ]
// in k-steps of 64 columns.  Roles:
//   warps 0-15  dequantise: warp w owns m-tile block j = 2(w%4) + (w/4)%2 of
//               the unit (TMEM lanes 16j..16j+15, inside the warp's lane
//               quarter) on the k-steps of parity w/8.  It streams its
//               block's packed bytes through a private cp.async ring, turns
//               each k-step into signed fp16 times the scale (one rounding:
//               s * 2^alpha * q), and stores the 16 x 64 tile into the
//               stage's TMEM columns (tcgen05.st 16x256b).
//   warp 16     TMA: the BN x 64 tile of the activation operand X (fp16,
//               128-byte swizzle) into the stage's shared-memory buffer.
//   warp 17     MMA: one thread issues tcgen05.mma kind::f16 (M=128, N=BN,
//               K=16 x 4) with A from TMEM and B from shared memory into one
//               of two fp32 TMEM accumulators, commits each stage back to the
//               producers and each finished unit to the epilogue.
//   warps 18-21 epilogue: tcgen05.ld of the accumulator (warp lane quarter =
//               32 rows), times 2^-c_t per token, optional logits, target
//               logit, and per-token (max, sum exp, first argmax) over the
//               128 rows, written as one partial per (token, 128-row tile).
// A merge kernel folds the partials into LSE, argmax and cross-entropy.
// Every mbarrier wait is bounded (kWaitLimitNs); on expiry the CTA raises
// ARCHEAD_STATUS_WAIT_TIMEOUT, skips its remaining work and frees its TMEM.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "device.cuh"
#include "tc_params.h"
#include "tcgen05.cuh"

namespace archead {

namespace {

constexpr uint32_t kTmemCols = 512;
static_assert(kTcMaxStages % 2 == 0, "stage parity");

struct TcSmem {
  uint8_t* bst;        // [stages][bstage_bytes], 1024-byte aligned
  uint8_t* rings;      // [kTcDeqWarps][ring][2 x kTcSlotBytes]
  float4* epi;         // [4][kTcMaxBN] per-warp (max, sum, idx) of the current unit
  float* etile;        // [4][32 x 33] per-warp transpose tiles of the epilogue
  uint64_t* full;      // [kTcMaxStages] dequant warps + TMA -> MMA
  uint64_t* empty;     // [kTcMaxStages] MMA -> dequant warps + TMA
  uint64_t* accf;      // [2] MMA -> epilogue
  uint64_t* acce;      // [2] epilogue -> MMA
  uint32_t* tmem;      // TMEM base address
  int* abort_flag;
};

__device__ __forceinline__ TcSmem tc_smem(uint8_t* base, const TcParams& p) {
  TcSmem s;
  s.bst = base;
  s.rings = base + p.ring_off;
  s.epi = reinterpret_cast<float4*>(base + p.epi_off);
  s.etile = reinterpret_cast<float*>(base + p.epi_off + 4 * kTcMaxBN * 16);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + p.bar_off);
  s.full = bars;
  s.empty = bars + kTcMaxStages;
  s.accf = bars + 2 * kTcMaxStages;
  s.acce = bars + 2 * kTcMaxStages + 2;
  s.tmem = reinterpret_cast<uint32_t*>(bars + 2 * kTcMaxStages + 4);
  s.abort_flag = reinterpret_cast<int*>(s.tmem + 1);
  return s;
}

__device__ __forceinline__ bool tc_aborted(const TcSmem& s) {
  return *reinterpret_cast<volatile int*>(s.abort_flag) != 0;
}

// Bounded, warp-uniform wait on an mbarrier phase; on expiry raises the
// timeout status and the block's abort flag.
__device__ __forceinline__ bool tc_wait_warp(const TcSmem& s, uint64_t* bar, uint32_t parity, uint32_t* status) {
  bool ok = true;
  if (tc_aborted(s)) ok = false;
  else ok = mbar_wait(smem_addr(bar), parity);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && (threadIdx.x & 31) == 0 && !tc_aborted(s)) {
    *reinterpret_cast<volatile int*>(s.abort_flag) = 1;
    atomicOr(status, static_cast<uint32_t>(ARCHEAD_STATUS_WAIT_TIMEOUT));
  }
  return ok;
}

// The same, with the common case (the phase has completed) in one try and one
// vote; the abort flag is read only when the phase is still pending.
__device__ __forceinline__ bool tc_wait_fast(const TcSmem& s, uint64_t* bar, uint32_t parity, uint32_t* status) {
  if (__all_sync(0xffffffffu, mbar_try_wait(smem_addr(bar), parity))) return true;
  return tc_wait_warp(s, bar, parity, status);
}

// Shared-memory loads by 32-bit address (ordered after the copy waits and the
// warp barrier before them).
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}

// ------------------------------------------------------- dequantising warps
// Packed bytes of one k-step of one m-tile block -> ring slot (kTcSlotBytes):
//   residual   [0,512) codes, [512, 512 + 32 * groups) group scales
//   core       [0,512) low nibbles, [512,640) fifth bits, [640,672) s_L
//   correction [0,1024) two 32-column chunks, [1024,1056) s_A
constexpr int kSlotResScales = 512, kSlotCoreHi = 512, kSlotCoreScales = 640, kSlotCorrScales = 1024;

__device__ __forceinline__ void issue_step(const TcParams& p, uint32_t dst, const uint8_t* blk, int ks, int lane) {
  if (ks < p.ks_core) {
    cp_async16(dst + lane * 16, blk + p.off_res + ks * kResChunkBytes + lane * 16);
    const int gsh = p.g_log2;
    const int g0 = (ks * kTcBK) >> gsh;
    const int nbytes = (gsh >= 6 ? 1 : (kTcBK >> gsh)) * kSresGroupBytes;
    if (lane * 16 < nbytes)
      cp_async16(dst + kSlotResScales + lane * 16, blk + p.off_sres + g0 * kSresGroupBytes + lane * 16);
  } else if (ks < p.ks_corr) {
    const int c = ks - p.ks_core;
    cp_async16(dst + lane * 16, blk + p.off_Lnib + c * kLNibChunkBytes + lane * 16);
    if (lane < 8) cp_async16(dst + kSlotCoreHi + lane * 16, blk + p.off_Lhi + c * kLHiChunkBytes + lane * 16);
    if (lane < 2) cp_async16(dst + kSlotCoreScales + lane * 16, blk + p.off_sL + lane * 16);
  } else {
    const int a = 2 * (ks - p.ks_corr);
    cp_async16(dst + lane * 16, blk + p.off_A + a * kAChunkBytes + lane * 16);
    if (a + 1 < p.n_A) cp_async16(dst + 512 + lane * 16, blk + p.off_A + (a + 1) * kAChunkBytes + lane * 16);
    if (lane < 2) cp_async16(dst + kSlotCorrScales + lane * 16, blk + p.off_sA + lane * 16);
  }
}

// Scale pair (row gr, row gr + 8) of a slot -> two half2 (s, s) times 2^e.
__device__ __forceinline__ void scale_pair(const uint8_t* at, float mul, uint32_t& s0, uint32_t& s1) {
  const float2 f = half2_bits_to_float2(*reinterpret_cast<const uint32_t*>(at));
  s0 = pack_half2(f.x * mul, f.x * mul);
  s1 = pack_half2(f.y * mul, f.y * mul);
}

// Fragment registers (p order) of one k16 step -> tcgen05.st order, scaled.
__device__ __forceinline__ void place(const uint32_t (&a)[4], uint32_t s0, uint32_t s1, uint32_t* r) {
  r[0] = hmul2_bits(a[0], s0);   // lane gr,     column 2cc     (k 2cc, 2cc+1)
  r[1] = hmul2_bits(a[2], s0);   // lane gr,     column 2cc + 1 (k 2cc+8, 2cc+9)
  r[2] = hmul2_bits(a[1], s1);   // lane gr + 8, column 2cc
  r[3] = hmul2_bits(a[3], s1);   // lane gr + 8, column 2cc + 1
}

// Residual scale groups per 64-column k-step, fixed at compile time: GM = 0
// (g >= 64: one group, whose scales the slot holds), 1 (g = 32: two), 2
// (g = 16: four).  k16 step st uses local group st >> (2 - GM).
template <int GM>
__device__ __forceinline__ void dequant_residual(const uint8_t* slot, float sc, int lane, uint32_t (&r)[16]) {
  const int gr = lane >> 2;
  const uint4 c = *reinterpret_cast<const uint4*>(slot + lane * 16);
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  uint32_t s0 = 0, s1 = 0;
#pragma unroll
  for (int st = 0; st < 4; ++st) {
    if (st % (4 >> GM) == 0) scale_pair(slot + kSlotResScales + (st >> (2 - GM)) * kSresGroupBytes + gr * 4, sc, s0, s1);
    uint32_t a[4];
    unpack_int4_signed(w[st], a);
    place(a, s0, s1, r + 4 * st);
  }
}

// The same in two parts, so that a stage's shared-memory loads can all be in
// flight before any unpacking: the codes (16 bytes at slot + code_off,
// code_off = 16 lane) and this lane's scale pair of each local group (at
// slot + scale_off, scale_off = kSlotResScales + 4 gr) of one k-step ...
template <int GM>
struct ResidualRaw {
  uint4 c;
  uint32_t s[1 << GM];
};
template <int GM>
__device__ __forceinline__ ResidualRaw<GM> load_residual(uint32_t slot, uint32_t code_off, uint32_t scale_off) {
  ResidualRaw<GM> x;
  x.c = lds128(slot + code_off);
#pragma unroll
  for (int g = 0; g < (1 << GM); ++g) x.s[g] = lds32(slot + scale_off + g * kSresGroupBytes);
  return x;
}
// ... then the tcgen05.st operands from them.
template <int GM>
__device__ __forceinline__ void dequant_residual_raw(const ResidualRaw<GM>& x, float sc, uint32_t (&r)[16]) {
  const uint32_t w[4] = {x.c.x, x.c.y, x.c.z, x.c.w};
  uint32_t s0 = 0, s1 = 0;
#pragma unroll
  for (int st = 0; st < 4; ++st) {
    if (st % (4 >> GM) == 0) {
      const float2 f = half2_bits_to_float2(x.s[st >> (2 - GM)]);
      s0 = pack_half2(f.x * sc, f.x * sc);
      s1 = pack_half2(f.y * sc, f.y * sc);
    }
    uint32_t a[4];
    unpack_int4_signed(w[st], a);
    place(a, s0, s1, r + 4 * st);
  }
}

__device__ __forceinline__ void dequant_core(const TcParams& p, const uint8_t* slot, int lane, uint32_t (&r)[16]) {
  const int gr = lane >> 2;
  const uint4 n = *reinterpret_cast<const uint4*>(slot + lane * 16);
  const uint32_t hb = *reinterpret_cast<const uint32_t*>(slot + kSlotCoreHi + lane * 4);
  uint32_t s0, s1;
  scale_pair(slot + kSlotCoreScales + gr * 4, p.sc_L, s0, s1);
  uint32_t a[4];
  unpack_int5_signed<0>(n.x, hb, a);
  place(a, s0, s1, r + 0);
  unpack_int5_signed<1>(n.y, hb, a);
  place(a, s0, s1, r + 4);
  unpack_int5_signed<2>(n.z, hb, a);
  place(a, s0, s1, r + 8);
  unpack_int5_signed<3>(n.w, hb, a);
  place(a, s0, s1, r + 12);
}

__device__ __forceinline__ void dequant_corr(const TcParams& p, const uint8_t* slot, bool second, int lane,
                                             uint32_t (&r)[16]) {
  const int gr = lane >> 2;
  uint32_t s0, s1;
  scale_pair(slot + kSlotCorrScales + gr * 4, p.sc_A, s0, s1);
  const uint4 c0 = *reinterpret_cast<const uint4*>(slot + lane * 16);
  uint32_t a[4];
  unpack_int8_signed(c0.x, c0.y, a);
  place(a, s0, s1, r + 0);
  unpack_int8_signed(c0.z, c0.w, a);
  place(a, s0, s1, r + 4);
  if (second) {
    const uint4 c1 = *reinterpret_cast<const uint4*>(slot + 512 + lane * 16);
    unpack_int8_signed(c1.x, c1.y, a);
    place(a, s0, s1, r + 8);
    unpack_int8_signed(c1.z, c1.w, a);
    place(a, s0, s1, r + 12);
  } else {
#pragma unroll
    for (int i = 8; i < 16; ++i) r[i] = 0u;
  }
}

// Block pointer of m-tile block j in this CTA's unit ordinal ui, or null when
// the unit is past the end or the block past the vocabulary.
__device__ __forceinline__ const uint8_t* unit_block(const TcParams& p, int ui, int n_my, int j) {
  if (ui >= n_my) return nullptr;
  const int u = static_cast<int>(blockIdx.x) + ui * static_cast<int>(gridDim.x);
  const int mt16 = (u / p.n_nt) * 8 + j;
  return mt16 < p.n_mtiles ? p.mtiles + static_cast<size_t>(mt16) * p.mblk_bytes : nullptr;
}

template <int GM>
__device__ __forceinline__ void dequant_step(const TcParams& p, const uint8_t* slot, int ks, int lane,
                                             uint32_t (&r)[16]) {
  if (ks < p.ks_core) dequant_residual<GM>(slot, p.sc_res, lane, r);
  else if (ks < p.ks_corr) dequant_core(p, slot, lane, r);
  else dequant_corr(p, slot, 2 * (ks - p.ks_corr) + 1 < p.n_A, lane, r);
}

// Warp w dequantises m-tile block j = 2(w%4) + (w/4)%2 of every unit (TMEM
// lanes 16j..16j+15 lie in the warp's lane quarter w%4) on the global stages
// g = ui * n_st + st of parity w/8; a stage buffer has a fixed parity (the
// buffer count is even), so each buffer is filled by the same eight warps.  R:
// ring slots, each the packed bytes of one stage (two k-steps), filled R - 1
// of the warp's stages ahead with 16-byte cp.async per lane.  (One bulk copy
// per piece, issued by one lane, measured slower: the copy engine queues many
// 512-byte copies.)  The stages whose two k-steps are both residual (all but a
// few per unit) run a loop of their own with no per-stage segment tests.
template <int R, int GM>
__device__ void dequant_loop(const TcParams& p, const TcSmem& sm, uint32_t tmem_base, int w, int lane) {
  constexpr uint32_t kPair = 2 * kTcSlotBytes;
  const int j = 2 * (w & 3) + ((w >> 2) & 1);
  const int par = w >> 3;
  const uint32_t ring_s = smem_addr(sm.rings) + static_cast<uint32_t>(w) * R * kPair;
  const uint8_t* ring = sm.rings + static_cast<size_t>(w) * R * kPair;
  const int n_my = (p.n_units - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                   static_cast<int>(gridDim.x);
  const int n_st = p.n_st;
  const int n_rst = p.ks_core >> 1;   // stages of two residual k-steps

  // Prefetch cursor: unit ordinal pu, stage pst, R - 1 of this warp's stages
  // ahead.  A residual stage is the codes of two k-steps (1024 contiguous
  // bytes, 16 per lane) and the scales of each (lanes below 2 kPieces).
  constexpr int kPieces = 2 << GM;                  // 16-byte scale pieces per k-step
  const int kk = lane / kPieces, piece = lane % kPieces;
  const bool scale_lane = lane < 2 * kPieces;
  const uint32_t code_dst = 16u * lane, scale_dst = kk * kTcSlotBytes + kSlotResScales + piece * 16;
  int pu = 0, pst = par;
  const uint8_t* pblk = nullptr;
  const uint8_t* pcode = nullptr;    // this lane's codes of k-step 0 of the unit
  const uint8_t* pscale = nullptr;   // its scale piece of group 0
  auto rebase = [&]() {
    pblk = unit_block(p, pu, n_my, j);
    if (pblk != nullptr) {
      pcode = pblk + p.off_res + 16 * lane;
      pscale = pblk + p.off_sres + 16 * piece;
    }
  };
  rebase();
  uint32_t pslot = 0;
  auto issue_next = [&]() {
    if (pu < n_my) {
      if (pblk != nullptr) {
        const uint32_t dst = ring_s + pslot * kPair;
        const int ks0 = 2 * pst;
        if (pst < n_rst) {
          const uint8_t* c = pcode + ks0 * kResChunkBytes;
          cp_async16(dst + code_dst, c);
          cp_async16(dst + kTcSlotBytes + code_dst, c + kResChunkBytes);
          if (scale_lane) cp_async16(dst + scale_dst, pscale + (((ks0 + kk) * kTcBK) >> p.g_log2) * kSresGroupBytes);
        } else {
          issue_step(p, dst, pblk, ks0, lane);
          if (ks0 + 1 < p.n_ks) issue_step(p, dst + kTcSlotBytes, pblk, ks0 + 1, lane);
        }
      }
      pst += 2;
      if (pst >= n_st) {
        pst -= n_st;
        ++pu;
        rebase();
      }
    }
    cp_async_commit();
    pslot = pslot + 1 == R ? 0u : pslot + 1;
  };
#pragma unroll 1
  for (int k = 0; k < R - 1; ++k) issue_next();

  const uint32_t tmem_row = tmem_base + (static_cast<uint32_t>(16 * j) << 16) + p.acol0;
  const uint32_t code_off = 16u * lane, scale_off = kSlotResScales + 4u * (lane >> 2);
  int s = par;
  uint32_t ph = 0;
  uint32_t slot_i = 0;
  // After a stage: the next ring slot and stage buffer.
  auto advance = [&]() {
    slot_i = slot_i + 1 == R ? 0u : slot_i + 1;
    s += 2;
    if (s >= p.stages) {
      s -= p.stages;
      ph ^= 1u;
    }
  };
  for (int ui = 0; ui < n_my; ++ui) {
    const uint8_t* blk = unit_block(p, ui, n_my, j);
    int st = (par + ui * n_st) & 1;   // global stage ui * n_st + st has parity par
    // Residual stages.
    for (; st < n_rst; st += 2) {
      issue_next();   // into the slot the previous stage freed
      if (!tc_wait_fast(sm, &sm.empty[s], ph ^ 1u, p.status)) goto done;
      tc_fence_after();
      cp_async_wait<R - 1>();
      __syncwarp();
      const uint32_t ta = tmem_row + static_cast<uint32_t>(s) * 64u;
      // One k-step at a time into TMEM (a store reads its registers when it
      // issues), so only one k-step's 16 result registers are live.
      if (blk != nullptr) {
        const uint32_t slot = ring_s + slot_i * kPair;
        const ResidualRaw<GM> x0 = load_residual<GM>(slot, code_off, scale_off);
        const ResidualRaw<GM> x1 = load_residual<GM>(slot + kTcSlotBytes, code_off, scale_off);
        uint32_t r[16];
        dequant_residual_raw<GM>(x0, p.sc_res, r);
        tmem_st_16x256b_x4(ta, r);
        dequant_residual_raw<GM>(x1, p.sc_res, r);
        tmem_st_16x256b_x4(ta + 32u, r);
      } else {
        uint32_t r[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) r[i] = 0u;
        tmem_st_16x256b_x4(ta, r);
        tmem_st_16x256b_x4(ta + 32u, r);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();   // every lane is done reading the slot and storing to TMEM
      if (lane == 0) mbar_arrive(smem_addr(&sm.full[s]));
      advance();
    }
    // The rest: a residual / core boundary, core and correction k-steps.
    for (; st < n_st; st += 2) {
      issue_next();
      if (!tc_wait_warp(sm, &sm.empty[s], ph ^ 1u, p.status)) goto done;
      tc_fence_after();
      cp_async_wait<R - 1>();
      __syncwarp();
      const int ks0 = 2 * st;
      const bool two = ks0 + 1 < p.n_ks;
      const uint32_t ta = tmem_row + static_cast<uint32_t>(s) * 64u;
      uint32_t r[16];
      if (blk == nullptr) {
#pragma unroll
        for (int i = 0; i < 16; ++i) r[i] = 0u;
        tmem_st_16x256b_x4(ta, r);
        if (two) tmem_st_16x256b_x4(ta + 32u, r);
      } else {
        const uint8_t* slot = ring + slot_i * kPair;
        dequant_step<GM>(p, slot, ks0, lane, r);
        tmem_st_16x256b_x4(ta, r);
        if (two) {
          dequant_step<GM>(p, slot + kTcSlotBytes, ks0 + 1, lane, r);
          tmem_st_16x256b_x4(ta + 32u, r);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&sm.full[s]));
      advance();
    }
  }
done:
  cp_async_wait_all();
}

template <int R>
__device__ void dequant_warp(const TcParams& p, const TcSmem& sm, uint32_t tmem_base, int w, int lane) {
  if (p.g_log2 >= 6) dequant_loop<R, 0>(p, sm, tmem_base, w, lane);
  else if (p.g_log2 == 5) dequant_loop<R, 1>(p, sm, tmem_base, w, lane);
  else dequant_loop<R, 2>(p, sm, tmem_base, w, lane);
}

// ---------------------------------------------------------------- TMA warp
// Stage buffer: two BN x 64 tiles of X (one per k-step), 128-byte swizzle.  The
// whole warp walks the stages; one elected lane issues.
__device__ void tma_warp(const TcParams& p, const TcSmem& sm, const CUtensorMap* xmap, int lane) {
  grid_dependency_wait();   // X and 2^-c_t come from the activation kernel
  const int n_my = (p.n_units - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                   static_cast<int>(gridDim.x);
  const uint32_t bst = smem_addr(sm.bst);
  int s = 0;
  uint32_t ph = 0;
  for (int ui = 0; ui < n_my; ++ui) {
    const int u = static_cast<int>(blockIdx.x) + ui * static_cast<int>(gridDim.x);
    const int y = (u % p.n_nt) * p.BN;
    for (int st = 0; st < p.n_st; ++st) {
      if (!tc_wait_warp(sm, &sm.empty[s], ph ^ 1u, p.status)) return;
      const int ks0 = 2 * st;
      const bool two = ks0 + 1 < p.n_ks;
      if (elect_one()) {
        const uint32_t bar = smem_addr(&sm.full[s]);
        const uint32_t dst = bst + static_cast<uint32_t>(s) * 2u * p.bstage_bytes;
        mbar_arrive_expect_tx(bar, (two ? 2u : 1u) * static_cast<uint32_t>(p.BN) * 128u);
        tma_load_2d(dst, xmap, ks0 * kTcBK, y, bar);
        if (two) tma_load_2d(dst + p.bstage_bytes, xmap, (ks0 + 1) * kTcBK, y, bar);
      }
      __syncwarp();
      if (++s == p.stages) {
        s = 0;
        ph ^= 1u;
      }
    }
  }
}

// ---------------------------------------------------------------- MMA warp
// The whole warp walks the stages (warp-uniform descriptors); one elected lane
// issues the MMAs and the commits that track them.
// The issue cost of a tcgen05.mma is mostly the instructions that prepare its
// operands, so everything per MMA is an immediate offset from two running
// values: the stage's A column in TMEM and its B descriptor (both advanced by a
// constant per stage and reset when the buffer index wraps).
__device__ void mma_warp(const TcParams& p, const TcSmem& sm, uint32_t tmem_base, int lane) {
  const int n_my = (p.n_units - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                   static_cast<int>(gridDim.x);
  const uint32_t idesc = tc_idesc_f16(kTcBM, p.BN);
  const uint64_t bd0 = smem_desc_k128(smem_addr(sm.bst));   // buffer 0, first k-step
  const uint32_t bstep = p.bstage_bytes >> 4;                // descriptor units per X tile (k-step)
  const uint32_t a_first = tmem_base + p.acol0;
  int s = 0;
  uint32_t ph = 0;
  uint64_t bd = bd0;
  uint32_t ad = a_first;
  for (int ui = 0; ui < n_my; ++ui) {
    const uint32_t a = static_cast<uint32_t>(ui) & 1u;
    if (!tc_wait_warp(sm, &sm.acce[a], ((static_cast<uint32_t>(ui) >> 1) & 1u) ^ 1u, p.status)) return;
    tc_fence_after();
    const uint32_t d = tmem_base + a * p.acc_stride;
    // The wait for stage st + 1 sits between issuing stage st's MMAs and
    // committing them, so its latency overlaps the tensor work.
    if (!tc_wait_warp(sm, &sm.full[s], ph, p.status)) return;
    for (int st = 0; st < p.n_st; ++st) {
      tc_fence_after();
      const bool two = 2 * st + 1 < p.n_ks;
      const uint32_t acc0 = st != 0 ? 1u : 0u;
      const bool leader = elect_one();   // the same lane issues the MMAs and the commit that tracks them
      if (leader) {
        tc_mma_ts(d, ad, bd, idesc, acc0);
        tc_mma_ts(d, ad + 8u, bd + 2u, idesc, 1u);
        tc_mma_ts(d, ad + 16u, bd + 4u, idesc, 1u);
        tc_mma_ts(d, ad + 24u, bd + 6u, idesc, 1u);
        if (two) {
          const uint64_t b1 = bd + bstep;
          tc_mma_ts(d, ad + 32u, b1, idesc, 1u);
          tc_mma_ts(d, ad + 40u, b1 + 2u, idesc, 1u);
          tc_mma_ts(d, ad + 48u, b1 + 4u, idesc, 1u);
          tc_mma_ts(d, ad + 56u, b1 + 6u, idesc, 1u);
        }
      }
      __syncwarp();
      const int sc = s;
      if (++s == p.stages) {
        s = 0;
        ph ^= 1u;
        ad = a_first;
        bd = bd0;
      } else {
        ad += 64u;
        bd += 2u * bstep;
      }
      const bool more = st + 1 < p.n_st;
      const bool ok = !more || tc_wait_warp(sm, &sm.full[s], ph, p.status);
      if (leader) tc_commit(smem_addr(&sm.empty[sc]));
      __syncwarp();
      if (!ok) return;
    }
    if (elect_one()) tc_commit(smem_addr(&sm.accf[a]));
    __syncwarp();
  }
}

// ----------------------------------------------------------- epilogue warps
// Warp q owns accumulator rows 32q..32q+31 (its TMEM lane quarter).  Per chunk
// of 32 token columns it loads its 32 x 32 block, transposes it through a
// private padded tile in shared memory, and lane c then folds token column c
// over the 32 rows on its own: max and first argmax, then sum of exp, the
// target logit if it falls in these rows, and the logits row segment if asked.
// The four warps' states of a token are merged into one partial per
// (token, 128-row tile).
__device__ void epilogue_warps(const TcParams& p, const TcSmem& sm, uint32_t tmem_base, int ew, int lane) {
  grid_dependency_wait();   // 2^-c_t, and the previous call's readers of the outputs
  const int q = (kTcDeqWarps + 2 + ew) & 3;   // TMEM lane quarter of this warp
  float* tile = sm.etile + q * (32 * 33);
  const int n_my = (p.n_units - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                   static_cast<int>(gridDim.x);
  bool ok = true;
  for (int ui = 0; ui < n_my; ++ui) {
    const int u = static_cast<int>(blockIdx.x) + ui * static_cast<int>(gridDim.x);
    const int mt = u / p.n_nt, tb = (u % p.n_nt) * p.BN;
    const uint32_t a = static_cast<uint32_t>(ui) & 1u;
    if (ok) ok = tc_wait_warp(sm, &sm.accf[a], (static_cast<uint32_t>(ui) >> 1) & 1u, p.status);
    if (ok) {
      tc_fence_after();
      const int v0 = mt * kTcBM + 32 * q;
      const int nrow = min(32, p.V - v0);          // rows of this warp inside the vocabulary
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + a * p.acc_stride;
      const int ncol = min(p.BN, p.T - tb);
      for (int c0 = 0; c0 < ncol; c0 += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c0), r);
        tmem_ld_wait();
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) tile[jj * 33 + lane] = __uint_as_float(r[jj]);
        __syncwarp();
        const int col = c0 + lane;
        if (col < ncol && nrow > 0) {
          const int t = tb + col;
          const float inv = __ldg(p.cinv + t);
          float y[32];
          float m = -INFINITY;
          int idx = 0x7fffffff;
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            y[k] = tile[lane * 33 + k] * inv;
            if (k < nrow && y[k] > m) {
              m = y[k];
              idx = v0 + k;
            }
          }
          float e = 0.f;
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (k < nrow) e += __expf(y[k] - m);
          if (p.targets != nullptr) {
            const int tg = __ldg(p.targets + t) - p.row0 - v0;   // row within this warp's 32
            if (tg >= 0 && tg < nrow) p.tgt[t] = tile[lane * 33 + tg] * inv;
          }
          if (p.logits != nullptr) {
            float* dst = p.logits + static_cast<size_t>(t) * p.V + v0;
            if (nrow == 32 && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
#pragma unroll
              for (int k = 0; k < 32; k += 4) *reinterpret_cast<float4*>(dst + k) = make_float4(y[k], y[k + 1], y[k + 2], y[k + 3]);
            } else {
              for (int k = 0; k < nrow; ++k) dst[k] = tile[lane * 33 + k] * inv;
            }
          }
          sm.epi[q * kTcMaxBN + col] = make_float4(m, e, __int_as_float(idx), 0.f);
        }
        __syncwarp();
      }
      tc_fence_before();
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&sm.acce[a]));
    // The four warps' states of each token -> one partial per (token, tile).
    named_bar_sync(1, 128);
    const int col = ew * 32 + lane;
    if (ok && col < p.BN && tb + col < p.T) {
      LseState st = lse_init();
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        if (mt * kTcBM + 32 * w >= p.V) continue;   // rows past the vocabulary: no state
        const float4 e = sm.epi[w * kTcMaxBN + col];
        st = lse_merge(st, LseState{e.x, e.y, __float_as_int(e.z)});
      }
      p.partials[static_cast<size_t>(tb + col) * p.n_mt128 + mt] = make_float4(st.m, st.s, __int_as_float(st.idx), 0.f);
    }
    named_bar_sync(1, 128);
  }
}

}  // namespace

// 22 warps: an SM sub-partition holds up to six of them, and its 16,384
// registers allow 80 per thread.
template <int R>
__global__ void __launch_bounds__(kTcWarps * 32, 1)
    tc_kernel(const TcParams p, const __grid_constant__ CUtensorMap xmap) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const TcSmem sm = tc_smem(base, p);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcMaxStages; ++s) {
      mbar_init(smem_addr(&sm.full[s]), kTcDeqWarps / 2 + 1);   // the eight warps of the stage's parity + TMA
      mbar_init(smem_addr(&sm.empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_addr(&sm.accf[a]), 1);
      mbar_init(smem_addr(&sm.acce[a]), 4);
    }
    *sm.abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kTcDeqWarps + 1) {
    tmem_alloc(smem_addr(sm.tmem), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *sm.tmem;

  if (warp < kTcDeqWarps) dequant_warp<R>(p, sm, tmem_base, warp, lane);
  else if (warp == kTcDeqWarps) tma_warp(p, sm, &xmap, lane);
  else if (warp == kTcDeqWarps + 1) mma_warp(p, sm, tmem_base, lane);
  else epilogue_warps(p, sm, tmem_base, warp - kTcDeqWarps - 2, lane);

  tc_fence_before();
  __syncthreads();
  if (warp == kTcDeqWarps + 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// Per-token fold of the partials: LSE, first argmax, cross-entropy.  One
// block per token: a thread folds the partials m = tid, tid + 256, ... (loads
// of a round issued together), then the warps (shuffle tree) and the block's
// eight warp states in warp order, so the order is fixed whatever the timing.
constexpr int kMergeThreads = 256;
constexpr int kMergeRound = 8;   // partials a thread loads before folding any
__global__ void __launch_bounds__(kMergeThreads) tc_merge_kernel(const float4* partials, int n_mt128, int T,
                                                                 const int32_t* targets, const float* tgt, int V,
                                                                 int row0, float* lse, int32_t* argmax, float* ce,
                                                                 float4* shard_out) {
  __shared__ float4 ws[kMergeThreads / 32];
  const int t = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  grid_dependency_wait();
  const float4* part = partials + static_cast<size_t>(t) * n_mt128;
  LseState a = lse_init();
  for (int m0 = 0; m0 < n_mt128; m0 += kMergeThreads * kMergeRound) {
    float4 q[kMergeRound];
#pragma unroll
    for (int u = 0; u < kMergeRound; ++u) {
      const int m = m0 + static_cast<int>(threadIdx.x) + kMergeThreads * u;
      q[u] = m < n_mt128 ? __ldcg(part + m) : make_float4(-INFINITY, 0.f, __int_as_float(0x7fffffff), 0.f);
    }
#pragma unroll
    for (int u = 0; u < kMergeRound; ++u) a = lse_merge(a, LseState{q[u].x, q[u].y, __float_as_int(q[u].z)});
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) a = lse_merge(a, lse_shfl_xor(a, o));
  if (lane == 0) ws[warp] = make_float4(a.m, a.s, __int_as_float(a.idx), 0.f);
  __syncthreads();
  if (threadIdx.x == 0) {
    a = lse_init();
#pragma unroll 1
    for (int w = 0; w < kMergeThreads / 32; ++w) a = lse_merge(a, LseState{ws[w].x, ws[w].y, __float_as_int(ws[w].z)});
    const float l = a.m + logf(a.s);
    const int gidx = a.idx + row0;
    // target logit when the target row is one of this head's rows
    const int tl = targets != nullptr ? targets[t] - row0 : -1;
    const float tv = (tl >= 0 && tl < V) ? __ldcg(tgt + t) : __int_as_float(0x7fc00000);
    if (lse != nullptr) lse[t] = l;
    if (argmax != nullptr) argmax[t] = gidx;
    if (ce != nullptr) ce[t] = l - tv;
    if (shard_out != nullptr) shard_out[t] = make_float4(l, a.m, __int_as_float(gidx), tv);
  }
}

// ------------------------------------------------------------------- host
// TMEM: two accumulators of acc_stride columns, then one 64-column A tile (two
// k-steps) per stage buffer; the buffers use what the accumulators leave of the
// 512 columns.  Shared memory: two X tiles per stage buffer, the dequantising
// warps' rings (as many slots as fit, kTcMinRing..kTcMaxRing), the epilogue
// tiles and the barriers.
namespace {
constexpr uint32_t kTcBarBytes = 256;
size_t plan_bytes(const TcParams& p) { return static_cast<size_t>(p.bar_off) + kTcBarBytes + 1024; }
}  // namespace

void tc_smem_plan(TcParams& p) {
  p.acc_stride = static_cast<uint32_t>((p.BN + 31) / 32 * 32);
  p.acol0 = 2 * p.acc_stride;
  p.stages = static_cast<int32_t>(std::min<uint32_t>(kTcMaxStages, (kTmemCols - p.acol0) / 64)) & ~1;
  p.bstage_bytes = static_cast<uint32_t>(p.BN) * 128u;   // one X tile; multiple of 2048 (BN % 16 == 0)
  p.ring_off = static_cast<uint32_t>(p.stages) * 2u * p.bstage_bytes;
  for (p.ring = kTcMaxRing; p.ring > kTcMinRing; --p.ring) {
    p.epi_off = p.ring_off + kTcDeqWarps * p.ring * 2 * kTcSlotBytes;
    p.bar_off = p.epi_off + 4 * kTcMaxBN * 16 + 4 * 32 * 33 * 4;
    if (plan_bytes(p) <= static_cast<size_t>(kTcSmemBudget)) return;
  }
  p.epi_off = p.ring_off + kTcDeqWarps * p.ring * 2 * kTcSlotBytes;
  p.bar_off = p.epi_off + 4 * kTcMaxBN * 16 + 4 * 32 * 33 * 4;
}

size_t tc_smem_bytes(const TcParams& p) { return plan_bytes(p); }

size_t tc_smem_max() {
  size_t m = 0;
  for (int bn = 16; bn <= kTcMaxBN; bn += 16) {
    TcParams p{};
    p.BN = bn;
    tc_smem_plan(p);
    m = std::max(m, tc_smem_bytes(p));
  }
  return m;
}

namespace {
const void* tc_kernel_for(int ring) {
  switch (ring) {
    case 2: return reinterpret_cast<const void*>(&tc_kernel<2>);
    case 3: return reinterpret_cast<const void*>(&tc_kernel<3>);
    case 4: return reinterpret_cast<const void*>(&tc_kernel<4>);
    default: return reinterpret_cast<const void*>(&tc_kernel<5>);
  }
}
}  // namespace

cudaError_t tc_set_attributes() {
  const int smem = static_cast<int>(tc_smem_max());
  cudaError_t e = cudaSuccess;
  for (int r = kTcMinRing; r <= kTcMaxRing && e == cudaSuccess; ++r)
    e = cudaFuncSetAttribute(tc_kernel_for(r), cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  return e;
}

namespace {
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiled g_encode = nullptr;
std::once_flag g_encode_once;
}  // namespace

// Tensor map of X [T, Kc] fp16: boxes of 64 columns x BN rows, 128-byte swizzle.
cudaError_t tc_encode_xmap(CUtensorMap* map, const uint16_t* xop, int T, int Kc, int BN) {
  std::call_once(g_encode_once, []() {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiled>(fn);
  });
  if (g_encode == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(Kc), static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(Kc) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTcBK), static_cast<cuuint32_t>(BN)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(xop), dims, strides,
                              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t launch_tc(const TcParams& p, const CUtensorMap& map, int grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kTcWarps * 32);
  cfg.dynamicSmemBytes = tc_smem_bytes(p);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[] = {const_cast<TcParams*>(&p), const_cast<CUtensorMap*>(&map)};
  return cudaLaunchKernelExC(&cfg, tc_kernel_for(p.ring), args);
}

cudaError_t launch_tc_merge(const float4* partials, int n_mt128, int T, const int32_t* targets, const float* tgt,
                            int V, int row0, float* lse, int32_t* argmax, float* ce, float4* shard_out,
                            cudaStream_t stream) {
  // Launched as a programmatic dependent of the tensor-core kernel: its blocks
  // take the SMs that kernel frees and wait (griddepcontrol.wait) for its
  // partials.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(T);
  cfg.blockDim = dim3(kMergeThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tc_merge_kernel, partials, n_mt128, T, targets, tgt, V, row0, lse, argmax, ce,
                            shard_out);
}

// Per token, fold the states of n vocabulary shards (stacked in increasing row
// order): LSE over all rows, the first maximum, and the target logit of the one
// shard that holds the target.
__global__ void __launch_bounds__(256) shard_merge_kernel(const float4* parts, int n, int T, float* lse,
                                                          int32_t* argmax, float* ce) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  float M = -INFINITY;
  for (int r = 0; r < n; ++r) M = fmaxf(M, parts[static_cast<size_t>(r) * T + t].x);
  float s = 0.f, best = -INFINITY, tv = __int_as_float(0x7fc00000);
  int idx = 0x7fffffff;
  for (int r = 0; r < n; ++r) {
    const float4 q = parts[static_cast<size_t>(r) * T + t];
    s += expf(q.x - M);
    const int qi = __float_as_int(q.z);
    if (q.y > best || (q.y == best && qi < idx)) {
      best = q.y;
      idx = qi;
    }
    if (q.w == q.w) tv = q.w;   // not NaN: this shard holds the target row
  }
  const float l = M + logf(s);
  if (lse != nullptr) lse[t] = l;
  if (argmax != nullptr) argmax[t] = idx;
  if (ce != nullptr) ce[t] = l - tv;
}

cudaError_t launch_shard_merge(const float4* parts, int n, int T, float* lse, int32_t* argmax, float* ce,
                               cudaStream_t stream) {
  shard_merge_kernel<<<(T + 255) / 256, 256, 0, stream>>>(parts, n, T, lse, argmax, ce);
  return cudaGetLastError();
}

}  // namespace archead
