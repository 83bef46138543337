// sm_100a device helpers: mbarriers, bulk copies, dependent-launch control,
// the m16n8k16 fp16 tensor-core fragment op, and exact code -> fp16 unpacking.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "layout.h"
#include "params.h"

namespace archead {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// One try: the thread may sleep up to kSuspendHintNs inside the instruction and
// wakes as soon as the phase completes, so a waiting warp costs no issue slots.
constexpr uint32_t kSuspendHintNs = 20000;
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "n"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}
// Waits for the phase with the given parity to complete; false after limit_ns.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
}

// ------------------------------------------------------------- bulk copies
// Global -> this CTA's shared memory, completion counted on `bar` (bytes).
// Both addresses 16-byte aligned, bytes a multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// 16-byte asynchronous copy global -> shared through L2 only (LSU path); the
// calling thread tracks completion with commit / wait groups.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// The same with an L2 cache policy (createpolicy): data read once per launch
// is marked evict-first, so what the launch reuses (its own instructions, the
// activations, the partials) stays in L2 while the packed head streams through.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void cp_async16_hint(uint32_t dst, const void* src, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// ------------------------------------------------- programmatic launch order
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Completion ticket: one gpu-scope acquire-release add, returning the old
// value.  The release half publishes the calling thread's earlier writes and,
// cumulatively, those ordered before them by a block or warp barrier; the
// acquire half orders the caller's later reads (and, after a barrier, its
// block's) after every earlier releaser's writes.
__device__ __forceinline__ unsigned ticket_acq_rel(unsigned* counter) {
  unsigned prev;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(counter) : "memory");
  return prev;
}

// ------------------------------------------------------------ named barrier
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------- tensor core
// D += A(16x16, row) * B(16x8, col), fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------- unpacking
// (x & mask) | bits in one LOP3.
template <uint32_t kMask, uint32_t kBits>
__device__ __forceinline__ uint32_t and_or(uint32_t x) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "n"(kMask), "n"(kBits));
  return r;
}
__device__ __forceinline__ uint32_t and_or_r(uint32_t x, uint32_t mask, uint32_t bits) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "r"(mask), "r"(bits));
  return r;
}
template <int kShift>
__device__ __forceinline__ uint32_t shift_to(uint32_t x) {
  if constexpr (kShift >= 0) return x >> kShift;
  else return x << (-kShift);
}

// fp16 fragment unpacking.  A 4-bit field placed under the fp16 exponent of
// 1024 (0x6400, mantissa step 1 at bit 0) reads as 1024 + u; the field at bits
// 4-7 under the exponent of 64 (0x5400, mantissa step 1 at bit 4) reads as
// 64 + u with no shift at all.  So per k16 step the A columns 2cc, 2cc+1
// (registers a0, a1) carry the offset code plus 1024 and the columns 2cc+8,
// 2cc+9 (a2, a3) the code plus 64, all exact in fp16; the tensor core
// multiplies exact integers and the constant part (offset, plus 1024 or 64)
// is removed once per scale group in fp32.  Keeping the 1024 costs
// accumulation precision only: the products are exact and the fp32
// accumulator carries the larger constant (an emulation with truncation after
// every addition puts the resulting logit error below a quarter of the parity
// tolerance), and it saves two instructions per k16 step.
constexpr float kBiasLo = 1024.f;
constexpr float kBiasHi = 64.f;
constexpr float kInt8Offset = 128.f;          // offset-binary INT8 after the 1024 is subtracted
constexpr uint32_t kHalf1024x2 = 0x64006400u;

__device__ __forceinline__ uint32_t hsub2_bits(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Offset-binary INT4 word: nibbles of (a0, a2, a1, a3) at bits 0, 4, 8, 12 (low
// columns) and 16, 20, 24, 28 (high columns).
__device__ __forceinline__ void unpack_int4_biased(uint32_t w, uint32_t (&a)[4]) {
  const uint32_t w8 = w >> 8;
  a[0] = and_or<0x000F000Fu, 0x64006400u>(w);
  a[2] = and_or<0x00F000F0u, 0x54005400u>(w);
  a[1] = and_or<0x000F000Fu, 0x64006400u>(w8);
  a[3] = and_or<0x00F000F0u, 0x54005400u>(w8);
}

// Offset-binary INT5 codes of k16 step S: low nibbles as for INT4 in w, the
// fifth bit of the low / high column of position q (q = 0..3 for a0, a2, a1,
// a3) at bits 4S+q / 4S+q+16 of hb.  The fifth bit goes to bit 4 (under 1024)
// or bit 8 (under 64, whose mantissa step is at bit 4).
template <int S>
__device__ __forceinline__ void unpack_int5_biased(uint32_t w, uint32_t hb, uint32_t (&a)[4]) {
  const uint32_t w8 = w >> 8;
  a[0] = and_or_r(shift_to<4 * S + 0 - 4>(hb), 0x00100010u, and_or<0x000F000Fu, 0x64006400u>(w));
  a[2] = and_or_r(shift_to<4 * S + 1 - 8>(hb), 0x01000100u, and_or<0x00F000F0u, 0x54005400u>(w));
  a[1] = and_or_r(shift_to<4 * S + 2 - 4>(hb), 0x00100010u, and_or<0x000F000Fu, 0x64006400u>(w8));
  a[3] = and_or_r(shift_to<4 * S + 3 - 8>(hb), 0x01000100u, and_or<0x00F000F0u, 0x54005400u>(w8));
}

// Offset-binary INT8 bytes (row gr col c, row gr col c+1, row gr+8 col c,
// row gr+8 col c+1) of w0 (columns c) and w1 (columns c+8): one byte permute
// per pair puts each byte under the exponent of 1024, one subtraction removes it.
__device__ __forceinline__ void unpack_int8_biased(uint32_t w0, uint32_t w1, uint32_t (&a)[4]) {
  a[0] = hsub2_bits(__byte_perm(w0, 0x64646464u, 0x4140u), kHalf1024x2);
  a[1] = hsub2_bits(__byte_perm(w0, 0x64646464u, 0x4342u), kHalf1024x2);
  a[2] = hsub2_bits(__byte_perm(w1, 0x64646464u, 0x4140u), kHalf1024x2);
  a[3] = hsub2_bits(__byte_perm(w1, 0x64646464u, 0x4342u), kHalf1024x2);
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t bits) {
  __half2 h = *reinterpret_cast<__half2*>(&bits);
  return __half22float2(h);
}

// ------------------------------------------------------ online log-sum-exp
// Running (max, sum of exp(y - max), index of the first maximum).
struct LseState {
  float m;
  float s;
  int idx;
};
__device__ __forceinline__ LseState lse_init() { return LseState{-INFINITY, 0.f, 0x7fffffff}; }
// Elements arrive in increasing index order per thread, so a strict > keeps
// the lowest index among equal maxima.
// The fast exponential is enough here: each term carries a relative error of a
// few ulp, far inside the LSE tolerance, and the maximum itself is exact.
__device__ __forceinline__ void lse_push(LseState& st, float y, int v) {
  if (y > st.m) {
    st.s = st.s * __expf(st.m - y) + 1.f;
    st.m = y;
    st.idx = v;
  } else {
    st.s += __expf(y - st.m);
  }
}
// Merge of two states, with the same fast exponential (a state with no
// element, s = 0, contributes nothing and its exp(-inf - m) is not used).
__device__ __forceinline__ LseState lse_merge(const LseState& a, const LseState& b) {
  LseState r;
  r.m = fmaxf(a.m, b.m);
  const float sa = (a.s == 0.f) ? 0.f : a.s * __expf(a.m - r.m);
  const float sb = (b.s == 0.f) ? 0.f : b.s * __expf(b.m - r.m);
  r.s = sa + sb;
  if (a.m > b.m) r.idx = a.idx;
  else if (b.m > a.m) r.idx = b.idx;
  else r.idx = min(a.idx, b.idx);
  return r;
}
__device__ __forceinline__ LseState lse_shfl_idx(const LseState& a, int src) {
  LseState o;
  o.m = __shfl_sync(0xffffffffu, a.m, src);
  o.s = __shfl_sync(0xffffffffu, a.s, src);
  o.idx = __shfl_sync(0xffffffffu, a.idx, src);
  return o;
}
__device__ __forceinline__ LseState lse_shfl_xor(const LseState& a, int mask) {
  LseState o;
  o.m = __shfl_xor_sync(0xffffffffu, a.m, mask);
  o.s = __shfl_xor_sync(0xffffffffu, a.s, mask);
  o.idx = __shfl_xor_sync(0xffffffffu, a.idx, mask);
  return o;
}

// --------------------------------------------------------------- sampling
// Philox4x64-10 (Salmon, Moraes, Dror, Shaw, SC 2011) from its definition:
// ten rounds of two 64 x 64 -> 128-bit multiplies, the key bumped by the Weyl
// constants between rounds.  Counter (c0, c1, 0, 0), key (k0, 0).
__device__ __forceinline__ void philox4x64_10(uint64_t c0, uint64_t c1, uint64_t k0, uint64_t (&out)[4]) {
  constexpr uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
  constexpr uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
  uint64_t c2 = 0, c3 = 0, k1 = 0;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t hi0 = __umul64hi(M0, c0), lo0 = M0 * c0;
    const uint64_t hi1 = __umul64hi(M1, c2), lo1 = M1 * c2;
    c0 = hi1 ^ c1 ^ k0;
    c1 = lo1;
    c2 = hi0 ^ c3 ^ k1;
    c3 = lo0;
    k0 += W0;
    k1 += W1;
  }
  out[0] = c0;
  out[1] = c1;
  out[2] = c2;
  out[3] = c3;
}

// Standard Gumbel draw from the top 23 bits k of a word: u = (k + 1/2) / 2^23
// (exact in fp32, strictly inside (0, 1)), G = -log(-log(u)).
__device__ __forceinline__ float gumbel_of(uint64_t w) {
  const float u = (static_cast<float>(static_cast<uint32_t>(w >> 41)) + 0.5f) * (1.0f / 8388608.0f);
  return -logf(-logf(u));
}

// Running first maximum (value, row) of the perturbed logits y / tau + G.
struct PickState {
  float z;
  int idx;
};
__device__ __forceinline__ PickState pick_init() { return PickState{-INFINITY, 0x7fffffff}; }
__device__ __forceinline__ void pick_push(PickState& s, float z, int v) {
  if (z > s.z) {
    s.z = z;
    s.idx = v;
  }
}
__device__ __forceinline__ PickState pick_merge(const PickState& a, const PickState& b) {
  if (a.z > b.z) return a;
  if (b.z > a.z) return b;
  return PickState{a.z, min(a.idx, b.idx)};
}
__device__ __forceinline__ PickState pick_shfl_xor(const PickState& a, int mask) {
  return PickState{__shfl_xor_sync(0xffffffffu, a.z, mask), __shfl_xor_sync(0xffffffffu, a.idx, mask)};
}
__device__ __forceinline__ PickState pick_shfl_idx(const PickState& a, int src) {
  return PickState{__shfl_sync(0xffffffffu, a.z, src), __shfl_sync(0xffffffffu, a.idx, src)};
}

}  // namespace archead
