// sm_100a device helpers: mbarriers, bulk copies, dependent-launch control,
// the m16n8k16 bf16 tensor-core fragment op, and exact code -> bf16 unpacking.
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

#include "layout.h"

namespace archead {

// A bounded wait gives up after this long (a legitimate wait is microseconds).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

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
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Waits for the phase with the given parity to complete; false after kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 15u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) return false;
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

// ------------------------------------------------- programmatic launch order
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------ named barrier
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------- tensor core
// D += A(16x16, row) * B(16x8, col), bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
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
// a * 1 + c on bf16 pairs (exact here: the operands are small integers).
__device__ __forceinline__ uint32_t bf16x2_add_const(uint32_t a, uint32_t c) {
  uint32_t r;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(0x3F803F80u), "r"(c));
  return r;
}

// bf16 bit patterns used below: 0x4300 = 128.0, 0xC308 = -136.0, 0xC310 = -144.0.
// A nibble u placed under the exponent of 128 gives 128 + u exactly.

// Offset-binary INT4 word (8 codes) -> the four A-fragment registers.
__device__ __forceinline__ void unpack_int4(uint32_t w, uint32_t (&a)[4]) {
  a[0] = bf16x2_add_const(and_or<0x000F000Fu, 0x43004300u>(w), 0xC308C308u);
  a[1] = bf16x2_add_const(and_or<0x000F000Fu, 0x43004300u>(w >> 4), 0xC308C308u);
  a[2] = bf16x2_add_const(and_or<0x000F000Fu, 0x43004300u>(w >> 8), 0xC308C308u);
  a[3] = bf16x2_add_const(and_or<0x000F000Fu, 0x43004300u>(w >> 12), 0xC308C308u);
}

template <int kShift>
__device__ __forceinline__ uint32_t shift_to(uint32_t x) {
  if constexpr (kShift >= 0) return x >> kShift;
  else return x << (-kShift);
}

// Offset-binary INT5 codes of k16 step S: low nibbles in w, fifth bits in hb.
template <int S>
__device__ __forceinline__ void unpack_int5(uint32_t w, uint32_t hb, uint32_t (&a)[4]) {
  const uint32_t t0 = and_or<0x000F000Fu, 0x43004300u>(w);
  const uint32_t t1 = and_or<0x000F000Fu, 0x43004300u>(w >> 4);
  const uint32_t t2 = and_or<0x000F000Fu, 0x43004300u>(w >> 8);
  const uint32_t t3 = and_or<0x000F000Fu, 0x43004300u>(w >> 12);
  a[0] = bf16x2_add_const(and_or_r(shift_to<4 * S + 0 - 4>(hb), 0x00100010u, t0), 0xC310C310u);
  a[1] = bf16x2_add_const(and_or_r(shift_to<4 * S + 1 - 4>(hb), 0x00100010u, t1), 0xC310C310u);
  a[2] = bf16x2_add_const(and_or_r(shift_to<4 * S + 2 - 4>(hb), 0x00100010u, t2), 0xC310C310u);
  a[3] = bf16x2_add_const(and_or_r(shift_to<4 * S + 3 - 4>(hb), 0x00100010u, t3), 0xC310C310u);
}

// Two offset-binary INT8 codes (bytes b, b+1 of w) -> one bf16 pair, exact:
// 0x4B0000uu is the float 2^23 + u, and 2^23 + 128 is subtracted.
template <int kByte>
__device__ __forceinline__ float int8_offset_to_float(uint32_t w) {
  return __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7650u | kByte)) - 8388736.0f;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ void unpack_int8_pair_words(uint32_t w0, uint32_t w1, uint32_t (&a)[4]) {
  a[0] = pack_bf16x2(int8_offset_to_float<0>(w0), int8_offset_to_float<1>(w0));
  a[1] = pack_bf16x2(int8_offset_to_float<2>(w0), int8_offset_to_float<3>(w0));
  a[2] = pack_bf16x2(int8_offset_to_float<0>(w1), int8_offset_to_float<1>(w1));
  a[3] = pack_bf16x2(int8_offset_to_float<2>(w1), int8_offset_to_float<3>(w1));
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
__device__ __forceinline__ void lse_push(LseState& st, float y, int v) {
  if (y > st.m) {
    st.s = st.s * expf(st.m - y) + 1.f;
    st.m = y;
    st.idx = v;
  } else {
    st.s += expf(y - st.m);
  }
}
__device__ __forceinline__ LseState lse_merge(const LseState& a, const LseState& b) {
  LseState r;
  r.m = fmaxf(a.m, b.m);
  const float sa = (a.s == 0.f) ? 0.f : a.s * expf(a.m - r.m);
  const float sb = (b.s == 0.f) ? 0.f : b.s * expf(b.m - r.m);
  r.s = sa + sb;
  if (a.m > b.m) r.idx = a.idx;
  else if (b.m > a.m) r.idx = b.idx;
  else r.idx = min(a.idx, b.idx);
  return r;
}
__device__ __forceinline__ LseState lse_shfl_xor(const LseState& a, int mask) {
  LseState o;
  o.m = __shfl_xor_sync(0xffffffffu, a.m, mask);
  o.s = __shfl_xor_sync(0xffffffffu, a.s, mask);
  o.idx = __shfl_xor_sync(0xffffffffu, a.idx, mask);
  return o;
}

}  // namespace archead
