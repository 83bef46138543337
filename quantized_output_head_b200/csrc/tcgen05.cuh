// sm_100a tensor-memory helpers for the tensor-core forward: TMEM allocation,
// tcgen05 MMA with A in tensor memory and B in shared memory, TMEM loads and
// stores, the tcgen05 fences, and the 2-D TMA tile load (single CTA, no
// cluster broadcast).  Also the exact code -> signed fp16 unpacking the
// dequantising warps use (scales are applied to fp16 there, once per weight).
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "device.cuh"

namespace archead {

// ------------------------------------------------------------ TMEM alloc
// Executed by one whole warp; writes the base address to shared memory.
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// --------------------------------------------------------------- ordering
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Arrives once on the mbarrier when every tcgen05 op this thread issued so far
// has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// One lane of a converged warp (the same lane every time the whole warp runs
// it): MMA and TMA issue sit under it so the loop around them stays
// warp-uniform.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "elect.sync _|P, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// ------------------------------------------------------------------- MMA
// D[tmem] = A[tmem] * B[smem]^T (+ D when accumulate != 0), kind::f16.
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor of kind::f16: fp16 A and B, both K-major, fp32 D,
// M x N tile (M = 128 here, N a multiple of 16 up to 256).
__host__ __device__ constexpr uint32_t tc_idesc_f16(int M, int N) {
  return (1u << 4)                                   // D format: f32
         | (0u << 7) | (0u << 10)                    // A, B format: f16
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// Shared-memory matrix descriptor of a K-major operand tile stored with the
// 128-byte swizzle: rows of 128 bytes (64 fp16), 8-row atoms of 1024 bytes.
// The tile base must be 1024-byte aligned; advancing along K inside the atom
// adds the byte offset to the start address (32 bytes per K = 16 step).
__device__ __forceinline__ uint64_t smem_desc_k128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);          // start address
  d |= static_cast<uint64_t>(1u) << 16;                         // leading byte offset (unused here)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;                 // stride byte offset: 8 rows
  d |= static_cast<uint64_t>(1u) << 46;                         // descriptor version
  d |= static_cast<uint64_t>(2u) << 61;                         // 128-byte swizzle
  return d;
}

// ------------------------------------------------------------ TMEM access
// 16 lanes x 256 bits, repeated 4 times along the columns: thread (gr, cc) of
// the warp supplies, for repetition i, (lane gr, col 8i + 2cc), (lane gr,
// col 8i + 2cc + 1), (lane gr + 8, col 8i + 2cc), (lane gr + 8, col 8i + 2cc + 1).
__device__ __forceinline__ void tmem_st_16x256b_x4(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bits, 16 columns: thread i gets lane (base + i), columns c..c+15.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
// 32 lanes x 32 bits, 32 columns: thread i gets lane (base + i), columns c..c+31.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------- TMA
// One 2-D tile of `map` at element coordinates (x, y) into this CTA's shared
// memory, completion counted in bytes on `bar`.  x * element size must be a
// multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// ------------------------------------------------- signed fp16 unpacking
// Offset-binary fields placed under the fp16 exponents of 1024 (low nibble) or
// 64 (nibble at bits 4-7, mantissa step at bit 4) read as base + offset code;
// one exact fp16 subtraction of base + offset leaves the signed code.
constexpr uint32_t kH2_1032 = 0x64086408u;   // 1024 + 8   (INT4 under 1024)
constexpr uint32_t kH2_72 = 0x54805480u;     // 64 + 8     (INT4 under 64)
constexpr uint32_t kH2_1040 = 0x64106410u;   // 1024 + 16  (INT5 under 1024)
constexpr uint32_t kH2_80 = 0x55005500u;     // 64 + 16    (INT5 under 64)
constexpr uint32_t kH2_1152 = 0x64806480u;   // 1024 + 128 (INT8 under 1024)

__device__ __forceinline__ uint32_t hmul2_bits(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// INT4 word of one k16 step (nibble positions as in the decode layout) ->
// signed fp16 fragment registers a[p] (p = 0..3 as in the m16n8k16 A operand).
__device__ __forceinline__ void unpack_int4_signed(uint32_t w, uint32_t (&a)[4]) {
  const uint32_t w8 = w >> 8;
  a[0] = hsub2_bits(and_or<0x000F000Fu, 0x64006400u>(w), kH2_1032);
  a[2] = hsub2_bits(and_or<0x00F000F0u, 0x54005400u>(w), kH2_72);
  a[1] = hsub2_bits(and_or<0x000F000Fu, 0x64006400u>(w8), kH2_1032);
  a[3] = hsub2_bits(and_or<0x00F000F0u, 0x54005400u>(w8), kH2_72);
}

// INT5 codes of k16 step S (low nibbles in w, fifth bits in hb) -> signed fp16.
template <int S>
__device__ __forceinline__ void unpack_int5_signed(uint32_t w, uint32_t hb, uint32_t (&a)[4]) {
  const uint32_t w8 = w >> 8;
  a[0] = hsub2_bits(and_or_r(shift_to<4 * S + 0 - 4>(hb), 0x00100010u, and_or<0x000F000Fu, 0x64006400u>(w)),
                    kH2_1040);
  a[2] = hsub2_bits(and_or_r(shift_to<4 * S + 1 - 8>(hb), 0x01000100u, and_or<0x00F000F0u, 0x54005400u>(w)),
                    kH2_80);
  a[1] = hsub2_bits(and_or_r(shift_to<4 * S + 2 - 4>(hb), 0x00100010u, and_or<0x000F000Fu, 0x64006400u>(w8)),
                    kH2_1040);
  a[3] = hsub2_bits(and_or_r(shift_to<4 * S + 3 - 8>(hb), 0x01000100u, and_or<0x00F000F0u, 0x54005400u>(w8)),
                    kH2_80);
}

// INT8 words of one k16 step (w0: columns c, c+1; w1: columns c+8, c+9; bytes
// row gr, row gr, row gr+8, row gr+8) -> signed fp16.
__device__ __forceinline__ void unpack_int8_signed(uint32_t w0, uint32_t w1, uint32_t (&a)[4]) {
  a[0] = hsub2_bits(__byte_perm(w0, 0x64646464u, 0x4140u), kH2_1152);
  a[1] = hsub2_bits(__byte_perm(w0, 0x64646464u, 0x4342u), kH2_1152);
  a[2] = hsub2_bits(__byte_perm(w1, 0x64646464u, 0x4140u), kH2_1152);
  a[3] = hsub2_bits(__byte_perm(w1, 0x64646464u, 0x4342u), kH2_1152);
}

// Position of logical column k (0..15) of a 16-column block in the operand
// order of the tensor-core path: the dequantising warps store fragment
// registers (a0, a2) of row gr into TMEM columns (2cc, 2cc + 1), so TMEM
// element e of the block holds column 2*(e/4) + (e & 1) + 8*((e/2) & 1).
__host__ __device__ constexpr int tc_kpos(int k) { return 4 * ((k & 7) >> 1) + 2 * (k >> 3) + (k & 1); }

}  // namespace archead
