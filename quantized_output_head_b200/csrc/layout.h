// Device layout of a packed ARCHead head (host and device code).
//
// The component list is the one of §3.3 of "ARCHead: Activation-Metric
// Residual Correction for Large Language Model Output Heads": SC4 residual
// codes and fp16 group scales, INT5 left / INT8 right core factors with row
// scales, INT8 correction factors with row / group scales, and shape metadata.
// This file fixes how those bytes sit in HBM for the sm_100a kernels.
//
// Vocabulary rows are grouped in "m-tiles" of 16 rows (the M extent of one
// m16n8k16 tensor-core fragment).  Every per-row byte of an m-tile (the INT4
// residual, its scales, the INT5 core factor, the INT8 correction factor and
// their row scales) is stored in ONE contiguous block, so a single bulk copy
// streams an m-tile from HBM to shared memory.  Inside a block the codes are
// pre-permuted so that lane l of a warp reads, with one 16-byte load, exactly
// the A-operand fragments of m16n8k16 it owns for four consecutive k16 steps:
//   lane l = 4*gr + cc;  fragment register p (p = 0..3) holds the pair
//   (row gr + 8*(p&1), col k0 + 2*cc + 8*(p>>1)) and the column after it.
// Codes are stored in offset binary (code + 8 for INT4, code + 16 for INT5,
// code + 128 for INT8), so one mask-and-OR under an fp16 exponent turns a field
// into an exact fp16 number (bias + offset code).
//
// m-tile block (all offsets multiples of 16 bytes):
//   res   [d/64 chunks][32 lanes][4 words]   word s = k16 step s of the chunk;
//          register p sits at nibble position q = (0, 2, 1, 3)[p]: bits
//          4q..4q+3 hold the low column, bits 4q+16..4q+19 the high column
//                                                               (512 B / chunk)
//   Lnib  [r_c'/64 chunks][32][4 words]      same, low 4 bits of (code + 16)
//   Lhi   [r_c'/64 chunks][32 lanes] u32     bit 4s+q / 4s+q+16 = bit 4 of the
//          low / high column of position q at step s            (128 B / chunk)
//   A     [r_r'/32 chunks][32][2 steps][2 words]  word 2s+h: bytes
//          (row gr col c, row gr col c+1, row gr+8 col c, row gr+8 col c+1),
//          c = k0 + 2cc + 8h                                   (512 B / chunk)
//   s_res [d/g groups][8 gr][2] fp16          (row gr, row gr+8)  (32 B / group)
//   s_L   [8 gr][2] fp16,  s_A [8 gr][2] fp16                      (32 B each)
// Rows at or beyond V (vocabulary padded to a multiple of 16), and columns
// beyond r_c / r_r (ranks padded to 64 / 32), hold code 0 and scale 0.
//
// After the m-tile blocks: R [r_c'][d] int8 and s_R [r_c'] fp16, B [r_r'][d]
// int8 and s_B [r_r'][d/g_B] fp16, plain row-major (read by the low-rank
// prologue), each region 256-byte aligned.
#pragma once
#include <stdint.h>

#include "archead.h"

namespace archead {

constexpr int kMT = 16;                 // vocabulary rows per m-tile
constexpr int kResChunkK = 64;          // residual columns per 16-byte lane load
constexpr int kResChunkBytes = 512;
constexpr int kLChunkK = 64;
constexpr int kLNibChunkBytes = 512;
constexpr int kLHiChunkBytes = 128;
constexpr int kAChunkK = 32;
constexpr int kAChunkBytes = 512;
constexpr int kSresGroupBytes = 32;

struct Layout {
  int32_t V, d, r_c, r_r, g, g_B;
  int32_t Vp, n_mtiles;                 // vocabulary padded to 16 rows
  int32_t rcp, rrp, Kz;                 // ranks padded to 64 / 32; Kz = rcp + rrp
  int32_t n_res, n_L, n_A, n_groups, g_steps;
  uint32_t off_res, off_Lnib, off_Lhi, off_A, off_sres, off_sL, off_sA, mblk_bytes;
  uint64_t off_R, off_sR, off_B, off_sB, arena_bytes;
};

inline uint64_t round_up(uint64_t x, uint64_t m) { return (x + m - 1) / m * m; }

inline bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

// Fills *L for a supported shape; returns false otherwise.
inline bool make_layout(const archead_desc& D, Layout* L) {
  if (D.V < 1 || D.d < 64 || D.d % 64 != 0 || D.r_c < 0 || D.r_r < 0) return false;
  if (!is_pow2(D.g) || D.g < 16 || D.d % D.g != 0) return false;
  if (D.g_B < 1 || D.d % D.g_B != 0) return false;
  if (D.V > (1 << 30) || D.d > (1 << 16) || D.r_c > 8192 || D.r_r > 8192) return false;
  Layout o{};
  o.V = D.V; o.d = D.d; o.r_c = D.r_c; o.r_r = D.r_r; o.g = D.g; o.g_B = D.g_B;
  o.Vp = (int32_t)round_up(D.V, kMT);
  o.n_mtiles = o.Vp / kMT;
  o.rcp = (int32_t)round_up(D.r_c, kLChunkK);
  o.rrp = (int32_t)round_up(D.r_r, kAChunkK);
  o.Kz = o.rcp + o.rrp;
  o.n_res = D.d / kResChunkK;
  o.n_L = o.rcp / kLChunkK;
  o.n_A = o.rrp / kAChunkK;
  o.n_groups = D.d / D.g;
  o.g_steps = D.g / 16;
  uint32_t off = 0;
  o.off_res = off;  off += (uint32_t)o.n_res * kResChunkBytes;
  o.off_Lnib = off; off += (uint32_t)o.n_L * kLNibChunkBytes;
  o.off_Lhi = off;  off += (uint32_t)o.n_L * kLHiChunkBytes;
  o.off_A = off;    off += (uint32_t)o.n_A * kAChunkBytes;
  o.off_sres = off; off += (uint32_t)o.n_groups * kSresGroupBytes;
  o.off_sL = off;   off += 32;
  o.off_sA = off;   off += 32;
  o.mblk_bytes = off;
  uint64_t a = round_up((uint64_t)o.n_mtiles * o.mblk_bytes, 256);
  o.off_R = a;  a += round_up((uint64_t)o.rcp * D.d, 256);
  o.off_sR = a; a += round_up((uint64_t)o.rcp * 2, 256);
  o.off_B = a;  a += round_up((uint64_t)o.rrp * D.d, 256);
  o.off_sB = a; a += round_up((uint64_t)o.rrp * (D.d / D.g_B) * 2, 256);
  o.arena_bytes = a;
  *L = o;
  return true;
}

// Eq. 10 payload bytes (format arithmetic, INT5 at 5 bits and INT4 at 4 bits).
inline uint64_t eq10_bytes(const archead_desc& D) {
  const uint64_t V = D.V, d = D.d, rc = D.r_c, rr = D.r_r;
  return (V * rc * 5 + 7) / 8 + 2 * V + rc * d + 2 * rc + (V * d + 1) / 2 +
         2 * V * (d / D.g) + V * rr + 2 * V + rr * d + 2 * rr * (d / D.g_B);
}

}  // namespace archead
