// Low-rank prologue of the factored forward (ARCHead paper, §3.2 Eq. 7 and
// the same factoring of the core of Eq. 3):
//   z_c[t,k] = s_R[k] sum_j R[k,j] h[t,j]                k < r_c
//   z_r[t,k] = sum_j s_B[k, j/g_B] B[k,j] h[t,j]         k < r_r
// accumulated in fp32.  For the fp16 tensor-core pass each token gets a power
// of two: E_t with max_j |h[t,j]| < 2^E_t.  z is stored scaled by
// 2^(kScaleExp - E_t - e_B), where 2^e_B bounds the L1 norm of every
// dequantised R / B row (so |scaled z| < 2^kScaleExp), as an fp16 pair: the
// rounded value and the rounded remainder.  One block per output row k, which
// it streams once per pass of up to kPT tokens; every block finds max|h_t|
// itself from the h it reads, and block 0 publishes E_t.  The kernel also
// resets the decode kernel's completion ticket and checks the target ids.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "device.cuh"
#include "params.h"

namespace archead {

constexpr int kPT = 8;        // tokens per pass over a row
constexpr int kRowWarps = 4;  // warps that share one output row (one block)
constexpr int kU = 4;         // 16-column pieces per lane in flight per batch

// One block of kRowWarps warps per output row (the whole grid starts at once
// and finishes in about one memory latency, so decode blocks do not start late
// on the SMs that hold prologue blocks): lane l of warp w takes the 16-column
// pieces j = 16 (l + 32 (w + kRowWarps u)), loads a batch of kU of them (and
// then each token's h for them) before using any, and the warps' partial sums
// and maxima of |h| meet in shared memory.
__global__ void __launch_bounds__(32 * kRowWarps) prologue_kernel(const PrologueParams p) {
  // Let the dependent decode grid start streaming the packed head right away;
  // it waits (griddepcontrol.wait) before it reads anything written here.
  grid_launch_dependents();
  __shared__ float s_acc[kRowWarps][kPT], s_max[kRowWarps][kPT];
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.counter = 0u;
  if (p.targets != nullptr) {
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < p.T; t += gridDim.x * blockDim.x) {
      const int v = p.targets[t];
      if (v < 0 || v >= p.v_total) atomicOr(p.status, static_cast<uint32_t>(ARCHEAD_STATUS_BAD_TARGET));
    }
  }
  const int row = blockIdx.x;   // block 0 also publishes E_t
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool has_row = row < p.Kz;   // false only for the lone block of a head without low-rank rows
  const bool core = row < p.rcp;
  const int k = core ? row : row - p.rcp;
  const int8_t* codes = has_row ? (core ? p.R : p.B) + static_cast<size_t>(k) * p.d : nullptr;
  const uint16_t* sb = (has_row && !core) ? p.s_B + static_cast<size_t>(k) * (p.d / p.g_B) : nullptr;
  const float s_row = (has_row && core) ? __half2float(__ushort_as_half(p.s_R[k])) : 1.f;
  constexpr int kStride = 16 * 32 * kRowWarps;   // columns between a lane's pieces
  for (int tb = 0; tb < p.T; tb += kPT) {
    const int nt = min(kPT, p.T - tb);
    float acc[kPT], hmax[kPT];
#pragma unroll
    for (int t = 0; t < kPT; ++t) acc[t] = hmax[t] = 0.f;
    for (int j0 = 16 * (lane + 32 * warp); j0 < p.d; j0 += kStride * kU) {
      // codes of the batch -> fp32, times the B group scale (per element where
      // a group boundary falls inside a piece)
      float cf[kU][16];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int j = j0 + kStride * u;
        const int4 cv = (has_row && j < p.d) ? *reinterpret_cast<const int4*>(codes + j) : make_int4(0, 0, 0, 0);
        const int8_t* c8 = reinterpret_cast<const int8_t*>(&cv);
#pragma unroll
        for (int e = 0; e < 16; ++e) cf[u][e] = static_cast<float>(c8[e]);
        if (sb != nullptr && j < p.d) {
          if (j / p.g_B == (j + 15) / p.g_B) {
            const float sc = __half2float(__ushort_as_half(sb[j / p.g_B]));
#pragma unroll
            for (int e = 0; e < 16; ++e) cf[u][e] *= sc;
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) cf[u][e] *= __half2float(__ushort_as_half(sb[(j + e) / p.g_B]));
          }
        }
      }
#pragma unroll
      for (int t = 0; t < kPT; ++t) {
        if (t < nt) {
          const uint16_t* h = p.hidden + static_cast<size_t>(tb + t) * p.d;
          uint4 hv[kU][2];
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int j = j0 + kStride * u;
            hv[u][0] = j < p.d ? *reinterpret_cast<const uint4*>(h + j) : make_uint4(0, 0, 0, 0);
            hv[u][1] = j < p.d ? *reinterpret_cast<const uint4*>(h + j + 8) : make_uint4(0, 0, 0, 0);
          }
          float a = acc[t], m = hmax[t];
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const uint32_t w[8] = {hv[u][0].x, hv[u][0].y, hv[u][0].z, hv[u][0].w,
                                   hv[u][1].x, hv[u][1].y, hv[u][1].z, hv[u][1].w};
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float lo = __uint_as_float(w[q] << 16), hi = __uint_as_float(w[q] & 0xFFFF0000u);
              m = fmaxf(m, fmaxf(fabsf(lo), fabsf(hi)));
              a = fmaf(cf[u][2 * q], lo, a);
              a = fmaf(cf[u][2 * q + 1], hi, a);
            }
          }
          acc[t] = a;
          hmax[t] = m;
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kPT; ++t) {
      float a = acc[t], m = hmax[t];
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      }
      if (lane == 0) {
        s_acc[warp][t] = a;
        s_max[warp][t] = m;
      }
    }
    __syncthreads();
    if (threadIdx.x < nt) {
      const int t = threadIdx.x;
      float a = 0.f, m = 0.f;
#pragma unroll
      for (int w = 0; w < kRowWarps; ++w) {
        a += s_acc[w][t];
        m = fmaxf(m, s_max[w][t]);
      }
      int E = 0;
      frexpf(m, &E);   // max|h_t| < 2^E (E = 0 when max|h_t| = 0)
      const int tg = tb + t;
      if (row == 0) p.escale[tg] = E;
      if (has_row) {
        const float z = ldexpf(a * s_row, kScaleExp - E - p.e_B);
        const __half hi = __float2half_rn(z);
        const __half lo = __float2half_rn(z - __half2float(hi));
        p.zhi[static_cast<size_t>(tg) * p.Kz + row] = __half_as_ushort(hi);
        p.zlo[static_cast<size_t>(tg) * p.Kz + row] = __half_as_ushort(lo);
      }
    }
    __syncthreads();
  }
}

cudaError_t launch_prologue(const PrologueParams& p, cudaStream_t stream) {
  // One block per row of (R | B); a head with no low-rank rows still runs one
  // block for E_t (its row 0 is then a zero row of the padded R).
  const int grid = p.Kz > 0 ? p.Kz : 1;
  prologue_kernel<<<grid, 32 * kRowWarps, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace archead
