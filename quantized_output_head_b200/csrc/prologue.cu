// Low-rank prologue of the factored forward (ARCHead paper, §3.2 Eq. 7 and
// the same factoring of the core of Eq. 3):
//   z_c[t,k] = s_R[k] sum_j R[k,j] h[t,j]                k < r_c
//   z_r[t,k] = sum_j s_B[k, j/g_B] B[k,j] h[t,j]         k < r_r
// accumulated in fp32.  For the fp16 tensor-core pass each token gets a power
// of two: E_t with max_j |h[t,j]| < 2^E_t.  z is stored scaled by
// 2^(kScaleExp - E_t - e_B), where 2^e_B bounds the L1 norm of every
// dequantised R / B row (so |scaled z| < 2^kScaleExp), as an fp16 pair: the
// rounded value and the rounded remainder.  One warp per output row k, which it
// streams once per pass of up to kPT tokens; every warp finds max|h_t| itself
// from the h rows it reads, and warp 0 of block 0 publishes E_t.  The kernel
// also resets the decode kernel's completion ticket and checks the target ids.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "device.cuh"
#include "params.h"

namespace archead {

constexpr int kPT = 8;   // tokens per pass over a row

// Warp per output row; each pass streams the row once for up to kPT tokens.
__global__ void __launch_bounds__(256) prologue_kernel(const PrologueParams p) {
  // Let the dependent decode grid start streaming the packed head right away;
  // it waits (griddepcontrol.wait) before it reads anything written here.
  grid_launch_dependents();
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.counter = 0u;
  if (p.targets != nullptr) {
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < p.T; t += gridDim.x * blockDim.x) {
      const int v = p.targets[t];
      if (v < 0 || v >= p.v_total) atomicOr(p.status, static_cast<uint32_t>(ARCHEAD_STATUS_BAD_TARGET));
    }
  }
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const bool publisher = row == 0;
  const bool has_row = row < p.Kz;
  if (!has_row && !publisher) return;
  const bool core = row < p.rcp;
  const int k = core ? row : row - p.rcp;
  const int8_t* codes = has_row ? (core ? p.R : p.B) + static_cast<size_t>(k) * p.d : nullptr;
  const int ngB = p.d / p.g_B;
  const float s_row = (has_row && core) ? __half2float(__ushort_as_half(p.s_R[k])) : 1.f;
  for (int tb = 0; tb < p.T; tb += kPT) {
    const int nt = min(kPT, p.T - tb);
    float acc[kPT], hmax[kPT];
#pragma unroll
    for (int t = 0; t < kPT; ++t) acc[t] = hmax[t] = 0.f;
#pragma unroll 1
    for (int j = lane * 16; j < p.d; j += 32 * 16) {
      float c[16];
      if (has_row) {
        const int4 cv = *reinterpret_cast<const int4*>(codes + j);
        const int8_t* c8 = reinterpret_cast<const int8_t*>(&cv);
        if (core) {
#pragma unroll
          for (int e = 0; e < 16; ++e) c[e] = static_cast<float>(c8[e]);
        } else {
          const uint16_t* sb = p.s_B + static_cast<size_t>(k) * ngB;
          const int g0 = j / p.g_B;
          if (g0 == (j + 15) / p.g_B) {   // the 16 columns share one group scale
            const float sc = __half2float(__ushort_as_half(sb[g0]));
#pragma unroll
            for (int e = 0; e < 16; ++e) c[e] = sc * static_cast<float>(c8[e]);
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              c[e] = __half2float(__ushort_as_half(sb[(j + e) / p.g_B])) * static_cast<float>(c8[e]);
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) c[e] = 0.f;
      }
#pragma unroll
      for (int t = 0; t < kPT; ++t) {
        if (t < nt) {
          const uint16_t* h = p.hidden + static_cast<size_t>(tb + t) * p.d + j;
          const uint4 hv0 = *reinterpret_cast<const uint4*>(h);
          const uint4 hv1 = *reinterpret_cast<const uint4*>(h + 8);
          const uint32_t w[8] = {hv0.x, hv0.y, hv0.z, hv0.w, hv1.x, hv1.y, hv1.z, hv1.w};
          float a = acc[t], m = hmax[t];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float lo = __uint_as_float(w[q] << 16), hi = __uint_as_float(w[q] & 0xFFFF0000u);
            m = fmaxf(m, fmaxf(fabsf(lo), fabsf(hi)));
            a = fmaf(c[2 * q], lo, a);
            a = fmaf(c[2 * q + 1], hi, a);
          }
          acc[t] = a;
          hmax[t] = m;
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kPT; ++t) {
      if (t < nt) {
        float a = acc[t], m = hmax[t];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
          a += __shfl_xor_sync(0xffffffffu, a, o);
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        }
        int E = 0;
        frexpf(m, &E);   // max|h_t| < 2^E (E = 0 when max|h_t| = 0)
        if (lane == 0) {
          const int tg = tb + t;
          if (publisher) p.escale[tg] = E;
          if (has_row) {
            const float z = ldexpf(a * s_row, kScaleExp - E - p.e_B);
            const __half hi = __float2half_rn(z);
            const __half lo = __float2half_rn(z - __half2float(hi));
            p.zhi[static_cast<size_t>(tg) * p.Kz + row] = __half_as_ushort(hi);
            p.zlo[static_cast<size_t>(tg) * p.Kz + row] = __half_as_ushort(lo);
          }
        }
      }
    }
  }
}

cudaError_t launch_prologue(const PrologueParams& p, cudaStream_t stream) {
  const int rows_per_block = 8;
  const int grid = p.Kz > 0 ? (p.Kz + rows_per_block - 1) / rows_per_block : 1;
  prologue_kernel<<<grid, 32 * rows_per_block, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace archead
