// Decode kernel: the packed-head forward (ARCHead paper, §3.2 Eq. 7) for up
// to 8 tokens per launch, streaming the packed head once from HBM.
//
// Per vocabulary row v and token t it forms
//   y[t,v] = sum_g s_res[v,g] (sum_{j in g} q[v,j] h[t,j])          residual (SC4)
//          + s_L[v] sum_k L[v,k] z_c[t,k]                         core (Eq. 3)
//          + s_A[v] sum_k A[v,k] z_r[t,k]                         correction (Eq. 4-6)
// with z_c, z_r from the prologue kernel.  The codes are unpacked to exact
// bf16 integers in registers and multiplied on the tensor cores (m16n8k16,
// vocabulary rows as M, tokens as N, fp32 accumulation); the fp16 group and
// row scales are applied to the fp32 partial sums, so no rounding of a scaled
// weight ever happens.  z is fed as a bf16 high part plus a bf16 remainder.
//
// Block organisation (one block per SM, persistent over m-tiles):
//   warp 0            producer: bulk-copies whole m-tile blocks HBM -> SMEM
//                     into a ring of `stages` slots (full/empty mbarriers)
//   residual warps    each owns kCRes 64-column chunks of d for every m-tile;
//                     the h fragments of its columns live in registers
//   core warps        each owns kCL 64-column chunks of r_c'
//   correction warps  each owns kCA 32-column chunks of r_r'
// Per m-tile the warps' 16 x 8 partial tiles are summed through SMEM, and
// threads 0..16*nt-1 of the consumers push the finished logits into a running
// log-sum-exp / argmax state (and write logits when asked).  At the end every
// block writes one partial per token; the last block to finish (atomic
// ticket, no spinning) merges them into LSE, argmax and CE.
#include <cuda_runtime.h>

#include "device.cuh"
#include "params.h"

namespace archead {

namespace {

struct SmemView {
  uint8_t* stages;
  float* red;        // [2][nw_work][16][8]
  uint64_t* full;    // [stages]
  uint64_t* empty;   // [stages]
  int* flags;        // [0] abort, [1] last block
};

__device__ __forceinline__ SmemView smem_view(uint8_t* smem, const DecodeParams& p) {
  SmemView v;
  v.stages = smem;
  v.red = reinterpret_cast<float*>(smem + static_cast<size_t>(p.stages) * p.mblk_bytes);
  v.full = reinterpret_cast<uint64_t*>(v.red + 2 * p.nw_work * 128);
  v.empty = v.full + p.stages;
  v.flags = reinterpret_cast<int*>(v.empty + p.stages);
  return v;
}

__device__ __forceinline__ void raise_timeout(const SmemView& sv, uint32_t* status) {
  *reinterpret_cast<volatile int*>(sv.flags) = 1;
  atomicOr(status, static_cast<uint32_t>(ARCHEAD_STATUS_WAIT_TIMEOUT));
}

// ----------------------------------------------------------------- producer
__device__ void producer(const DecodeParams& p, const SmemView& sv, int n_my) {
  const int S = p.stages;
  int issued = 0;
  for (int i = 0; i < n_my; ++i) {
    const int s = i % S;
    const int u = i / S;
    if (u > 0 && !mbar_wait(smem_addr(&sv.empty[s]), (u - 1) & 1)) {
      raise_timeout(sv, p.status);
      break;
    }
    if (*reinterpret_cast<volatile int*>(sv.flags)) break;
    const uint32_t full = smem_addr(&sv.full[s]);
    mbar_arrive_expect_tx(full, p.mblk_bytes);
    const uint8_t* src = p.mtiles + (static_cast<size_t>(blockIdx.x) + static_cast<size_t>(i) * gridDim.x) * p.mblk_bytes;
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

// --------------------------------------------------------- per-role tiles
template <int CRES>
__device__ __forceinline__ void residual_tile(const uint8_t* stg, const DecodeParams& p, int wres, int lane,
                                              const uint32_t (&hf)[CRES][4][2], int last_k16, float (&acc)[4]) {
  const int gr = lane >> 2;
  const int gmask = (1 << p.g_steps_log2) - 1;
  float tmp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < CRES; ++c) {
    const int chunk = wres * CRES + c;
    if (chunk < p.n_res) {
      const uint4 nib = *reinterpret_cast<const uint4*>(stg + p.off_res + chunk * kResChunkBytes + lane * 16);
      const uint32_t wv[4] = {nib.x, nib.y, nib.z, nib.w};
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        uint32_t a[4];
        unpack_int4(wv[s], a);
        mma_bf16_16816(tmp, a, hf[c][s][0], hf[c][s][1]);
        const int k16 = chunk * 4 + s;
        if (((k16 + 1) & gmask) == 0 || k16 == last_k16) {
          const int grp = k16 >> p.g_steps_log2;
          const float2 sc = half2_bits_to_float2(
              *reinterpret_cast<const uint32_t*>(stg + p.off_sres + grp * kSresGroupBytes + gr * 4));
          acc[0] = fmaf(sc.x, tmp[0], acc[0]);
          acc[1] = fmaf(sc.x, tmp[1], acc[1]);
          acc[2] = fmaf(sc.y, tmp[2], acc[2]);
          acc[3] = fmaf(sc.y, tmp[3], acc[3]);
          tmp[0] = tmp[1] = tmp[2] = tmp[3] = 0.f;
        }
      }
    }
  }
}

__device__ __forceinline__ void core_tile(const uint8_t* stg, const DecodeParams& p, int wl, int lane,
                                          const uint32_t (&zf)[kCL][4][2][2], float (&acc)[4]) {
  const int gr = lane >> 2;
#pragma unroll
  for (int c = 0; c < kCL; ++c) {
    const int chunk = wl * kCL + c;
    if (chunk < p.n_L) {
      const uint4 nib = *reinterpret_cast<const uint4*>(stg + p.off_Lnib + chunk * kLNibChunkBytes + lane * 16);
      const uint32_t hb = *reinterpret_cast<const uint32_t*>(stg + p.off_Lhi + chunk * kLHiChunkBytes + lane * 4);
      uint32_t a[4];
      unpack_int5<0>(nib.x, hb, a);
      mma_bf16_16816(acc, a, zf[c][0][0][0], zf[c][0][0][1]);
      mma_bf16_16816(acc, a, zf[c][0][1][0], zf[c][0][1][1]);
      unpack_int5<1>(nib.y, hb, a);
      mma_bf16_16816(acc, a, zf[c][1][0][0], zf[c][1][0][1]);
      mma_bf16_16816(acc, a, zf[c][1][1][0], zf[c][1][1][1]);
      unpack_int5<2>(nib.z, hb, a);
      mma_bf16_16816(acc, a, zf[c][2][0][0], zf[c][2][0][1]);
      mma_bf16_16816(acc, a, zf[c][2][1][0], zf[c][2][1][1]);
      unpack_int5<3>(nib.w, hb, a);
      mma_bf16_16816(acc, a, zf[c][3][0][0], zf[c][3][0][1]);
      mma_bf16_16816(acc, a, zf[c][3][1][0], zf[c][3][1][1]);
    }
  }
  const float2 sc = half2_bits_to_float2(*reinterpret_cast<const uint32_t*>(stg + p.off_sL + gr * 4));
  acc[0] *= sc.x;
  acc[1] *= sc.x;
  acc[2] *= sc.y;
  acc[3] *= sc.y;
}

__device__ __forceinline__ void correction_tile(const uint8_t* stg, const DecodeParams& p, int wa, int lane,
                                                const uint32_t (&zf)[kCA][2][2][2], float (&acc)[4]) {
  const int gr = lane >> 2;
#pragma unroll
  for (int c = 0; c < kCA; ++c) {
    const int chunk = wa * kCA + c;
    if (chunk < p.n_A) {
      const uint4 w = *reinterpret_cast<const uint4*>(stg + p.off_A + chunk * kAChunkBytes + lane * 16);
      uint32_t a[4];
      unpack_int8_pair_words(w.x, w.y, a);
      mma_bf16_16816(acc, a, zf[c][0][0][0], zf[c][0][0][1]);
      mma_bf16_16816(acc, a, zf[c][0][1][0], zf[c][0][1][1]);
      unpack_int8_pair_words(w.z, w.w, a);
      mma_bf16_16816(acc, a, zf[c][1][0][0], zf[c][1][0][1]);
      mma_bf16_16816(acc, a, zf[c][1][1][0], zf[c][1][1][1]);
    }
  }
  const float2 sc = half2_bits_to_float2(*reinterpret_cast<const uint32_t*>(stg + p.off_sA + gr * 4));
  acc[0] *= sc.x;
  acc[1] *= sc.x;
  acc[2] *= sc.y;
  acc[3] *= sc.y;
}

// B-operand fragment (16 x 8, column = token) from a row-major bf16 matrix:
// lane (gr, cc) holds rows k0 + 2cc, +1 and k0 + 2cc + 8, +9 of token gr.
__device__ __forceinline__ void load_b_frag(const uint16_t* base, size_t ld, int k0, int lane, int nt,
                                            bool valid, uint32_t& b0, uint32_t& b1) {
  const int gr = lane >> 2, cc = lane & 3;
  if (valid && gr < nt) {
    const uint16_t* r = base + static_cast<size_t>(gr) * ld + k0 + 2 * cc;
    b0 = *reinterpret_cast<const uint32_t*>(r);
    b1 = *reinterpret_cast<const uint32_t*>(r + 8);
  } else {
    b0 = 0u;
    b1 = 0u;
  }
}

enum Role { kRoleRes = 0, kRoleCore = 1, kRoleCorr = 2, kRoleIdle = 3 };

// The consumer loop of one role.  Returns this thread's running LSE state.
template <int ROLE, int CRES>
__device__ LseState consumer_loop(const DecodeParams& p, const SmemView& sv, int n_my, int ridx, int cw,
                                  int ctid, int lane) {
  const int S = p.stages;
  const int nthreads = p.nw_cons * 32;
  const int t0 = p.t0;
  // Fragments of the B operand, fixed for the whole launch.
  uint32_t hf[CRES][4][2];
  uint32_t zc[kCL][4][2][2];
  uint32_t za[kCA][2][2][2];
  int last_k16 = 0;
  if constexpr (ROLE == kRoleRes) {
    const uint16_t* hb = p.hidden + static_cast<size_t>(t0) * p.d;
#pragma unroll
    for (int c = 0; c < CRES; ++c) {
      const int chunk = ridx * CRES + c;
#pragma unroll
      for (int s = 0; s < 4; ++s)
        load_b_frag(hb, p.d, chunk * kResChunkK + s * 16, lane, p.nt, chunk < p.n_res, hf[c][s][0], hf[c][s][1]);
    }
    last_k16 = min((ridx + 1) * CRES, p.n_res) * 4 - 1;
  }
  grid_dependency_wait();   // prologue output and the previous launch on this workspace
  if constexpr (ROLE == kRoleCore) {
    const uint16_t* zh = p.zhi + static_cast<size_t>(t0) * p.Kz;
    const uint16_t* zl = p.zlo + static_cast<size_t>(t0) * p.Kz;
#pragma unroll
    for (int c = 0; c < kCL; ++c) {
      const int chunk = ridx * kCL + c;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const int k0 = chunk * kLChunkK + s * 16;
        load_b_frag(zh, p.Kz, k0, lane, p.nt, chunk < p.n_L, zc[c][s][0][0], zc[c][s][0][1]);
        load_b_frag(zl, p.Kz, k0, lane, p.nt, chunk < p.n_L, zc[c][s][1][0], zc[c][s][1][1]);
      }
    }
  }
  if constexpr (ROLE == kRoleCorr) {
    const uint16_t* zh = p.zhi + static_cast<size_t>(t0) * p.Kz;
    const uint16_t* zl = p.zlo + static_cast<size_t>(t0) * p.Kz;
#pragma unroll
    for (int c = 0; c < kCA; ++c) {
      const int chunk = ridx * kCA + c;
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int k0 = p.rcp + chunk * kAChunkK + s * 16;
        load_b_frag(zh, p.Kz, k0, lane, p.nt, chunk < p.n_A, za[c][s][0][0], za[c][s][0][1]);
        load_b_frag(zl, p.Kz, k0, lane, p.nt, chunk < p.n_A, za[c][s][1][0], za[c][s][1][1]);
      }
    }
  }

  // Epilogue slot of this thread: (row e_row of each m-tile, token e_t).
  const int e_row = ctid & 15;
  const int e_t = ctid >> 4;
  const bool e_active = ctid < 16 * p.nt;
  const int target = (e_active && p.targets != nullptr) ? p.targets[t0 + e_t] : -1;
  LseState st = lse_init();

  for (int i = 0; i < n_my; ++i) {
    const int s = i % S;
    const uint8_t* stg = sv.stages + static_cast<size_t>(s) * p.mblk_bytes;
    bool ok = (*reinterpret_cast<volatile int*>(sv.flags) == 0) && mbar_wait(smem_addr(&sv.full[s]), (i / S) & 1);
    ok = __all_sync(0xffffffffu, ok);   // the tensor-core ops below need the whole warp
    if (!ok && lane == 0) raise_timeout(sv, p.status);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (ok) {
      if constexpr (ROLE == kRoleRes) residual_tile<CRES>(stg, p, ridx, lane, hf, last_k16, acc);
      if constexpr (ROLE == kRoleCore) core_tile(stg, p, ridx, lane, zc, acc);
      if constexpr (ROLE == kRoleCorr) correction_tile(stg, p, ridx, lane, za, acc);
    }
    if constexpr (ROLE != kRoleIdle) {
      const int gr = lane >> 2, cc = lane & 3;
      float* r = sv.red + ((i & 1) * p.nw_work + cw) * 128;
      *reinterpret_cast<float2*>(r + gr * 8 + 2 * cc) = make_float2(acc[0], acc[1]);
      *reinterpret_cast<float2*>(r + (gr + 8) * 8 + 2 * cc) = make_float2(acc[2], acc[3]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&sv.empty[s]));
    named_bar_sync(1, nthreads);
    if (e_active) {
      const float* r = sv.red + (i & 1) * p.nw_work * 128 + e_row * 8 + e_t;
      float y = 0.f;
      for (int w = 0; w < p.nw_work; ++w) y += r[w * 128];
      const int v = (static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x)) * kMT + e_row;
      if (v < p.V) {
        lse_push(st, y, v);
        if (p.logits != nullptr) p.logits[static_cast<size_t>(t0 + e_t) * p.V + v] = y;
        if (v == target) p.tgt[t0 + e_t] = y;
      }
    }
  }
  return st;
}

}  // namespace

template <int CRES>
__global__ void __launch_bounds__(kMaxDecodeWarps * 32, 1) decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const SmemView sv = smem_view(smem, p);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_my = (p.n_mtiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                   static_cast<int>(gridDim.x);
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(smem_addr(&sv.full[s]), 1);
      mbar_init(smem_addr(&sv.empty[s]), p.nw_cons);
    }
    sv.flags[0] = 0;
    sv.flags[1] = 0;
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) producer(p, sv, n_my);
    return;
  }

  const int cw = warp - 1;
  const int ctid = threadIdx.x - 32;
  const int nthreads = p.nw_cons * 32;
  LseState st;
  if (cw < p.nw_res) {
    st = consumer_loop<kRoleRes, CRES>(p, sv, n_my, cw, cw, ctid, lane);
  } else if (cw < p.nw_res + p.nw_L) {
    st = consumer_loop<kRoleCore, CRES>(p, sv, n_my, cw - p.nw_res, cw, ctid, lane);
  } else if (cw < p.nw_work) {
    st = consumer_loop<kRoleCorr, CRES>(p, sv, n_my, cw - p.nw_res - p.nw_L, cw, ctid, lane);
  } else {
    st = consumer_loop<kRoleIdle, CRES>(p, sv, n_my, 0, cw, ctid, lane);
  }

  // Block partial per token: threads 16t..16t+15 hold token t (one half-warp).
  const int e_row = ctid & 15, e_t = ctid >> 4;
  if (cw < 4) {
#pragma unroll
    for (int m = 8; m >= 1; m >>= 1) st = lse_merge(st, lse_shfl_xor(st, m));
    if (e_row == 0 && e_t < p.nt) {
      p.partials[static_cast<size_t>(p.t0 + e_t) * gridDim.x + blockIdx.x] =
          make_float4(st.m, st.s, __int_as_float(st.idx), 0.f);
      __threadfence();
    }
  }
  named_bar_sync(1, nthreads);
  if (ctid == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(p.counter, 1u);
    sv.flags[1] = (prev == gridDim.x - 1) ? 1 : 0;
  }
  named_bar_sync(1, nthreads);
  if (sv.flags[1] == 0) return;

  // Last block: merge the per-block partials of every token of this launch.
  __threadfence();
  for (int t = cw; t < p.nt; t += p.nw_cons) {
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
        const int target = p.targets[tg];
        p.ce[tg] = (target >= 0 && target < p.V) ? lse - __ldcg(p.tgt + tg) : __int_as_float(0x7fc00000);
      }
    }
  }
  named_bar_sync(1, nthreads);
  if (ctid == 0) *p.counter = 0u;
}

template __global__ void decode_kernel<4>(const DecodeParams);
template __global__ void decode_kernel<8>(const DecodeParams);

size_t decode_smem_bytes(int stages, uint32_t mblk_bytes, int nw_work) {
  return static_cast<size_t>(stages) * mblk_bytes + static_cast<size_t>(2) * nw_work * 128 * 4 +
         static_cast<size_t>(2) * stages * 8 + 16;
}

cudaError_t decode_set_attributes(int cres, size_t smem) {
  const void* fn = (cres == 4) ? reinterpret_cast<const void*>(&decode_kernel<4>)
                               : reinterpret_cast<const void*>(&decode_kernel<8>);
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
}

cudaError_t launch_decode(int cres, const DecodeParams& p, int grid, size_t smem, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3((1 + p.nw_cons) * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cres == 4) return cudaLaunchKernelEx(&cfg, decode_kernel<4>, p);
  return cudaLaunchKernelEx(&cfg, decode_kernel<8>, p);
}

}  // namespace archead
