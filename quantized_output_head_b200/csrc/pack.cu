// archead_pack_load: the conversion step of the ARCHead paper (§3.3).  The
// canonical packed components (the registered tensors of the state dict) are
// validated, re-laid out into the m-tile blocks described in layout.h, and
// copied into the caller's device arena.  The dense head never reaches this
// library.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>
#include <thread>
#include <vector>

#include "handle.h"

namespace archead {
namespace {

bool fp16_finite(uint16_t b) { return (b & 0x7C00u) != 0x7C00u; }

double half_to_double(uint16_t b) {
  const int e = (b >> 10) & 0x1F, m = b & 0x3FF;
  const double v = (e == 0) ? std::ldexp(static_cast<double>(m), -24) : std::ldexp(1024.0 + m, e - 25);
  return (b & 0x8000u) ? -v : v;
}

bool codes_in_range(const int8_t* p, size_t n, int lo, int hi) {
  for (size_t i = 0; i < n; ++i)
    if (p[i] < lo || p[i] > hi) return false;
  return true;
}

bool scales_finite(const uint16_t* p, size_t n) {
  for (size_t i = 0; i < n; ++i)
    if (!fp16_finite(p[i])) return false;
  return true;
}

struct Src {
  const Layout& L;
  const archead_host_components& C;
  int code_q(int r, int c) const { return (r < L.V) ? C.q[static_cast<size_t>(r) * L.d + c] : 0; }
  int code_L(int r, int c) const {
    return (r < L.V && c < L.r_c) ? C.L[static_cast<size_t>(r) * L.r_c + c] : 0;
  }
  int code_A(int r, int c) const {
    return (r < L.V && c < L.r_r) ? C.A[static_cast<size_t>(r) * L.r_r + c] : 0;
  }
  uint16_t s_res(int r, int grp) const { return (r < L.V) ? C.s_res[static_cast<size_t>(r) * L.n_groups + grp] : 0; }
  uint16_t s_L(int r) const { return (r < L.V && L.r_c > 0) ? C.s_L[r] : 0; }
  uint16_t s_A(int r) const { return (r < L.V && L.r_r > 0) ? C.s_A[r] : 0; }
};

// Row and column of fragment register p (p = 0..3: a0..a3; low column of the
// pair) for lane (gr, cc) at k16 step base k0, and the nibble position q of
// that register in a packed word (a0, a2, a1, a3 at q = 0, 1, 2, 3).
inline int frag_row(int v0, int gr, int p) { return v0 + gr + 8 * (p & 1); }
inline int frag_col(int k0, int cc, int p) { return k0 + 2 * cc + 8 * (p >> 1); }
inline int nib_pos(int p) { return (p == 1) ? 2 : (p == 2) ? 1 : p; }

void pack_mtile(const Src& S, int mt, uint8_t* blk) {
  const Layout& L = S.L;
  const int v0 = mt * kMT;
  for (int lane = 0; lane < 32; ++lane) {
    const int gr = lane >> 2, cc = lane & 3;
    // SC4 residual, offset binary (code + 8).
    for (int ch = 0; ch < L.n_res; ++ch) {
      uint32_t* dst = reinterpret_cast<uint32_t*>(blk + L.off_res + ch * kResChunkBytes + lane * 16);
      for (int s = 0; s < 4; ++s) {
        const int k0 = ch * kResChunkK + s * 16;
        uint32_t w = 0;
        for (int p = 0; p < 4; ++p) {
          const int r = frag_row(v0, gr, p), c = frag_col(k0, cc, p);
          const uint32_t lo = static_cast<uint32_t>(S.code_q(r, c) + 8);
          const uint32_t hi = static_cast<uint32_t>(S.code_q(r, c + 1) + 8);
          const int q = nib_pos(p);
          w |= (lo << (4 * q)) | (hi << (4 * q + 16));
        }
        dst[s] = w;
      }
    }
    // INT5 core factor: low nibble plane and fifth-bit plane of (code + 16).
    for (int ch = 0; ch < L.n_L; ++ch) {
      uint32_t* dst = reinterpret_cast<uint32_t*>(blk + L.off_Lnib + ch * kLNibChunkBytes + lane * 16);
      uint32_t hb = 0;
      for (int s = 0; s < 4; ++s) {
        const int k0 = ch * kLChunkK + s * 16;
        uint32_t w = 0;
        for (int p = 0; p < 4; ++p) {
          const int r = frag_row(v0, gr, p), c = frag_col(k0, cc, p);
          const uint32_t lo = static_cast<uint32_t>(S.code_L(r, c) + 16);
          const uint32_t hi = static_cast<uint32_t>(S.code_L(r, c + 1) + 16);
          const int q = nib_pos(p);
          w |= ((lo & 15u) << (4 * q)) | ((hi & 15u) << (4 * q + 16));
          hb |= ((lo >> 4) << (4 * s + q)) | ((hi >> 4) << (4 * s + q + 16));
        }
        dst[s] = w;
      }
      *reinterpret_cast<uint32_t*>(blk + L.off_Lhi + ch * kLHiChunkBytes + lane * 4) = hb;
    }
    // INT8 correction factor, offset binary (code + 128).
    for (int ch = 0; ch < L.n_A; ++ch) {
      uint8_t* dst = blk + L.off_A + ch * kAChunkBytes + lane * 16;
      for (int s = 0; s < 2; ++s) {
        const int k0 = ch * kAChunkK + s * 16;
        for (int h = 0; h < 2; ++h) {
          const int c = k0 + 2 * cc + 8 * h;
          uint8_t* b = dst + s * 8 + h * 4;
          b[0] = static_cast<uint8_t>(S.code_A(v0 + gr, c) + 128);
          b[1] = static_cast<uint8_t>(S.code_A(v0 + gr, c + 1) + 128);
          b[2] = static_cast<uint8_t>(S.code_A(v0 + gr + 8, c) + 128);
          b[3] = static_cast<uint8_t>(S.code_A(v0 + gr + 8, c + 1) + 128);
        }
      }
    }
  }
  // Scales: (row gr, row gr + 8) pairs.
  for (int gr = 0; gr < 8; ++gr) {
    for (int grp = 0; grp < L.n_groups; ++grp) {
      uint16_t* d = reinterpret_cast<uint16_t*>(blk + L.off_sres + grp * kSresGroupBytes + gr * 4);
      d[0] = S.s_res(v0 + gr, grp);
      d[1] = S.s_res(v0 + gr + 8, grp);
    }
    uint16_t* dl = reinterpret_cast<uint16_t*>(blk + L.off_sL + gr * 4);
    dl[0] = S.s_L(v0 + gr);
    dl[1] = S.s_L(v0 + gr + 8);
    uint16_t* da = reinterpret_cast<uint16_t*>(blk + L.off_sA + gr * 4);
    da[0] = S.s_A(v0 + gr);
    da[1] = S.s_A(v0 + gr + 8);
  }
}

bool plan_decode(archead_handle* h, int smem_optin) {
  const Layout& L = h->L;
  const int nw_res = (L.n_res + kCRes - 1) / kCRes;
  const int nw_L = (L.n_L + kCL - 1) / kCL;
  const int nw_A = (L.n_A + kCA - 1) / kCA;
  const int nw_work = nw_res + nw_L + nw_A;
  if (kEpiWarps + nw_work > kMaxDecodeWarps) return false;
  // The rings and slots of the widest launch (8 tokens) must fit.
  DecodeParams dp{};
  dp.nw_res = nw_res;
  dp.nw_L = nw_L;
  dp.nw_A = nw_A;
  dp.nw_work = nw_work;
  dp.nt = kDecodeTokens;
  dp.slots = 4;
  dp.mg = 1;
  decode_smem_plan(dp, L.g_steps);
  if (decode_smem_bytes(dp) > static_cast<size_t>(smem_optin)) return false;
  h->nw_res = nw_res;
  h->nw_L = nw_L;
  h->nw_A = nw_A;
  h->nw_work = nw_work;
  h->smem_optin = smem_optin;
  return true;
}

// Smallest e with 2^e >= the largest L1 norm of a dequantised R or B row.
int row_norm_exponent(const Layout& L, const archead_host_components& C) {
  double bmax = 0.0;
  const size_t d = L.d;
  for (int k = 0; k < L.r_c; ++k) {
    double a = 0.0;
    for (size_t j = 0; j < d; ++j) a += std::abs(static_cast<double>(C.R[k * d + j]));
    bmax = std::max(bmax, a * half_to_double(C.s_R[k]));
  }
  const size_t ngB = d / L.g_B;
  for (int k = 0; k < L.r_r; ++k) {
    double a = 0.0;
    for (size_t j = 0; j < d; ++j)
      a += std::abs(static_cast<double>(C.B[k * d + j])) * half_to_double(C.s_B[k * ngB + j / L.g_B]);
    bmax = std::max(bmax, a);
  }
  if (bmax <= 0.0) return 0;
  int e = 0;
  std::frexp(bmax, &e);   // bmax < 2^e
  return e;
}

// Smallest e with x < 2^e (x > 0); 0 for x == 0.
int exp_above(double x) {
  if (!(x > 0.0)) return 0;
  int e = 0;
  std::frexp(x, &e);
  return e;
}

double max_abs_half(const uint16_t* s, size_t n) {
  double m = 0.0;
  for (size_t i = 0; i < n; ++i) m = std::max(m, std::abs(half_to_double(s[i])));
  return m;
}

// Weight exponents of the tensor-core path: each dequantised segment times
// 2^alpha|beta|gamma stays below 2^kScaleExp (|q| <= 8, |L| <= 16, |A| <= 128),
// and mseg keeps the activation side below 2^kScaleExp too (z rows are bounded
// by 2^(E_t + e_B)).
void plan_tc(archead_handle* h, const archead_host_components& C, int smem_optin) {
  const Layout& L = h->L;
  h->tc_alpha = kScaleExp - exp_above(8.0 * max_abs_half(C.s_res, static_cast<size_t>(L.V) * L.n_groups));
  h->tc_beta = L.r_c > 0 ? kScaleExp - exp_above(16.0 * max_abs_half(C.s_L, L.V)) : 0;
  h->tc_gamma = L.r_r > 0 ? kScaleExp - exp_above(128.0 * max_abs_half(C.s_A, L.V)) : 0;
  int m = h->tc_alpha;
  if (L.r_c > 0) m = std::min(m, h->tc_beta - h->e_B);
  if (L.r_r > 0) m = std::min(m, h->tc_gamma - h->e_B);
  h->tc_mseg = m;
  // The activation kernel folds the group scales of B at 64-column block ends.
  h->tc_ok = (L.g_B % kTcBK == 0) && tc_smem_max() <= static_cast<size_t>(smem_optin);
}

}  // namespace
}  // namespace archead

using namespace archead;

extern "C" ARCHEAD_API size_t archead_packed_bytes(const archead_desc* desc) {
  Layout L;
  if (desc == nullptr || !make_layout(*desc, &L)) return 0;
  return static_cast<size_t>(eq10_bytes(*desc));
}

extern "C" ARCHEAD_API size_t archead_arena_bytes(const archead_desc* desc) {
  Layout L;
  if (desc == nullptr || !make_layout(*desc, &L)) return 0;
  return static_cast<size_t>(L.arena_bytes);
}

namespace archead {
namespace {

int validate(const Layout& L, const archead_host_components& C) {
  const size_t V = L.V, d = L.d, rc = L.r_c, rr = L.r_r;
  if (C.q == nullptr || C.s_res == nullptr) return ARCHEAD_EINVAL;
  if (rc > 0 && (C.L == nullptr || C.s_L == nullptr || C.R == nullptr || C.s_R == nullptr)) return ARCHEAD_EINVAL;
  if (rr > 0 && (C.A == nullptr || C.s_A == nullptr || C.B == nullptr || C.s_B == nullptr)) return ARCHEAD_EINVAL;
  // Code ranges of the narrow formats and finite scales (INT8 codes are in range by type).
  if (!codes_in_range(C.q, V * d, -8, 7)) return ARCHEAD_EINVAL;
  if (rc > 0 && !codes_in_range(C.L, V * rc, -16, 15)) return ARCHEAD_EINVAL;
  if (!scales_finite(C.s_res, V * L.n_groups)) return ARCHEAD_EINVAL;
  if (rc > 0 && (!scales_finite(C.s_L, V) || !scales_finite(C.s_R, rc))) return ARCHEAD_EINVAL;
  if (rr > 0 && (!scales_finite(C.s_A, V) || !scales_finite(C.s_B, rr * (d / L.g_B)))) return ARCHEAD_EINVAL;
  return ARCHEAD_OK;
}

// Writes the whole arena image (arena_bytes, zero-filled by the caller).
void build_image(const Layout& L, const archead_host_components& C, uint8_t* img) {
  const size_t d = L.d, rc = L.r_c, rr = L.r_r;
  const Src S{L, C};
  const int nthr = std::max(1, std::min<int>(16, static_cast<int>(std::thread::hardware_concurrency())));
  std::vector<std::thread> pool;
  for (int t = 0; t < nthr; ++t) {
    pool.emplace_back([&, t]() {
      for (int mt = t; mt < L.n_mtiles; mt += nthr) pack_mtile(S, mt, img + static_cast<size_t>(mt) * L.mblk_bytes);
    });
  }
  for (auto& th : pool) th.join();
  for (size_t k = 0; k < rc; ++k) {
    std::memcpy(img + L.off_R + k * d, C.R + k * d, d);
    reinterpret_cast<uint16_t*>(img + L.off_sR)[k] = C.s_R[k];
  }
  const size_t ngB = d / L.g_B;
  for (size_t k = 0; k < rr; ++k) {
    std::memcpy(img + L.off_B + k * d, C.B + k * d, d);
    std::memcpy(img + L.off_sB + k * ngB * 2, C.s_B + k * ngB, ngB * 2);
  }
}

}  // namespace
}  // namespace archead

extern "C" ARCHEAD_API int archead_pack_image(const archead_desc* desc, const archead_host_components* comps,
                                              void* host_image, size_t image_bytes) {
  if (desc == nullptr || comps == nullptr || host_image == nullptr) return ARCHEAD_EINVAL;
  Layout L;
  if (!make_layout(*desc, &L)) return ARCHEAD_EUNSUP;
  if (image_bytes < L.arena_bytes) return ARCHEAD_ENOMEM;
  const int v = validate(L, *comps);
  if (v != ARCHEAD_OK) return v;
  std::memset(host_image, 0, L.arena_bytes);
  build_image(L, *comps, static_cast<uint8_t*>(host_image));
  return ARCHEAD_OK;
}

extern "C" ARCHEAD_API int archead_pack_load(const archead_desc* desc, const archead_host_components* comps,
                                             void* dev_arena, size_t arena_bytes, archead_stream_t stream,
                                             archead_handle** out) {
  if (desc == nullptr || comps == nullptr || dev_arena == nullptr || out == nullptr) return ARCHEAD_EINVAL;
  *out = nullptr;
  Layout L;
  if (!make_layout(*desc, &L)) return ARCHEAD_EUNSUP;
  if (reinterpret_cast<uintptr_t>(dev_arena) % 256 != 0) return ARCHEAD_EALIGN;
  if (arena_bytes < L.arena_bytes) return ARCHEAD_ENOMEM;
  const int v = validate(L, *comps);
  if (v != ARCHEAD_OK) return v;

  int dev = 0, major = 0, minor = 0, sms = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return set_cuda_error(e);
  if (major != 10 || minor != 0) return ARCHEAD_EUNSUP;

  archead_handle* h = new (std::nothrow) archead_handle{};
  if (h == nullptr) return ARCHEAD_ENOMEM;
  h->L = L;
  h->arena = static_cast<const uint8_t*>(dev_arena);
  h->device = dev;
  h->num_sms = sms;
  h->grid = std::min(sms, L.n_mtiles);
  if (!plan_decode(h, optin)) {
    delete h;
    return ARCHEAD_EUNSUP;
  }
  h->e_B = row_norm_exponent(L, *comps);
  h->row0 = 0;
  h->v_total = L.V;
  h->wait_limit_ns = kWaitLimitNs;
  h->test_stall = 0;
  h->graphs = nullptr;
  plan_tc(h, *comps, optin);
  e = decode_set_attributes(L.g_steps, static_cast<size_t>(optin));
  if (e == cudaSuccess && h->tc_ok) e = tc_set_attributes();
  if (e != cudaSuccess) {
    delete h;
    return set_cuda_error(e);
  }
  uint8_t* img = static_cast<uint8_t*>(std::calloc(L.arena_bytes, 1));
  if (img == nullptr) {
    delete h;
    return ARCHEAD_ENOMEM;
  }
  build_image(L, *comps, img);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  e = cudaMemcpyAsync(dev_arena, img, L.arena_bytes, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  std::free(img);
  if (e != cudaSuccess) {
    delete h;
    return set_cuda_error(e);
  }
  h->graphs = host_graph_cache_new();
  if (h->graphs == nullptr) {
    delete h;
    return ARCHEAD_ENOMEM;
  }
  *out = h;
  return ARCHEAD_OK;
}

extern "C" ARCHEAD_API void archead_free(archead_handle* handle) {
  if (handle == nullptr) return;
  host_graph_cache_free(handle->graphs);
  delete handle;
}
