// GPU construction of an ARCHead packed head: the activation metric of §3.1
// (Eq. 1-2), the quantised core of §3.2 (Eq. 3) and the activation-metric
// correction (Eq. 4-5 with INT8 factors), in the order of Algorithm 1 (§3.4)
// of "ARCHead: Activation-Metric Residual Correction for Large Language Model
// Output Heads".
//
// Everything is IEEE fp64.  Dense products go to cuBLAS (DGEMM, DSYRK, DSYMM),
// the two symmetric eigenproblems per head (C_lam, and a Gram matrix per
// truncated SVD) to cuSOLVER (DSYEVD); conversions, damping, the columns of
// T_p, the choice and sign of singular vectors and the quantisers are the
// kernels below.
//
// Storage: callers pass row-major matrices.  cuBLAS and cuSOLVER are
// column-major, so a row-major X [m, n] is handed to them as the column-major
// n x m matrix X^T; every call below is written with that in mind (noted
// beside each).
#include <cublas_v2.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cusolverDn.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>

#include "archead_build.h"

namespace {

thread_local char g_err[320] = "";

void set_err(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

#define CK_CUDA(x)                                                          \
  do {                                                                      \
    const cudaError_t e_ = (x);                                             \
    if (e_ != cudaSuccess) {                                                \
      set_err("%s: %s", #x, cudaGetErrorString(e_));                        \
      return ARCHEAD_ECUDA;                                                 \
    }                                                                       \
  } while (0)
#define CK_BLAS(x)                                                          \
  do {                                                                      \
    const cublasStatus_t e_ = (x);                                          \
    if (e_ != CUBLAS_STATUS_SUCCESS) {                                      \
      set_err("%s: cuBLAS status %d", #x, static_cast<int>(e_));            \
      return ARCHEAD_ECUDA;                                                 \
    }                                                                       \
  } while (0)
#define CK_SOLVER(x)                                                        \
  do {                                                                      \
    const cusolverStatus_t e_ = (x);                                        \
    if (e_ != CUSOLVER_STATUS_SUCCESS) {                                    \
      set_err("%s: cuSOLVER status %d", #x, static_cast<int>(e_));          \
      return ARCHEAD_ECUDA;                                                 \
    }                                                                       \
  } while (0)
#define CK(x)                 \
  do {                        \
    const int s_ = (x);       \
    if (s_ != ARCHEAD_OK) return s_; \
  } while (0)

// ----------------------------------------------------------------- kernels
constexpr int kThreads = 256;

int grid_for(size_t n) {
  const size_t b = (n + kThreads - 1) / kThreads;
  return static_cast<int>(b < 148 * 64 ? (b > 0 ? b : 1) : 148 * 64);
}

__global__ void to_f64_kernel(const float* __restrict__ x, double* __restrict__ y, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    y[i] = static_cast<double>(x[i]);
}

// b = a - b, elementwise.
__global__ void rsub_kernel(const double* __restrict__ a, double* __restrict__ b, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    b[i] = a[i] - b[i];
}

// Eq. 2: C_lam = C + lam * mean(diag C) * I, on the diagonal of the d x d
// matrix in place.  One block of 1024 threads.
__global__ void damp_kernel(double* C, int d, double lam) {
  __shared__ double part[1024];
  double s = 0.0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) s += C[static_cast<size_t>(i) * d + i];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (static_cast<int>(threadIdx.x) < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  const double add = lam * (part[0] / d);
  for (int i = threadIdx.x; i < d; i += blockDim.x) C[static_cast<size_t>(i) * d + i] += add;
}

// Eq. 2: the powers Lambda^p and Lambda^-p of the eigenvalues.
__global__ void powers_kernel(const double* __restrict__ w, int d, double p, double* __restrict__ fp,
                              double* __restrict__ fm) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < d) {
    fp[i] = pow(w[i], p);
    fm[i] = pow(w[i], -p);
  }
}

// Q diag(fp) and Q diag(fm): column i of the column-major eigenvector matrix
// (eigenvector i) times fp[i], resp. fm[i].
__global__ void scale_columns_kernel(const double* __restrict__ Q, const double* __restrict__ fp,
                                     const double* __restrict__ fm, int d, double* __restrict__ Qp,
                                     double* __restrict__ Qm) {
  const size_t n = static_cast<size_t>(d) * d;
  for (size_t e = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t col = e / d;
    Qp[e] = Q[e] * fp[col];
    Qm[e] = Q[e] * fm[col];
  }
}

// The r eigenvectors of the largest eigenvalues (DSYEVD orders them
// ascending: columns n-1, n-2, ... of the column-major d x n matrix Q) as
// columns 0..r-1 of Vr (column-major d x r), in descending order, each negated
// when its first entry of largest magnitude is negative.  One block per vector.
__global__ void top_vectors_kernel(const double* __restrict__ Q, int d, int n, int r, double* __restrict__ Vr) {
  __shared__ double best_v[kThreads];
  __shared__ int best_i[kThreads];
  const int i = blockIdx.x;
  if (i >= r) return;
  const double* src = Q + static_cast<size_t>(n - 1 - i) * d;
  double bv = -1.0;
  int bi = INT_MAX;
  for (int j = threadIdx.x; j < d; j += blockDim.x) {   // increasing j: '>' keeps the first maximum
    const double a = fabs(src[j]);
    if (a > bv) {
      bv = a;
      bi = j;
    }
  }
  best_v[threadIdx.x] = bv;
  best_i[threadIdx.x] = bi;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (static_cast<int>(threadIdx.x) < w) {
      const double ov = best_v[threadIdx.x + w];
      const int oi = best_i[threadIdx.x + w];
      if (ov > best_v[threadIdx.x] || (ov == best_v[threadIdx.x] && oi < best_i[threadIdx.x])) {
        best_v[threadIdx.x] = ov;
        best_i[threadIdx.x] = oi;
      }
    }
    __syncthreads();
  }
  const int j0 = best_i[0];
  const double sgn = (j0 < d && src[j0] < 0.0) ? -1.0 : 1.0;
  double* dst = Vr + static_cast<size_t>(i) * d;
  for (int j = threadIdx.x; j < d; j += blockDim.x) dst[j] = sgn * src[j];
}

// Standard normal entries of the randomised SVD's test matrix, a function of
// the seed and the entry's index only: SplitMix64 (Steele, Lea, Flood 2014)
// of seed + 2i and seed + 2i + 1 gives two 53-bit uniforms in (0, 1), and the
// Box-Muller transform the normal deviate.
__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  x += 0x9E3779B97F4A7C15ull;
  x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
  x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
  return x ^ (x >> 31);
}
__global__ void gaussian_kernel(double* __restrict__ x, size_t n, uint64_t seed) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const double u1 = (static_cast<double>(splitmix64(seed + 2 * i) >> 11) + 0.5) * 0x1.0p-53;
    const double u2 = (static_cast<double>(splitmix64(seed + 2 * i + 1) >> 11) + 0.5) * 0x1.0p-53;
    x[i] = sqrt(-2.0 * log(u1)) * cospi(2.0 * u2);
  }
}

// Symmetric quantiser, one warp per group of G consecutive elements of a row:
// s = fp16(amax / qmax); codes clamp(rint(x / s), qmin, qmax) with the
// fp16-rounded s; s = 0 gives codes 0.  dq (may alias x) receives codes * s.
__global__ void quantize_kernel(const double* x, int rows, int cols, int G, int qmin, int qmax,
                                int8_t* __restrict__ codes, uint16_t* __restrict__ scales, double* dq) {
  const int ng = cols / G;
  const long long gid = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
  if (gid >= static_cast<long long>(rows) * ng) return;   // whole warps leave together
  const int lane = threadIdx.x & 31;
  const long long row = gid / ng;
  const int grp = static_cast<int>(gid - row * ng);
  const size_t off = static_cast<size_t>(row) * cols + static_cast<size_t>(grp) * G;
  double amax = 0.0;
  for (int j = lane; j < G; j += 32) amax = fmax(amax, fabs(x[off + j]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const __half sh = __double2half(amax / static_cast<double>(qmax));
  const double s = static_cast<double>(__half2float(sh));
  if (lane == 0) scales[gid] = __half_as_ushort(sh);
  for (int j = lane; j < G; j += 32) {
    double c = 0.0;
    if (s > 0.0) c = fmin(fmax(rint(x[off + j] / s), static_cast<double>(qmin)), static_cast<double>(qmax));
    codes[off + j] = static_cast<int8_t>(c);
    if (dq != nullptr) dq[off + j] = c * s;   // each lane rewrites only the elements it read
  }
}

int launch_quantize(const double* x, int rows, int cols, int bits, int G, int8_t* codes, uint16_t* scales,
                    double* dq, cudaStream_t st) {
  int qmin, qmax;
  switch (bits) {
    case 4: qmin = -8; qmax = 7; break;
    case 5: qmin = -16; qmax = 15; break;
    case 8: qmin = -128; qmax = 127; break;
    default:
      set_err("quantise: bits must be 4, 5 or 8 (got %d)", bits);
      return ARCHEAD_EINVAL;
  }
  if (rows <= 0 || cols <= 0 || G <= 0 || cols % G != 0) {
    set_err("quantise: rows %d, cols %d, group %d", rows, cols, G);
    return ARCHEAD_EINVAL;
  }
  const long long groups = static_cast<long long>(rows) * (cols / G);
  const long long blocks = (groups + kThreads / 32 - 1) / (kThreads / 32);
  quantize_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, st>>>(x, rows, cols, G, qmin, qmax, codes,
                                                                      scales, dq);
  CK_CUDA(cudaGetLastError());
  return ARCHEAD_OK;
}

// ----------------------------------------------------------- library state
// cuBLAS and cuSOLVER handles, created on a thread's first call on a device
// and kept for the life of the process (creating and destroying them on every
// call measured sporadic stalls of 0.3-1.3 s on builds of ~0.4 s); each call
// binds them to its stream.
struct Handles {
  cublasHandle_t blas = nullptr;
  cusolverDnHandle_t solver = nullptr;
};

constexpr int kMaxDevices = 64;

int get_handles(cudaStream_t st, const Handles** out) {
  thread_local Handles cache[kMaxDevices];
  int dev = 0;
  CK_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) {
    set_err("device %d out of range", dev);
    return ARCHEAD_EINVAL;
  }
  Handles& h = cache[dev];
  if (h.blas == nullptr) CK_BLAS(cublasCreate(&h.blas));
  if (h.solver == nullptr) CK_SOLVER(cusolverDnCreate(&h.solver));
  CK_BLAS(cublasSetStream(h.blas, st));
  CK_SOLVER(cusolverDnSetStream(h.solver, st));
  *out = &h;
  return ARCHEAD_OK;
}

// Solver scratch (doubles) for a d x d eigendecomposition, and for the
// randomised SVD's Householder QR of up to d columns.
int eig_lwork(cusolverDnHandle_t h, int d, int* lwork) {
  int le = 0, lq = 0, lo = 0;
  CK_SOLVER(cusolverDnDsyevd_bufferSize(h, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_LOWER, d, nullptr, d,
                                        nullptr, &le));
  CK_SOLVER(cusolverDnDgeqrf_bufferSize(h, d, d, nullptr, d, &lq));
  CK_SOLVER(cusolverDnDorgqr_bufferSize(h, d, d, d, nullptr, d, nullptr, &lo));
  *lwork = std::max(le, std::max(lq, lo));
  return ARCHEAD_OK;
}

// Workspace plan (fp64 unless noted), each region 256-byte aligned:
//   big0 [V * d]            dense head W
//   big1 [max(V, N) * d]    H, then W - A_c B_c, then E
//   fac  [V * rmax]         A_c, then A_w
//   vec  [d * rmax]         right singular vectors (B_c, V_w)
//   vec2 [d * rmax]         T_p V_w, then B_w
//   mat  [5][d * d]         eigenproblem / Gram, T_p, T_p^-1, two scratch
//   w [d], fp [d], fm [d], eig [lwork], info (int)
struct Plan {
  double *big0, *big1, *fac, *vec, *vec2, *mat[5], *w, *fp, *fm, *eig;
  int* info;
  size_t bytes;
};

size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

Plan make_plan(uint8_t* base, long long V, long long d, long long N, long long rmax, long long lwork) {
  Plan p{};
  size_t off = 0;
  auto take = [&](size_t elems, size_t elem_bytes) -> void* {
    void* ptr = base ? base + off : nullptr;
    off += align256(elems * elem_bytes);
    return ptr;
  };
  p.big0 = static_cast<double*>(take(V * d, 8));
  p.big1 = static_cast<double*>(take((V > N ? V : N) * d, 8));
  p.fac = static_cast<double*>(take(V * rmax, 8));
  p.vec = static_cast<double*>(take(d * rmax, 8));
  p.vec2 = static_cast<double*>(take(d * rmax, 8));
  for (int i = 0; i < 5; ++i) p.mat[i] = static_cast<double*>(take(d * d, 8));
  p.w = static_cast<double*>(take(d, 8));
  p.fp = static_cast<double*>(take(d, 8));
  p.fm = static_cast<double*>(take(d, 8));
  p.eig = static_cast<double*>(take(lwork > 0 ? lwork : 1, 8));
  p.info = static_cast<int*>(take(1, 4));
  p.bytes = off;
  return p;
}

// Symmetric eigendecomposition in place (lower triangle of the column-major
// d x d matrix A in, eigenvectors out; eigenvalues ascending into w); the
// host reads the solver's status after a stream synchronisation.
int eigh(const Handles& h, double* A, int d, double* w, double* work, int lwork, int* info, cudaStream_t st) {
  CK_SOLVER(cusolverDnDsyevd(h.solver, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_LOWER, d, A, d, w, work,
                             lwork, info));
  int hinfo = 0;
  CK_CUDA(cudaMemcpyAsync(&hinfo, info, sizeof(int), cudaMemcpyDeviceToHost, st));
  CK_CUDA(cudaStreamSynchronize(st));
  if (hinfo != 0) {
    set_err("cusolverDnDsyevd: info %d (d = %d)", hinfo, d);
    return ARCHEAD_ECUDA;
  }
  return ARCHEAD_OK;
}

// Method of the two rank-r factorisations (archead_svd_opts).
struct SvdOpts {
  int method = ARCHEAD_SVD_EXACT;
  int oversample = 0, power_iters = 0;
  uint64_t seed = 0;
};

// Columns of the randomised method's sketch: k = min(d, r + oversample, above
// 64 rounded up to a multiple of 64: the solver's blocked QR measured up to 2x
// slower on other widths); 0 when the sketch would not fit beside its k x k
// projection in a d x d region (k (d + k) > d^2), where the exact method is
// used instead.
int sketch_cols(int d, int r, const SvdOpts& o) {
  if (o.method != ARCHEAD_SVD_RANDOMIZED) return 0;
  long long k = static_cast<long long>(r) + o.oversample;
  if (k > 64) k = (k + 63) / 64 * 64;
  k = std::min<long long>(d, k);
  return k * (d + k) <= static_cast<long long>(d) * d ? static_cast<int>(k) : 0;
}

// Householder QR of the column-major d x k matrix Y, replaced by its Q factor.
int orthonormalise(const Handles& h, const Plan& pl, int lwork, double* Y, int d, int k) {
  int lq = 0, lo = 0;
  CK_SOLVER(cusolverDnDgeqrf_bufferSize(h.solver, d, k, Y, d, &lq));
  CK_SOLVER(cusolverDnDorgqr_bufferSize(h.solver, d, k, k, Y, d, pl.fp, &lo));
  if (lq > lwork || lo > lwork) {
    set_err("orthonormalise: QR scratch %d / %d > %d", lq, lo, lwork);
    return ARCHEAD_ENOMEM;
  }
  CK_SOLVER(cusolverDnDgeqrf(h.solver, d, k, Y, d, pl.fp, pl.eig, lwork, pl.info));
  CK_SOLVER(cusolverDnDorgqr(h.solver, d, k, k, Y, d, pl.fp, pl.eig, lwork, pl.info));
  return ARCHEAD_OK;
}

// The r right singular vectors of M from its d x d Gram matrix G = M^T M
// (lower triangle, column-major), as columns of Vr (column-major d x r), in
// descending order of the singular value, signs as top_vectors_kernel fixes
// them.  s1, s2: d x d scratch regions.  Exact: the eigendecomposition of G
// (G is overwritten).  Randomised (ARCHead paper §3.2 Eq. 4; Halko, Martinsson
// and Tropp 2011, subspace iteration and Rayleigh-Ritz on G): Y = G Omega with
// a Gaussian Omega of k columns; power_iters times Q = qr(Y), Y = G Q; then
// Q = qr(Y), the k x k projection Q^T G Q, its eigenvectors Phi, and the Ritz
// vectors Q Phi of the r largest Ritz values.
int right_vectors(const Handles& h, const Plan& pl, int lwork, double* G, double* s1, double* s2, int d, int r,
                  const SvdOpts& o, double* Vr, cudaStream_t st) {
  const int k = sketch_cols(d, r, o);
  if (k == 0) {
    CK(eigh(h, G, d, pl.w, pl.eig, lwork, pl.info, st));
    top_vectors_kernel<<<r, kThreads, 0, st>>>(G, d, d, r, Vr);
    CK_CUDA(cudaGetLastError());
    return ARCHEAD_OK;
  }
  const double zero = 0.0, one = 1.0;
  double* Y = s1;                                        // d x k: the sketch, then Q
  double* P = s1 + static_cast<size_t>(d) * k;           // k x k projection (fits: k (d + k) <= d^2)
  double* Z = s2;                                        // d x k: G Q, then the Ritz vectors
  gaussian_kernel<<<grid_for(static_cast<size_t>(d) * k), kThreads, 0, st>>>(Z, static_cast<size_t>(d) * k, o.seed);
  CK_CUDA(cudaGetLastError());
  CK_BLAS(cublasDsymm(h.blas, CUBLAS_SIDE_LEFT, CUBLAS_FILL_MODE_LOWER, d, k, &one, G, d, Z, d, &zero, Y, d));
  for (int it = 0; it < o.power_iters; ++it) {
    CK(orthonormalise(h, pl, lwork, Y, d, k));
    CK_BLAS(cublasDsymm(h.blas, CUBLAS_SIDE_LEFT, CUBLAS_FILL_MODE_LOWER, d, k, &one, G, d, Y, d, &zero, Z, d));
    CK_CUDA(cudaMemcpyAsync(Y, Z, static_cast<size_t>(d) * k * sizeof(double), cudaMemcpyDeviceToDevice, st));
  }
  CK(orthonormalise(h, pl, lwork, Y, d, k));
  CK_BLAS(cublasDsymm(h.blas, CUBLAS_SIDE_LEFT, CUBLAS_FILL_MODE_LOWER, d, k, &one, G, d, Y, d, &zero, Z, d));
  CK_BLAS(cublasDgemm(h.blas, CUBLAS_OP_T, CUBLAS_OP_N, k, k, d, &one, Y, d, Z, d, &zero, P, k));
  int lk = 0;
  CK_SOLVER(cusolverDnDsyevd_bufferSize(h.solver, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_LOWER, k, P, k, pl.w,
                                        &lk));
  if (lk > lwork) {
    set_err("right_vectors: eigensolver scratch %d > %d", lk, lwork);
    return ARCHEAD_ENOMEM;
  }
  CK(eigh(h, P, k, pl.w, pl.eig, lwork, pl.info, st));
  CK_BLAS(cublasDgemm(h.blas, CUBLAS_OP_N, CUBLAS_OP_N, d, k, k, &one, Y, d, P, k, &zero, Z, d));
  top_vectors_kernel<<<r, kThreads, 0, st>>>(Z, d, k, r, Vr);
  CK_CUDA(cudaGetLastError());
  return ARCHEAD_OK;
}

// §3.1 Eq. 1-2 into Tp, Ti (column-major d x d; both symmetric).  Uses
// big1 (H in fp64), mat[0] (C, then Q), mat[3], mat[4] (Q Lambda^{+-p}).
int metric_impl(const Handles& h, const Plan& pl, int lwork, int d, int N, const float* H, double lam, double p,
                double* Tp, double* Ti, cudaStream_t st) {
  const size_t nh = static_cast<size_t>(N) * d;
  to_f64_kernel<<<grid_for(nh), kThreads, 0, st>>>(H, pl.big1, nh);
  CK_CUDA(cudaGetLastError());
  // Row-major H [N, d] is the column-major d x N matrix H^T: H^T (H^T)^T / N = C.
  const double inv_n = 1.0 / N, zero = 0.0, one = 1.0;
  CK_BLAS(cublasDsyrk(h.blas, CUBLAS_FILL_MODE_LOWER, CUBLAS_OP_N, d, N, &inv_n, pl.big1, d, &zero, pl.mat[0], d));
  damp_kernel<<<1, 1024, 0, st>>>(pl.mat[0], d, lam);
  CK_CUDA(cudaGetLastError());
  CK(eigh(h, pl.mat[0], d, pl.w, pl.eig, lwork, pl.info, st));
  double wmin = 0.0;
  CK_CUDA(cudaMemcpyAsync(&wmin, pl.w, sizeof(double), cudaMemcpyDeviceToHost, st));
  CK_CUDA(cudaStreamSynchronize(st));
  if (!(wmin > 0.0)) {
    set_err("damped covariance is not positive definite (smallest eigenvalue %g)", wmin);
    return ARCHEAD_EINVAL;
  }
  powers_kernel<<<(d + kThreads - 1) / kThreads, kThreads, 0, st>>>(pl.w, d, p, pl.fp, pl.fm);
  scale_columns_kernel<<<grid_for(static_cast<size_t>(d) * d), kThreads, 0, st>>>(pl.mat[0], pl.fp, pl.fm, d,
                                                                                 pl.mat[3], pl.mat[4]);
  CK_CUDA(cudaGetLastError());
  // T_p = (Q Lambda^p) Q^T, T_p^-1 = (Q Lambda^-p) Q^T.
  CK_BLAS(cublasDgemm(h.blas, CUBLAS_OP_N, CUBLAS_OP_T, d, d, d, &one, pl.mat[3], d, pl.mat[0], d, &zero, Tp, d));
  CK_BLAS(cublasDgemm(h.blas, CUBLAS_OP_N, CUBLAS_OP_T, d, d, d, &one, pl.mat[4], d, pl.mat[0], d, &zero, Ti, d));
  return ARCHEAD_OK;
}

// §3.2 Eq. 4-5 and the INT8 factors.  E row-major [V, d] (the column-major
// d x V matrix E^T).  Uses mat[0] (E^T E), mat[3] (E^T E T_p), mat[4]
// (T_p E^T E T_p, then its eigenvectors), vec (V_w), vec2, fac.
int correction_impl(const Handles& h, const Plan& pl, int lwork, int V, int d, int r_r, int g_B, const double* E,
                    const double* Tp, const double* Ti, const SvdOpts& svd, int8_t* A, uint16_t* s_A, int8_t* B,
                    uint16_t* s_B, cudaStream_t st) {
  const double zero = 0.0, one = 1.0;
  // The right singular vectors of E T_p are the eigenvectors of its Gram
  // matrix (E T_p)^T (E T_p) = T_p (E^T E) T_p.
  CK_BLAS(cublasDsyrk(h.blas, CUBLAS_FILL_MODE_LOWER, CUBLAS_OP_N, d, V, &one, E, d, &zero, pl.mat[0], d));
  CK_BLAS(cublasDsymm(h.blas, CUBLAS_SIDE_LEFT, CUBLAS_FILL_MODE_LOWER, d, d, &one, pl.mat[0], d, Tp, d, &zero,
                      pl.mat[3], d));
  CK_BLAS(cublasDgemm(h.blas, CUBLAS_OP_N, CUBLAS_OP_N, d, d, d, &one, Tp, d, pl.mat[3], d, &zero, pl.mat[4], d));
  CK(right_vectors(h, pl, lwork, pl.mat[4], pl.mat[0], pl.mat[3], d, r_r, svd, pl.vec, st));
  // Z = T_p V_w (d x r_r); A_w = U S = E T_p V_w = E Z, row-major [V, r_r] =
  // the column-major r_r x V matrix Z^T E^T.
  CK_BLAS(cublasDgemm(h.blas, CUBLAS_OP_N, CUBLAS_OP_N, d, r_r, d, &one, Tp, d, pl.vec, d, &zero, pl.vec2, d));
  CK_BLAS(cublasDgemm(h.blas, CUBLAS_OP_T, CUBLAS_OP_N, r_r, V, d, &one, pl.vec2, d, E, d, &zero, pl.fac, r_r));
  // B_w = V_w^T T_p^-1, row-major [r_r, d] = the column-major d x r_r matrix
  // (T_p^-1)^T V_w.
  CK_BLAS(cublasDgemm(h.blas, CUBLAS_OP_T, CUBLAS_OP_N, d, r_r, d, &one, Ti, d, pl.vec, d, &zero, pl.vec2, d));
  CK(launch_quantize(pl.fac, V, r_r, 8, r_r, A, s_A, nullptr, st));
  CK(launch_quantize(pl.vec2, r_r, d, 8, g_B, B, s_B, nullptr, st));
  return ARCHEAD_OK;
}

bool valid_desc(const archead_desc* x) {
  if (!x) return false;
  const int lim = x->V < x->d ? x->V : x->d;
  return x->V >= 1 && x->d >= 1 && x->r_c >= 0 && x->r_r >= 0 && x->r_c <= lim && x->r_r <= lim &&
         x->g >= 1 && x->g_B >= 1 && x->d % x->g == 0 && x->d % x->g_B == 0;
}

int query_lwork(int d, int* lwork) {
  const Handles* hp = nullptr;
  CK(get_handles(nullptr, &hp));
  const Handles& h = *hp;
  return eig_lwork(h.solver, d, lwork);
}

int check_ws(const Plan& need, const void* ws, size_t ws_bytes) {
  if (!ws) {
    set_err("workspace is null");
    return ARCHEAD_EINVAL;
  }
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) {
    set_err("workspace is not 256-byte aligned");
    return ARCHEAD_EALIGN;
  }
  if (ws_bytes < need.bytes) {
    set_err("workspace has %zu bytes, %zu needed", ws_bytes, need.bytes);
    return ARCHEAD_ENOMEM;
  }
  return ARCHEAD_OK;
}

}  // namespace

extern "C" {

ARCHEAD_API const char* archead_build_last_error(void) { return g_err; }

ARCHEAD_API size_t archead_build_workspace_bytes(const archead_desc* desc, int32_t n_calib) {
  if (!valid_desc(desc) || n_calib < 1) return 0;
  int lwork = 0;
  if (query_lwork(desc->d, &lwork) != ARCHEAD_OK) return 0;
  const int rmax = desc->r_c > desc->r_r ? desc->r_c : desc->r_r;
  return make_plan(nullptr, desc->V, desc->d, n_calib, rmax > 0 ? rmax : 1, lwork).bytes;
}

ARCHEAD_API int archead_build_quantize(const double* x, int32_t rows, int32_t cols, int32_t bits, int32_t group,
                                       int8_t* codes, uint16_t* scales, archead_stream_t stream) {
  g_err[0] = '\0';
  if (!x || !codes || !scales) {
    set_err("quantise: null pointer");
    return ARCHEAD_EINVAL;
  }
  return launch_quantize(x, rows, cols, bits, group == 0 ? cols : group, codes, scales, nullptr,
                         reinterpret_cast<cudaStream_t>(stream));
}

ARCHEAD_API int archead_build_metric(int32_t d, int32_t n_calib, const float* H, double lam, double p,
                                     double* T_p, double* T_p_inv, void* workspace, size_t ws_bytes,
                                     archead_stream_t stream) {
  g_err[0] = '\0';
  if (d < 1 || n_calib < 1 || !H || !T_p || !T_p_inv || !(lam >= 0.0) || !std::isfinite(p)) {
    set_err("metric: bad argument");
    return ARCHEAD_EINVAL;
  }
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Handles* hp = nullptr;
  CK(get_handles(st, &hp));
  const Handles& h = *hp;
  int lwork = 0;
  CK(eig_lwork(h.solver, d, &lwork));
  const Plan need = make_plan(nullptr, 1, d, n_calib, 1, lwork);
  CK(check_ws(need, workspace, ws_bytes));
  const Plan pl = make_plan(static_cast<uint8_t*>(workspace), 1, d, n_calib, 1, lwork);
  CK(metric_impl(h, pl, lwork, d, n_calib, H, lam, p, T_p, T_p_inv, st));
  CK_CUDA(cudaStreamSynchronize(st));
  return ARCHEAD_OK;
}

}  // extern "C"

namespace {

// archead_svd_opts -> SvdOpts (null: exact); false on a bad option.
bool read_svd(const archead_svd_opts* o, SvdOpts* out) {
  *out = SvdOpts{};
  if (o == nullptr) return true;
  if ((o->method != ARCHEAD_SVD_EXACT && o->method != ARCHEAD_SVD_RANDOMIZED) || o->oversample < 0 ||
      o->power_iters < 0 || o->power_iters > 64)
    return false;
  out->method = o->method;
  out->oversample = o->oversample;
  out->power_iters = o->power_iters;
  out->seed = o->seed;
  return true;
}

int build_correction(const archead_desc* desc, const double* E, const double* T_p, const double* T_p_inv,
                     const archead_svd_opts* svd_opts, int8_t* A, uint16_t* s_A, int8_t* B, uint16_t* s_B,
                     void* workspace, size_t ws_bytes, archead_stream_t stream) {
  g_err[0] = '\0';
  SvdOpts svd;
  if (!read_svd(svd_opts, &svd)) {
    set_err("correction: bad SVD options");
    return ARCHEAD_EINVAL;
  }
  if (!valid_desc(desc) || desc->r_r < 1 || !E || !T_p || !T_p_inv || !A || !s_A || !B || !s_B) {
    set_err("correction: bad argument");
    return ARCHEAD_EINVAL;
  }
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Handles* hp = nullptr;
  CK(get_handles(st, &hp));
  const Handles& h = *hp;
  int lwork = 0;
  CK(eig_lwork(h.solver, desc->d, &lwork));
  const Plan need = make_plan(nullptr, desc->V, desc->d, 1, desc->r_r, lwork);
  CK(check_ws(need, workspace, ws_bytes));
  const Plan pl = make_plan(static_cast<uint8_t*>(workspace), desc->V, desc->d, 1, desc->r_r, lwork);
  CK(correction_impl(h, pl, lwork, desc->V, desc->d, desc->r_r, desc->g_B, E, T_p, T_p_inv, svd, A, s_A, B, s_B,
                     st));
  CK_CUDA(cudaStreamSynchronize(st));
  return ARCHEAD_OK;
}

int build_head(const archead_desc* desc, const float* W, const float* H, int32_t n_calib, double lam, double p,
               const archead_svd_opts* svd_opts, const archead_device_components* out, void* workspace,
               size_t ws_bytes, archead_stream_t stream) {
  g_err[0] = '\0';
  SvdOpts svd;
  if (!read_svd(svd_opts, &svd)) {
    set_err("build_head: bad SVD options");
    return ARCHEAD_EINVAL;
  }
  if (!valid_desc(desc) || desc->r_c + desc->r_r < 1 || !W || !H || n_calib < 1 || !out || !out->q ||
      !out->s_res || !(lam >= 0.0) || !std::isfinite(p)) {
    set_err("build_head: bad argument");
    return ARCHEAD_EINVAL;
  }
  const int V = desc->V, d = desc->d, r_c = desc->r_c, r_r = desc->r_r;
  if ((r_c > 0 && (!out->L || !out->s_L || !out->R || !out->s_R)) ||
      (r_r > 0 && (!out->A || !out->s_A || !out->B || !out->s_B))) {
    set_err("build_head: null component pointer");
    return ARCHEAD_EINVAL;
  }
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Handles* hp = nullptr;
  CK(get_handles(st, &hp));
  const Handles& h = *hp;
  int lwork = 0;
  CK(eig_lwork(h.solver, d, &lwork));
  const int rmax = r_c > r_r ? r_c : r_r;
  const Plan need = make_plan(nullptr, V, d, n_calib, rmax, lwork);
  CK(check_ws(need, workspace, ws_bytes));
  const Plan pl = make_plan(static_cast<uint8_t*>(workspace), V, d, n_calib, rmax, lwork);
  double* Tp = pl.mat[1];
  double* Ti = pl.mat[2];
  const double zero = 0.0, one = 1.0, minus_one = -1.0;
  const size_t nw = static_cast<size_t>(V) * d;

  // A rank-0 branch is an empty sum: its per-row scales are fp16 zero.
  if (r_c == 0 && out->s_L) CK_CUDA(cudaMemsetAsync(out->s_L, 0, static_cast<size_t>(V) * sizeof(uint16_t), st));
  if (r_r == 0 && out->s_A) CK_CUDA(cudaMemsetAsync(out->s_A, 0, static_cast<size_t>(V) * sizeof(uint16_t), st));

  // Eq. 1-2: the damped activation metric.
  CK(metric_impl(h, pl, lwork, d, n_calib, H, lam, p, Tp, Ti, st));

  // Eq. 3: the rank-r_c core.  Row-major W [V, d] is the column-major d x V
  // matrix W^T; its Gram matrix W^T W has the right singular vectors of W as
  // eigenvectors, and A_c = U S = W V_c.
  to_f64_kernel<<<grid_for(nw), kThreads, 0, st>>>(W, pl.big0, nw);
  CK_CUDA(cudaGetLastError());
  CK_CUDA(cudaMemcpyAsync(pl.big1, pl.big0, nw * sizeof(double), cudaMemcpyDeviceToDevice, st));
  if (r_c > 0) {
    CK_BLAS(cublasDsyrk(h.blas, CUBLAS_FILL_MODE_LOWER, CUBLAS_OP_N, d, V, &one, pl.big0, d, &zero, pl.mat[0], d));
    // V_c, column-major d x r_c: also B_c = V_c^T as a row-major [r_c, d].
    CK(right_vectors(h, pl, lwork, pl.mat[0], pl.mat[3], pl.mat[4], d, r_c, svd, pl.vec, st));
    // A_c row-major [V, r_c] = the column-major r_c x V matrix V_c^T W^T.
    CK_BLAS(cublasDgemm(h.blas, CUBLAS_OP_T, CUBLAS_OP_N, r_c, V, d, &one, pl.vec, d, pl.big0, d, &zero, pl.fac,
                        r_c));
    // W - A_c B_c: column-major (W - A_c B_c)^T = W^T - B_c^T A_c^T = W^T - V_c (A_c^T).
    CK_BLAS(cublasDgemm(h.blas, CUBLAS_OP_N, CUBLAS_OP_N, d, V, r_c, &minus_one, pl.vec, d, pl.fac, r_c, &one,
                        pl.big1, d));
    // Q5(A_c) per row, Q8(B_c) per row; both replaced by their dequantised values.
    CK(launch_quantize(pl.fac, V, r_c, 5, r_c, out->L, out->s_L, pl.fac, st));
    CK(launch_quantize(pl.vec, r_c, d, 8, d, out->R, out->s_R, pl.vec, st));
  }
  // Q_SC4 of the residual, replaced by its dequantised values.
  CK(launch_quantize(pl.big1, V, d, 4, desc->g, out->q, out->s_res, pl.big1, st));
  // E = W - W_d = (W - Q_SC4(.)) - L_hat R_hat.
  rsub_kernel<<<grid_for(nw), kThreads, 0, st>>>(pl.big0, pl.big1, nw);
  CK_CUDA(cudaGetLastError());
  if (r_c > 0)
    CK_BLAS(cublasDgemm(h.blas, CUBLAS_OP_N, CUBLAS_OP_N, d, V, r_c, &minus_one, pl.vec, d, pl.fac, r_c, &one,
                        pl.big1, d));

  // Eq. 4-5: the activation-metric correction of E.
  if (r_r > 0)
    CK(correction_impl(h, pl, lwork, V, d, r_r, desc->g_B, pl.big1, Tp, Ti, svd, out->A, out->s_A, out->B,
                       out->s_B, st));
  CK_CUDA(cudaStreamSynchronize(st));
  return ARCHEAD_OK;
}

}  // namespace

extern "C" {

ARCHEAD_API int archead_build_correction(const archead_desc* desc, const double* E, const double* T_p,
                                         const double* T_p_inv, int8_t* A, uint16_t* s_A, int8_t* B,
                                         uint16_t* s_B, void* workspace, size_t ws_bytes,
                                         archead_stream_t stream) {
  return build_correction(desc, E, T_p, T_p_inv, nullptr, A, s_A, B, s_B, workspace, ws_bytes, stream);
}

ARCHEAD_API int archead_build_correction_svd(const archead_desc* desc, const double* E, const double* T_p,
                                             const double* T_p_inv, const archead_svd_opts* svd, int8_t* A,
                                             uint16_t* s_A, int8_t* B, uint16_t* s_B, void* workspace,
                                             size_t ws_bytes, archead_stream_t stream) {
  return build_correction(desc, E, T_p, T_p_inv, svd, A, s_A, B, s_B, workspace, ws_bytes, stream);
}

ARCHEAD_API int archead_build_head(const archead_desc* desc, const float* W, const float* H, int32_t n_calib,
                                   double lam, double p, const archead_device_components* out, void* workspace,
                                   size_t ws_bytes, archead_stream_t stream) {
  return build_head(desc, W, H, n_calib, lam, p, nullptr, out, workspace, ws_bytes, stream);
}

ARCHEAD_API int archead_build_head_svd(const archead_desc* desc, const float* W, const float* H, int32_t n_calib,
                                       double lam, double p, const archead_svd_opts* svd,
                                       const archead_device_components* out, void* workspace, size_t ws_bytes,
                                       archead_stream_t stream) {
  return build_head(desc, W, H, n_calib, lam, p, svd, out, workspace, ws_bytes, stream);
}

}  // extern "C"
