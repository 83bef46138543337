/*
 * archead_build.h -- C ABI of the GPU construction of an ARCHead packed head
 * (libarchead_build.so), the step that produces the components archead.h
 * consumes.
 *
 * Source: "ARCHead: Activation-Metric Residual Correction for Large Language
 * Model Output Heads" (arXiv 2608.02703).
 *   §3.1 Eq. 1   C = H^T H / N from N calibration hidden states H [N, d]
 *   §3.1 Eq. 2   C_lam = C + lam * mean(diag C) * I = Q Lambda Q^T,
 *                T_p = Q Lambda^p Q^T,  T_p^-1 = Q Lambda^-p Q^T
 *   §3.2 Eq. 3   W_d = Q5(A_c) Q8(B_c) + Q_SC4(W - A_c B_c), A_c B_c of rank r_c
 *   §3.2 Eq. 4-5 E = W - W_d;  E T_p ~ U S V^T (rank r_r);  A_w = U S,
 *                B_w = V^T T_p^-1;  INT8 A_w per row, B_w per group of g_B
 *   §3.4 (Algorithm 1) the same steps in this order.
 *
 * Readings of points the paper leaves open (the same ones the CPU oracle takes):
 *   - the rank-r_c core A_c B_c is the exact truncated SVD of W with
 *     A_c = U S and B_c = V^T (Eq. 3 names no metric for it);
 *   - both truncated SVDs are exact by default (the paper's randomised SVD
 *     approximates this; archead_build_head_svd runs the randomised one);
 *     they are computed from the d x d Gram matrices W^T W and T_p E^T E T_p,
 *     whose eigenvectors are the right singular vectors, with the left factor
 *     as W V (resp. E T_p V);
 *   - each singular pair's sign is fixed so that the largest-magnitude entry
 *     of the right singular vector is positive (first index on ties);
 *   - quantisers are symmetric: s = fp16(amax / qmax), codes
 *     clamp(rint(x / s), qmin, qmax) with the fp16-rounded s (round half to
 *     even), s = 0 and codes 0 for an all-zero group; qmax = 7, 15, 127 and
 *     qmin = -8, -16, -128 for 4, 5 and 8 bits.
 *
 * Conventions
 *   - Return value: ARCHEAD_OK or a negative ARCHEAD_E* code of archead.h;
 *     archead_build_last_error() describes the last failure of this thread.
 *   - All matrices are row-major device buffers owned by the caller.  Scratch
 *     comes from the caller's workspace (archead_build_workspace_bytes,
 *     256-byte aligned); the only device memory allocated inside a call is
 *     what the cuBLAS and cuSOLVER handles reserve for themselves: the
 *     library creates one of each on a thread's first call on a device and
 *     keeps them for the life of the process.
 *   - Arithmetic is IEEE fp64 (cuBLAS DGEMM / DSYRK / DSYMM for the dense
 *     products, cuSOLVER DSYEVD for the symmetric eigenproblems, this
 *     library's kernels for everything else).
 *   - archead_build_quantize is asynchronous on the stream; the other calls
 *     synchronise the stream before they return (they read the eigensolver's
 *     status and the smallest eigenvalue of C_lam on the host).
 */
#ifndef ARCHEAD_BUILD_H
#define ARCHEAD_BUILD_H

#include <stddef.h>
#include <stdint.h>

#include "archead.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Device destinations of the canonical components (same names, shapes and
 * code ranges as archead_host_components). */
typedef struct archead_device_components {
  int8_t* L;   uint16_t* s_L;     /* [V, r_c], [V]           */
  int8_t* R;   uint16_t* s_R;     /* [r_c, d], [r_c]         */
  int8_t* q;   uint16_t* s_res;   /* [V, d],   [V, d / g]    */
  int8_t* A;   uint16_t* s_A;     /* [V, r_r], [V]           */
  int8_t* B;   uint16_t* s_B;     /* [r_r, d], [r_r, d / g_B] */
} archead_device_components;

/* Bytes of workspace archead_build_head needs for this shape and n_calib
 * calibration rows (also enough for archead_build_metric and
 * archead_build_correction of the same d, V and ranks).  Needs a current CUDA
 * device (it sizes the eigensolver's scratch).  0 on an invalid shape or a
 * failed query. */
ARCHEAD_API size_t archead_build_workspace_bytes(const archead_desc* desc, int32_t n_calib);

/* Symmetric b-bit quantiser of §3.2 (the one Eq. 3 and the INT8 factors use):
 * x [rows, cols] fp64 -> codes int8 [rows, cols] and fp16 scale bits
 * [rows, cols / group]; group = 0 means one scale per row.  bits in {4, 5, 8};
 * group must divide cols.  Asynchronous.  EINVAL on a bad argument. */
ARCHEAD_API int archead_build_quantize(const double* x, int32_t rows, int32_t cols, int32_t bits, int32_t group,
                                       int8_t* codes, uint16_t* scales, archead_stream_t stream);

/* §3.1 Eq. 1-2: T_p and T_p^-1 [d, d] (fp64) from calibration states H
 * [n_calib, d] (fp32).  lam >= 0, any real p.  EINVAL when C_lam is not
 * positive definite (its smallest eigenvalue <= 0). */
ARCHEAD_API int archead_build_metric(int32_t d, int32_t n_calib, const float* H, double lam, double p,
                                     double* T_p, double* T_p_inv, void* workspace, size_t ws_bytes,
                                     archead_stream_t stream);

/* §3.2 Eq. 4-5 and the INT8 storage of the factors: from the core's
 * remainder E [V, d] (fp64) and T_p, T_p^-1 [d, d], the codes and scales of
 * A (per row) and B (per group of g_B along d).  Uses desc->V, d, r_r, g_B. */
ARCHEAD_API int archead_build_correction(const archead_desc* desc, const double* E, const double* T_p,
                                         const double* T_p_inv, int8_t* A, uint16_t* s_A, int8_t* B,
                                         uint16_t* s_B, void* workspace, size_t ws_bytes,
                                         archead_stream_t stream);

/* Algorithm 1 end to end: from the dense head W [V, d] (fp32) and calibration
 * states H [n_calib, d] (fp32), every component of the packed head, written
 * to the caller's device buffers in `out` (those of a rank-0 branch may be
 * null; its per-row scales, if given, are set to fp16 zero).
 * desc: g and g_B divide d; 0 <= r_c, r_r <= min(V, d); r_c + r_r >= 1.
 * EINVAL on a bad argument or a C_lam that is not positive definite, EALIGN /
 * ENOMEM on a misaligned / too small workspace, ECUDA on a failed CUDA,
 * cuBLAS or cuSOLVER call (archead_build_last_error names it). */
ARCHEAD_API int archead_build_head(const archead_desc* desc, const float* W, const float* H, int32_t n_calib,
                                   double lam, double p, const archead_device_components* out, void* workspace,
                                   size_t ws_bytes, archead_stream_t stream);

/* Method of the two rank-r truncated SVDs (the core of Eq. 3 and E T_p of
 * Eq. 4).
 *   ARCHEAD_SVD_EXACT       the full eigendecomposition of the d x d Gram
 *                           matrix (the readings above; archead_build_head
 *                           and archead_build_correction use it).
 *   ARCHEAD_SVD_RANDOMIZED  the randomised truncated SVD that §3.2 Eq. 4
 *                           prescribes (used for both factorisations): on the
 *                           Gram matrix G = M^T M, a Gaussian test matrix of
 *                           k = min(d, r + oversample, rounded up to a
 *                           multiple of 64 above 64) columns, power_iters
 *                           steps of subspace iteration (Householder QR, then
 *                           G Q), a last QR, and the eigenvectors of the k x k
 *                           projection Q^T G Q mapped back (Rayleigh-Ritz;
 *                           Halko, Martinsson and Tropp 2011).  The r Ritz
 *                           vectors of the largest Ritz values, signs as
 *                           above, replace the exact right singular vectors;
 *                           the rest of the build is unchanged.  When
 *                           k (d + k) > d^2 the exact method is used.  The
 *                           test matrix is a function of seed and the entry
 *                           index (SplitMix64, Box-Muller), so builds repeat.
 * oversample >= 0, 0 <= power_iters <= 64; EINVAL otherwise. */
enum { ARCHEAD_SVD_EXACT = 0, ARCHEAD_SVD_RANDOMIZED = 1 };
typedef struct archead_svd_opts {
  int32_t method;        /* ARCHEAD_SVD_EXACT or ARCHEAD_SVD_RANDOMIZED */
  int32_t oversample;    /* extra sketch columns beyond r */
  int32_t power_iters;   /* subspace iteration steps */
  uint64_t seed;         /* of the Gaussian test matrix */
} archead_svd_opts;

/* archead_build_correction / archead_build_head with the SVD method of svd
 * (NULL: exact).  Same arguments, workspace and errors otherwise. */
ARCHEAD_API int archead_build_correction_svd(const archead_desc* desc, const double* E, const double* T_p,
                                             const double* T_p_inv, const archead_svd_opts* svd, int8_t* A,
                                             uint16_t* s_A, int8_t* B, uint16_t* s_B, void* workspace,
                                             size_t ws_bytes, archead_stream_t stream);
ARCHEAD_API int archead_build_head_svd(const archead_desc* desc, const float* W, const float* H, int32_t n_calib,
                                       double lam, double p, const archead_svd_opts* svd,
                                       const archead_device_components* out, void* workspace, size_t ws_bytes,
                                       archead_stream_t stream);

/* Description of this thread's last failure ("" if none). */
ARCHEAD_API const char* archead_build_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* ARCHEAD_BUILD_H */
