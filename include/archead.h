/*
 * archead.h -- C ABI of the B200 (sm_100a) library for the forward pass of an
 * ARCHead packed LM-head.
 *
 * Source: "ARCHead: Activation-Metric Residual Correction for Large Language
 * Model Output Heads" (arXiv 2608.02703).
 *   §3.2 Eq. 3   W_d   = Q5(A_c) Q8(B_c) + Q_SC4(W - A_c B_c)   quantised core
 *   §3.2 Eq. 6   W_hat = W_d + A_w B_w                           with INT8 A_w, B_w
 *   §3.2 Eq. 7   Y_hat = H W_d^T + (H B_w^T) A_w^T               factored forward
 *   §3.3         the module registers only the packed tensors and shape metadata;
 *                the dense head is discarded after conversion.
 *
 * In this library's names:
 *   L  [V, r_c]  INT5 codes of Q5(A_c), one fp16 scale per row     s_L [V]
 *   R  [r_c, d]  INT8 codes of Q8(B_c), one fp16 scale per row     s_R [r_c]
 *   q  [V, d]    signed INT4 residual codes (SC4)                  s_res [V, d/g]
 *   A  [V, r_r]  INT8 codes of A_w, one fp16 scale per row         s_A [V]
 *   B  [r_r, d]  INT8 codes of B_w, one fp16 scale per d-group     s_B [r_r, d/g_B]
 * and for hidden states h [T, d] (bf16) the logits are
 *   y[t,v] = s_L[v] sum_k L[v,k] z_c[t,k] + sum_j s_res[v,j/g] q[v,j] h[t,j]
 *          + s_A[v] sum_k A[v,k] z_r[t,k],
 *   z_c[t,k] = s_R[k] sum_j R[k,j] h[t,j],  z_r[t,k] = sum_j s_B[k,j/g_B] B[k,j] h[t,j].
 * The dense V x d head is never formed on the device.
 *
 * Conventions for every call
 *   - Return value: ARCHEAD_OK (0) or a negative ARCHEAD_E* code.  No C++
 *     exception crosses this boundary.
 *   - Device pointers are plain CUDA device addresses owned by the caller; the
 *     library allocates no device memory (the host-buffer forms may keep
 *     captured CUDA graphs and one stream per handle, driver resources that
 *     archead_free releases).  Host pointers are only read during the call
 *     (or, for the *_host entry points, until it returns).
 *   - Forward calls are asynchronous on the given stream and never synchronise
 *     the host (except archead_lse_argmax_host, which is the host-buffer form).
 *     A fault inside a kernel surfaces at the caller's next synchronisation.
 *   - Alignment: arena and workspace 256 bytes, hidden 16 bytes, every other
 *     device buffer 4 bytes; otherwise ARCHEAD_EALIGN.
 *   - The kernels are built for sm_100a only; pack_load returns ARCHEAD_EUNSUP
 *     on any other device.
 */
#ifndef ARCHEAD_H
#define ARCHEAD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ARCHEAD_API __attribute__((visibility("default")))

typedef struct CUstream_st* archead_stream_t; /* == cudaStream_t; NULL = legacy default stream */

enum {
  ARCHEAD_OK = 0,
  ARCHEAD_EINVAL = -1,   /* null pointer, bad shape, T <= 0, code out of range, bad scale */
  ARCHEAD_EALIGN = -2,   /* a pointer is not aligned as required */
  ARCHEAD_EUNSUP = -3,   /* shape or device the compiled kernels do not support */
  ARCHEAD_ECUDA = -4,    /* a CUDA runtime call failed: see archead_last_cuda_error() */
  ARCHEAD_ENOMEM = -5,   /* a host allocation failed, or a caller buffer is too small */
  ARCHEAD_ETIMEOUT = -6  /* a bounded device-side wait expired (read back by archead_workspace_status) */
};

/* Device-side status bits written into the workspace by the kernels. */
enum {
  ARCHEAD_STATUS_WAIT_TIMEOUT = 1, /* a pipeline wait gave up; that call's outputs are invalid */
  ARCHEAD_STATUS_BAD_TARGET = 2    /* a target id was outside [0, V); its CE is NaN */
};

/* Shape metadata of one packed head (§3.3: "group size and shape metadata").
 * Supported: V >= 1; d a positive multiple of 64; g a power of two >= 16
 * dividing d; g_B >= 1 dividing d; r_c >= 0; r_r >= 0. */
typedef struct archead_desc {
  int32_t V, d, r_c, r_r, g, g_B;
} archead_desc;

/* Canonical packed components in host memory, row-major, one code per int8
 * element holding the two's-complement value; scales are IEEE fp16 bit
 * patterns.  Ranges: L in [-16,15], q in [-8,7], R / A / B in [-128,127].
 * The list is the state-dict component list of §3.3. */
typedef struct archead_host_components {
  const int8_t* L;   const uint16_t* s_L;    /* [V, r_c],  [V]          */
  const int8_t* R;   const uint16_t* s_R;    /* [r_c, d],  [r_c]        */
  const int8_t* q;   const uint16_t* s_res;  /* [V, d],    [V, d/g]     */
  const int8_t* A;   const uint16_t* s_A;    /* [V, r_r],  [V]          */
  const int8_t* B;   const uint16_t* s_B;    /* [r_r, d],  [r_r, d/g_B] */
} archead_host_components;

typedef struct archead_handle archead_handle;

/* §3.3 Eq. 10: bytes(ARCHead) = sum_i numel(theta_i) * element_size(theta_i)
 * over the registered components, with INT5 and INT4 codes at 5 and 4 bits:
 *   V(5 r_c/8 + 2 + d/2 + 2d/g + r_r + 2) + r_c(d + 2) + r_r(d + 2d/g_B).
 * Returns 0 for an unsupported or null desc. */
ARCHEAD_API size_t archead_packed_bytes(const archead_desc* desc);

/* Device bytes the packed arena needs: the Eq. 10 payload in the kernels'
 * tile layout plus padding (vocabulary rounded up to 16 rows, r_c to 64,
 * r_r to 32, segments to 16 and regions to 256 bytes).  0 if unsupported. */
ARCHEAD_API size_t archead_arena_bytes(const archead_desc* desc);

/* Validate the components, re-lay them out for the kernels and copy them into
 * the caller-owned device arena (>= archead_arena_bytes, 256-byte aligned, on
 * the current device).  This is the conversion step of §3.3: afterwards the
 * arena is immutable and the host arrays may be freed.  Synchronises `stream`
 * before returning (the host staging buffer is released).  On success *out is
 * a new host-side handle that points into the arena without owning it; free it
 * with archead_free.  Codes out of range, or inf / NaN scales: ARCHEAD_EINVAL. */
ARCHEAD_API int archead_pack_load(const archead_desc* desc, const archead_host_components* comps,
                                  void* dev_arena, size_t arena_bytes, archead_stream_t stream,
                                  archead_handle** out);

/* Host-side form of the conversion: validate the components and write the
 * arena image (the exact bytes archead_pack_load copies to the device) into
 * host memory of >= archead_arena_bytes bytes.  The image can be stored and
 * later copied into an arena as is; it is position independent.  Same error
 * codes as archead_pack_load; no CUDA call is made. */
ARCHEAD_API int archead_pack_image(const archead_desc* desc, const archead_host_components* comps,
                                   void* host_image, size_t image_bytes);

/* Which kernel a forward call with T tokens runs its vocabulary pass on:
 *   ARCHEAD_KERNEL_DECODE        the streaming decode kernel (up to 8 tokens
 *                                per launch, mma.sync fragments in registers);
 *   ARCHEAD_KERNEL_TENSOR_CORE   the tcgen05 kernel (T >= 9 and g_B a multiple
 *                                of 64): weights dequantised into tensor
 *                                memory, 128 rows x up to 128 tokens per unit.
 * Both compute Eq. 7 of §3.2; -1 if handle is null or T <= 0.  (A library
 * query with no counterpart in the paper.) */
enum { ARCHEAD_KERNEL_DECODE = 0, ARCHEAD_KERNEL_TENSOR_CORE = 1 };
ARCHEAD_API int archead_forward_kernel(const archead_handle* handle, int32_t T);

/* Workspace bytes one forward call with T tokens needs (256-byte aligned
 * scratch, caller-owned; reused across calls on one stream).  Holds the
 * low-rank prologue output z (decode kernel) or the fp16 activation operand
 * [h | z] (tensor-core kernel), per-block log-sum-exp partials, completion
 * tickets and the status word.  Zero-fill a workspace once before its first
 * use (the status word is sticky; every ticket is back at zero when a call
 * ends); afterwards the calls keep it consistent.
 * Calls that share a workspace must be ordered (same stream).  0 if handle is
 * null or T <= 0. */
ARCHEAD_API size_t archead_workspace_bytes(const archead_handle* handle, int32_t T);

/* Logits of Eq. 7 for T tokens.
 *   hidden   [T, d] bf16 bit patterns, row-major, device.
 *   logits   [T, V] fp32, row-major, device; may be NULL.
 *   argmax   [T] int32, device, lowest index of the row maximum; may be NULL.
 * At least one of logits / argmax must be non-NULL. */
ARCHEAD_API int archead_logits(const archead_handle* handle, const uint16_t* hidden, int32_t T,
                               float* logits, int32_t* argmax,
                               void* workspace, size_t workspace_bytes, archead_stream_t stream);

/* Fused vocabulary-wide epilogue (the head feeds softmax directly, §1): per
 * token, without writing the [T, V] logits,
 *   lse[t]    = log sum_v exp(y[t,v])                    fp32, device, required
 *   argmax[t] = lowest v attaining max_v y[t,v]          int32, device, required
 *   ce[t]     = lse[t] - y[t, targets[t]]                fp32, device; NULL to skip
 * targets [T] int32 in [0, V), device; required when ce is non-NULL.  A
 * target outside [0, V) gives ce = NaN and sets ARCHEAD_STATUS_BAD_TARGET.
 * log_softmax(y)[t,v] = y[t,v] - lse[t]. */
ARCHEAD_API int archead_logits_lse_argmax(const archead_handle* handle, const uint16_t* hidden,
                                          int32_t T, const int32_t* targets, float* lse,
                                          int32_t* argmax, float* ce, void* workspace,
                                          size_t workspace_bytes, archead_stream_t stream);

/* Host-buffer form of archead_logits_lse_argmax: hidden [T, d] and targets [T]
 * are HOST pointers (pinned memory recommended), copied to the device inside
 * the workspace; lse / argmax / ce are HOST pointers filled before return.
 * workspace must be >= archead_host_workspace_bytes(handle, T).  Synchronises
 * the stream.  An output in pinned (page-locked, device-mapped) host memory is
 * written there by the kernels, with no copy after them; outputs in pageable
 * memory go through the workspace and a device-to-host copy.  When every host buffer is
 * pinned, the call's fixed sequence (copies in, the forward launches, any
 * copies out) is captured once per distinct set of arguments (the last four
 * are kept per handle) and replayed with one graph launch; otherwise, or if
 * the capture fails, it runs directly. */
ARCHEAD_API size_t archead_host_workspace_bytes(const archead_handle* handle, int32_t T);
ARCHEAD_API int archead_lse_argmax_host(const archead_handle* handle, const uint16_t* hidden_host,
                                        int32_t T, const int32_t* targets_host, float* lse_host,
                                        int32_t* argmax_host, float* ce_host, void* workspace,
                                        size_t workspace_bytes, archead_stream_t stream);

/* Host-buffer form of archead_logits: hidden [T, d] bf16 is a HOST pointer
 * (pinned memory recommended) copied to the device inside the workspace; the
 * logits [T, V] fp32 and argmax [T] int32 are HOST pointers filled before
 * return (either may be NULL, not both).  workspace (device, 256-byte
 * aligned) must be >= archead_host_logits_workspace_bytes(handle, T): it
 * stages the hidden states (and logits bound for pageable memory) on the
 * device.  Synchronises the stream.  Pinned outputs, the logits included, are
 * written by the kernels and pinned buffers take the captured sequence, as in
 * archead_lse_argmax_host. */
ARCHEAD_API size_t archead_host_logits_workspace_bytes(const archead_handle* handle, int32_t T);
ARCHEAD_API int archead_logits_host(const archead_handle* handle, const uint16_t* hidden_host, int32_t T,
                                    float* logits_host, int32_t* argmax_host, void* workspace,
                                    size_t workspace_bytes, archead_stream_t stream);

/* Allocation-free form of archead_logits_lse_argmax, for callers that may not
 * allocate device memory when they run the head (for example while a CUDA
 * graph is being captured under an allocator that forbids it, or inside a
 * host framework that owns all device memory).  Same arguments and results,
 * without the workspace: scratch comes from a fixed array of
 * archead_static_workspace_capacity() bytes (2 MiB) in the library's own device
 * memory, held by every GPU that loads the library until the process exits.
 * The first call on a device, with that device current, looks the array up
 * (cudaGetSymbolAddress) and clears its status word with an asynchronous
 * memset on `stream`, so make that first call before any stream capture.  A
 * new context on the device (after cudaDeviceReset) is noticed by its handle
 * and set up again the same way.  All calls on a device share the array:
 * calls that may overlap on the GPU race.  A T whose workspace would not fit
 * the array returns ARCHEAD_ENOMEM.  (No counterpart in the paper: a library
 * convenience.) */
ARCHEAD_API size_t archead_static_workspace_capacity(void);
ARCHEAD_API int archead_logits_lse_argmax_static(const archead_handle* handle, const uint16_t* hidden,
                                                 int32_t T, const int32_t* targets, float* lse,
                                                 int32_t* argmax, float* ce, archead_stream_t stream);

/* Status word of the fixed array behind archead_logits_lse_argmax_static on
 * the current device: the OR of ARCHEAD_STATUS_* bits its calls raised since
 * the last clear (a timed-out wait, or a target id outside [0, V) whose CE is
 * NaN).  clear != 0 resets it, ordered on `stream`.  Synchronises `stream`.
 * Returns ARCHEAD_ETIMEOUT if ARCHEAD_STATUS_WAIT_TIMEOUT is set.  (No
 * counterpart in the paper.) */
ARCHEAD_API int archead_static_workspace_status(int clear, archead_stream_t stream, uint32_t* status_out);

/* Temperature sampling fused into the vocabulary pass (a consumer of the
 * logits of Eq. 7 with no counterpart in the paper): for each token t,
 *   sampled[t] = first argmax over rows v of  y[t,v] / temperature + G[t,v],
 * G[t,v] = -log(-log(u)), u = (k + 1/2) / 2^23 with k the top 23 bits of word
 * (v mod 4) of Philox4x64-10 (Salmon et al., SC 2011) at counter
 * (offset + t, v / 4, 0, 0) and key (seed, 0); v is the global row (see the
 * vocabulary shards below).  This draws v with probability
 * softmax(y[t] / temperature)_v (Gumbel-max).  lse and argmax (of the
 * untempered logits) may be NULL.  Runs on the decode kernel for every T;
 * same workspace and stream rules as archead_logits_lse_argmax.  EINVAL unless
 * 0 < temperature < inf. */
ARCHEAD_API int archead_sample(const archead_handle* handle, const uint16_t* hidden, int32_t T, float temperature,
                               uint64_t seed, uint64_t offset, int32_t* sampled, float* lse, int32_t* argmax,
                               void* workspace, size_t workspace_bytes, archead_stream_t stream);

/* Vocabulary shards (one process per GPU, each holding a contiguous range of
 * vocabulary rows; R, B and their scales replicated).  The rows of Eq. 7 of
 * §3.2 are independent, so a shard computes its logits alone and only the
 * per-token softmax statistics cross GPUs.  (A library extension for
 * vocabulary-parallel serving; the paper runs on one GPU.)
 *
 * archead_set_vocab_shard: this head holds global rows
 *   [row_offset, row_offset + V) of a vocabulary of vocab_total rows.  After it,
 *   argmax ids are global, target ids are global ids in [0, vocab_total) (others
 *   raise ARCHEAD_STATUS_BAD_TARGET; a target in another shard is not an error),
 *   and the forward entry points report over this shard's rows (CE is NaN when
 *   the target is elsewhere).  EINVAL unless 0 <= row_offset, row_offset is a
 *   multiple of 16 and row_offset + V <= vocab_total.
 * archead_shard_partials: per token t, partials[4t .. 4t+3] = (log-sum-exp over
 *   this shard's rows, the largest logit, the global row of its first
 *   occurrence as int32 bits, the target logit or NaN when the target row is
 *   in another shard or targets is NULL).  partials is device memory, 16-byte
 *   aligned; same workspace and stream rules as archead_logits_lse_argmax.
 * archead_merge_shards: partials of n_shards shards stacked [n_shards][T][4]
 *   in increasing row order (an all-gather in rank order when ranks hold
 *   increasing row ranges) -> LSE over all rows, first argmax, CE = LSE - the
 *   target logit (NaN if no shard held the target).  Any output may be NULL,
 *   not all three.  Device pointers; no workspace. */
ARCHEAD_API int archead_set_vocab_shard(archead_handle* handle, int32_t row_offset, int32_t vocab_total);
ARCHEAD_API int archead_shard_partials(const archead_handle* handle, const uint16_t* hidden, int32_t T,
                                       const int32_t* targets, float* partials, void* workspace,
                                       size_t workspace_bytes, archead_stream_t stream);
ARCHEAD_API int archead_merge_shards(const float* partials, int32_t n_shards, int32_t T, float* lse,
                                     int32_t* argmax, float* ce, archead_stream_t stream);

/* Sampling across vocabulary shards (with archead_set_vocab_shard):
 * archead_sample_partials: per token t, sample_partials[2t .. 2t+1] = (the
 *   largest y[t,v] / temperature + G[t,v] over this shard's rows, the global
 *   row of its first occurrence as int32 bits), G drawn for the global row v
 *   exactly as archead_sample draws it, so a pick does not depend on how the
 *   vocabulary is split.  sample_partials: device, 8-byte aligned, [T][2]
 *   floats (also scratch for the call).  Same arguments, workspace and
 *   stream rules as archead_sample otherwise.
 * archead_merge_sample_shards: pairs of n_shards shards stacked
 *   [n_shards][T][2] in increasing row order -> sampled[t], the first maximum
 *   over all rows: the id archead_sample returns for the unsharded head.
 *   Device pointers; no workspace. */
ARCHEAD_API int archead_sample_partials(const archead_handle* handle, const uint16_t* hidden, int32_t T,
                                        float temperature, uint64_t seed, uint64_t offset, float* sample_partials,
                                        void* workspace, size_t workspace_bytes, archead_stream_t stream);
ARCHEAD_API int archead_merge_sample_shards(const float* sample_partials, int32_t n_shards, int32_t T,
                                            int32_t* sampled, archead_stream_t stream);

/* Read (and with clear != 0, reset) the device status word of a workspace:
 * a bitwise OR of ARCHEAD_STATUS_* since the last clear.  Synchronises the
 * stream.  Returns ARCHEAD_ETIMEOUT if ARCHEAD_STATUS_WAIT_TIMEOUT is set. */
ARCHEAD_API int archead_workspace_status(void* workspace, int clear, archead_stream_t stream,
                                         uint32_t* status_out);

/* Optional profiling hook: when both are non-NULL (cudaEvent_t handles), every
 * later forward call on this handle records `before` on its stream just before
 * the first vocabulary-pass launch and `after` just after the last one, so
 * cudaEventElapsedTime(before, after) is the device time of the vocabulary
 * pass alone (the low-rank prologue or activation kernel and the final
 * per-token fold excluded).  NULL, NULL switches it off. */
ARCHEAD_API int archead_set_profile_events(archead_handle* handle, void* before, void* after);

/* Test support for the decode kernel's bounded waits (no counterpart in the
 * paper).  Every pipeline wait of the decode kernel gives up after
 * wait_limit_ns (2 s unless set here), raises ARCHEAD_STATUS_WAIT_TIMEOUT in
 * the workspace status word and makes its block skip the remaining work, so
 * the call's outputs are invalid but the context stays usable.  With
 * stall != 0, later decode-kernel calls on this handle first wait on a
 * barrier that nothing completes, so the limit expires on purpose.  EINVAL if
 * handle is NULL or wait_limit_ns is 0.  Restore with (2000000000, 0). */
ARCHEAD_API int archead_test_decode_waits(archead_handle* handle, uint64_t wait_limit_ns, int stall);

/* Free a handle and the captured sequences of its host-buffer calls (the arena
 * stays with the caller). */
ARCHEAD_API void archead_free(archead_handle* handle);

/* The last cudaError_t seen by a call that returned ARCHEAD_ECUDA (thread-local). */
ARCHEAD_API int archead_last_cuda_error(void);

/* Static text for a status code. */
ARCHEAD_API const char* archead_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* ARCHEAD_H */
