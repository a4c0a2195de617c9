/*
 * kronq.h -- C ABI of libkronq, the sm_100a (B200) implementation of the
 * KronQ per-layer quantization path.
 *
 * The path, in the order the KronQ pages run it:
 *   1. kronq_covariance     H_X = X^T X / N, H_G = G^T G / N
 *   2. kronq_biip_rotate    bidirectional incoherence processing of W, H_X, H_G
 *   3. kronq_sensitivity    s = tr(H_G) tr(H_X)
 *   4. kronq_cholesky_inv   damping and the inverse Cholesky factor of H_X
 *   5. kronq_quantize_layer column-wise OBS quantization with lazy block updates
 *   6. kronq_pack           2/4-bit codes packed into 32-bit words
 * plus kronq_unpack and kronq_layer_loss (a measurement helper).
 *
 * Conventions shared by every call
 *   - Matrices are row-major and contiguous unless a leading dimension is
 *     passed.  W is m x n (m = d_out rows, n = d_in columns).
 *   - Every data pointer is a DEVICE pointer owned by the caller; the library
 *     keeps no pointer after the call returns and allocates no device memory.
 *     Scratch memory comes from the caller's workspace (ws, ws_bytes), at
 *     least kronq_workspace_size() bytes, 256-byte aligned.
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).  Argument errors are detected on the host
 *     and returned before anything is launched.
 *   - Numerical failures found on the device (a non-positive pivot, a wait
 *     that timed out) are written to the optional device word `info`
 *     (0 = fine, otherwise a negative KRONQ_ERR_* code; the first error
 *     wins).  Read it after synchronising the stream.
 *   - Return value: KRONQ_OK or a negative KRONQ_ERR_* code.
 */
#ifndef KRONQ_H
#define KRONQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum kronq_status {
  KRONQ_OK = 0,
  KRONQ_ERR_INVALID_ARG = -1,  /* null pointer, bad shape, misalignment, group not dividing n */
  KRONQ_ERR_UNSUPPORTED = -2,  /* valid request this build does not handle (3-bit packing, a width with no transform) */
  KRONQ_ERR_NOT_PD = -3,       /* damped H_X not positive definite (device-side, via info) */
  KRONQ_ERR_CUDA = -4,         /* a CUDA runtime call failed */
  KRONQ_ERR_TIMEOUT = -5,      /* a bounded wait inside a kernel gave up (device-side, via info) */
  KRONQ_ERR_WORKSPACE = -6     /* workspace missing or smaller than kronq_workspace_size() */
};

/* --incoh_mode of the pages (KronQ README (GitHub), "Mapping paper results to flags"). */
enum kronq_incoh_mode {
  KRONQ_MODE_FULL = 0,        /* both rescales, both rotations */
  KRONQ_MODE_NO_RESCALE = 1,  /* both rotations, no diagonal rescale */
  KRONQ_MODE_SU_ONLY = 2,     /* output side only: S_G and U */
  KRONQ_MODE_SV_ONLY = 3      /* input side only: S_X and V */
};

/* Human-readable name of a status code (static string, never NULL). */
const char* kronq_status_string(int status);

/* ABI version of this header (major * 100 + minor): 101. */
int kronq_abi_version(void);

/* Number of kernels this library has launched in this process (all devices,
 * all streams; a host-side counter, for measurement). */
uint64_t kronq_launch_count(void);

/*
 * Launch timing, a measurement helper (the pages have no counterpart; it
 * lets a benchmark attribute time to kernels that run inside one call).
 * While enabled, the library records a CUDA event pair on the launching
 * stream around every launch of the categories below; kronq_timing_read
 * waits for the recorded events of the current device and returns the
 * summed device time in ms and the number of launches of one category.
 * kronq_timing_enable(on) clears the records (on = 0 also stops recording).
 * Events are created by the library (cudaEventCreate) and reused; do not
 * enable timing while a stream is being captured into a CUDA graph.
 * Recording adds a few microseconds of host time per timed launch.
 */
enum kronq_timer {
  KRONQ_TIMER_LAZY_UPDATE = 0,  /* the solver's lazy block updates (tensor-core GEMMs) */
  KRONQ_TIMER_CHOL_UPDATE = 1,  /* the inverse Cholesky's trailing updates (tensor-core GEMMs) */
  KRONQ_TIMER_CHOL_PANEL = 2,   /* the inverse Cholesky's panel factorisations */
  KRONQ_TIMER_OBS_BLOCK = 3,    /* the solver's 128-column block kernels */
  KRONQ_TIMER_COUNT = 4
};
int kronq_timing_enable(int on);
int kronq_timing_read(int category, double* total_ms, uint64_t* launches);

/*
 * Workspace, in bytes, that kronq_biip_rotate, kronq_cholesky_inv,
 * kronq_quantize_layer and kronq_layer_loss need for a layer of m x n.
 * Returns 0 for invalid sizes.
 */
size_t kronq_workspace_size(int64_t m, int64_t n, int bits, int group, int block);

/*
 * H = alpha * A^T A + beta * H   (d x d, fp32, full symmetric matrix written)
 *
 * KronQ summary (hyper.ai), "Method" (Eq. 7): H_X = E[x x^T] over the
 * calibration activations and H_G = E[g g^T] over the output gradients.
 * With alpha = 1/N over N rows this is the mean; calling it once per chunk of
 * rows with alpha = 1/N_total and beta = 0 for the first chunk and 1 after
 * streams the sum.
 *
 * A     : N x d bf16 (raw bf16 bits), row-major with leading dimension lda
 *         (elements); lda >= d, lda % 8 == 0, A 16-byte aligned.
 * H     : d x d fp32, leading dimension ldh >= d, ldh % 4 == 0, 16-byte aligned.
 *         When beta == 0, H is write-only (its old contents may be NaN).
 * N = 0 : H = beta * H.   d = 0 : no-op.   0 < d < 64: KRONQ_ERR_UNSUPPORTED.
 * info  : optional device int32 (KRONQ_ERR_TIMEOUT on a stuck pipeline).
 * Tensor cores (tcgen05, TMEM accumulators, TMA-fed); only tiles on or above
 * the diagonal are computed; each writes its elements and their mirror
 * images.  When beta != 0 the old H must be symmetric (its upper triangle is
 * read).
 */
int kronq_covariance(const uint16_t* A, int64_t N, int64_t d, int64_t lda,
                     float* H, int64_t ldh, float alpha, float beta,
                     int32_t* info, void* stream);

/*
 * s = tr(H_G) * tr(H_X)   (fp64 sums of the diagonals)
 *
 * KronQ summary (hyper.ai), "Method" (Eq. 14): the sublayer sensitivity,
 * taken after BiIP; sublayers with a larger s receive more bits.
 * H_X: n x n fp32 (leading dim n), H_G: m x m fp32 (leading dim m).
 * out  : DEVICE pointer to 3 doubles: {s, tr(H_X), tr(H_G)}.
 */
int kronq_sensitivity(const float* H_X, int64_t n, const float* H_G, int64_t m,
                      double* out, void* stream);

/*
 * Bidirectional incoherence processing, in place.
 *
 * KronQ summary (hyper.ai), "Method", Eqs. 11-12: diagonal rescale on both
 * sides, then W' = U W V^T, H_X' = V H_X V^T, H_G' = U H_G U^T with
 * randomized Hadamard transforms U = T_m D_u, V = T_n D_v.
 * Rescale: S_X[j] = (H_X[j,j] / ||W[:,j]||^2)^alpha first, then
 * S_G[i] = (H_G[i,i] / ||(W S_X)[i,:]||^2)^alpha; W <- S_G W S_X,
 * H_X <- S_X^-1 H_X S_X^-1, H_G <- S_G^-1 H_G S_G^-1 (a zero diagonal or norm
 * gives a scale of 1).  T_d = C_q (x) H_{2^k}/sqrt(2^k) for d = q 2^k, q odd,
 * C_q the orthonormal DCT-II.
 *
 * W      : m x n fp32, overwritten by W'.   H_X: n x n fp32.   H_G: m x m fp32.
 * sign_u : m int8 (+1/-1), sign_v: n int8.
 * mode   : enum kronq_incoh_mode.
 * S_X, S_G : outputs (n and m fp32) when inverse == 0.
 * inverse = 1 : apply the exact inverse to W only (W = S_G^-1 U^T W' V S_X^-1,
 *          S_X and S_G are then inputs; H_X and H_G may be NULL).
 * Widths: m, n multiples of 16 (KRONQ_ERR_INVALID_ARG otherwise); for
 *         d = q 2^k (q odd) the transform runs as (C_q (x) H_{2^(k-k2)})
 *         (x) H_{2^k2} with 2^k2 = min(2^k, 4096): q <= 63 and
 *         q 2^(k-k2) <= 64 are required (KRONQ_ERR_UNSUPPORTED otherwise;
 *         4096, 8192, 11008, 14336 and 28672 are all covered).
 */
int kronq_biip_rotate(float* W, int64_t m, int64_t n, float* H_X, float* H_G,
                      const int8_t* sign_u, const int8_t* sign_v,
                      float alpha, int mode, int inverse,
                      float* S_X, float* S_G, void* ws, size_t ws_bytes, void* stream);

/*
 * Damping and the inverse Cholesky factor.
 *
 * KronQ review (pith.science), appendix, Algorithm 2, steps 1-2:
 * H_d = H + damp_rel * mean(diag(H)) * I, then U_c upper triangular with
 * H_d^-1 = U_c^T U_c and a positive diagonal.  Computed as a reverse-order
 * Cholesky factorisation of H_d followed by a triangular inverse (fp32).
 *
 * H    : n x n fp32 symmetric (not modified).  U_c: n x n fp32 output
 *        (strictly lower part set to 0).  May not alias H.
 * info : optional device int32, KRONQ_ERR_NOT_PD if a pivot is <= 0 (U_c is
 *        then undefined).
 */
int kronq_cholesky_inv(const float* H, int64_t n, float damp_rel, float* U_c,
                       int32_t* info, void* ws, size_t ws_bytes, void* stream);

/*
 * Column-wise OBS quantization (GPTQ-style) of the rotated weights.
 *
 * KronQ summary (hyper.ai), "Method", Prop. 1: H_G cancels in the column
 * update, so each row is solved with H_X's factor alone.  KronQ review
 * (pith.science), appendix, Algorithm 2: blocks of B columns with an error
 * buffer E and lazy updates of the trailing columns.
 * Grid (asymmetric, b bits): lo = min(0, min w), hi = max(0, max w),
 * scale = (hi - lo)/(2^b - 1), zero = round(-lo/scale); per-channel from the
 * whole row before the loop, per group at the group's first column from the
 * error-updated weights.  q = clamp(round(w/scale) + zero, 0, 2^b - 1)
 * (round half to even, in fp32); e = (w - scale (q - zero)) / U_c[j,j];
 * W[:, k] -= e U_c[j, k] for k > j.
 *
 * W      : m x n fp32, the rotated weights; overwritten (scratch).
 * U_c    : n x n fp32 upper factor from kronq_cholesky_inv.
 * bits   : 2, 3, 4 or 8.  group: -1 (per-channel), 32, 64 or 128.  block: 128.
 * codes  : m x n uint8 output.   scales: m x G fp32, zeros: m x G uint8
 *          (G = 1 per-channel, n/group otherwise).
 * W_hat  : optional m x n fp32 output of the dequantized weights (NULL: skip).
 * n must be a multiple of 128.
 */
int kronq_quantize_layer(float* W, int64_t m, int64_t n, const float* U_c,
                         int bits, int group, int block,
                         uint8_t* codes, float* scales, uint8_t* zeros, float* W_hat,
                         int32_t* info, void* ws, size_t ws_bytes, void* stream);

/* Options of kronq_quantize_layer_opt (bit flags). */
enum kronq_quant_option {
  KRONQ_QUANT_CLIP = 1   /* --w_clip: clip-ratio search for every grid */
};

/*
 * kronq_quantize_layer with options.  options = 0 is kronq_quantize_layer.
 *
 * KRONQ_QUANT_CLIP: the README's --w_clip (KronQ README (GitHub),
 * "Reproduce from scratch"; the pages name the flag without defining it).
 * Reading taken: each grid (per row before the loop, or per group at its
 * first column) is the first of the shrunk ranges [p lo, p hi],
 * p = 1 - i/100 for i = 0 .. 79, with the least squared error
 * sum (w - w_hat)^2 over the row or group; the candidate grids and the
 * differences are fp32 operations, the squares are summed in fp64.
 * Other bits set: KRONQ_ERR_INVALID_ARG.  Everything else as
 * kronq_quantize_layer.
 */
int kronq_quantize_layer_opt(float* W, int64_t m, int64_t n, const float* U_c,
                             int bits, int group, int block, int options,
                             uint8_t* codes, float* scales, uint8_t* zeros, float* W_hat,
                             int32_t* info, void* ws, size_t ws_bytes, void* stream);

/*
 * The --act_order column order (KronQ README (GitHub), "Reproduce from
 * scratch"; undefined on the pages).  Reading taken: columns in descending
 * order of diag(H), equal values in increasing column order (NaN last).
 * perm[k] = the column quantized k-th.  To quantize in that order: permute
 * the columns of W and both sides of H_X with kronq_permute, factor the
 * permuted H_X with kronq_cholesky_inv, run the solver, and scatter the
 * codes (and W_hat) back with KRONQ_UNPERM_COLS; with groups, a group is g
 * consecutive columns of the permuted order (scales / zeros are indexed by
 * those groups).
 * H: n x n fp32 device (only the diagonal is read).  perm: n int32 device.
 */
int kronq_act_order(const float* H, int64_t n, int32_t* perm, void* stream);

/* kronq_permute modes. */
enum kronq_perm_mode {
  KRONQ_PERM_COLS = 0,    /* dst[r][k] = src[r][perm[k]]          */
  KRONQ_UNPERM_COLS = 1,  /* dst[r][perm[k]] = src[r][k]          */
  KRONQ_PERM_SYM = 2      /* dst[a][b] = src[perm[a]][perm[b]], m == n, fp32 */
};

/*
 * Column (or symmetric) permutation of an m x n row-major matrix of 1-byte
 * (codes) or 4-byte (fp32) elements; src and dst are distinct device
 * buffers.  perm: n int32 device, a permutation of 0 .. n-1; entries out of
 * range are skipped and reported as KRONQ_ERR_INVALID_ARG in the optional
 * device word info.  Not in the pages: the plumbing of --act_order.
 */
int kronq_permute(const void* src, void* dst, int64_t m, int64_t n, int elem_bytes,
                  const int32_t* perm, int mode, int32_t* info, void* stream);

/*
 * Deployment matvec of a quantized layer: y = W_hat x in the original space,
 * straight from the packed codes, with the BiIP transforms applied to the
 * vectors (KronQ README (GitHub): the fused dequant + BiIP matvec of the
 * deploy path, batch-1 decode).  With W' = U S_G W S_X V^T (KronQ summary
 * (hyper.ai), "Method", Eqs. 11-12):
 *     y = S_G^-1 U^T ( W_hat' ( V S_X^-1 x ) ),
 *     W_hat'[i][j] = scale[i][g(j)] (code[i][j] - zero[i][g(j)]).
 *
 * packed : m x (n bits/32) uint32 from kronq_pack, 16-byte aligned.
 * bits   : 2 or 4.  group: -1 (per-channel), 32, 64 or 128.
 * scales, zeros : m x G as written by kronq_quantize_layer (no act_order:
 *          the columns of the codes are in the transform's order).
 * S_X (n), S_G (m), sign_u (m), sign_v (n), mode : as used and written by
 *          kronq_biip_rotate (S_X, S_G 16-byte, the signs 4-byte aligned).
 * x      : batch x n fp32, y: batch x m fp32 (16-byte aligned); batch 1, 2,
 *          4 or 8.  n a multiple of 64, m of 16.
 * ws     : at least kronq_deploy_workspace_size(m, n, batch) bytes.
 */
size_t kronq_deploy_workspace_size(int64_t m, int64_t n, int64_t batch);
int kronq_deploy_matvec(const uint32_t* packed, int64_t m, int64_t n, int bits, int group,
                        const float* scales, const uint8_t* zeros,
                        const float* S_X, const float* S_G,
                        const int8_t* sign_u, const int8_t* sign_v, int mode,
                        const float* x, int64_t batch, float* y,
                        void* ws, size_t ws_bytes, void* stream);

/*
 * kronq_quantize_layer without a workspace: for callers that cannot allocate
 * device memory while they run (a host framework that owns the allocator,
 * memory planned once at start-up, or a loop where cudaMalloc/cudaFree would
 * synchronise the device).  The KronQ pages have no counterpart; this is a
 * deployment variant of the same solver.
 *
 * Same arguments and meaning as kronq_quantize_layer, minus (ws, ws_bytes).
 * The solver's scratch (its m x 128 error block and the current block's
 * n x 128 slab of U_c, both as bf16 hi / lo planes) lives in a static 64 MiB
 * device array inside the library (every GPU that loads the library holds it
 * until the process exits), so m and n may each be at most 32768
 * (KRONQ_ERR_UNSUPPORTED above that).  That array always holds the one-level
 * lazy update's scratch; when the two-level update's (1024-column
 * super-blocks, about 4 (m + n) KiB) does not also fit in it -- e.g.
 * m = n = 8192, or m = 16384 with n = 4096, or any n of 14592 or more --
 * the call runs the one-level update (K = 128 trailing updates after every
 * block).  The codes agree with
 * kronq_quantize_layer's up to floating-point summation order (the parity
 * bar, >= 99.9 % identical); the one-level update is slower on wide layers.  The library looks up the array's device
 * address once per device, during the first call made on that device; make
 * that first call before any stream capture.  All calls share the array:
 * calls whose work can overlap on the GPU (different streams without
 * ordering, several host threads) race on it and must be serialised by the
 * caller.  Nothing in it needs to start zeroed.  Allocates nothing.
 */
int kronq_quantize_layer_noalloc(float* W, int64_t m, int64_t n, const float* U_c,
                                 int bits, int group, int block,
                                 uint8_t* codes, float* scales, uint8_t* zeros, float* W_hat,
                                 int32_t* info, void* stream);

/*
 * GPTAQ asymmetric calibration (optional: the drift-corrected objective).
 *
 * KronQ summary (hyper.ai), "Method": building on GPTAQ, the objective is
 * corrected for input drift -- the quantized layer sees X~ (its input in
 * the partly quantized model) while its target is the full-precision W X.
 * KronQ review (pith.science), appendix, Algorithm 2, step 3:
 * P = alpha (Delta X X^T L) (.) M_U L^T, L <- InverseCholesky(H_X), M_U the
 * upper-triangular mask.  Readings: Delta X = X - X~; the solver's H_X is
 * the covariance of X~; L = U_c^T (H_d^-1 = L L^T); M_U keeps the diagonal;
 * after column p is quantized, each later column k receives
 * -delta_p U_c[p][k] + w_p P[p][k] with w_p the value the quantizer saw.
 * Sequence: kronq_drift_covariance -> kronq_biip_rotate (on W, H~, H_G) ->
 * kronq_biip_rotate_input (on Delta X X^T, with that call's S_X) ->
 * kronq_cholesky_inv (on H~') -> kronq_gptaq_correction ->
 * kronq_quantize_layer_gptaq.  Workspace: kronq_gptaq_workspace_size bytes
 * (it covers every call of the sequence).
 */
size_t kronq_gptaq_workspace_size(int64_t m, int64_t n);

/* H = X~^T X~ / N and A = (X - X~)^T X~ / N (both n x n fp32, full) from the
 * two calibration inputs side by side: XqX is N x 2n bf16 (row stride ld
 * >= 2n elements, 16-byte aligned rows), row t = [x~_t, x_t].  One
 * covariance of the 2n-wide rows (into the workspace), then the two blocks;
 * A is the difference of two fp32 sums, so its absolute error is that of H
 * (about 1e-5 of |H|).  Errors as kronq_covariance. */
int kronq_drift_covariance(const void* XqX, int64_t N, int64_t n, int64_t ld, float* H, float* A,
                           int32_t* info, void* ws, size_t ws_bytes, void* stream);

/* The input side of BiIP applied to A (n x n fp32, in place):
 * A <- V S_X^-1 A S_X^-1 V^T with the S_X a kronq_biip_rotate call returned
 * and its sign_v; mode as there (SU_ONLY leaves A unchanged, NO_RESCALE
 * only rotates, SV_ONLY and FULL rescale and rotate). */
int kronq_biip_rotate_input(float* A, int64_t n, const float* S_X, const int8_t* sign_v, int mode,
                            void* ws, size_t ws_bytes, void* stream);

/* P (n x n fp32 out, upper triangular) = alpha ((A U_c^T) (.) M_U) U_c, i.e.
 * alpha (Delta X X^T L) (.) M_U L^T with L = U_c^T; tensor-core products at
 * fp32 accuracy.  n a multiple of 4, at most 32768; pointers 16-byte
 * aligned; P must not alias A or U_c. */
int kronq_gptaq_correction(const float* A, const float* U_c, int64_t n, float alpha, float* P,
                           int32_t* info, void* ws, size_t ws_bytes, void* stream);

/* kronq_quantize_layer with the GPTAQ term P (n x n fp32, from
 * kronq_gptaq_correction): same arguments otherwise; group -1 or 128;
 * n <= 32768.  With P = 0 the codes are those of kronq_quantize_layer. */
int kronq_quantize_layer_gptaq(float* W, int64_t m, int64_t n, const float* U_c, const float* P,
                               int bits, int group, int block,
                               uint8_t* codes, float* scales, uint8_t* zeros, float* W_hat,
                               int32_t* info, void* ws, size_t ws_bytes, void* stream);

/*
 * Pack b-bit codes into 32-bit words (b = 2 or 4).
 *
 * KronQ README (GitHub), "Model zoo": W4 / W2 stored as packed int4 / int2;
 * 3-bit is not packable (KRONQ_ERR_UNSUPPORTED).  Code (i, j) goes to word
 * (i, floor(j b / 32)), bits [(j mod 32/b) b, +b).  Rows take
 * ceil(n b / 32) words; spare high bits are 0.  Codes must be < 2^b.
 * codes: m x n uint8.  packed: m x ceil(n b/32) uint32, 4-byte aligned.
 */
int kronq_pack(const uint8_t* codes, int64_t m, int64_t n, int bits,
               uint32_t* packed, void* stream);

/* Exact inverse of kronq_pack. */
int kronq_unpack(const uint32_t* packed, int64_t m, int64_t n, int bits,
                 uint8_t* codes, void* stream);

/*
 * Layer loss tr(H_G dW H_X dW^T), dW = W_ref - W_hat (a measurement helper,
 * not on the quantization path).  KronQ summary (hyper.ai), "Method": the
 * Kronecker-factored objective.  All inputs fp32 device; loss_out: DEVICE
 * double.  Workspace: kronq_workspace_size(m, n, ...) bytes.
 */
int kronq_layer_loss(const float* W_ref, const float* W_hat, int64_t m, int64_t n,
                     const float* H_X, const float* H_G, double* loss_out,
                     void* ws, size_t ws_bytes, void* stream);

/*
 * Failure-detection self test: one CTA waits on an mbarrier that nothing
 * arrives on, through the same bounded wait the pipelined kernels use, with
 * a limit of limit_ns (1 .. 2e9).  Expected outcome: *info (device int32,
 * caller-zeroed) becomes KRONQ_ERR_TIMEOUT and the kernel returns; the
 * context stays usable.  Not part of the quantization path.
 */
int kronq_selftest_wait(int32_t* info, int64_t limit_ns, void* stream);

/*
 * Waits for the work queued on `stream` and reports how it ended (a host
 * convenience; the pages have no counterpart).  Returns KRONQ_ERR_CUDA when
 * the stream's work raised a CUDA error; otherwise, when `info` is given
 * (the device word passed to the earlier calls), its value: 0 (KRONQ_OK) or
 * the first numerical failure those calls recorded (KRONQ_ERR_NOT_PD,
 * KRONQ_ERR_TIMEOUT).  `info` is only read.  Blocks the calling thread.
 */
int kronq_sync_status(void* stream, const int32_t* info);

#ifdef __cplusplus
}
#endif

#endif /* KRONQ_H */
