/*
 * signmuon.h -- C ABI of libsignmuon.so, the B200 (sm_100a) Sign-Muon step.
 *
 * The method is the one described in the technical summary of "SignMuon:
 * Communication-Efficient Distributed Muon Optimization" (arXiv 2605.16311),
 * section 2, "Algorithmic flow (distributed)", steps 1-5:
 *   1. every worker m updates its momentum M^(m) from its gradient G^(m) and
 *      computes the polar factor U^(m) with Newton-Schulz iterations;
 *   2. it takes the entrywise sign S^(m) = sign(U^(m));
 *   3. the signs are exchanged as an integer sum (int8) or as 1-bit packed
 *      buffers;
 *   4. the majority vote sign(sum_m S^(m)) updates W <- W - eta * vote;
 *   5. optionally, a local polar step on the voted matrix.
 * Here the M workers are M buffers on one GPU, so step 3's collective is the
 * local M-way reduction inside signmuon_vote_update.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All pointers named "device" point to device memory of the current CUDA
 *   device; arrays of pointers (type `const void* const*` etc.) are HOST
 *   arrays whose elements are device pointers.  The library copies what it
 *   needs into the caller's device workspace.
 * - Ownership: the caller owns every buffer, including the workspace.  The
 *   library allocates no memory and keeps no state between calls (the one
 *   exception is the fixed scratch array of signmuon_momentum_norm_noalloc,
 *   described at its declaration).
 * - Units: a "unit" is one (matrix i, worker m) pair; per-unit arrays have
 *   n_mats * n_workers entries, indexed i * n_workers + m.
 * - Matrices are row-major.  Dense fp32/bf16/int8 buffers have row stride
 *   `cols`.  bf16 Newton-Schulz buffers (the "X" buffers and the vote matrix)
 *   have row stride signmuon_x_ld(cols) elements (cols rounded up to 8).
 * - Packed sign buffers: row-major uint32 words, ceil(cols/32) words per row;
 *   bit j of word w in row r is entry (r, 32w + j); a set bit is +1; bits
 *   past the last column are 0.  A buffer holds signmuon_packed_words(shape)
 *   words (the row-major words, rounded up to a multiple of 4).
 * - int8 sign buffers: row-major int8 in {-1, +1}, row stride cols.
 * - sign(0) = sign(-0) = +1 and a NaN maps to +1 (the test is "u < 0").
 * - Every buffer pointer must be 16-byte aligned (SIGNMUON_ERR_ALIGNMENT),
 *   except the inv_norm input of the Newton-Schulz calls (one float per
 *   unit, 4-byte aligned: it may point into a larger per-unit array).
 * - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *   enqueued asynchronously; no entry point synchronises the host except
 *   signmuon_device_error.
 * - Errors: arguments are validated before anything is enqueued and a
 *   status is returned; nothing is launched when validation fails.  Launch
 *   failures return SIGNMUON_ERR_CUDA.  Kernels never trap: a kernel that
 *   gives up waiting (a bounded wait ran out) records a nonzero code in the
 *   first word of the workspace it was given, readable with
 *   signmuon_device_error.
 */
#ifndef SIGNMUON_H_
#define SIGNMUON_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum signmuon_status {
  SIGNMUON_OK = 0,
  SIGNMUON_ERR_INVALID_ARG = 1,  /* null pointer, size <= 0, count out of range */
  SIGNMUON_ERR_ALIGNMENT = 2,    /* a buffer is not 16-byte aligned             */
  SIGNMUON_ERR_UNSUPPORTED = 3,  /* valid request this library cannot run      */
  SIGNMUON_ERR_WORKSPACE = 4,    /* workspace null or smaller than required     */
  SIGNMUON_ERR_CUDA = 5          /* a CUDA call or kernel launch failed        */
} signmuon_status;

typedef enum signmuon_dtype { SIGNMUON_F32 = 0, SIGNMUON_BF16 = 1 } signmuon_dtype;

/* What the last Newton-Schulz iteration writes. */
typedef enum signmuon_ns_out {
  SIGNMUON_OUT_PACK1 = 0,     /* 1-bit packed signs, one buffer per unit        */
  SIGNMUON_OUT_INT8 = 1,      /* int8 +-1 signs, one buffer per unit             */
  SIGNMUON_OUT_UPDATE_W = 2,  /* W <- W - eta * U in place (n_workers must be 1) */
  SIGNMUON_OUT_U_F32 = 3      /* the polar estimate U itself, fp32 [rows, cols]  */
} signmuon_ns_out;

typedef struct signmuon_shape {
  int32_t rows;
  int32_t cols;
} signmuon_shape;

#define SIGNMUON_MAX_WORKERS 127

/* Human-readable name of a status code (static storage). */
const char* signmuon_status_string(int status);

/* Library ABI version (incremented on any signature change). */
int signmuon_abi_version(void);

/* Text of the CUDA error behind the most recent SIGNMUON_ERR_CUDA returned to
 * the calling thread ("no error" if none); static storage. */
const char* signmuon_last_error_string(void);

/* Row stride, in elements, of a bf16 Newton-Schulz buffer with `cols` columns:
 * cols rounded up to a multiple of 8 (16 bytes, the TMA stride granule). */
int32_t signmuon_x_ld(int32_t cols);

/* Words (uint32) of one packed sign buffer of this shape: rows*ceil(cols/32)
 * rounded up to a multiple of 4.  Returns -1 for an invalid shape. */
int64_t signmuon_packed_words(signmuon_shape shape);

/* Reads (synchronously: waits for the device) the error word a kernel left
 * in `workspace` (device pointer given to an earlier call) and clears it.
 * *code = 0 means no kernel gave up.  Returns SIGNMUON_ERR_CUDA if the copy
 * fails. */
signmuon_status signmuon_device_error(void* workspace, uint32_t* code, void* stream);

/* ------------------------------------------------------------------------
 * Step 1a: momentum and Frobenius normalisation.
 * Source: SignMuon summary, section 2 "Algorithmic flow", step 1 (each
 * worker updates its local momentum) and section 4 "nanoGPT" (Frobenius
 * scaling of the Newton-Schulz input).
 *
 * For every unit u = i*n_workers + m (matrix i has shapes[i]):
 *   mom[u]    <- beta * mom[u] + (1 - beta) * grad[u]          (fp32, in place)
 *   x_bf16[u] <- bf16(mom[u])  (row stride signmuon_x_ld(cols); pad columns
 *                               are not written)
 *   inv_norm[u] <- 1 / (||mom[u]||_F + 1e-7)                   (fp32)
 * so that the Newton-Schulz input is X0 = inv_norm[u] * x_bf16[u].
 * The norm is reduced in a fixed order (bit-reproducible run to run).
 *
 * grad: per-unit device pointers, dtype grad_dtype, [rows, cols].
 * mom: per-unit device fp32 [rows, cols], updated in place.
 * x_bf16: per-unit device bf16 [rows, x_ld].
 * inv_norm: device fp32 [n_mats * n_workers].
 * workspace: device, >= signmuon_momentum_workspace_bytes(...) bytes.
 * ---------------------------------------------------------------------- */
size_t signmuon_momentum_workspace_bytes(const signmuon_shape* shapes, int n_mats,
                                         int n_workers);
signmuon_status signmuon_momentum_norm(const signmuon_shape* shapes, int n_mats, int n_workers,
                                       signmuon_dtype grad_dtype, const void* const* grad,
                                       float* const* mom, float beta, void* const* x_bf16,
                                       float* inv_norm, void* workspace, size_t ws_bytes,
                                       void* stream);

/* ------------------------------------------------------------------------
 * Steps 1a-2 for k = 0 (the majority-vote Signum / SignSGD baseline),
 * fused: the momentum update and the signs of X0 = M / (||M||_F + 1e-7)
 * in one pass, without the bf16 copy of M.
 * Source: SignMuon summary, section 4 (the Signum / SignSGD baselines the
 * summary compares against) and section 2 "Algorithmic flow" steps 1-3.
 *
 * mom[u] and inv_norm[u] are updated exactly as by signmuon_momentum_norm.
 * signs[u] receives sign(X0) (+1 for 0, -0 and NaN), which is sign(mom[u])
 * when the norm is finite and +1 everywhere when it is not (X0 is then NaN
 * or zero in every entry):
 *   int8_out == 0: packed words (signmuon_packed_words words per unit, bit
 *                  j of word w in row r = entry (r, 32w + j), 1 = +1); every
 *                  cols must be a multiple of 32 (else SIGNMUON_ERR_UNSUPPORTED,
 *                  and signmuon_momentum_norm + signmuon_newton_schulz_batched
 *                  with k = 0 serve); trailing pad words are not written.
 *   int8_out != 0: int8 [rows, cols], any shape.
 * The signs equal those of signmuon_newton_schulz_batched with k = 0 except
 * for |M| below about 5e-41, where that path's bf16 copy of M (or its
 * product with inv_norm) underflows to -0; this call reads the fp32 momentum
 * itself and keeps those signs, as the fp64 definition does.
 * Arguments, alignment and workspace as for signmuon_momentum_norm.
 * ---------------------------------------------------------------------- */
signmuon_status signmuon_momentum_sign(const signmuon_shape* shapes, int n_mats, int n_workers,
                                       signmuon_dtype grad_dtype, const void* const* grad,
                                       float* const* mom, float beta, int int8_out,
                                       void* const* signs, float* inv_norm, void* workspace,
                                       size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Step 1a, spectral variant: spectral scaling of the Newton-Schulz input.
 * Source: SignMuon summary, section 4 "nanoGPT" (the method is robust to
 * Frobenius vs spectral scaling of the normalisation).
 *
 * For every unit, sigma_est is estimated by `iters` power iterations on
 * X^T X, X = x_bf16[u] ([rows, signmuon_x_ld(cols)] bf16, as written by
 * signmuon_momentum_norm), from the start vector v0 = 1/sqrt(cols):
 *   z = X^T X v,  v <- z / ||z||,  sigma_est = sqrt(||z||) of the last step;
 * then inv_norm[u] <- 1 / (sigma_est + 1e-7), replacing the Frobenius value
 * so that signmuon_newton_schulz_batched starts from X0 = X / sigma_est.
 * sigma_est never exceeds the largest singular value of X.  A zero matrix
 * gives inv_norm = 1e7 (X0 = 0).  1 <= iters <= 1000.  Sums are taken in a
 * fixed order (bit-reproducible run to run).
 * workspace: device, >= signmuon_spectral_workspace_bytes(...) bytes.
 * ---------------------------------------------------------------------- */
size_t signmuon_spectral_workspace_bytes(const signmuon_shape* shapes, int n_mats, int n_workers);
signmuon_status signmuon_spectral_norm(const signmuon_shape* shapes, int n_mats, int n_workers,
                                       const void* const* x_bf16, int iters, float* inv_norm,
                                       void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Step 1b-2: k Newton-Schulz iterations, then the entrywise sign.
 * Source: SignMuon summary, section 2 "Core mechanism" item 1 and
 * "Algorithmic flow" steps 1-2 (and step 5 for SIGNMUON_OUT_UPDATE_W).
 *
 * For every unit, starting from X = inv_norm[u] * x_bf16[u], k times:
 *   rows <= cols:  A = X X^T,  B = b A + c A^2,  X <- a X + B X
 *   rows >  cols:  A = X^T X,  B = b A + c A^2,  X <- a X + X B
 * on the tensor cores (bf16 operands, fp32 accumulation, bf16 between
 * iterations).  The kernels store Q = A + b/(2c) I in fp16 and form
 * B' = c Q Q + (a - b^2/(4c)) I = a I + b A + c A^2 (bf16) when c != 0 and
 * |b/(2c)| <= 4 (otherwise they store A and form a I + b A + c A A), and
 * compute X <- B' X (X B'): the same map with the a X term folded into the
 * product.  Of the symmetric Q and B' only the
 * 256x256 blocks on and above the diagonal are computed and stored in the
 * workspace.
 * The last iteration's epilogue writes, per out_mode:
 *   PACK1:    out[u] = packed sign(U)   (uint32, signmuon_packed_words words)
 *   INT8:     out[u] = int8 sign(U)     ([rows, cols])
 *   U_F32:    out[u] = U                (fp32 [rows, cols])
 *   UPDATE_W: w[i] <- w[i] - eta * U    (w_dtype [rows, cols], in place;
 *             requires n_workers == 1; `out` is ignored and may be NULL)
 * k = 0 writes the same outputs from U = X0.
 *
 * x_bf16 buffers are CLOBBERED (used as one of the two iterate buffers).
 * Coefficients a, b, c are the caller's (the Python step class passes
 * 3.4445, -4.7750, 2.0315).  k must be in [0, 64].
 * workspace: device; signmuon_newton_schulz_workspace_bytes(..., 0) bytes
 * run all units at once, any size >= the value for minimal=1 runs them in
 * successive waves.
 * ---------------------------------------------------------------------- */
size_t signmuon_newton_schulz_workspace_bytes(const signmuon_shape* shapes, int n_mats,
                                              int n_workers, int minimal);
signmuon_status signmuon_newton_schulz_batched(
    const signmuon_shape* shapes, int n_mats, int n_workers, void* const* x_bf16,
    const float* inv_norm, int k, float a, float b, float c, signmuon_ns_out out_mode,
    void* const* out, signmuon_dtype w_dtype, void* const* w, float eta, void* workspace,
    size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Step 1b-2 split in two: plan once, run every step.
 * Same computation as signmuon_newton_schulz_batched (which is exactly
 * plan followed by run); the split only moves per-call host work off the
 * step: encoding eight TMA tensor maps per unit and uploading the unit table
 * (1152 bytes per unit) happen once, in plan, instead of on every call.
 * An optimizer whose buffers persist from step to step plans once and then
 * calls run each step.
 *
 * plan: caller-owned HOST memory of signmuon_newton_schulz_plan_bytes(...)
 *   bytes, 8-byte aligned; plan() fills it, run() only reads it.  The plan
 *   records the device addresses of x_bf16, inv_norm, out (or w) and the
 *   workspace: all of them must stay allocated, and hold the same shapes,
 *   for as long as the plan is run.  After any of them moves, plan again.
 * plan() validates and documents its arguments as signmuon_newton_schulz_
 *   batched does, then writes the unit table into `workspace` with work
 *   enqueued on `stream`; run() enqueues the k iterations on `stream`, which
 *   must be ordered after that upload (the same stream, or synchronised).
 * run() reads inv_norm and x_bf16 at the time it executes (stream order),
 *   so each step's momentum kernel may refill them in place.
 * Two runs of plans that share a workspace must not overlap in time (they
 *   share the A / B' / P buffers); a later plan() on the same workspace
 *   overwrites the unit table of an earlier one, invalidating it.
 * Errors: SIGNMUON_ERR_INVALID_ARG for a NULL plan, a plan buffer smaller
 *   than plan_bytes, a plan not filled by a successful plan(), or k outside
 *   [0, 64]; the other codes as for signmuon_newton_schulz_batched.  A failed
 *   plan() leaves the plan unusable (run() rejects it).
 * ---------------------------------------------------------------------- */
size_t signmuon_newton_schulz_plan_bytes(int n_mats, int n_workers);
signmuon_status signmuon_newton_schulz_plan(
    const signmuon_shape* shapes, int n_mats, int n_workers, void* const* x_bf16,
    const float* inv_norm, signmuon_ns_out out_mode, void* const* out, signmuon_dtype w_dtype,
    void* const* w, void* workspace, size_t ws_bytes, void* plan, size_t plan_bytes,
    void* stream);
signmuon_status signmuon_newton_schulz_run(const void* plan, int k, float a, float b, float c,
                                           float eta, void* stream);

/* ------------------------------------------------------------------------
 * Step 2-3 standalone: entrywise sign of a matrix, packed or int8.
 * Source: SignMuon summary, section 2 "Algorithmic flow", steps 2-3 and
 * "Communication efficiency" (1 bit per entry, or 8 bits with int8).
 *
 * u: device [rows, ld_u] of u_dtype (ld_u >= cols, in elements).
 * out: device; packed (signmuon_packed_words words, pad bits 0 and trailing
 * pad words 0) when int8_out == 0, else int8 [rows, cols].
 * ---------------------------------------------------------------------- */
signmuon_status signmuon_sign_pack(signmuon_shape shape, signmuon_dtype u_dtype, const void* u,
                                   int64_t ld_u, int int8_out, void* out, void* stream);

/* ------------------------------------------------------------------------
 * Steps 3-4: majority vote over the M workers' signs and the update.
 * Source: SignMuon summary, section 2 "Core mechanism" item 3 (integer sum
 * then sign) and "Algorithmic flow" step 4 (W <- W - eta * vote).
 *
 * For every matrix i, with c = number of workers whose sign is +1:
 *   vote = +1 if 2c > M, -1 if 2c < M, 0 on a tie (even M).
 * signs: per-unit device buffers, packed (int8_in == 0) or int8.
 * Update mode (vote_bf16 == NULL):  w[i] <- w[i] - eta * vote, computed
 *   exactly and rounded once to w_dtype (round to nearest even).
 * Vote-out mode (vote_bf16 != NULL): w is not touched; writes the vote as
 *   bf16 {-1, 0, +1} to vote_bf16[i] ([rows, signmuon_x_ld(cols)]), its
 *   number of non-zeros to nnz[i] (device int64) and 1/sqrt(nnz) (0 when
 *   nnz = 0) to vote_inv_norm[i] (device fp32): the input of the optional
 *   local polar step (signmuon_newton_schulz_batched with n_workers = 1,
 *   k = 1, out_mode = SIGNMUON_OUT_UPDATE_W).
 * 1 <= n_workers <= SIGNMUON_MAX_WORKERS.
 * workspace: device, >= signmuon_vote_workspace_bytes(...) bytes.
 * ---------------------------------------------------------------------- */
size_t signmuon_vote_workspace_bytes(const signmuon_shape* shapes, int n_mats, int n_workers);
signmuon_status signmuon_vote_update(const signmuon_shape* shapes, int n_mats, int n_workers,
                                     int int8_in, const void* const* signs,
                                     signmuon_dtype w_dtype, void* const* w, float eta,
                                     void* const* vote_bf16, int64_t* nnz, float* vote_inv_norm,
                                     void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Allocation-free variant of signmuon_momentum_norm.
 * The paper has no counterpart: this is a deployment convenience.
 *
 * Same inputs, outputs and results as signmuon_momentum_norm, but the
 * scratch it needs (unit table and per-block partial sums) lives in a 1 MiB
 * device array inside the library rather than in a caller workspace.  It is
 * meant for callers that cannot allocate device memory around the step, e.g.
 * an optimizer embedded in a runtime whose allocator already owns the whole
 * device, or a loop that must avoid cudaMalloc/cudaFree because they
 * synchronise the device.  The call itself allocates nothing.
 *
 * Limits: n_mats * n_workers <= 1170 units, and at most 245760 blocks of
 * 4096 elements in total (sum over units of ceil(rows*cols/4096)), i.e.
 * about 1.0e9 momentum elements; larger requests return
 * SIGNMUON_ERR_WORKSPACE without enqueuing anything.
 * The array (1 MiB) is held on every GPU that loads the library until the
 * process exits.  The first call on each device looks up the array's device
 * address (once per device, with that device current); make that first call
 * before any stream capture.  The address is cached for the life of the
 * process and belongs to the device's primary context: after
 * cudaDeviceReset it is stale, so do not call this entry point again in
 * that process.  All calls share the array and each call
 * rewrites what it reads, so nothing needs clearing, but calls whose kernels
 * can overlap on the GPU (different streams with no ordering) race on it.
 * ---------------------------------------------------------------------- */
signmuon_status signmuon_momentum_norm_noalloc(const signmuon_shape* shapes, int n_mats, int n_workers,
                                               signmuon_dtype grad_dtype, const void* const* grad,
                                               float* const* mom, float beta, void* const* x_bf16,
                                               float* inv_norm, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SIGNMUON_H_ */
