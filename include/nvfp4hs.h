/*
 * nvfp4hs.h -- C ABI of the B200 (sm_100a) library for Hessian-weighted NVFP4
 * block-scale selection.
 *
 * The method (H-Scale summary, sec. 3 "Method" and sec. B "Implementation
 * Pseudocode"; ScaleSweep summary, sec. 2 "Theoretical Bounds" and sec. 3
 * "Implementation"): for a weight matrix W[out, in] quantized to NVFP4 (16
 * E2M1 values share one E4M3 scale, one FP32 scale per tensor),
 *   1. h_j = sum_t x_tj^2 over calibration activations X[tokens, in]
 *      (the diagonal of X^T X, the per-channel second-order proxy);
 *   2. S = amax(|W|) / (Q * 6), Q = 448 (standard) or 256 (ScaleSweep);
 *   3. per 16-element group along `in`: base code b = E4M3(absmax / 6 / S);
 *      candidate codes b+lo .. b+hi (clamped to the 126 positive finite E4M3
 *      codes), each scored by sum_j h_j (w_j - q_j)^2 with q the E2M1
 *      round-to-nearest-even reconstruction at that scale; the smallest score
 *      wins, ties to the lowest offset;
 *   4. the group is quantized once with the winner and packed.
 *
 * Conventions shared by every call
 *   - All array pointers are DEVICE pointers owned by the caller, except where
 *     a parameter says "host".  The library allocates nothing.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call only enqueues work and returns; results are valid
 *     once the stream has reached that point.
 *   - bf16 inputs are raw bfloat16 bit patterns (uint16), row-major with a
 *     leading dimension in ELEMENTS.
 *   - Arguments are checked on the host before anything is enqueued; a failed
 *     check enqueues nothing and returns a negative nvfp4_status.  A CUDA
 *     launch error returns NVFP4_ERR_CUDA.  No C++ exception crosses the ABI.
 *   - Calls are re-entrant: concurrent calls on different streams are safe as
 *     long as they do not share output or workspace buffers.
 *   - Packed layout: codes[r, j/2] holds element j of row r in its low nibble
 *     when j is even and in its high nibble when j is odd; a nibble is
 *     (sign << 3) | k with k the E2M1 magnitude index (0,0.5,1,1.5,2,3,4,6) and
 *     the sign bit set only for a negative nonzero value.  scales[r, j/16] is
 *     the E4M3 bit pattern of group j/16 (0 for an all-zero group).  This is
 *     4.5 bits per weight (Replay-the-Curvature summary, sec. 1).
 */
#ifndef NVFP4HS_H
#define NVFP4HS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum nvfp4_status {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = -1,  /* NULL where not allowed, negative size, bad q_max/flag */
    NVFP4_ERR_SHAPE = -2,        /* in % 16 != 0, leading dimension < in, too large     */
    NVFP4_ERR_ALIGN = -3,        /* a pointer or leading dimension breaks the alignment */
    NVFP4_ERR_WINDOW = -4,       /* lo/hi outside the supported sweep window            */
    NVFP4_ERR_NONFINITE = -5,    /* written to a device status word: Inf/NaN in W       */
    NVFP4_ERR_CUDA = -6,         /* a CUDA runtime call or kernel launch failed         */
    NVFP4_ERR_WORKSPACE = -7,    /* workspace NULL or smaller than the queried size     */
    NVFP4_ERR_CAPTURE = -8,      /* a call that stages host tables, on a capturing stream */
    NVFP4_ERR_NUMERIC = -9       /* written to a device status word: a Cholesky failed  */
} nvfp4_status;

/* Library version (major*10000 + minor*100 + patch). */
int nvfp4_version(void);

/* Bounds checks (debugging aid; no counterpart on the pages).  A library built
 * with -DNVFP4HS_CHECKS checks every global-memory address of the per-step
 * kernels (diagonal Hessian, global scale, sweep, dequantize) against the
 * extent of its buffer that the call's size arguments imply; an address
 * outside is counted, the first is recorded, and the access goes to a dummy
 * buffer instead (no fault, no write to memory the call does not own).
 * nvfp4_debug_checks_compiled() is 1 in such a build, 0 otherwise.
 * nvfp4_debug_checks() synchronises with the device, writes the number of
 * failed checks and the first one ((site << 48) | (byte offset + 1); 0 when
 * none), and clears them if reset is 1; in a build without checks it writes
 * zeros. */
int nvfp4_debug_checks_compiled(void);
int nvfp4_debug_checks(unsigned long long* first, unsigned int* count, int reset);

/* The cudaError_t behind the calling thread's most recent NVFP4_ERR_CUDA. */
int nvfp4_last_cuda_error(void);

/* ------------------------------------------------------------------------
 * Step 1: diagonal Hessian proxy (H-Scale summary, sec. B: h = diag(X^T X);
 * sec. 3 "Hessian-guided objective").
 *
 * h[j] = (accumulate ? h[j] : 0) + sum_{t < tokens} X[t * ldx + j]^2.
 *   X          bf16 [tokens, ldx], 16-byte aligned; ldx % 8 == 0; ldx >= in.
 *   tokens     >= 0 (0 leaves h unchanged with accumulate, else zeroes it).
 *   in         > 0, in % 8 == 0.
 *   h          float [in], 4-byte aligned.  Products are exact in FP32; sums are
 *              FP32 in short runs, FP32 per thread, FP64 across threads, so the
 *              result is within ~1e-6 relative of the exact sum for any input.
 *   workspace  device scratch of at least nvfp4_diag_hessian_workspace_size()
 *              bytes, 256-byte aligned; holds per-thread partial sums.  Its
 *              contents need not be initialised and are garbage afterwards.
 * Deterministic: the summation order depends only on (tokens, in) and the
 * number of SMs of the current device.
 * ------------------------------------------------------------------------ */
size_t nvfp4_diag_hessian_workspace_size(int64_t tokens, int64_t in);
int nvfp4_diag_hessian(const void* X, int64_t tokens, int64_t in, int64_t ldx, float* h,
                       int accumulate, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Step 2: FP32 global scale (ScaleSweep summary, sec. 2: S = max|x| / (Q*6)).
 *
 * amax = max |W|; S = fl32(amax / fl32(q_max * 6)), S = 0 when amax = 0.
 *   W          bf16 [out, ldw], 16-byte aligned; ldw % 8 == 0; in % 8 == 0.
 *   q_max      > 0 and finite (448: E4M3 max; 256: ScaleSweep's choice).
 *   S          float, device scalar (written).
 *   amax       float, device scalar, may be NULL.
 *   status     int, device scalar, may be NULL: NVFP4_OK, or NVFP4_ERR_NONFINITE
 *              when W holds an Inf or NaN (S and amax are then NaN).
 *   workspace  at least nvfp4_global_scale_workspace_size() bytes, 256-byte
 *              aligned; no initialisation needed.
 * ------------------------------------------------------------------------ */
size_t nvfp4_global_scale_workspace_size(int64_t out, int64_t in);
int nvfp4_global_scale(const void* W, int64_t out, int64_t in, int64_t ldw, float q_max,
                       float* S, float* amax, int* status, void* workspace,
                       size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Step 2 without caller-provided scratch.  (The method's pages have no
 * counterpart: this is a deployment convenience.)
 *
 * Same arguments, result and status word as nvfp4_global_scale, minus the
 * workspace.  For callers that cannot allocate device memory -- plugin hooks
 * handed tensors but no allocator, or code under a hard memory cap or inside
 * a pre-planned memory pool -- the per-CTA partial maxima go to a 64 KiB
 * array compiled into the library, which every GPU that loads the library
 * holds until the process exits.  Nothing is allocated.
 *   - Every call looks up the array's device address in the current context
 *     (cudaGetSymbolAddress), so a cudaDeviceReset or another context on the
 *     same device never leaves it a stale address.  The first call on a device
 *     also makes the runtime load the library's device code there: make that
 *     first call before any stream capture.
 *   - CUDA failures (device query, address lookup, launch) return
 *     NVFP4_ERR_CUDA with the code kept for nvfp4_last_cuda_error().
 *   - All calls share the array: calls that overlap on the GPU (different
 *     streams without ordering between them) race and must not be issued.
 *   - The array needs no initialisation; it is not cleared.
 *   - A problem whose partials would not fit the array returns
 *     NVFP4_ERR_WORKSPACE (never on current GPUs: one 4-byte partial per CTA).
 * ------------------------------------------------------------------------ */
int nvfp4_global_scale_noalloc(const void* W, int64_t out, int64_t in, int64_t ldw, float q_max,
                               float* S, float* amax, int* status, void* stream);

/* ------------------------------------------------------------------------
 * Steps 3-4: windowed scale sweep + quantize + pack (H-Scale summary, sec. 3
 * "Group-wise scale selection", "Efficient scale search"; sec. B
 * "HScaleGroupQuantize"; ScaleSweep summary, sec. 3).
 *
 *   W          bf16 [out, ldw], 16-byte aligned; ldw % 8 == 0; in % 16 == 0.
 *   h          float [in], 16-byte aligned, non-negative; NULL = plain MSE
 *              (h == 1).
 *   S          float device scalar from nvfp4_global_scale (or the caller's).
 *   lo, hi     offset window, -16 <= lo <= 0 <= hi <= 15, hi - lo <= 15.
 *              H-Scale default [-9,+6]; ScaleSweep MSE [-3,+7], WMSE [-8,+7].
 *   codes      uint8 [out, in/2], 8-byte aligned (written).
 *   scales     uint8 [out, in/16] (written).
 *   chosen_offset  int8 [out, in/16] or NULL: winning offset k (the lowest k
 *              reaching the winning code; 0 for an all-zero group).
 * The loss is evaluated in FP32; the decision of every element's E2M1 code and
 * of the base code follows IEEE round-to-nearest-even as the definition does,
 * so results agree with an exact evaluation except where two candidates' losses
 * are within ~1e-7 relative of each other.
 * Scheduling: where in/16 is a multiple of 32 and every row lane of the grid
 * would take four rows or more, rows are handed out at run time from counters
 * the library keeps in device memory (one per 32-group column strip).  The
 * counters form 64 slots that launches take in turn; before a launch, its
 * stream waits for an event the library recorded after the slot's previous
 * launch (free on the same stream), so launches sharing a slot never
 * overlap, and each launch zeroes its slot before it ends.  A launch being
 * captured into a CUDA graph uses a fixed row stride.  The bytes written do
 * not depend on the order rows are taken in.  The library serialises its own
 * slot bookkeeping (a mutex per device).
 * ------------------------------------------------------------------------ */
int nvfp4_scale_sweep_quantize(const void* W, int64_t out, int64_t in, int64_t ldw,
                               const float* h, const float* S, int lo, int hi,
                               uint8_t* codes, uint8_t* scales, int8_t* chosen_offset,
                               void* stream);

/* Test support: device address and size in bytes of the run-time row
 * counters of nvfp4_scale_sweep_quantize on the current device, read-only for
 * the caller: 64 slots of 258 uint32 words (256 strip counters, a count of
 * finished CTAs, a count of launches the slot has served).  Returns NVFP4_OK,
 * NVFP4_ERR_INVALID_ARG for NULL outputs, NVFP4_ERR_CUDA without a device. */
int nvfp4_debug_row_counters(void** ptr, size_t* bytes);

/* ------------------------------------------------------------------------
 * Full sweep: every one of the 126 positive E4M3 codes is a candidate --
 * the exhaustive search that ScaleSweep summary sec. 2 calls too costly for
 * routine use, here as the reference for window-recovery statistics (how much
 * of the full search's gain a window keeps).  Arguments as
 * nvfp4_scale_sweep_quantize without the window; ties go to the lowest code;
 * chosen_offset (if not NULL) receives code - base code.
 * ------------------------------------------------------------------------ */
int nvfp4_scale_sweep_quantize_full(const void* W, int64_t out, int64_t in, int64_t ldw,
                                    const float* h, const float* S, uint8_t* codes,
                                    uint8_t* scales, int8_t* chosen_offset, void* stream);

/* ------------------------------------------------------------------------
 * Grouped and batched forms: one launch for many matrices, as in a
 * mixture-of-experts layer whose experts each see their own slice of the
 * calibration tokens and get their own h and S.  Each computes exactly what
 * the single-matrix call computes for every member (bit-identical outputs for
 * the global scale and the sweep; h to the same tolerance, summed in a
 * different fixed order).
 * ------------------------------------------------------------------------ */

/* Diagonal Hessian per expert (H-Scale summary, sec. B; one statistic per
 * expert).  The rows are cut into about one wave of equal slices that never
 * straddle two experts; each slice's sums land in the workspace and are added
 * per expert in a fixed order.  X holds the experts' calibration rows back to
 * back:
 *   expert e owns rows row_offsets[e] .. row_offsets[e+1]-1 of X[total_tokens, ldx].
 *   row_offsets  DEVICE int64 [experts+1], non-decreasing, within [0, total_tokens]
 *                (offsets outside that are clamped; a decreasing table gives
 *                undefined h but never an out-of-bounds access), 8-byte aligned.
 *   experts      1 .. 65535.
 *   h            float [experts, in] (row e = expert e), accumulate as above.
 *   workspace    at least nvfp4_diag_hessian_grouped_workspace_size() bytes,
 *                256-byte aligned; contents need no initialisation.  The size
 *                depends on the current device's SM count (0 without a device).
 * Other arguments as nvfp4_diag_hessian. */
size_t nvfp4_diag_hessian_grouped_workspace_size(int64_t total_tokens, int64_t experts, int64_t in);
int nvfp4_diag_hessian_grouped(const void* X, const int64_t* row_offsets, int64_t experts,
                               int64_t total_tokens, int64_t in, int64_t ldx, float* h,
                               int accumulate, void* workspace, size_t workspace_bytes,
                               void* stream);

/* One weight matrix of a batch: device pointer, shape, leading dimension. */
typedef struct nvfp4_matrix_desc {
    const void* W;
    int64_t out, in, ldw;
} nvfp4_matrix_desc;

/* Global scale of n matrices (ScaleSweep summary, sec. 2), one per matrix.
 *   descs        HOST array of n descriptors (read before the call returns).
 *   S            DEVICE float [n]; amax, status: DEVICE [n] or NULL.
 *   workspace    at least nvfp4_global_scale_batched_workspace_size(descs, n)
 *                bytes, 256-byte aligned: a device copy of the table plus one
 *                partial maximum per CTA.
 * Each descriptor is checked as nvfp4_global_scale checks its arguments.
 * The table is staged from host memory, so the call cannot be captured into
 * a CUDA graph: on a capturing stream it returns NVFP4_ERR_CAPTURE and
 * enqueues nothing. */
size_t nvfp4_global_scale_batched_workspace_size(const nvfp4_matrix_desc* descs, int64_t n);
int nvfp4_global_scale_batched(const nvfp4_matrix_desc* descs, int64_t n, float q_max, float* S,
                               float* amax, int* status, void* workspace,
                               size_t workspace_bytes, void* stream);

/* One matrix of a batched sweep: the arguments of nvfp4_scale_sweep_quantize. */
typedef struct nvfp4_sweep_desc {
    const void* W;
    int64_t out, in, ldw;
    const float* h;          /* NULL = plain MSE; all NULL or all non-NULL */
    const float* S;          /* device scalar */
    uint8_t* codes;
    uint8_t* scales;
    int8_t* chosen_offset;   /* may be NULL */
} nvfp4_sweep_desc;

/* Windowed sweep of n matrices with one window [lo, hi] (H-Scale summary,
 * sec. 3 and B).
 *   descs        HOST array of n descriptors (read before the call returns).
 *   workspace    at least nvfp4_scale_sweep_quantize_batched_workspace_size(n)
 *                bytes, 256-byte aligned (a device copy of the table).
 * A batch mixing NULL and non-NULL h returns NVFP4_ERR_INVALID_ARG.  As for
 * nvfp4_global_scale_batched, a capturing stream returns NVFP4_ERR_CAPTURE. */
size_t nvfp4_scale_sweep_quantize_batched_workspace_size(int64_t n);
int nvfp4_scale_sweep_quantize_batched(const nvfp4_sweep_desc* descs, int64_t n, int lo, int hi,
                                       void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * A layer in one call: steps 1-4 for several projections that share
 * calibration inputs (for example an MLP's gate and up projections reading
 * one input, its down projection another).  For every input k,
 * h_k = diag(X_k^T X_k) as nvfp4_diag_hessian writes it (not accumulated);
 * for every weight j, S_j as nvfp4_global_scale writes it, then the windowed
 * sweep of nvfp4_scale_sweep_quantize with the h of its input (input = -1:
 * plain MSE).  The bytes written equal those of the per-step calls.
 *
 * The library orders the work itself: the first weight swept has its S and
 * its input's h computed first; the other reductions, which are bound by HBM
 * bandwidth, are streamed by an extra warp in each CTA of earlier sweeps,
 * which are bound by FP32 arithmetic (H-Scale summary, sec. 4 "Efficiency
 * and Hardware Deployment": the added cost is the offline search and one
 * activation pass).  A reduction that no earlier sweep can carry (the
 * sweep's row length is not a multiple of 512 elements, or it is short) runs
 * on its own before it is needed.  The sweep order is the one with the
 * lowest estimated time (HBM bytes of the reductions run on their own
 * against the sweeps' FP32 work): among all permutations for up to four
 * weights; for more, each weight is tried first with the others in the order
 * given.  Ties keep the order given.  Every order writes the same bytes as
 * long as no two weights' outputs (S, amax, status, codes, scales,
 * chosen_offset) overlap each other or any input, which the call requires.
 * nvfp4_quantize_layer_order writes the order chosen: order[j] = the index of
 * the weight swept j-th (it needs the device, for its SM count; no launch).
 *
 *   weights    n_weights descriptors: W bf16 [out, ldw] (16-byte aligned,
 *              ldw % 8 == 0, in % 16 == 0, out and in > 0); input in
 *              [-1, n_inputs) with inputs[input].in == in; S device scalar
 *              (written); amax, status nullable device scalars (status: 0, or
 *              NVFP4_ERR_NONFINITE when W holds Inf/NaN, as
 *              nvfp4_global_scale); codes [out, in/2] 8-byte aligned; scales
 *              [out, in/16]; chosen_offset [out, in/16] or NULL.
 *   inputs     n_inputs descriptors: X bf16 [tokens, ldx] (16-byte aligned,
 *              in % 8 == 0, tokens >= 0); h float [in], 16-byte aligned
 *              (written).
 *   q_max      448 or 256 as for nvfp4_global_scale; lo, hi as for the sweep.
 *   workspace  device, 256-byte aligned, at least
 *              nvfp4_quantize_layer_workspace_size(...) bytes (which depends
 *              on the device; 0 for invalid descriptors or no device).
 *   sweep_events  NULL, or 2 * n_weights cudaEvent_t (as void*) created by
 *              the caller on this device: events[2j] and events[2j+1] are
 *              recorded on `stream` right before and after weight j's sweep
 *              launch (with the reductions it carries), for timing.
 * Descriptors are read on the host during the call.  Asynchronous on
 * `stream`.  Returns NVFP4_OK or the status of the first failing check.
 * ------------------------------------------------------------------------ */
typedef struct {
  const void* W;
  int64_t out, in, ldw;
  int input;
  float* S;
  float* amax;
  int* status;
  uint8_t* codes;
  uint8_t* scales;
  int8_t* chosen_offset;
} nvfp4_layer_weight;

typedef struct {
  const void* X;
  int64_t tokens, in, ldx;
  float* h;
} nvfp4_layer_input;

size_t nvfp4_quantize_layer_workspace_size(const nvfp4_layer_weight* weights, int n_weights,
                                           const nvfp4_layer_input* inputs, int n_inputs);
int nvfp4_quantize_layer_order(const nvfp4_layer_weight* weights, int n_weights,
                               const nvfp4_layer_input* inputs, int n_inputs, int lo, int hi,
                               int* order);
int nvfp4_quantize_layer(const nvfp4_layer_weight* weights, int n_weights,
                         const nvfp4_layer_input* inputs, int n_inputs, float q_max, int lo,
                         int hi, void* workspace, size_t workspace_bytes,
                         void* const* sweep_events, void* stream);

/* ------------------------------------------------------------------------
 * Several consecutive layers in one call (H-Scale summary, sec. 4
 * "Efficiency and Hardware Deployment": the added cost is one activation pass
 * and the offline search, which a model-wide pass should pay once).  Each
 * layer is the argument set of nvfp4_quantize_layer, its weights' `input`
 * indexing its own inputs.  The call is nvfp4_quantize_layer over all the
 * layers' weights (in layer order) and inputs together: the results are the
 * per-step calls' bytes, and the reductions of a later layer -- its inputs'
 * h and its weights' S -- are streamed beside the sweeps of earlier layers,
 * so that only the first swept weight's S and its input's h run on their own
 * (in a single-layer call, each layer would run those two alone and its last
 * sweep would carry nothing).
 *   layers       n_layers HOST descriptors (read during the call).
 *   sweep_events NULL or 2 * (total weights) events, weights counted across
 *                the layers in order, as for nvfp4_quantize_layer.
 * Workspace, alignment, status and error rules are nvfp4_quantize_layer's;
 * an `input` outside its own layer's inputs returns NVFP4_ERR_INVALID_ARG.
 * ------------------------------------------------------------------------ */
typedef struct {
  const nvfp4_layer_weight* weights;
  int n_weights;
  const nvfp4_layer_input* inputs;
  int n_inputs;
} nvfp4_layer;

size_t nvfp4_quantize_layers_workspace_size(const nvfp4_layer* layers, int n_layers);
int nvfp4_quantize_layers(const nvfp4_layer* layers, int n_layers, float q_max, int lo, int hi,
                          void* workspace, size_t workspace_bytes, void* const* sweep_events,
                          void* stream);

/* ------------------------------------------------------------------------
 * H-Scale as GPTQ's local quantizer (H-Scale summary, sec. B "Implementation"
 * and "GPTQ Integration": H-Scale replaces only the local quantization call;
 * GPTQ's inverse-Cholesky processing, error computation and propagation are
 * unchanged).  GPTQ in the given column order on W with the calibration
 * inputs X:
 *   H = X^T X; a column whose diagonal is 0 gets H_jj = 1 and zero weights;
 *   H += damp * mean(diag H) * I (GPTQ's usual damp is 0.01);
 *   U = the upper Cholesky factor of H^-1;
 *   column by column: quantize w_j, err = (w_j - q_j) / U_jj, and w_k -= err U_jk
 *   for every later column k.
 * The local call: at the first column of each 16-column group, every row's
 * scale code for the group is the windowed sweep's choice (weighted by
 * h = diag(X^T X), or plain MSE if weighted == 0) on the group's current,
 * error-updated FP32 weights, with S = the global scale of the original W;
 * each column of the group is then quantized at its turn with that scale.
 *
 *   W        bf16 [out, ldw], 16-byte aligned, ldw % 8 == 0; in % 16 == 0;
 *            out, in > 0; out < 2^31, in <= 16 * 65535.
 *   X        bf16 [tokens, ldx], 16-byte aligned, ldx % 8 == 0; tokens >= 0,
 *            ldx >= in; tokens, ldx < 2^31 (the GEMM's int sizes).
 *   codes, scales, S, h  the NVFP4 result ([out, in/2], [out, in/16]), the
 *            global scale and diag(X^T X) (as nvfp4_diag_hessian writes it).
 *   status   nullable device int: 0, NVFP4_ERR_NONFINITE (W holds Inf/NaN), or
 *            NVFP4_ERR_NUMERIC (the damped Hessian's Cholesky failed in FP32).
 *   workspace  nvfp4_gptq_workspace_size(out, in, tokens) bytes, 256-byte
 *            aligned (it holds H and its Cholesky factor, the FP32 sums P
 *            [out, in] of the propagated errors, a batch's errors and
 *            factor rows for the update GEMMs in FP16 and the solver's
 *            scratch: about 4 in^2 + out (4 in + 3072) + 3200 in bytes plus
 *            32 MiB).
 * Steps: no inverse is formed.  The lower Cholesky factor of the reversed H
 * gives H = R R^T with R upper (U = R^-1), and the columns run in the
 * equivalent R form: W - Q = Err U, so Err = (W - Q) R, and a group's current
 * weights are W_grp + ((W - Q)[:, <grp] R[<grp, grp]) R_grp^-1 with R_grp the
 * group's 16 x 16 diagonal block.  h, S, the block inverses and the batches
 * of columns are this library's kernels; X^T X and the batches' updates of
 * later columns' sums are GEMMs (cuBLAS; the updates as three FP16
 * tensor-core products of split, power-of-two-scaled FP32 operands with FP32
 * accumulation, about 2^-21 relative per product), the Cholesky factor comes
 * from cuSOLVER.  The first call on a device creates the
 * library's cuBLAS and cuSOLVER handles there, which hold a little device
 * memory until the process exits; every call's scratch is the caller's
 * workspace.  Calls are serialised on the host; asynchronous on `stream`.
 * Results are FP32 GPTQ: they follow an FP64 evaluation of the same steps
 * until a quantization decision flips, which a row then carries into its
 * later columns.
 * ------------------------------------------------------------------------ */
size_t nvfp4_gptq_workspace_size(int64_t out, int64_t in, int64_t tokens);
int nvfp4_gptq_quantize(const void* W, int64_t out, int64_t in, int64_t ldw, const void* X,
                        int64_t tokens, int64_t ldx, float q_max, int lo, int hi, float damp,
                        int weighted, uint8_t* codes, uint8_t* scales, float* S, float* h,
                        int* status, void* workspace, size_t workspace_bytes, void* stream);

/* Opt-in phase timing of nvfp4_gptq_quantize, for profiling without external
 * tools.  nvfp4_gptq_set_timing(1) starts it (and clears what was recorded);
 * each later call records CUDA event pairs on its own stream around its
 * phases (a few hundred per call, up to 8192 pairs in all; the events are
 * created on the device current at the first nvfp4_gptq_set_timing(1) of the
 * process, and calls on other devices are not timed).  nvfp4_gptq_phase_times waits for the recorded
 * events and writes ms[p], the milliseconds spent in phase p summed over
 * the timed calls, for p < n (at most NVFP4_GPTQ_PHASES); it returns
 * NVFP4_ERR_WORKSPACE if the pairs ran out (the sums are then partial).
 * nvfp4_gptq_set_timing(0) stops recording.  Host calls, serialised with
 * nvfp4_gptq_quantize. */
enum nvfp4_gptq_phase {
    NVFP4_GPTQ_PHASE_REDUCTIONS = 0,  /* h and S                                    */
    NVFP4_GPTQ_PHASE_GRAM = 1,        /* X^T X                                      */
    NVFP4_GPTQ_PHASE_FACTOR = 2,      /* damping, Cholesky factor, block inverses   */
    NVFP4_GPTQ_PHASE_BATCH = 3,       /* batch kernels: local call, quantization,
                                         propagation inside a batch                 */
    NVFP4_GPTQ_PHASE_SPLIT = 4,       /* FP16 splits of the factor's rows           */
    NVFP4_GPTQ_PHASE_UPDATE = 5,      /* update GEMMs of later columns' sums        */
    NVFP4_GPTQ_PHASES = 6
};
int nvfp4_gptq_set_timing(int on);
int nvfp4_gptq_phase_times(float* ms, int n);

/* The local call of nvfp4_gptq_quantize on its own: the windowed sweep of an
 * FP32 matrix W [out, ldw] (in % 16 == 0; h NULL = plain MSE; S a device
 * scalar), each group quantized at its chosen scale -- the same device code
 * GPTQ runs on its error-updated columns.  codes 8-byte aligned. */
int nvfp4_scale_sweep_quantize_f32(const float* W, int64_t out, int64_t in, int64_t ldw,
                                   const float* h, const float* S, int lo, int hi,
                                   uint8_t* codes, uint8_t* scales, void* stream);

/* ------------------------------------------------------------------------
 * A mixture-of-experts layer in one call: two batches of expert matrices, each
 * batch reading one expert-contiguous calibration input (for example every
 * expert's gate and up projections reading the routed tokens' hidden states,
 * then every expert's down projection reading their activations).
 *   first_input.h, second_input.h  = the grouped diagonal Hessian of each
 *                    input, as nvfp4_diag_hessian_grouped writes it (not
 *                    accumulated);
 *   S[0 .. n_first + n_second)  = the global scale of every matrix, first
 *                    batch then second, as nvfp4_global_scale_batched writes
 *                    it (amax and status too, both nullable);
 *   both batches' sweeps, as nvfp4_scale_sweep_quantize_batched writes them.
 * The bytes written equal those of the grouped and batched calls.  One batch
 * is swept first, its input's h computed on its own beforehand; the other
 * input's diagonal Hessian is streamed by a fifth warp in every CTA of that
 * sweep, which is bound by FP32 arithmetic, and the other batch is swept last.
 * The call picks the order with the lower estimated time (HBM bytes of the
 * reduction run on its own against the sweeps' FP32 work; see
 * nvfp4_quantize_grouped_layer_order).  `second` goes first only if none of
 * its h point into first_input.h.  Either order writes the same bytes, as
 * long as no matrix's outputs overlap another's or any input (required).
 *
 *   first, second  sweep descriptors as for nvfp4_scale_sweep_quantize_batched
 *              (out, in > 0); descriptor i of `first` has S == S + i, of
 *              `second` S == S + n_first + i.  Their h may point into the
 *              inputs' h (the first batch into first_input.h, the second into
 *              either), or be NULL for a whole batch (plain MSE).
 *   first_input, second_input  X bf16 [total_tokens, ldx] with row_offsets
 *              int64 [experts + 1] on the device (as for
 *              nvfp4_diag_hessian_grouped); h float [experts, in], 16-byte
 *              aligned (written).
 *   workspace  device, 256-byte aligned, at least
 *              nvfp4_quantize_grouped_layer_workspace_size(...) bytes (device
 *              dependent; 0 for invalid arguments or no device).
 *   sweep_events  NULL or 4 cudaEvent_t (as void*): [0], [1] recorded on
 *              `stream` right before and after the sweep launch of `first`,
 *              [2], [3] around that of `second` (the one swept first includes
 *              what it streams), for timing.
 * Asynchronous on `stream`; descriptors are read on the host during the call
 * and staged from host memory, so a capturing stream returns
 * NVFP4_ERR_CAPTURE with nothing enqueued.
 *
 * nvfp4_quantize_grouped_layer_order returns which batch that call, with the
 * same arguments, sweeps first: 0 for `first`, 1 for `second`, or a negative
 * status.  It reads only the descriptors' sizes and h pointers on the host
 * (no CUDA call).
 * ------------------------------------------------------------------------ */
typedef struct {
  const void* X;
  const int64_t* row_offsets;
  int64_t total_tokens, in, ldx;
  float* h;
} nvfp4_grouped_input;

size_t nvfp4_quantize_grouped_layer_workspace_size(const nvfp4_sweep_desc* first, int64_t n_first,
                                                   const nvfp4_sweep_desc* second, int64_t n_second,
                                                   const nvfp4_grouped_input* first_input,
                                                   const nvfp4_grouped_input* second_input,
                                                   int64_t experts, float* S);
int nvfp4_quantize_grouped_layer_order(const nvfp4_sweep_desc* first, int64_t n_first,
                                       const nvfp4_sweep_desc* second, int64_t n_second,
                                       const nvfp4_grouped_input* first_input,
                                       const nvfp4_grouped_input* second_input, int64_t experts,
                                       float* S, int lo, int hi);
int nvfp4_quantize_grouped_layer(const nvfp4_sweep_desc* first, int64_t n_first,
                                 const nvfp4_sweep_desc* second, int64_t n_second,
                                 const nvfp4_grouped_input* first_input,
                                 const nvfp4_grouped_input* second_input, int64_t experts,
                                 float q_max, int lo, int hi, float* S, float* amax, int* status,
                                 void* workspace, size_t workspace_bytes,
                                 void* const* sweep_events, void* stream);

/* ------------------------------------------------------------------------
 * Online activation quantization (ScaleSweep summary, sec. 1-3 and
 * "Experimental Results": in the W+A settings the activations are NVFP4 too,
 * their scales chosen with the MSE objective and the [-3, +7] window).  One
 * launch does, for every token row t of A:
 *   S[t] = fl32(amax_t / fl32(q_max * 6))   (0 for an all-zero row), then
 *   the windowed sweep of nvfp4_scale_sweep_quantize on that row alone, with
 *   h == 1 and the scale S[t].
 * The page does not say how the activations' FP32 scale is set; the reading
 * taken is a dynamic scale per token by the weight-tensor formula, so a row's
 * results do not depend on the other rows.
 *   A          bf16 [tokens, lda], 16-byte aligned; lda % 8 == 0; in % 16 == 0.
 *   q_max      > 0 and finite (ScaleSweep uses 256).
 *   lo, hi     as nvfp4_scale_sweep_quantize; [-3, +7] on the page.
 *   S          float [tokens] (written).
 *   codes      uint8 [tokens, in/2], 8-byte aligned; scales uint8 [tokens, in/16];
 *   chosen_offset  int8 [tokens, in/16] or NULL.
 *   status     int, device scalar, may be NULL: the call first sets it to
 *              NVFP4_OK (an asynchronous memset on `stream`); a row holding Inf
 *              or NaN sets it to NVFP4_ERR_NONFINITE and gets S[t] = NaN and
 *              zero codes, scales and offsets.
 * Layout of codes and scales as for a weight matrix [tokens, in].
 * ------------------------------------------------------------------------ */
int nvfp4_quantize_activations(const void* A, int64_t tokens, int64_t in, int64_t lda,
                               float q_max, int lo, int hi, float* S, uint8_t* codes,
                               uint8_t* scales, int8_t* chosen_offset, int* status,
                               void* stream);

/* ------------------------------------------------------------------------
 * Scale bytes in the tensor-core layout.  The pages return groups "in native
 * NVFP4 representation" (H-Scale summary, sec. 3); a Blackwell block-scaled
 * NVFP4 GEMM reads the codes as they are (two E2M1 values per byte, element
 * 2k in the low nibble) but wants the E4M3 scales tiled:
 *   rows padded to a multiple of 128 and columns to a multiple of 4 (padding
 *   bytes 0); 128 x 4 blocks of 512 bytes stored block-row by block-row;
 *   inside a block, scale (r, c) at byte (r % 32) * 16 + (r / 32) * 4 + c.
 * This is the 16-element E4M3 scale-vector layout of cuBLASLt's NVFP4 GEMM.
 *   scales     uint8 [rows, ld] (row-major as written by the sweep), cols <= ld.
 *   cols       in / 16 (scales per row).
 *   out        uint8 [nvfp4_blocked_scales_size(rows, cols)], 16-byte aligned.
 * ------------------------------------------------------------------------ */
size_t nvfp4_blocked_scales_size(int64_t rows, int64_t cols);
int nvfp4_scales_to_blocked(const uint8_t* scales, int64_t rows, int64_t cols, int64_t ld,
                            uint8_t* out, void* stream);

/* ------------------------------------------------------------------------
 * Dequantize (NVFP4 decode, H-Scale summary sec. 3: effective scale = global
 * x local): W_out[r, j] = sign * fl32(g[k] * v(scale)) * S, float [out, in].
 *   codes [out, in/2] 8-byte aligned; scales [out, in/16]; S device scalar;
 *   W_out 16-byte aligned; in % 16 == 0.
 * ------------------------------------------------------------------------ */
int nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* S,
                     int64_t out, int64_t in, float* W_out, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4HS_H */
