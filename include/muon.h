/*
 * muon.h -- C ABI of the B200 (sm_100a) Muon optimizer step.
 *
 * What the library computes (Modded-NanoGPT news article, "Muon optimizer"
 * section):
 *   - the lessons paragraph: Nesterov momentum on the gradient, with the
 *     orthogonalisation applied after the momentum, run in bf16;
 *   - the zeroth_power_via_newtonschulz5 listing: X = G / (||G||_F + eps),
 *     transpose when rows > cols, `ns_steps` quintic iterations
 *     A = X X^T, B = b A + c A A, X = a X + B X with
 *     (a, b, c) = (3.4445, -4.7750, 2.0315), transpose back;
 *   - the update itself (the article's formula did not survive extraction;
 *     the plainest reading is used): buf <- mu*buf + g, G = g + mu*buf,
 *     W <- W - lr * NS5(G).
 *
 * Conventions shared by every entry point
 *   - Matrices are fp32, row-major, contiguous; matrix i has shapes[2i] rows
 *     and shapes[2i+1] columns.  Only 2-D matrices can be expressed.
 *   - All pointers inside the pointer arrays are DEVICE pointers on the
 *     current CUDA device, owned by the caller.  The pointer arrays and the
 *     shapes array themselves are HOST memory, read during the call only.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous with respect to the host: results are ready once the
 *     stream has reached this call.
 *   - Argument errors are detected on the host, before anything is launched,
 *     and returned synchronously.  Errors found by kernels (a bounded wait
 *     that ran out) are recorded in a per-(device, stream) status word; they
 *     are returned by the next call on that stream, by muon_sync_status(), and
 *     described by muon_last_error().  Kernels never trap.
 *   - The library keeps, per (device, stream), a workspace in device memory
 *     (bf16 iterates, Gram and polynomial matrices, norms, TMA descriptors).
 *     It is allocated by the first call that needs it (cudaMalloc, which is
 *     not allowed during stream capture: make the first call for a given set
 *     of shapes outside capture) and freed by muon_release().
 *   - Matrices with short side <= 128 and long side <= 512, or with both
 *     sides <= 256, run their whole step in one fused launch (one CTA per
 *     matrix, a cluster of two CTAs per matrix for both sides <= 256, or -- for
 *     at most 37 matrices with short side <= 128 and long side above 256 -- a
 *     cluster of four CTAs per matrix) and use no workspace.  The others
 *     run the momentum/norm/cast prologue, then every Newton-Schulz phase and
 *     the weight update in one chained launch (short side <= 1024), or one
 *     launch per phase (larger matrices).
 *   - Concurrent calls on different streams use different workspaces; calls
 *     on one stream are serialised by the stream.
 *   - NaN / Inf in the inputs propagate to the outputs; nothing checks them.
 */
#ifndef MUON_B200_H
#define MUON_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MUON_OK = 0,
  MUON_ERR_INVALID_ARG = -1,  /* null pointer, n <= 0, ns_steps < 0, bad flag  */
  MUON_ERR_SHAPE = -2,        /* a dimension <= 0 or too large for int32 math  */
  MUON_ERR_CUDA = -3,         /* a CUDA runtime / driver call failed           */
  MUON_ERR_NOMEM = -4,        /* workspace allocation failed                   */
  MUON_ERR_TIMEOUT = -5,      /* a kernel gave up on a bounded wait            */
  MUON_ERR_DEVICE = -6,       /* no usable sm_100 device                       */
  MUON_ERR_UNSUPPORTED = -7   /* configuration this build does not handle      */
} muon_status;

/* Default quintic coefficients, step count and eps of the NS5 listing. */
#define MUON_NS_A 3.4445f
#define MUON_NS_B (-4.7750f)
#define MUON_NS_C 2.0315f
#define MUON_NS_STEPS 5
#define MUON_NS_EPS 1e-7f

/*
 * One Muon step over n independent weight matrices (Nesterov momentum,
 * NS5 with the listing's defaults, W -= lr*O).
 *   params[i]        in/out  W_i, updated in place.
 *   grads[i]         in      g_i, read only.
 *   momentum_bufs[i] in/out  buf_i (fp32 state), updated in place to
 *                            mu*buf_i + g_i.
 *   shapes           in      2n int64: rows_i, cols_i.
 *   ns_steps         >= 0    quintic iterations (5 in the listing; 0 gives
 *                            O = G/(||G||_F + eps) rounded to bf16).
 * Returns MUON_OK or a muon_status error code.
 */
int muon_step(float* const* params, const float* const* grads, float* const* momentum_bufs,
              const int64_t* shapes, int n, float lr, float mu, int ns_steps, void* stream);

/*
 * muon_step with every constant of the method exposed: quintic coefficients
 * (a, b, c), eps added to the Frobenius norm, and nesterov (1: G = g + mu*buf
 * after the buffer update, as in the lessons paragraph; 0: G = buf).
 */
int muon_step_ex(float* const* params, const float* const* grads, float* const* momentum_bufs,
                 const int64_t* shapes, int n, float lr, float mu, int ns_steps,
                 float a, float b, float c, float eps, int nesterov, void* stream);

/*
 * muon_step_ex with e4m3 (fp8) operands in the first `fp8_iters` quintic
 * iterations (0 <= fp8_iters <= 2; 0 is muon_step_ex).  A reduced-precision
 * variant, not the method as the article states it (its lessons paragraph
 * runs the iteration in bf16); the fp8 training results quoted on the
 * Karpathy-tweets page (llm.c, tensorwise vs rowwise scaling) motivate it.
 *   - Which products read e4m3 operands: the A A product of iterations
 *     0 .. fp8_iters-1 and the X X^T product of iterations 1 .. fp8_iters-1.
 *     They take e4m3 copies of their operands scaled by a power of two (fixed
 *     per iteration from bounds on the singular values, see the source) and
 *     accumulate in fp32; the epilogues still work in fp32 and write the bf16
 *     results as before, plus the e4m3 copies.  The update B X keeps bf16
 *     operands in every iteration (an e4m3 iterate would move its singular
 *     vectors, which no later iteration corrects), and so does iteration 0's
 *     X X^T (the first iterate is stored before the norm of G is known).
 *   - Error: the same as the bf16 path's to within a few 1e-4 relative
 *     Frobenius (about 1e-2 against exact NS5 on Gaussian, tall and
 *     ill-conditioned inputs); e4m3 in a third iteration would not stay
 *     within 3e-2.
 *   - Applies where the phases run as separate launches (groups with a
 *     short side above 1024), where it is faster (3-7 % on the GPT-2-XL set and
 *     the 2048 / 4096 square batches).  Groups that run in the chained launch
 *     (short side <= 1024) and the matrices the fused single-CTA and CTA-pair
 *     kernels run whole keep bf16 operands: there the e4m3 copies cost more
 *     than the shorter products save (measured slower on every such set), so
 *     for them this call is muon_step_ex.
 *   - Workspace: the e4m3 copies take kp*lp + kp*kp more bytes per matrix
 *     (kp, lp: short and long side rounded up to 128) than muon_workspace_size
 *     reports.
 * Returns MUON_ERR_INVALID_ARG for fp8_iters outside [0, 2], else as muon_step_ex.
 */
int muon_step_fp8(float* const* params, const float* const* grads, float* const* momentum_bufs,
                  const int64_t* shapes, int n, float lr, float mu, int ns_steps, float a, float b, float c,
                  float eps, int nesterov, int fp8_iters, void* stream);

/*
 * The two halves of a Muon step for a data-parallel run that exchanges the
 * orthogonalised update in bf16 instead of the fp32 weights (half the bytes
 * on the interconnect; the speedrun of the Modded-NanoGPT article trains on 8
 * GPUs).  Every rank computes O for the matrices it owns with
 * muon_update_bf16, the ranks all-gather the bf16 O, and every rank applies
 * all of them with muon_apply_bf16, so that every replica of W receives the
 * same update.  (A deployment variant: the article has no exchange.)
 *
 * muon_update_bf16: momentum and NS5 as in muon_step_ex, W untouched.
 *   grads[i]         in      g_i (fp32, m x n), read only.
 *   momentum_bufs[i] in/out  buf_i, updated in place as by muon_step_ex.
 *   O[i]             out     NS5(G_i) rounded to bf16 (round to nearest
 *                            even), m x n row-major, 2-byte bf16 bit
 *                            patterns, caller-owned device memory.
 * The update goes through a library-held fp32 scratch of sum(m*n) floats
 * (allocated by the first call that needs it, freed by muon_release) before
 * its rounding to bf16.
 */
int muon_update_bf16(const float* const* grads, float* const* momentum_bufs, uint16_t* const* O,
                     const int64_t* shapes, int n, float mu, int ns_steps, float a, float b, float c,
                     float eps, int nesterov, void* stream);

/*
 * muon_apply_bf16: W_i <- W_i - lr * O_i for bf16 O_i (m x n row-major,
 * 2-byte bf16 bit patterns, read only), one fused multiply-add in fp32 per
 * element.  params[i] in/out: W_i, updated in place.
 */
int muon_apply_bf16(float* const* params, const uint16_t* const* O, const int64_t* shapes, int n, float lr,
                    void* stream);

/*
 * NS5 alone (the zeroth_power_via_newtonschulz5 listing): O_i = NS5(G_i)
 * with the listing's defaults and `ns_steps` iterations.  G_i is read only,
 * O_i (m x n fp32, caller-owned device memory) is overwritten.
 */
int muon_orthogonalize(const float* const* G, float* const* O, const int64_t* shapes, int n,
                       int ns_steps, void* stream);

/*
 * muon_step on HOST buffers: params, grads and momentum_bufs point to host
 * memory (pinned memory gives full PCIe bandwidth; pageable works).  The
 * library copies the inputs to device staging buffers, runs the step and
 * copies W and buf back, all on `stream`, and returns after the stream has
 * finished (the host buffers hold the results on return).
 */
int muon_step_host(float* const* params, const float* const* grads, float* const* momentum_bufs,
                   const int64_t* shapes, int n, float lr, float mu, int ns_steps, void* stream);

/*
 * muon_step without any device allocation.  (Not part of the method: the
 * article has no counterpart; this is a deployment variant of muon_step.)
 *
 * For callers that cannot call cudaMalloc -- code running inside a custom
 * allocator or a memory-pool callback, or a process whose device memory is
 * budgeted up front so that a new allocation could fail or deadlock.  The
 * caller passes the same inputs and outputs as to muon_step (device
 * pointers, updated in place); all scratch (bf16 iterates, Gram and
 * polynomial matrices, norm partials, tensor-map table, status word) lives
 * in one static device array of 64 MiB that every GPU loading this library
 * holds until the process exits.
 *   - Limit: one call takes at most 320 matrices over at most 16 padded
 *     shapes, and their scratch (the muon_workspace_size layout) must fit in
 *     64 MiB minus a 64 KiB table, e.g. one GPT-2-124M layer (4 x 768x768,
 *     768x3072, 3072x768).  Larger requests return MUON_ERR_UNSUPPORTED with
 *     the required size in muon_last_error(); nothing is launched.  Matrices
 *     the fused kernels run whole (short side <= 128 and long side <= 512,
 *     or both sides <= 256) use no scratch and do not count.
 *   - The array is part of this library's device code: it comes into being
 *     when that code is loaded on a device, which with CUDA's lazy module
 *     loading (the default) is the first call of this library on that device
 *     -- any entry point, this one included.  That first load allocates the
 *     array and the code, so make one call on each device (this entry point
 *     with real buffers, or any other) before entering a context that must not
 *     allocate, and before any stream capture.  Each call then looks up the
 *     array's device address with the device current, which allocates
 *     nothing.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind; each call clears what must start at zero.  Calls that overlap
 *     on the GPU (e.g. on two streams) race on it: serialise them.
 *   - The call waits for earlier work on `stream` before it launches: it
 *     reads back the status word its kernels keep in the array.  A bounded
 *     wait that ran out in the previous call's kernels is returned here as
 *     MUON_ERR_TIMEOUT (nothing is launched; the word is cleared, so the next
 *     call runs normally).  The tensor-map table is copied from pageable host
 *     memory on `stream`.
 *   - muon_debug_set applies as for muon_step (wait bound, fault injection).
 *   - After cudaDeviceReset, call muon_release() before the next call.
 */
int muon_step_noalloc(float* const* params, const float* const* grads, float* const* momentum_bufs,
                      const int64_t* shapes, int n, float lr, float mu, int ns_steps, void* stream);

/* Bytes of device workspace a call with these shapes uses (0 on bad input). */
size_t muon_workspace_size(const int64_t* shapes, int n);

/* Waits for `stream`, then returns and clears the status its kernels recorded
 * (MUON_OK, MUON_ERR_TIMEOUT, ...). */
int muon_sync_status(void* stream);

/* Human-readable description of the last error seen by this thread. */
const char* muon_last_error(void);

/* Frees every cached workspace and staging buffer on every device and
 * forgets the per-device set-up (call it before cudaDeviceReset). */
void muon_release(void);

/* ---- measurement hooks (used by the benchmark; off by default) ---------- */

/* Kernel kinds reported by the profiling hooks. */
#define MUON_KIND_PROLOGUE 0
#define MUON_KIND_GRAM 1
#define MUON_KIND_POLY 2
#define MUON_KIND_UPDATE 3
#define MUON_KIND_UPDATE_APPLY 4
#define MUON_KIND_APPLY_X0 5
#define MUON_KIND_SMALL 6        /* fused single-CTA step of small matrices */
#define MUON_KIND_PAIR 7         /* fused CTA-pair step, 128 < short side <= 256, long side <= 256 */
#define MUON_KIND_CHAIN 8        /* every Newton-Schulz phase and the weight update, one chained launch */
#define MUON_KIND_O16 9          /* bf16 update exchange: fp32 -> bf16 rounding of O, or W -= lr * O */
#define MUON_KIND_QUAD 10        /* fused step on a cluster of four CTAs, short side <= 128, 256 < long side <= 512 */
#define MUON_NUM_KINDS 11

/* 1: bracket every kernel launch with CUDA events on its stream; 0: stop. */
int muon_profile_enable(int enable);
/* Synchronises the recorded events and adds, per kind, the summed device
 * milliseconds and the launch count into ms[kind] / launches[kind]
 * (arrays of nkinds entries); then forgets them. */
int muon_profile_read(double* ms, int64_t* launches, int nkinds);
/* Number of kernels this library has launched since it was loaded. */
int64_t muon_launch_count(void);
/* Clusters of two CTAs the chained launch runs on the current device (the
 * most that can be resident at once), or -1 if the device cannot be used. */
int muon_chain_clusters(void);

/* ---- test hooks -------------------------------------------------------- */

/* wait_limit_ns: bound of every device-side wait (0 keeps the default, 2 s).
 * flags bit 0: the next GEMM launch skips filling its first pipeline stage,
 * so its MMA warp's wait runs out and the call reports MUON_ERR_TIMEOUT
 * (fault injection that neither faults nor hangs the GPU).
 * flags bit 1: the same for the next CTA-pair launch, whose first product is
 * not issued, so both CTAs' waits for it run out.
 * flags bit 2 (kept until cleared): run the Newton-Schulz phases as one launch
 * per phase instead of the chained launch (for comparisons).
 * flags bit 3: the next four-CTA launch keeps back one CTA's first Gram
 * partial, so the waits of every CTA of its clusters run out.
 * flags bit 5 (bounds-checking build only, libmuon_b200_debug.so): the next
 * GEMM launch that runs one phase gets one tile index past the end of its grid
 * for every cluster; the device bounds checks stop it before it touches memory
 * and the call reports MUON_ERR_DEVICE. */
int muon_debug_set(int flags, int64_t wait_limit_ns);

/* Guard bands (a debugging aid).  With MUON_GUARD_BANDS=1 in the environment
 * when the library is loaded, the workspace layout leaves 4 KiB of a fixed
 * byte (0xA5) after every region of a group (iterates, Gram and polynomial
 * matrices, norm partials, scales, completion counters), written on `stream`
 * before the group's launches.  This call waits for `stream` and returns how
 * many of those bytes of the last group run on it no longer hold the fixed
 * byte (0: no launch wrote past the end of a region), MUON_ERR_UNSUPPORTED
 * when guard bands are off, or another MUON_ERR_* on failure.  Covers the
 * workspace of muon_step, muon_step_ex, muon_step_fp8's bf16 regions,
 * muon_orthogonalize and muon_update_bf16, not the static scratch of
 * muon_step_noalloc. */
int muon_guard_check(void* stream);

/* The work lists of the chained launch for these shapes and `ns_steps`, as
 * the library would build them for a device that holds `nclusters` clusters of
 * two CTAs at once (host only: no device is touched).  Covers the first group
 * of matrices (at most 320 matrices over 16 padded shapes; matrices the fused
 * kernels run whole take no part).  Item i is items[8i .. 8i+7] = {need,
 * matrix (the caller's index), shape class, index in class, tile row, tile
 * column, phase (0 Gram, 1 polynomial, 2 update, 3 the last update with
 * W -= lr*O), iteration}; cluster c runs
 * items [cluster_off[c], cluster_off[c + 1]) in order (cluster_off holds
 * nclusters + 1 entries).  *nitems receives the item count;
 * MUON_ERR_INVALID_ARG if `capacity` (in items) is smaller. */
int muon_chain_plan(const int64_t* shapes, int n, int ns_steps, int nclusters, int32_t* items, int64_t capacity,
                    int32_t* cluster_off, int64_t* nitems);

#ifdef __cplusplus
}
#endif

#endif /* MUON_B200_H */
