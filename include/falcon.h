/*
 * falcon.h -- C ABI of libfalcon.so: the Falcon family of normalised
 * first-order fast-weight updates (Fast Weight Attention) on sm_100a.
 *
 * Method (web pages on arXiv 2608.27763, cited by title and section):
 *   [EXPL] "Fast Weight Attention：用于持续学习的快速权重注意力", 核心方法 1-4
 *   [SUMM] "Fast Weight Attention for Continual Learning", 方法
 *   [NEWS] "借鉴40年前的设想！字节Seed提出快速权重注意力推进大模型持续学习", 02
 *
 * Per (batch b, head h) the state S is a d_v x d_k matrix, S_0 = 0.  With the
 * prefix-aligned pair (x_t, y_t) = (phi(k_{t-1}), v_t) ([SUMM] 输入与状态定义),
 * phi(k) = k/|k| (phi(0) = 0) and x_1 = 0:
 *   n_t     = |x_t|^2  (Falcon-3/3A: sum of |x_i|^2 over the window W_t)
 *   eta_t   = beta_t / (eps + n_t), 0 when n_t = 0   (NLMS step, [EXPL] 核心方法 2)
 *   alpha_t = max(1 - eta_t * lambda_h, 2^-20)        (positive decay, [NEWS] 02 (1))
 *   Falcon-1/2   S_t = alpha S_{t-1} + eta (y_t - S_{t-1} x_t) x_t^T
 *   Falcon-1A/2A S_t = alpha S_{t-1} + eta y_t x_t^T
 *   Falcon-3     S_t = alpha S_{t-1} + eta sum_{i in W_t} (y_i - S_{t-1} x_i) x_i^T
 *   Falcon-3A    S_t = alpha S_{t-1} + eta sum_{i in W_t} y_i x_i^T
 *   o_t = S_t q_t  (read after write)
 * W_t = {max(1, t-window+1), ..., t}.  Falcon-2/2A take beta (hence eta and
 * alpha) per value channel j, i.e. per row of S ([NEWS] 02 (2)).
 *
 * Conventions shared by every entry point:
 *  - All tensor arguments are DEVICE pointers (HOST pointers for
 *    falcon_fwd_host) to contiguous row-major arrays owned by the caller;
 *    the library never frees or retains them.
 *  - Calls only enqueue work on `stream` (0 = legacy default stream) and never
 *    synchronise.  A non-zero return means nothing was enqueued, except
 *    FALCON_ERR_LAUNCH, which reports cudaGetLastError() after a launch.
 *    Faults inside a kernel surface asynchronously on the stream.
 *  - Device values are not inspected by the host: lambda must lie in [0, 1)
 *    and beta should be >= 0; other values give results but no error.
 *  - Element types: falcon_dtype selects fp32 or bf16 for q, k, v, beta and
 *    out.  lambda, the state, x_prev and the window carry are always fp32.
 */
#ifndef FALCON_H
#define FALCON_H

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FALCON_F1 = 0,  /* regression, scalar NLMS step                      */
    FALCON_F2 = 1,  /* regression, one step per value channel            */
    FALCON_F3 = 2,  /* regression, sliding-window mini-batch of `window` */
    FALCON_F1A = 3, /* inner product, scalar step                        */
    FALCON_F2A = 4, /* inner product, per value channel                  */
    FALCON_F3A = 5  /* inner product, sliding window                     */
} falcon_variant;

/* The three equivalent computation forms ([EXPL] 核心方法 3; [SUMM] 计算形式与数值稳定). */
typedef enum {
    FALCON_RECURRENT = 0, /* token-by-token state update                    */
    FALCON_MASKED = 1,    /* all positions at once through a causal L x L mask */
    FALCON_CHUNK = 2      /* parallel inside chunks, state passed between    */
} falcon_form;

typedef enum { FALCON_F32 = 0, FALCON_BF16 = 1 } falcon_dtype;

/* Sample pairing: the prefix-aligned pair ([SUMM] 输入与状态定义) or the
 * same-step pair (phi(k_t), v_t) ([EXPL] 核心方法 1, warning paragraph). */
typedef enum { FALCON_PAIR_PREFIX = 0, FALCON_PAIR_SAME_STEP = 1 } falcon_pairing;

/* Feature map: L2 normalisation, or the identity (for special-case checks). */
typedef enum { FALCON_PHI_L2 = 0, FALCON_PHI_IDENTITY = 1 } falcon_phi;

enum {
    FALCON_OK = 0,
    FALCON_ERR_NULL = -1,        /* a required pointer is NULL                      */
    FALCON_ERR_ENUM = -2,        /* variant / form / dtype / pairing / phi invalid   */
    FALCON_ERR_SHAPE = -3,       /* B,H,L < 0, or d_k, d_v not in {16,32,64,128}     */
    FALCON_ERR_CHUNK = -4,       /* chunk not in {16,32,64} for the chunk form      */
    FALCON_ERR_WINDOW = -6,      /* window < 1 or > 8 for Falcon-3/3A               */
    FALCON_ERR_LAUNCH = -7,      /* a kernel launch failed (cudaGetLastError)       */
    FALCON_ERR_ALLOC = -8,       /* stream-ordered scratch allocation failed        */
    FALCON_ERR_UNSUPPORTED = -9, /* combination not supported (e.g. pairing+decode) */
    FALCON_ERR_SCRATCH = -10     /* problem needs more than the fixed scratch of
                                    falcon_fwd_masked_noalloc                      */
};

/*
 * falcon_fwd -- forward pass over whole sequences.
 *
 *   q, k     [B,H,L,d_k] dtype     queries and keys
 *   v        [B,H,L,d_v] dtype     values (targets y_t = v_t)
 *   beta     [B,H,L] dtype (Falcon-1/3/1A/3A) or [B,H,L,d_v] (Falcon-2/2A)
 *   lambda   [H] fp32              forgetting strength per head, in [0,1)
 *   eps      NLMS regulariser (>= 0)
 *   window   B_w for Falcon-3/3A (1..8); ignored otherwise
 *   chunk    chunk length for FALCON_CHUNK (16, 32 or 64); ignored otherwise
 *   out      [B,H,L,d_v] dtype     o_t = S_t q_t (written)
 *   final_state [B,H,d_v,d_k] fp32 S_L (written), may be NULL
 * S_0 = 0.  L may be 0 (out untouched, final_state zeroed) and need not be a
 * multiple of `chunk`.  Two paths draw stream-ordered scratch on `stream`
 * from a memory pool the library owns (one per device, kept mapped between
 * calls; see falcon_scratch_trim) and return FALCON_ERR_ALLOC if that fails:
 * FALCON_MASKED (about B*H*L*(window*d_v+2*d_v) floats) and the bf16
 * tensor-core chunk path, Falcon-1/1A with d_k = d_v = 64 and chunk 64
 * (32 KiB + 4 bytes per (b, h, chunk): the chunk-local results that the
 * second of its two kernels chains across chunks).
 */
int falcon_fwd(falcon_variant variant, falcon_form form, falcon_dtype dtype,
               const void *q, const void *k, const void *v, const void *beta,
               const float *lambda, float eps, int window,
               int B, int H, int L, int d_k, int d_v, int chunk,
               void *out, float *final_state, cudaStream_t stream);

/* falcon_fwd with the pairing and the feature map selectable. */
int falcon_fwd_ex(falcon_variant variant, falcon_form form, falcon_dtype dtype,
                  falcon_pairing pairing, falcon_phi phi,
                  const void *q, const void *k, const void *v, const void *beta,
                  const float *lambda, float eps, int window,
                  int B, int H, int L, int d_k, int d_v, int chunk,
                  void *out, float *final_state, cudaStream_t stream);

/*
 * falcon_fwd_host -- falcon_fwd_ex for inputs and outputs in HOST memory,
 * for one or several variants over the same inputs.  The library copies the
 * inputs to the device, runs the forward and copies the results back.  The
 * batch is cut into `slices` runs of whole batch rows; slice i's inputs go
 * host->device on a library-owned copy stream while slice i-1 computes on
 * `stream` and slice i-2's outputs go device->host on a second copy stream.
 *
 *   n_variants   1..6 entries of `variants`, all with the same beta layout
 *                (all per value channel, Falcon-2/2A, or none): every one is
 *                computed from the same inputs (FALCON_ERR_UNSUPPORTED
 *                otherwise, and for n_variants outside 1..6 or slices < 0)
 *   q, k, v, beta, lambda   as in falcon_fwd_ex, in host memory (page-locked
 *                memory lets the copies run asynchronously and overlap;
 *                pageable memory gives the same results without overlap,
 *                and its copies may block the calling thread)
 *   out          array of n_variants host pointers, out[i] [B,H,L,d_v] dtype
 *   final_state  NULL, or an array of n_variants host pointers (entries may
 *                be NULL), final_state[i] [B,H,d_v,d_k] fp32
 *   slices       number of slices, clamped to [1, min(B, 64)]; 0 lets the
 *                library choose (about one per 4 MiB of input, at most 8)
 *   every other argument as in falcon_fwd_ex.
 * The call returns once the work is enqueued.  The host buffers must stay
 * valid, and the inputs unchanged, until `stream` has passed the call's work;
 * the outputs are complete then (cudaStreamSynchronize(stream)).  The device
 * buffers (inputs, lambda, outputs and states: about the inputs' size plus
 * n_variants times the outputs') are one stream-ordered block from the
 * library's pool, freed on `stream` at the end of the call's work.  Argument
 * errors return before anything is enqueued.  An error after the first copy
 * (FALCON_ERR_LAUNCH, or a status of the per-slice forward) stops further
 * slices; the streams are still joined into `stream` and the block freed,
 * and the outputs are then incomplete.
 */
int falcon_fwd_host(int n_variants, const falcon_variant *variants, falcon_form form, falcon_dtype dtype,
                    falcon_pairing pairing, falcon_phi phi,
                    const void *q, const void *k, const void *v, const void *beta,
                    const float *lambda, float eps, int window,
                    int B, int H, int L, int d_k, int d_v, int chunk,
                    void *const *out, float *const *final_state, int slices, cudaStream_t stream);

/*
 * falcon_fwd_carry -- falcon_fwd over a segment that continues a sequence:
 * the recurrence picks up where an earlier segment (or a run of decode
 * steps) left off.  Chunks already hand a fixed-size state from one to the
 * next ([EXPL] 核心方法 3; [NEWS] 02 (2)); a segment boundary is the same
 * hand-off, plus the samples that straddle it.
 *
 *   initial_state [B,H,d_v,d_k] fp32, or NULL: S_0 of the segment (zeros)
 *   x_prev        [B,H,d_k] fp32, or NULL: phi(k) of the token before the
 *                 segment, i.e. x_1 of the segment under the prefix pair
 *                 (zeros: the start of a sequence)
 *   win           [B,H,window-1,d_k+d_v] fp32, Falcon-3/3A, or NULL: the
 *                 window-1 samples (x_i, y_i) before the segment, oldest
 *                 first (zeros where the sequence has fewer)
 * The carry has exactly the layout of the decode carry, so the final state of
 * one segment and falcon_decode_carry_from_prefill of its keys and values
 * continue it (or decode_step's in/out buffers after decoding).  Every other
 * argument is as in falcon_fwd; prefix pairing, L2 feature map.  Forms:
 * FALCON_RECURRENT and FALCON_CHUNK; FALCON_MASKED with a non-NULL carry
 * returns FALCON_ERR_UNSUPPORTED (with all three NULL this is falcon_fwd).
 * With L = 0 the final state is initial_state (or zeros).
 */
int falcon_fwd_carry(falcon_variant variant, falcon_form form, falcon_dtype dtype,
                     const void *q, const void *k, const void *v, const void *beta,
                     const float *lambda, float eps, int window,
                     int B, int H, int L, int d_k, int d_v, int chunk,
                     const float *initial_state, const float *x_prev, const float *win,
                     void *out, float *final_state, cudaStream_t stream);

/*
 * falcon_bwd -- the backward pass: gradients of a scalar loss with respect
 * to q, k, v, beta and lambda, given dL/d(out) and dL/d(final_state), for a
 * forward from S_0 = 0 with the same arguments.  The chunk form trains on the
 * recurrent function ([EXPL] 核心方法 3); this is its derivative, taken in
 * the recurrent form on the CUDA cores (fp32); shown here for one sample per
 * update (a window sums the same terms over its samples):
 *   dq_t = S_t^T do_t;  Gs_t = do_t q_t^T + alpha_{t+1} Gs_{t+1};
 *   dv_t = eta_t (Gs_t x_t);  the decays through dL/dG_t = do_t o_t - eta_t
 *   y_t (Gs_t x_t) (+ <dL/dS_L, S_L> at the last token) summed from t
 *   onwards (per value channel for Falcon-2A);
 *   then alpha = max(1 - eta lambda, 2^-20) (no gradient on the floor),
 *   eta = beta/(eps + |x|^2) and x = phi(k).
 *
 *   variant     any; window as in falcon_fwd (1..8 for Falcon-3/3A)
 *   dtype, q, k, v, beta, lambda, eps, B, H, L, pairing, phi: as in
 *               falcon_fwd_ex; d_k = d_v in {32, 64, 128} (other shapes:
 *               FALCON_ERR_UNSUPPORTED)
 *   dout        [B,H,L,d_v] dtype: dL/d(out)
 *   dstate      [B,H,d_v,d_k] fp32, or NULL (zero): dL/d(final_state)
 *   dq, dk      [B,H,L,d_k] fp32, written
 *   dv          [B,H,L,d_v] fp32, written
 *   dbeta       [B,H,L] (Falcon-1/3/1A/3A) or [B,H,L,d_v] (Falcon-2/2A) fp32, written
 *   dlambda     [H] fp32, written (summed over b), or NULL
 * The regression family's derivative needs S_{t-1} at every step: the
 * forward sweep keeps S every 32 tokens and the reverse sweep recomputes
 * each 32-token stretch from it.
 * Scratch: (2 L d + L + 5 L c) floats per (b,h), c = 1 or d_v, plus
 * (ceil(L/32) + 32) d^2 for the regression family (and under 64 floats of
 * alignment), stream-ordered from the library's pool (FALCON_ERR_ALLOC if
 * that fails).  Errors as in falcon_fwd.
 */
int falcon_bwd(falcon_variant variant, falcon_dtype dtype, falcon_pairing pairing, falcon_phi phi,
               const void *q, const void *k, const void *v, const void *beta, const float *lambda, float eps,
               int window, int B, int H, int L, int d_k, int d_v, const void *dout, const float *dstate,
               float *dq, float *dk, float *dv, float *dbeta, float *dlambda, cudaStream_t stream);

/*
 * falcon_decode_step -- one recurrent step for N independent sequences
 * ([EXPL] 核心方法 3: recurrent, O(d^2) per step, for inference).
 *
 *   q, k     [N,H,d_k] dtype, v [N,H,d_v] dtype, beta [N,H] or [N,H,d_v] dtype
 *   lambda   [H] fp32; eps, window as in falcon_fwd
 *   state    [N,H,d_v,d_k] fp32, in/out: S_{t-1} -> S_t
 *   x_prev   [N,H,d_k] fp32, in/out: phi(k_{t-1}) -> phi(k_t); zeros before
 *            the first token of a sequence
 *   win      [N,H,window-1,d_k+d_v] fp32, in/out, Falcon-3/3A only (NULL
 *            otherwise): the previous window-1 samples (x_i, y_i), oldest
 *            first; zeros where the sequence has fewer samples
 *   out      [N,H,d_v] dtype: o_t
 * Prefix pairing and the L2 feature map.  Each (n,h) is read and written by
 * exactly one thread block, so in-place carries are race-free.
 */
int falcon_decode_step(falcon_variant variant, falcon_dtype dtype,
                       const void *q, const void *k, const void *v, const void *beta,
                       const float *lambda, float eps, int window,
                       int N, int H, int d_k, int d_v,
                       float *state, float *x_prev, float *win, void *out,
                       cudaStream_t stream);

/*
 * falcon_decode_carry_from_prefill -- the decode carry after a prefill of L
 * tokens: x_prev = phi(k_L) and, for Falcon-3/3A, the samples (x_i, v_i),
 * i = L-window+2 .. L (zeros for i < 1).  k [B,H,L,d_k], v [B,H,L,d_v] dtype;
 * x_prev [B,H,d_k] and win [B,H,window-1,d_k+d_v] fp32 are written (win may
 * be NULL when window <= 1 or the variant has no window).  The final state of
 * the prefill comes from falcon_fwd's final_state.
 */
int falcon_decode_carry_from_prefill(falcon_variant variant, falcon_dtype dtype,
                                     const void *k, const void *v, int window,
                                     int B, int H, int L, int d_k, int d_v,
                                     float *x_prev, float *win, cudaStream_t stream);

/*
 * falcon_fwd_masked_noalloc -- the masked-parallel forward (prefix pair, L2
 * feature map) without any device allocation.  The paper has no counterpart;
 * this entry point exists for callers that may not allocate device memory:
 * a host that owns every device allocation and gives a plug-in only its
 * input and output buffers, or a service running under a fixed, pre-planned
 * memory budget.  falcon_fwd's masked form draws its scratch from
 * a stream-ordered pool; this one uses a fixed array of
 * FALCON_NOALLOC_SCRATCH_BYTES inside the library instead, which every GPU
 * that loads the library holds until the process exits.  Arguments, layouts
 * and results are those of falcon_fwd with form = FALCON_MASKED.
 *  - The problem must fit: B*H*L*(window_eff*d_v + 2*d_v) floats, window_eff
 *    = window for Falcon-3/3A and 1 otherwise, at most
 *    FALCON_NOALLOC_SCRATCH_BYTES/4; larger problems return
 *    FALCON_ERR_SCRATCH and enqueue nothing.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture.
 *  - Every call on a device shares the one array: calls that may overlap on
 *    the GPU (other streams, other host threads) race and must be serialised
 *    by the caller.  No state carries over between calls (every scratch
 *    element is written before it is read).
 *  - Never calls cudaMalloc, cudaMallocAsync, cudaFree or any allocating
 *    library routine.
 */
#define FALCON_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
int falcon_fwd_masked_noalloc(falcon_variant variant, falcon_dtype dtype,
                              const void *q, const void *k, const void *v, const void *beta,
                              const float *lambda, float eps, int window,
                              int B, int H, int L, int d_k, int d_v,
                              void *out, float *final_state, cudaStream_t stream);

/*
 * falcon_device_wait_timeouts -- diagnostic: how many thread blocks of the
 * tensor-core kernels on the current device gave up on a bounded wait for
 * their own tensor-core work (about 2 s per wait) since the library was
 * loaded (each wait gives up after 4e9 SM cycles, 2-4 s).  A block that
 * gives up skips its remaining chunks, frees its tensor
 * memory and exits, so the device stays usable; its outputs are then
 * incomplete.  Synchronises with the device.  Returns 0 and writes *count.
 */
int falcon_device_wait_timeouts(unsigned int *count);

/*
 * falcon_selftest_bounded_wait -- checks on the current device that the
 * bounded waits the tensor-core kernels use give up instead of hanging: one
 * block waits on a barrier phase that nothing completes, gives up after
 * 2 * `timeout_us` thousand SM cycles (between 1 and 2 times `timeout_us`
 * microseconds at SM clocks of 1-2 GHz) and exits normally.  Synchronises; writes
 * *gave_up = 1 when the wait gave up as it must (0 would mean it saw a
 * completion, -1 that the kernel did not run).
 */
int falcon_selftest_bounded_wait(unsigned int timeout_us, int *gave_up);

/*
 * falcon_scratch_trim -- returns the unused memory of the current device's
 * scratch pool (see falcon_fwd) to the driver.  Scratch still in use by
 * enqueued work is kept.  The pool grows again on the next call that needs
 * scratch.  Returns FALCON_OK, or FALCON_ERR_LAUNCH if the CUDA call fails.
 */
int falcon_scratch_trim(void);

/* Static description of a status code (never NULL). */
const char *falcon_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* FALCON_H */
