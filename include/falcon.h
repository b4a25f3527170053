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
 *  - Memory: the *_ws entry points run in a workspace the caller allocates
 *    (its size from the matching *_workspace_size query, 256-byte aligned)
 *    and allocate nothing.  The other entry points that need a workspace
 *    draw it stream-ordered (cudaMallocAsync) from the device's current
 *    memory pool and free it on the same stream; the library keeps no pool
 *    of its own, so what stays mapped between calls is the pool owner's
 *    choice (its release threshold).  Library-owned device memory is limited
 *    to a few diagnostic counters and the fixed array of
 *    falcon_fwd_masked_noalloc.
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
#include <stddef.h>

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
    FALCON_ERR_CHUNK = -4,       /* chunk not in {16,32,64} (or 128 where taken)     */
    FALCON_ERR_WINDOW = -6,      /* window < 1 or > 8 for Falcon-3/3A               */
    FALCON_ERR_LAUNCH = -7,      /* a kernel launch failed (cudaGetLastError)       */
    FALCON_ERR_ALLOC = -8,       /* stream-ordered scratch allocation failed        */
    FALCON_ERR_UNSUPPORTED = -9, /* combination not supported (e.g. pairing+decode) */
    FALCON_ERR_SCRATCH = -10,    /* problem needs more than the fixed scratch of
                                    falcon_fwd_masked_noalloc                      */
    FALCON_ERR_WORKSPACE = -11   /* the caller's workspace is NULL, smaller than its
                                    size query or not 256-byte aligned              */
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
 *   chunk    chunk length for FALCON_CHUNK (16, 32 or 64; 128 for Falcon-1/1A
 *            with bf16 inputs and d_k = d_v in {32, 64}); ignored otherwise
 *   out      [B,H,L,d_v] dtype     o_t = S_t q_t (written)
 *   final_state [B,H,d_v,d_k] fp32 S_L (written), may be NULL
 * S_0 = 0.  L may be 0 (out untouched, final_state zeroed) and need not be a
 * multiple of `chunk`.  Three paths need a workspace, drawn stream-ordered
 * on `stream` from the device's current memory pool (FALCON_ERR_ALLOC if
 * that fails; falcon_fwd_ws takes it from the caller instead):
 * FALCON_MASKED (about B*H*L*(window*d_v+2*d_v) floats on the CUDA cores;
 * Falcon-1/1A with bf16 inputs, d_k = d_v = 64 and L <= 65536 run on the
 * tensor cores, keeping 16 KiB per (b, h, 64-token block), and take the
 * larger of the two so that misaligned pointers can fall back), the bf16
 * tensor-core chunk path of Falcon-1/1A with d_k = d_v = 64 and chunk 64
 * (32 KiB + 4 bytes per (b, h, chunk): the chunk-local results that the
 * second of its two kernels chains across chunks) and that of Falcon-2A
 * with d_k = d_v = 128 and chunk 64 (96.5 KiB per (b, h, chunk)).
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
 * falcon_fwd_workspace_size -- bytes of device workspace a forward with
 * these arguments needs (0 when its kernels need none).  A host-only query:
 * nothing is enqueued.  Argument errors as in falcon_fwd_ex; *bytes is 0
 * then.
 */
int falcon_fwd_workspace_size(falcon_variant variant, falcon_form form, falcon_dtype dtype,
                              falcon_pairing pairing, falcon_phi phi, int window,
                              int B, int H, int L, int d_k, int d_v, int chunk, size_t *bytes);

/*
 * falcon_fwd_ws -- the forward (every form, pairing and feature map, with or
 * without the carry of falcon_fwd_carry_ex) in a workspace the caller owns:
 * the library allocates nothing.
 *   workspace        device memory, 256-byte aligned, at least the bytes
 *                    falcon_fwd_workspace_size gives for the same arguments
 *                    (may be NULL when that is 0); its contents on entry do
 *                    not matter, and it may be reused once `stream` has
 *                    passed the call's work
 *   workspace_bytes  its size; too small, misaligned or NULL when needed:
 *                    FALCON_ERR_WORKSPACE, nothing enqueued
 *   initial_state, x_prev, win   the carry of falcon_fwd_carry_ex, or NULL
 * Every other argument, and the results, as in falcon_fwd_carry_ex.
 */
int falcon_fwd_ws(falcon_variant variant, falcon_form form, falcon_dtype dtype,
                  falcon_pairing pairing, falcon_phi phi,
                  const void *q, const void *k, const void *v, const void *beta,
                  const float *lambda, float eps, int window,
                  int B, int H, int L, int d_k, int d_v, int chunk,
                  const float *initial_state, const float *x_prev, const float *win,
                  void *out, float *final_state, void *workspace, size_t workspace_bytes,
                  cudaStream_t stream);

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
 *                library choose (about one per 16 MiB of input, at most 8)
 *   every other argument as in falcon_fwd_ex.
 * The call returns once the work is enqueued.  The host buffers must stay
 * valid, and the inputs unchanged, until `stream` has passed the call's work;
 * the outputs are complete then (cudaStreamSynchronize(stream)).  The device
 * buffers (inputs, lambda, outputs and states: about the inputs' size plus
 * n_variants times the outputs', and the per-slice forward's workspace) are
 * one stream-ordered block from the device's current memory pool, freed on
 * `stream` at the end of the call's work (falcon_fwd_host_ws: the caller's
 * block instead).  Argument errors return before anything is enqueued.  An error after the first copy
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
 * falcon_fwd_host_workspace_size / falcon_fwd_host_ws -- falcon_fwd_host in
 * a device workspace the caller owns (256-byte aligned; the library then
 * allocates nothing).  The size depends on the arguments of the size query,
 * with_state != 0 when final states are wanted for every variant (a call
 * that wants fewer needs no more).  Too small, misaligned or NULL:
 * FALCON_ERR_WORKSPACE, nothing enqueued.  Everything else as falcon_fwd_host.
 */
int falcon_fwd_host_workspace_size(int n_variants, const falcon_variant *variants, falcon_form form,
                                   falcon_dtype dtype, falcon_pairing pairing, falcon_phi phi, int window,
                                   int B, int H, int L, int d_k, int d_v, int chunk, int with_state, int slices,
                                   size_t *bytes);
int falcon_fwd_host_ws(int n_variants, const falcon_variant *variants, falcon_form form, falcon_dtype dtype,
                       falcon_pairing pairing, falcon_phi phi,
                       const void *q, const void *k, const void *v, const void *beta,
                       const float *lambda, float eps, int window,
                       int B, int H, int L, int d_k, int d_v, int chunk,
                       void *const *out, float *const *final_state, int slices,
                       void *workspace, size_t workspace_bytes, cudaStream_t stream);

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
 * falcon_fwd_carry_ex -- falcon_fwd_carry with the pairing and the feature
 * map selectable.  Under the same-step pair ([EXPL] 核心方法 1, warning
 * paragraph) the segment's first sample is (phi(k_1), v_1) of the segment
 * itself, so x_prev is not read (it may be NULL); `win` holds the window-1
 * same-step samples before the segment, as falcon_decode_carry_from_prefill_ex
 * and falcon_decode_step_ex leave them.  phi applies to the segment's keys;
 * carried samples are used as given.
 */
int falcon_fwd_carry_ex(falcon_variant variant, falcon_form form, falcon_dtype dtype,
                        falcon_pairing pairing, falcon_phi phi,
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
 * Workspace: (2 L d + L + 5 L c) floats per (b,h), c = 1 or d_v, plus
 * (ceil(L/32) + 32) d^2 for the regression family (and under 64 floats of
 * alignment), stream-ordered from the device's current memory pool
 * (FALCON_ERR_ALLOC if that fails).  Errors as in falcon_fwd.
 */
int falcon_bwd(falcon_variant variant, falcon_dtype dtype, falcon_pairing pairing, falcon_phi phi,
               const void *q, const void *k, const void *v, const void *beta, const float *lambda, float eps,
               int window, int B, int H, int L, int d_k, int d_v, const void *dout, const float *dstate,
               float *dq, float *dk, float *dv, float *dbeta, float *dlambda, cudaStream_t stream);

/*
 * falcon_bwd_ex -- falcon_bwd with the form of the forward whose derivative
 * is taken.
 *   form  FALCON_RECURRENT: as falcon_bwd (every variant and shape above).
 *         FALCON_CHUNK: the chunk-parallel backward ([NEWS] 02 (2), the
 *         paragraph after the variant list: every variant trains in the
 *         chunk-parallel form), for Falcon-1 and Falcon-1A with bf16 inputs,
 *         d_k = d_v = 64 and chunk 64 (FALCON_ERR_UNSUPPORTED for other
 *         variants, dtypes or sizes; FALCON_ERR_CHUNK for another chunk; the
 *         recurrent form covers them).  The chunk-parallel forward (tensor
 *         cores) runs first and keeps the state entering every chunk; a
 *         reverse chain per head then carries dL/dS across chunk boundaries,
 *         G_c = g_C G_{c+1} - G_{c+1} Phi'_c^T + dO_c^T Qt_c, with the
 *         forward's per-chunk operators; every chunk's gradients (through
 *         the steps, the decays and the key normalisation too) then come at
 *         once from its inputs, its entering state and G_{c+1} (matrix form,
 *         TF32 tensor-core products with truncated operands, fp32
 *         accumulation; dlambda summed with float atomics, so its last bits
 *         may differ between runs).  q, k, v, dout, dq, dk and dv must be
 *         16-byte aligned (FALCON_ERR_UNSUPPORTED otherwise).
 *         FALCON_MASKED: FALCON_ERR_UNSUPPORTED.
 *   chunk 64 for FALCON_CHUNK; ignored otherwise
 * Every other argument and the results as in falcon_bwd; the workspace is
 * drawn stream-ordered from the device's current memory pool.
 */
int falcon_bwd_ex(falcon_variant variant, falcon_form form, falcon_dtype dtype, falcon_pairing pairing,
                  falcon_phi phi, const void *q, const void *k, const void *v, const void *beta,
                  const float *lambda, float eps, int window, int B, int H, int L, int d_k, int d_v, int chunk,
                  const void *dout, const float *dstate, float *dq, float *dk, float *dv, float *dbeta,
                  float *dlambda, cudaStream_t stream);

/*
 * falcon_bwd_workspace_size / falcon_bwd_ws -- falcon_bwd_ex in a workspace
 * the caller owns (256-byte aligned, at least the queried bytes; the library
 * then allocates nothing; FALCON_ERR_WORKSPACE when it is too small,
 * misaligned or NULL).  Everything else as falcon_bwd_ex.
 */
int falcon_bwd_workspace_size(falcon_variant variant, falcon_form form, falcon_dtype dtype, falcon_pairing pairing,
                              falcon_phi phi, int window, int B, int H, int L, int d_k, int d_v, int chunk,
                              size_t *bytes);
int falcon_bwd_ws(falcon_variant variant, falcon_form form, falcon_dtype dtype, falcon_pairing pairing,
                  falcon_phi phi, const void *q, const void *k, const void *v, const void *beta,
                  const float *lambda, float eps, int window, int B, int H, int L, int d_k, int d_v, int chunk,
                  const void *dout, const float *dstate, float *dq, float *dk, float *dv, float *dbeta,
                  float *dlambda, void *workspace, size_t workspace_bytes, cudaStream_t stream);

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
 * falcon_decode_step_ex -- falcon_decode_step with the pairing selectable.
 * Under the same-step pair ([EXPL] 核心方法 1, warning paragraph) the
 * step's sample is (phi(k_t), v_t): x_prev is not read and may be NULL (when
 * given it is still set to phi(k_t)); the window carry then holds the
 * previous window-1 same-step samples and receives (phi(k_t), v_t).
 */
int falcon_decode_step_ex(falcon_variant variant, falcon_dtype dtype, falcon_pairing pairing,
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
 * falcon_decode_carry_from_prefill_ex -- the same with the pairing
 * selectable.  Under the same-step pair the window holds the samples
 * (phi(k_i), v_i), i = L-window+2 .. L (zeros for i < 1), and x_prev (which
 * the same-step decode does not read) may be NULL; when given it is phi(k_L).
 */
int falcon_decode_carry_from_prefill_ex(falcon_variant variant, falcon_dtype dtype, falcon_pairing pairing,
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
 * that loads the library holds until the process exits.  Arguments and
 * layouts are those of falcon_fwd with form = FALCON_MASKED; it always runs
 * the CUDA-core masked kernel, so its results are bit for bit those of
 * falcon_fwd's masked form wherever that form runs on the CUDA cores too
 * (every shape but Falcon-1/1A with bf16 inputs and d_k = d_v = 64, which
 * falcon_fwd runs on the tensor cores: equal there within rounding).
 *  - The problem must fit: B*H*L*(window_eff*d_v + 2*d_v) floats, window_eff
 *    = window for Falcon-3/3A and 1 otherwise, at most
 *    FALCON_NOALLOC_SCRATCH_BYTES/4; larger problems return
 *    FALCON_ERR_SCRATCH and enqueue nothing.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture.  With lazy module loading the array itself is
 *    materialised when the library's device code is first loaded on that
 *    device, possibly during that first call: make it part of set-up, before
 *    a memory budget is fixed (a lookup that runs out of memory returns
 *    FALCON_ERR_ALLOC).
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
 * current memory pool, from which the allocating entry points draw their
 * workspace (see falcon_fwd), to the driver (cudaMemPoolTrimTo(pool, 0)).
 * Memory still in use by enqueued work is kept.  Returns FALCON_OK, or
 * FALCON_ERR_LAUNCH if the CUDA call fails.
 */
int falcon_scratch_trim(void);

/* Static description of a status code (never NULL). */
const char *falcon_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* FALCON_H */
