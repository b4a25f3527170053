// kernels.h -- internal launch interface between the C ABI (api.cu) and the
// kernels (the parameter blocks are in params.h).  Not installed; the public
// boundary is include/falcon.h.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "params.h"
#include "params_bwd.h"

namespace falcon {

template <typename T> int launch_recurrent(const FwdParams &p, cudaStream_t s);
template <typename T> int launch_span_chunk(const FwdParams &p, cudaStream_t s);
template <typename T> int launch_span_masked(const FwdParams &p, cudaStream_t s);
// bf16 chunk-parallel forward on tcgen05 as two kernels (every chunk's local
// part at once, then the per-head chain) over a stream-ordered workspace;
// returns 1 (nothing launched) for shapes it does not cover, so the caller
// falls back to the span kernel, and FALCON_ERR_ALLOC when the workspace
// cannot be had.
int launch_split_chunk(const FwdParams &p, cudaStream_t s);
// true when the shape is one the split kernels take (pointer alignment aside)
bool split_chunk_covers(const FwdParams &p);
// the workspace of the call: the per-chunk images and g_C (the backward
// keeps them, through split_chunk_images_ws_bytes, for its reverse chain)
size_t split_chunk_ws_bytes(const FwdParams &p);
size_t split_chunk_images_ws_bytes(const FwdParams &p);
// Number of tensor-core thread blocks that gave up on a bounded wait.
unsigned int split_wait_timeouts();
unsigned int decode_wait_timeouts();
// bf16 Falcon-2A chunk-parallel forward, d_k = d_v = 128, chunk 64, on
// tcgen05 (dS per chunk, state scan, outputs); returns 1 for shapes it does
// not cover.
int launch_pc_chunk(const FwdParams &p, cudaStream_t s);
bool pc_chunk_covers(const FwdParams &p);
size_t pc_chunk_ws_bytes(const FwdParams &p);
unsigned int pc_wait_timeouts();
// bf16 Falcon-2 chunk-parallel forward, d_k = d_v = 128, chunk 64, on tcgen05
// (one block per head, per-channel forward substitution); returns 1 for
// shapes it does not cover.
int launch_f2_chunk(const FwdParams &p, cudaStream_t s);
// Falcon-3 / Falcon-3A (bf16, d = 64, chunk 64, window 2-4): per-chunk
// images, then the split path's chain kernel on them
bool w_local_covers(const FwdParams &p);
size_t w_local_ws_bytes(const FwdParams &p);
// the chain kernel of the split path over per-chunk images [-Phi'^T (the
// regression family) | Qt | O0^T | B] (32 KB each, per (b*H + h, chunk)) and
// g_C, in stream order after the kernel that wrote them
int launch_chain_images(const FwdParams &p, const uint8_t *img, const float *gc, cudaStream_t s);
unsigned int f2_wait_timeouts();
// bf16 Falcon-3/3A chunk-parallel forward, d_k = d_v = 64, chunk 64, window
// 2..4, on tcgen05 (one block per head, the windowed system in token order);
// returns 1 for shapes it does not cover.
int launch_w_chunk(const FwdParams &p, cudaStream_t s);
unsigned int w_wait_timeouts();
// bf16 Falcon-1/1A chunk-parallel forward, d_k = d_v = 64, chunk 16, 32 or
// 128 (TF32 warp MMAs, one block per head); returns 1 for shapes it does not
// cover.
int launch_seq_chunk(const FwdParams &p, cudaStream_t s);
bool seq_chunk_covers(const FwdParams &p);
template <typename T> int launch_decode(const DecodeParams &p, cudaStream_t s);
// Backward pass of every variant (recurrent form, fp32), d_k = d_v in
// {32, 64, 128}; the arguments are validated by the caller.
template <typename T> int launch_bwd(const BwdParams &p, cudaStream_t s);
size_t bwd_ws_bytes(const BwdParams &p);
// The chunk-parallel backward (k_bwd_chunk.cu): the shapes it takes, its
// workspace, and its launch (forward with chunk states, reverse chain,
// per-chunk gradients: dq, dk, dv, dbeta and dlambda whole).
bool bwd_chunk_covers(const BwdParams &p);
size_t bwd_chunk_ws_bytes(const BwdParams &p);
int launch_bwd_chunk(const BwdParams &p, void *ws, cudaStream_t s);
template <typename T> int launch_carry(const CarryParams &p, cudaStream_t s);

// Stream-ordered scratch from the device's current memory pool
// (cudaMallocAsync); scratch_trim hands that pool's unused memory back.
cudaError_t scratch_alloc(void **ptr, size_t bytes, cudaStream_t s);
cudaError_t scratch_free(void *ptr, cudaStream_t s);
cudaError_t scratch_trim();

// Status codes the launchers return (the values of include/falcon.h).
constexpr int kErrAlloc = -8;
constexpr int kErrWorkspace = -11;
// The workspace of one call: the caller's block when `given` (checked to be
// at least `need` bytes and 256-byte aligned, else kErrWorkspace; nothing is
// allocated), else `need` bytes drawn stream-ordered on `s` (kErrAlloc if
// that fails).  *owned tells ws_release whether to free it on `s`.
int ws_acquire(int given, void *given_ptr, size_t given_bytes, size_t need, cudaStream_t s, void **ptr,
               bool *owned);
void ws_release(void *ptr, bool owned, cudaStream_t s);

// The argument checks of falcon_fwd_ex (FALCON_OK or the status it returns
// for them); nothing is enqueued.
int validate_fwd(int variant, int form, int dtype, int pairing, int phi, int window, int B, int H, int L, int d_k,
                 int d_v, int chunk);

// Scratch sizes (floats) of the masked-parallel form.
// The masked-parallel form of Falcon-1/1A (bf16, d = 64) on the tensor cores
// (k_masked_tc.cu): covered shapes, workspace, launch (1: not covered or
// misaligned pointers, the CUDA-core kernel takes it), give-ups of its waits.
bool masked_tc_covers(const FwdParams &p);
size_t masked_tc_ws_bytes(const FwdParams &p);
int launch_masked_tc(const FwdParams &p, void *ws, cudaStream_t s);
unsigned int masked_wait_timeouts();
size_t masked_ws_r_floats(const FwdParams &p);
size_t masked_ws_eg_floats(const FwdParams &p);

}  // namespace falcon
