// host.cu -- falcon_fwd_host: the forward on host buffers.  The batch is cut
// into slices; the slices' inputs go host -> device on a copy-in stream (all
// of them enqueued first), each slice's forward (every requested variant)
// runs on the caller's stream once its inputs have landed, and its outputs go
// device -> host on a copy-out stream, so that the copies of one slice
// overlap the compute and the opposite-direction copies of its neighbours.  Events order the three streams; the device buffers are one
// block: the caller's workspace (falcon_fwd_host_ws), or stream-ordered
// memory freed on the caller's stream once every copy has been joined back
// into it (falcon_fwd_host).
#include <cuda_runtime.h>

#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "../../include/falcon.h"
#include "kernels.h"

using namespace falcon;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxVariants = 6;
constexpr int kMaxSlices = 64;
std::mutex g_stream_mutex;
cudaStream_t g_copy_in[kMaxDevices], g_copy_out[kMaxDevices];
bool g_streams_made[kMaxDevices];

// The two copy streams of the current device (created once, non-blocking).
cudaError_t copy_streams(cudaStream_t *in, cudaStream_t *out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_stream_mutex);
    if (!g_streams_made[dev]) {
        e = cudaStreamCreateWithFlags(&g_copy_in[dev], cudaStreamNonBlocking);
        if (e != cudaSuccess) return e;
        e = cudaStreamCreateWithFlags(&g_copy_out[dev], cudaStreamNonBlocking);
        if (e != cudaSuccess) {
            cudaStreamDestroy(g_copy_in[dev]);
            return e;
        }
        g_streams_made[dev] = true;
    }
    *in = g_copy_in[dev];
    *out = g_copy_out[dev];
    return cudaSuccess;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool per_channel(int variant) { return variant == FALCON_F2 || variant == FALCON_F2A; }

// Default slice count: about one slice per 16 MiB of input, 1 to 8 slices.
// With copies running both ways the link, not the compute, sets the pace;
// smaller slices only add per-copy overhead (75.9 MB of input in 4 slices
// measured 2.0 ms a step, in 8 slices 2.27 ms).
int default_slices(size_t input_bytes, int B) {
    const size_t n = input_bytes >> 24;
    return static_cast<int>(std::max<size_t>(1, std::min<size_t>(n, static_cast<size_t>(std::min(B, 8)))));
}

struct Events {
    cudaEvent_t ev[2 * kMaxSlices + 3];
    int made = 0;
    cudaError_t make(int n) {
        for (; made < n; ++made) {
            const cudaError_t e = cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    // Recorded events are released once the device has passed them.
    ~Events() {
        for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);
    }
};

}  // namespace

namespace {

// Device layout of one falcon_fwd_host call: the inputs, lambda, and each
// variant's outputs and states (each array on a 256-byte boundary), then the
// workspace of the per-slice forward, which every slice and variant reuses in
// stream order.
struct HostLayout {
    size_t bq, bv, bb, bs;  // bytes per batch row
    size_t o_k, o_v, o_b, o_l, o_out[kMaxVariants], o_st[kMaxVariants];
    size_t o_inner, inner, total;
    int ns;
};

int host_layout(int n_variants, const falcon_variant *variants, falcon_form form, falcon_dtype dtype,
                falcon_pairing pairing, falcon_phi phi, int window, int B, int H, int L, int d_k, int d_v, int chunk,
                bool with_state, const bool *states, int slices, HostLayout *lay) {
    if (n_variants < 1 || n_variants > kMaxVariants || slices < 0) return FALCON_ERR_UNSUPPORTED;
    if (!variants) return FALCON_ERR_NULL;
    for (int i = 0; i < n_variants; ++i) {
        const int rc = validate_fwd(variants[i], form, dtype, pairing, phi, window, B, H, L, d_k, d_v, chunk);
        if (rc) return rc;
        if (per_channel(variants[i]) != per_channel(variants[0])) return FALCON_ERR_UNSUPPORTED;
    }
    HostLayout &y = *lay;
    const size_t es = dtype == FALCON_BF16 ? 2 : 4;
    y.bq = (size_t)H * L * d_k * es;
    y.bv = (size_t)H * L * d_v * es;
    y.bb = (size_t)H * L * (per_channel(variants[0]) ? d_v : 1) * es;
    y.bs = (size_t)H * d_v * d_k * sizeof(float);
    y.o_k = align256((size_t)B * y.bq);
    y.o_v = y.o_k + align256((size_t)B * y.bq);
    y.o_b = y.o_v + align256((size_t)B * y.bv);
    y.o_l = y.o_b + align256((size_t)B * y.bb);
    size_t total = y.o_l + align256((size_t)H * sizeof(float));
    for (int i = 0; i < n_variants; ++i) {
        y.o_out[i] = total;
        total += align256((size_t)B * y.bv);
        y.o_st[i] = total;
        if (with_state && states[i]) total += align256((size_t)B * y.bs);
    }
    int ns = slices > 0 ? std::min(slices, B) : default_slices((size_t)B * (2 * y.bq + y.bv + y.bb), B);
    y.ns = std::max(1, std::min(ns, kMaxSlices));
    int rows = 0;  // the largest slice
    for (int i = 0; i < y.ns; ++i)
        rows = std::max(rows, (int)((long long)(i + 1) * B / y.ns) - (int)((long long)i * B / y.ns));
    y.inner = 0;
    for (int i = 0; i < n_variants; ++i) {
        size_t need = 0;
        const int rc = falcon_fwd_workspace_size(variants[i], form, dtype, pairing, phi, window, rows, H, L, d_k,
                                                 d_v, chunk, &need);
        if (rc) return rc;
        y.inner = std::max(y.inner, need);
    }
    y.o_inner = total;
    y.total = total + align256(y.inner);
    return FALCON_OK;
}

int fwd_host_impl(int n_variants, const falcon_variant *variants, falcon_form form, falcon_dtype dtype,
                  falcon_pairing pairing, falcon_phi phi, const void *q, const void *k, const void *v,
                  const void *beta, const float *lambda, float eps, int window, int B, int H, int L, int d_k,
                  int d_v, int chunk, void *const *out, float *const *final_state, int slices, int ws_given,
                  void *ws_ptr, size_t ws_bytes, cudaStream_t stream) {
    bool states[kMaxVariants] = {false};
    if (n_variants >= 1 && n_variants <= kMaxVariants && final_state)
        for (int i = 0; i < n_variants; ++i) states[i] = final_state[i] != nullptr;
    HostLayout lay;
    int lrc = host_layout(n_variants, variants, form, dtype, pairing, phi, window, B, H, L, d_k, d_v, chunk,
                          final_state != nullptr, states, slices, &lay);
    if (lrc) return lrc;
    if ((size_t)B * H == 0) return FALCON_OK;
    if (L > 0) {
        if (!q || !k || !v || !beta || !lambda || !out) return FALCON_ERR_NULL;
        for (int i = 0; i < n_variants; ++i)
            if (!out[i]) return FALCON_ERR_NULL;
    }
    const size_t bq = lay.bq, bv = lay.bv, bb = lay.bb, bs = lay.bs;
    const size_t o_k = lay.o_k, o_v = lay.o_v, o_b = lay.o_b, o_l = lay.o_l;
    const size_t *o_out = lay.o_out, *o_st = lay.o_st;
    const int ns = lay.ns;
    if (ws_given && (!ws_ptr || ws_bytes < lay.total || (reinterpret_cast<uintptr_t>(ws_ptr) & 255u) != 0))
        return FALCON_ERR_WORKSPACE;

    cudaStream_t s_in, s_out;
    if (copy_streams(&s_in, &s_out) != cudaSuccess) {
        cudaGetLastError();
        return FALCON_ERR_LAUNCH;
    }
    Events evs;
    if (evs.make(2 * ns + 3) != cudaSuccess) {
        cudaGetLastError();
        return FALCON_ERR_LAUNCH;
    }
    void *ws = nullptr;
    bool owned = false;
    lrc = ws_acquire(ws_given, ws_ptr, ws_bytes, lay.total, stream, &ws, &owned);
    if (lrc) return lrc;
    uint8_t *dev = static_cast<uint8_t *>(ws);
    cudaEvent_t ev_start = evs.ev[2 * ns], ev_done = evs.ev[2 * ns + 1], ev_in_tail = evs.ev[2 * ns + 2];

    // every cuda call is checked; after the first failure nothing more is
    // computed, but the streams are still joined and the block freed
    int rc = FALCON_OK;
    auto ok = [&](cudaError_t e) {
        if (e != cudaSuccess && rc == FALCON_OK) rc = FALCON_ERR_LAUNCH;
        return rc == FALCON_OK;
    };
    auto copy = [&](void *dst, const void *src, size_t bytes, cudaStream_t s) {
        if (bytes > 0 && rc == FALCON_OK) ok(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDefault, s));
    };
    const uint8_t *hq = static_cast<const uint8_t *>(q), *hk = static_cast<const uint8_t *>(k);
    const uint8_t *hv = static_cast<const uint8_t *>(v), *hb = static_cast<const uint8_t *>(beta);

    ok(cudaEventRecord(ev_start, stream));
    if (rc == FALCON_OK) ok(cudaStreamWaitEvent(s_in, ev_start, 0));
    if (rc == FALCON_OK) ok(cudaStreamWaitEvent(s_out, ev_start, 0));
    if (L > 0) copy(dev + o_l, lambda, (size_t)H * sizeof(float), s_in);
    // every slice's inputs are enqueued first, so that the copy-in stream
    // never waits for the host to enqueue a slice's forward
    for (int i = 0; i < ns && rc == FALCON_OK; ++i) {
        const int b0 = (int)((long long)i * B / ns), b1 = (int)((long long)(i + 1) * B / ns), nb = b1 - b0;
        if (L > 0) {
            copy(dev + b0 * bq, hq + b0 * bq, nb * bq, s_in);
            copy(dev + o_k + b0 * bq, hk + b0 * bq, nb * bq, s_in);
            copy(dev + o_v + b0 * bv, hv + b0 * bv, nb * bv, s_in);
            copy(dev + o_b + b0 * bb, hb + b0 * bb, nb * bb, s_in);
        }
        if (rc == FALCON_OK) ok(cudaEventRecord(evs.ev[2 * i], s_in));
    }
    for (int i = 0; i < ns && rc == FALCON_OK; ++i) {
        const int b0 = (int)((long long)i * B / ns), b1 = (int)((long long)(i + 1) * B / ns), nb = b1 - b0;
        cudaEvent_t ev_in = evs.ev[2 * i], ev_comp = evs.ev[2 * i + 1];
        if (rc == FALCON_OK) ok(cudaStreamWaitEvent(stream, ev_in, 0));
        for (int j = 0; j < n_variants && rc == FALCON_OK; ++j) {
            const bool st = final_state && final_state[j];
            const int r = falcon_fwd_ws(variants[j], form, dtype, pairing, phi, dev + b0 * bq, dev + o_k + b0 * bq,
                                        dev + o_v + b0 * bv, dev + o_b + b0 * bb,
                                        reinterpret_cast<const float *>(dev + o_l), eps, window, nb, H, L, d_k, d_v,
                                        chunk, nullptr, nullptr, nullptr, dev + o_out[j] + b0 * bv,
                                        st ? reinterpret_cast<float *>(dev + o_st[j] + b0 * bs) : nullptr,
                                        dev + lay.o_inner, lay.inner, stream);
            if (r != FALCON_OK) rc = r;
        }
        if (rc == FALCON_OK) ok(cudaEventRecord(ev_comp, stream));
        if (rc == FALCON_OK) ok(cudaStreamWaitEvent(s_out, ev_comp, 0));
        for (int j = 0; j < n_variants; ++j) {
            if (L > 0) copy(static_cast<uint8_t *>(out[j]) + b0 * bv, dev + o_out[j] + b0 * bv, nb * bv, s_out);
            if (final_state && final_state[j])
                copy(reinterpret_cast<uint8_t *>(final_state[j]) + b0 * bs, dev + o_st[j] + b0 * bs, nb * bs, s_out);
        }
    }
    // join both copy streams back into the caller's stream, then free
    bool joined = true;
    for (cudaEvent_t ev : {ev_in_tail, ev_done}) {
        cudaStream_t from = ev == ev_done ? s_out : s_in;
        if (cudaEventRecord(ev, from) != cudaSuccess || cudaStreamWaitEvent(stream, ev, 0) != cudaSuccess)
            joined = false;
    }
    if (!joined) {
        // without the join the block cannot be freed in stream order: wait here
        cudaStreamSynchronize(s_in);
        cudaStreamSynchronize(s_out);
        cudaStreamSynchronize(stream);
        if (rc == FALCON_OK) rc = FALCON_ERR_LAUNCH;
    }
    ws_release(ws, owned, stream);
    if (rc != FALCON_OK) cudaGetLastError();
    return rc;
}

}  // namespace

extern "C" int falcon_fwd_host(int n_variants, const falcon_variant *variants, falcon_form form, falcon_dtype dtype,
                               falcon_pairing pairing, falcon_phi phi, const void *q, const void *k, const void *v,
                               const void *beta, const float *lambda, float eps, int window, int B, int H, int L,
                               int d_k, int d_v, int chunk, void *const *out, float *const *final_state, int slices,
                               cudaStream_t stream) {
    return fwd_host_impl(n_variants, variants, form, dtype, pairing, phi, q, k, v, beta, lambda, eps, window, B, H,
                         L, d_k, d_v, chunk, out, final_state, slices, 0, nullptr, 0, stream);
}

extern "C" int falcon_fwd_host_workspace_size(int n_variants, const falcon_variant *variants, falcon_form form,
                                              falcon_dtype dtype, falcon_pairing pairing, falcon_phi phi,
                                              int window, int B, int H, int L, int d_k, int d_v, int chunk,
                                              int with_state, int slices, size_t *bytes) {
    if (!bytes) return FALCON_ERR_NULL;
    *bytes = 0;
    bool states[kMaxVariants];
    for (int i = 0; i < kMaxVariants; ++i) states[i] = with_state != 0;
    HostLayout lay;
    const int rc = host_layout(n_variants, variants, form, dtype, pairing, phi, window, B, H, L, d_k, d_v, chunk,
                               with_state != 0, states, slices, &lay);
    if (rc) return rc;
    *bytes = (size_t)B * H == 0 ? 0 : lay.total;
    return FALCON_OK;
}

extern "C" int falcon_fwd_host_ws(int n_variants, const falcon_variant *variants, falcon_form form,
                                  falcon_dtype dtype, falcon_pairing pairing, falcon_phi phi, const void *q,
                                  const void *k, const void *v, const void *beta, const float *lambda, float eps,
                                  int window, int B, int H, int L, int d_k, int d_v, int chunk, void *const *out,
                                  float *const *final_state, int slices, void *workspace, size_t workspace_bytes,
                                  cudaStream_t stream) {
    return fwd_host_impl(n_variants, variants, form, dtype, pairing, phi, q, k, v, beta, lambda, eps, window, B, H,
                         L, d_k, d_v, chunk, out, final_state, slices, 1, workspace, workspace_bytes, stream);
}
