// host.cu -- falcon_fwd_host: the forward on host buffers.  The batch is cut
// into slices; each slice's inputs go host -> device on a copy-in stream, its
// forward (every requested variant) runs on the caller's stream, and its
// outputs go device -> host on a copy-out stream, so that the copies of one
// slice overlap the compute and the opposite-direction copies of its
// neighbours.  Events order the three streams; the device buffers are one
// stream-ordered block of the library's pool, freed on the caller's stream
// once every copy has been joined back into it.
#include <cuda_runtime.h>

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

// Default slice count: about one slice per 4 MiB of input, 1 to 8 slices.
int default_slices(size_t input_bytes, int B) {
    const size_t n = input_bytes >> 22;
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

extern "C" int falcon_fwd_host(int n_variants, const falcon_variant *variants, falcon_form form, falcon_dtype dtype,
                               falcon_pairing pairing, falcon_phi phi, const void *q, const void *k, const void *v,
                               const void *beta, const float *lambda, float eps, int window, int B, int H, int L,
                               int d_k, int d_v, int chunk, void *const *out, float *const *final_state, int slices,
                               cudaStream_t stream) {
    if (n_variants < 1 || n_variants > kMaxVariants || slices < 0) return FALCON_ERR_UNSUPPORTED;
    if (!variants) return FALCON_ERR_NULL;
    for (int i = 0; i < n_variants; ++i) {
        const int rc = validate_fwd(variants[i], form, dtype, pairing, phi, window, B, H, L, d_k, d_v, chunk);
        if (rc) return rc;
        if (per_channel(variants[i]) != per_channel(variants[0])) return FALCON_ERR_UNSUPPORTED;
    }
    if ((size_t)B * H == 0) return FALCON_OK;
    if (L > 0) {
        if (!q || !k || !v || !beta || !lambda || !out) return FALCON_ERR_NULL;
        for (int i = 0; i < n_variants; ++i)
            if (!out[i]) return FALCON_ERR_NULL;
    }

    // bytes per batch row of every array, and the device block's layout
    const size_t es = dtype == FALCON_BF16 ? 2 : 4;
    const size_t bq = (size_t)H * L * d_k * es, bv = (size_t)H * L * d_v * es;
    const size_t bb = (size_t)H * L * (per_channel(variants[0]) ? d_v : 1) * es;
    const size_t bs = (size_t)H * d_v * d_k * sizeof(float);
    const size_t o_k = align256((size_t)B * bq), o_v = o_k + align256((size_t)B * bq);
    const size_t o_b = o_v + align256((size_t)B * bv), o_l = o_b + align256((size_t)B * bb);
    size_t o_out[kMaxVariants], o_st[kMaxVariants];
    size_t total = o_l + align256((size_t)H * sizeof(float));
    for (int i = 0; i < n_variants; ++i) {
        o_out[i] = total;
        total += align256((size_t)B * bv);
        o_st[i] = total;
        if (final_state && final_state[i]) total += align256((size_t)B * bs);
    }
    int ns = slices > 0 ? std::min(slices, B) : default_slices((size_t)B * (2 * bq + bv + bb), B);
    ns = std::min(ns, kMaxSlices);

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
    if (scratch_alloc(&ws, total, stream) != cudaSuccess) {
        cudaGetLastError();
        return FALCON_ERR_ALLOC;
    }
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
    for (int i = 0; i < ns && rc == FALCON_OK; ++i) {
        const int b0 = (int)((long long)i * B / ns), b1 = (int)((long long)(i + 1) * B / ns), nb = b1 - b0;
        cudaEvent_t ev_in = evs.ev[2 * i], ev_comp = evs.ev[2 * i + 1];
        if (L > 0) {
            copy(dev + b0 * bq, hq + b0 * bq, nb * bq, s_in);
            copy(dev + o_k + b0 * bq, hk + b0 * bq, nb * bq, s_in);
            copy(dev + o_v + b0 * bv, hv + b0 * bv, nb * bv, s_in);
            copy(dev + o_b + b0 * bb, hb + b0 * bb, nb * bb, s_in);
        }
        if (rc == FALCON_OK) ok(cudaEventRecord(ev_in, s_in));
        if (rc == FALCON_OK) ok(cudaStreamWaitEvent(stream, ev_in, 0));
        for (int j = 0; j < n_variants && rc == FALCON_OK; ++j) {
            const bool st = final_state && final_state[j];
            const int r = falcon_fwd_ex(variants[j], form, dtype, pairing, phi, dev + b0 * bq, dev + o_k + b0 * bq,
                                        dev + o_v + b0 * bv, dev + o_b + b0 * bb,
                                        reinterpret_cast<const float *>(dev + o_l), eps, window, nb, H, L, d_k, d_v,
                                        chunk, dev + o_out[j] + b0 * bv,
                                        st ? reinterpret_cast<float *>(dev + o_st[j] + b0 * bs) : nullptr, stream);
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
    scratch_free(ws, stream);
    if (rc != FALCON_OK) cudaGetLastError();
    return rc;
}
