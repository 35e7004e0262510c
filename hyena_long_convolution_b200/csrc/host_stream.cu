// host_stream.cu -- the long modal conv and the short FIR over inputs and
// outputs in host memory.  The sequence is streamed through two device
// staging slots in chunks, with the carried state (the modal state, or the
// FIR window) passed from chunk to chunk (Evo2-7B-262K model card, "Custom
// cache"; turboquant-evo2-int4 card, chunked prefill): while the scan of
// chunk i runs on the caller's stream, chunk i+1 is copied host->device on one
// copy stream and chunk i-1's output device->host on another, so the host
// link carries both directions at once.  Chunks of whole 128-token units (any
// chunk for the FIR) make the result equal to the single pass bit for bit.
#include <mutex>

#include "hyena_internal.h"

namespace {

constexpr int kSlots = 2;
constexpr int kMaxDevices = 64;

struct CopyStreams {
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, done = nullptr;
    cudaEvent_t loaded[kSlots] = {}, scanned[kSlots] = {}, stored[kSlots] = {};
};

std::mutex g_mutex;  // one enqueue sequence at a time (the events are shared)
CopyStreams g_streams[kMaxDevices];
bool g_ready[kMaxDevices] = {};

cudaError_t copy_streams(int dev, CopyStreams **out)
{
    if (!g_ready[dev]) {
        CopyStreams &c = g_streams[dev];
        cudaError_t e = cudaStreamCreateWithFlags(&c.h2d, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c.d2h, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.start, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.done, cudaEventDisableTiming);
        for (int s = 0; s < kSlots && e == cudaSuccess; ++s) {
            e = cudaEventCreateWithFlags(&c.loaded[s], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.scanned[s], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.stored[s], cudaEventDisableTiming);
        }
        if (e != cudaSuccess) return e;
        g_ready[dev] = true;
    }
    *out = &g_streams[dev];
    return cudaSuccess;
}

size_t align256(size_t x)
{
    return (x + 255) & ~static_cast<size_t>(255);
}

struct HostLayout {
    size_t modal, tensor, state, total;  // bytes
};

HostLayout host_layout(int B, int D, int N, int chunk)
{
    HostLayout h{};
    h.modal = align256(hyena_modal_long_conv_workspace_size(B, D, N));
    h.tensor = align256(static_cast<size_t>(B) * chunk * D * sizeof(hyena_bf16_t));
    h.state = align256(static_cast<size_t>(B) * D * N * sizeof(float));
    h.total = h.modal + static_cast<size_t>(kSlots) * 4 * h.tensor + h.state;
    return h;
}

// Rows t0 .. t0+rows-1 of every batch row of a host tensor (row stride ld)
// to / from a packed device slot [B][rows][D].
cudaError_t copy_rows(void *dst, size_t dpitch, const void *src, size_t spitch, int D, int rows, int B,
                      size_t dst_batch, size_t src_batch, cudaMemcpyKind kind, cudaStream_t st)
{
    for (int b = 0; b < B; ++b) {
        const cudaError_t e = cudaMemcpy2DAsync(static_cast<char *>(dst) + b * dst_batch, dpitch,
                                                static_cast<const char *>(src) + b * src_batch, spitch,
                                                static_cast<size_t>(D) * sizeof(hyena_bf16_t), rows, kind, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// The chunk loop shared by both operators.  `scan(i, last, x1, x2, x3, y,
// rows)` enqueues the computation of chunk i on `st` from the packed slot
// tensors ([B][rows][D], row stride D) and returns its status.
template <class Scan>
hyena_status_t stream_chunks(const hyena_bf16_t *x1, const hyena_bf16_t *x2, const hyena_bf16_t *x3, int64_t ld_x,
                             hyena_bf16_t *y, int64_t ld_y, int B, int L, int D, int chunk, unsigned char *slots,
                             size_t tensor_bytes, cudaStream_t st, const char *what, Scan scan)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        hyena::record_cuda_error(e, "cudaGetDevice");
        return HYENA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return HYENA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    CopyStreams *cs = nullptr;
    e = copy_streams(dev, &cs);
    if (e != cudaSuccess) {
        hyena::record_cuda_error(e, what);
        return HYENA_ERR_CUDA;
    }
    auto slot_tensor = [&](int s, int k) {
        return reinterpret_cast<hyena_bf16_t *>(slots + (static_cast<size_t>(s) * 4 + k) * tensor_bytes);
    };
    int launches = 0;
#define HS_TRY(expr)                                    \
    do {                                                \
        const cudaError_t e_ = (expr);                  \
        if (e_ != cudaSuccess) {                        \
            hyena::record_cuda_error(e_, what);         \
            return HYENA_ERR_CUDA;                      \
        }                                               \
    } while (0)
    // Everything before this call on the caller's stream (inputs, parameters,
    // state) comes first; the copy streams start from there.
    HS_TRY(cudaEventRecord(cs->start, st));
    HS_TRY(cudaStreamWaitEvent(cs->h2d, cs->start, 0));
    HS_TRY(cudaStreamWaitEvent(cs->d2h, cs->start, 0));
    const int nchunks = (L + chunk - 1) / chunk;
    const size_t dpitch = static_cast<size_t>(D) * sizeof(hyena_bf16_t);
    const size_t xpitch = static_cast<size_t>(ld_x) * sizeof(hyena_bf16_t);
    const size_t ypitch = static_cast<size_t>(ld_y) * sizeof(hyena_bf16_t);
    const hyena_bf16_t *xs[3] = {x1, x2, x3};
    for (int i = 0; i < nchunks; ++i) {
        const int s = i % kSlots;
        const int t0 = i * chunk;
        const int rows = (L - t0) < chunk ? (L - t0) : chunk;
        const size_t dbatch = static_cast<size_t>(rows) * dpitch;  // the slot holds [B][rows][D]
        // chunk i's inputs, once chunk i-2 (same slot) has been scanned
        if (i >= kSlots) HS_TRY(cudaStreamWaitEvent(cs->h2d, cs->scanned[s], 0));
        for (int k = 0; k < 3; ++k)
            HS_TRY(copy_rows(slot_tensor(s, k), dpitch, xs[k] + static_cast<size_t>(t0) * ld_x, xpitch, D, rows, B,
                             dbatch, static_cast<size_t>(L) * xpitch, cudaMemcpyHostToDevice, cs->h2d));
        HS_TRY(cudaEventRecord(cs->loaded[s], cs->h2d));
        // the scan of chunk i on the caller's stream, once its rows have
        // landed and chunk i-2's output has left the slot
        HS_TRY(cudaStreamWaitEvent(st, cs->loaded[s], 0));
        if (i >= kSlots) HS_TRY(cudaStreamWaitEvent(st, cs->stored[s], 0));
        const hyena_status_t r = scan(i, i == nchunks - 1, slot_tensor(s, 0), slot_tensor(s, 1), slot_tensor(s, 2),
                                      slot_tensor(s, 3), rows);
        if (r != HYENA_OK) return r;
        launches += hyena_last_launch_count();
        HS_TRY(cudaEventRecord(cs->scanned[s], st));
        // chunk i's output back to the host
        HS_TRY(cudaStreamWaitEvent(cs->d2h, cs->scanned[s], 0));
        HS_TRY(copy_rows(y + static_cast<size_t>(t0) * ld_y, ypitch, slot_tensor(s, 3), dpitch, D, rows, B,
                         static_cast<size_t>(L) * ypitch, dbatch, cudaMemcpyDeviceToHost, cs->d2h));
        HS_TRY(cudaEventRecord(cs->stored[s], cs->d2h));
    }
    // the caller's stream sees the last output on the host
    HS_TRY(cudaEventRecord(cs->done, cs->d2h));
    HS_TRY(cudaStreamWaitEvent(st, cs->done, 0));
#undef HS_TRY
    hyena::set_last_launches(launches);
    return HYENA_OK;
}

}  // namespace

extern "C" size_t hyena_modal_host_workspace_size(int B, int D, int N, int chunk)
{
    if (B < 1 || D < 1 || chunk < hyena::MT || chunk % hyena::MT != 0) return 0;
    if (hyena_modal_long_conv_workspace_size(B, D, N) == 0) return 0;
    return host_layout(B, D, N, chunk).total;
}

extern "C" hyena_status_t hyena_modal_long_conv_host(const hyena_bf16_t *x1, const hyena_bf16_t *x2,
                                                     const hyena_bf16_t *x3, int64_t ld_x,
                                                     const float *log_poles, const float *residues,
                                                     const float *Dskip, hyena_bf16_t *y, int64_t ld_y,
                                                     const float *state_in, float *state_out, int B, int L,
                                                     int D, int N, int chunk, void *workspace,
                                                     size_t workspace_bytes, void *stream)
{
    if (B < 1 || L < 0 || D < 1 || N < 1) return HYENA_ERR_INVALID_ARG;
    if (N > HYENA_MAX_MODES) return HYENA_ERR_UNSUPPORTED;
    if (chunk < hyena::MT || chunk % hyena::MT != 0) return HYENA_ERR_INVALID_ARG;
    if (L > 0 && (!x1 || !x2 || !x3 || !y)) return HYENA_ERR_INVALID_ARG;
    if (ld_x < D || ld_y < D) return HYENA_ERR_INVALID_ARG;
    if (D % 8) return HYENA_ERR_ALIGNMENT;
    const HostLayout lay = host_layout(B, D, N, chunk);
    if (workspace == nullptr || workspace_bytes < lay.total) return HYENA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return HYENA_ERR_ALIGNMENT;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    void *modal_ws = ws;
    unsigned char *slots = ws + lay.modal;
    float *carry = reinterpret_cast<float *>(slots + static_cast<size_t>(kSlots) * 4 * lay.tensor);
    if (L == 0)
        return hyena_modal_long_conv(nullptr, nullptr, nullptr, D, log_poles, residues, Dskip, nullptr, D,
                                     state_in, state_out, B, 0, D, N, modal_ws, lay.modal, stream);
    return stream_chunks(x1, x2, x3, ld_x, y, ld_y, B, L, D, chunk, slots, lay.tensor, static_cast<cudaStream_t>(stream),
                         "host-buffer modal conv",
                         [&](int i, bool last, const hyena_bf16_t *c1, const hyena_bf16_t *c2, const hyena_bf16_t *c3,
                             hyena_bf16_t *cy, int rows) {
                             // the first chunk synthesises the filter, the others reuse its table
                             if (i == 0)
                                 return hyena_modal_long_conv(c1, c2, c3, D, log_poles, residues, Dskip, cy, D,
                                                              state_in, last ? state_out : carry, B, rows, D, N,
                                                              modal_ws, lay.modal, stream);
                             return hyena_modal_long_conv_prepared(c1, c2, c3, D, cy, D, carry, last ? state_out : carry,
                                                                   B, rows, D, N, modal_ws, lay.modal, stream);
                         });
}

extern "C" size_t hyena_short_host_workspace_size(int B, int D, int K, int chunk)
{
    if (B < 1 || D < 1 || K < 1 || K > HYENA_MAX_TAPS || chunk < 1) return 0;
    const size_t tensor = align256(static_cast<size_t>(B) * chunk * D * sizeof(hyena_bf16_t));
    const size_t window = align256(static_cast<size_t>(B) * (K > 1 ? K - 1 : 1) * D * sizeof(float));
    return static_cast<size_t>(kSlots) * 4 * tensor + window;
}

extern "C" hyena_status_t hyena_short_conv_host(const hyena_bf16_t *x1, const hyena_bf16_t *x2,
                                                const hyena_bf16_t *x3, int64_t ld_x, const hyena_bf16_t *taps,
                                                const float *Dskip, hyena_bf16_t *y, int64_t ld_y,
                                                const float *hist_in, float *hist_out, int B, int L, int D, int K,
                                                int chunk, void *workspace, size_t workspace_bytes, void *stream)
{
    if (B < 1 || L < 0 || D < 1 || K < 1 || chunk < 1) return HYENA_ERR_INVALID_ARG;
    if (K > HYENA_MAX_TAPS) return HYENA_ERR_UNSUPPORTED;
    if (L > 0 && (!x1 || !x2 || !x3 || !y)) return HYENA_ERR_INVALID_ARG;
    if (ld_x < D || ld_y < D) return HYENA_ERR_INVALID_ARG;
    if (D % 8) return HYENA_ERR_ALIGNMENT;
    const size_t need = hyena_short_host_workspace_size(B, D, K, chunk);
    if (workspace == nullptr || workspace_bytes < need) return HYENA_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return HYENA_ERR_ALIGNMENT;
    unsigned char *slots = static_cast<unsigned char *>(workspace);
    const size_t tensor = align256(static_cast<size_t>(B) * chunk * D * sizeof(hyena_bf16_t));
    float *window = reinterpret_cast<float *>(slots + static_cast<size_t>(kSlots) * 4 * tensor);
    if (L == 0)
        return hyena_short_conv(nullptr, nullptr, nullptr, D, taps, Dskip, nullptr, D, hist_in, hist_out, B, 0, D, K,
                                stream);
    return stream_chunks(x1, x2, x3, ld_x, y, ld_y, B, L, D, chunk, slots, tensor, static_cast<cudaStream_t>(stream),
                         "host-buffer short conv",
                         [&](int i, bool last, const hyena_bf16_t *c1, const hyena_bf16_t *c2, const hyena_bf16_t *c3,
                             hyena_bf16_t *cy, int rows) {
                             return hyena_short_conv(c1, c2, c3, D, taps, Dskip, cy, D, i == 0 ? hist_in : window,
                                                     last ? hist_out : window, B, rows, D, K, stream);
                         });
}
