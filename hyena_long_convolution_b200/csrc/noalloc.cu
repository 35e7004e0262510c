// noalloc.cu -- the long modal conv for callers that cannot allocate device
// memory.  The scan's scratch (look-back slots, flags, coefficient table)
// lives in a fixed-size array that this library owns in device memory; the
// caller passes only inputs and outputs.
#include <cstdio>
#include <mutex>

#include "hyena_internal.h"

namespace {

// Fixed scratch shared by every call of hyena_modal_long_conv_noalloc in the
// process (per device).  Device globals start zero-filled, which is the state
// the scan kernel requires before its first launch; each launch leaves it
// ready for the next one.  Header words (unsigned int): [0] ticket, [1]
// finished CTAs, [2] error bits of the current call, [3] epoch (all as the
// workspace of hyena_modal_long_conv), [4] error bits of earlier calls not yet
// reported by hyena_modal_noalloc_check.
__device__ __align__(256) unsigned char g_modal_scratch[HYENA_NOALLOC_SCRATCH_BYTES];

constexpr int kStickyWord = 4;
constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once
// per device; the host-side symbol itself is not a device address).
void *scratch_for_device(int dev, cudaError_t *err)
{
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_modal_scratch);
        if (*err != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    *err = cudaSuccess;
    return g_scratch_ptr[dev];
}

hyena_status_t current_scratch(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        hyena::record_cuda_error(e, "cudaGetDevice");
        return HYENA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return HYENA_ERR_UNSUPPORTED;
    *out = scratch_for_device(dev, &e);
    if (*out == nullptr) {
        hyena::record_cuda_error(e, "allocation-free modal conv: scratch address");
        return HYENA_ERR_CUDA;
    }
    return HYENA_OK;
}

// Before each call: keep the previous call's error bits for the check call,
// clear them for this one, and zero this call's look-back flags, so that a
// flag word can never be a value another layout (B, D, N) left at that place.
// One block; the flags of one call are at most a few tens of KB.
__global__ void noalloc_prepare_kernel(unsigned int *hdr, unsigned long long *flags, size_t nflags)
{
    if (threadIdx.x == 0) {
        hdr[kStickyWord] |= hdr[2];
        hdr[2] = 0u;
    }
    for (size_t i = threadIdx.x; i < nflags; i += blockDim.x) flags[i] = 0ull;
}

}  // namespace

extern "C" hyena_status_t hyena_modal_long_conv_noalloc(const hyena_bf16_t *x1, const hyena_bf16_t *x2,
                                                        const hyena_bf16_t *x3, int64_t ld_x,
                                                        const float *log_poles, const float *residues,
                                                        const float *Dskip, hyena_bf16_t *y, int64_t ld_y,
                                                        const float *state_in, float *state_out, int B, int L,
                                                        int D, int N, void *stream)
{
    const size_t need = hyena_modal_long_conv_workspace_size(B, D, N);
    if (need == 0) return (N > HYENA_MAX_MODES) ? HYENA_ERR_UNSUPPORTED : HYENA_ERR_INVALID_ARG;
    if (need > static_cast<size_t>(HYENA_NOALLOC_SCRATCH_BYTES)) {
        char msg[160];
        snprintf(msg, sizeof msg, "allocation-free modal conv: B=%d, D=%d, N=%d need %zu bytes of scratch, limit %zu",
                 B, D, N, need, static_cast<size_t>(HYENA_NOALLOC_SCRATCH_BYTES));
        hyena::record_message(msg);
        return HYENA_ERR_WORKSPACE;
    }
    void *scratch = nullptr;
    const hyena_status_t st = current_scratch(&scratch);
    if (st != HYENA_OK) return st;
    if (L > 0) {
        const hyena::ModalLayout lay = hyena::modal_layout(B, D, N);
        unsigned char *base = static_cast<unsigned char *>(scratch);
        const size_t nflags = (lay.off_slots - lay.off_flags) / sizeof(unsigned long long);
        noalloc_prepare_kernel<<<1, 256, 0, static_cast<cudaStream_t>(stream)>>>(
            reinterpret_cast<unsigned int *>(base + lay.off_hdr),
            reinterpret_cast<unsigned long long *>(base + lay.off_flags), nflags);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) {
            hyena::record_cuda_error(e, "allocation-free modal conv: prepare scratch");
            return HYENA_ERR_CUDA;
        }
    }
    const hyena_status_t r = hyena_modal_long_conv(x1, x2, x3, ld_x, log_poles, residues, Dskip, y, ld_y, state_in,
                                                   state_out, B, L, D, N, scratch, HYENA_NOALLOC_SCRATCH_BYTES,
                                                   stream);
    if (r == HYENA_OK && L > 0) hyena::add_launches(1);  // the prepare kernel
    return r;
}

extern "C" hyena_status_t hyena_modal_noalloc_check(void *stream)
{
    void *scratch = nullptr;
    const hyena_status_t st = current_scratch(&scratch);
    if (st != HYENA_OK) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return HYENA_ERR_CUDA;
    unsigned int w[5] = {};
    if (cudaMemcpy(w, scratch, sizeof w, cudaMemcpyDeviceToHost) != cudaSuccess) return HYENA_ERR_CUDA;
    const unsigned int errors = w[2] | w[kStickyWord];
    if (errors == 0u) return HYENA_OK;
    unsigned int *hdr = static_cast<unsigned int *>(scratch);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(hdr + 2, 0, sizeof(unsigned int), s) != cudaSuccess ||
        cudaMemsetAsync(hdr + kStickyWord, 0, sizeof(unsigned int), s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return HYENA_ERR_CUDA;
    return HYENA_ERR_TIMEOUT;
}

extern "C" hyena_status_t hyena_modal_noalloc_scratch(void **device_ptr, size_t *bytes)
{
    if (device_ptr == nullptr || bytes == nullptr) return HYENA_ERR_INVALID_ARG;
    void *scratch = nullptr;
    const hyena_status_t st = current_scratch(&scratch);
    if (st != HYENA_OK) return st;
    *device_ptr = scratch;
    *bytes = HYENA_NOALLOC_SCRATCH_BYTES;
    return HYENA_OK;
}
