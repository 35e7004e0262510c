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
// ready for the next one.
__device__ __align__(256) unsigned char g_modal_scratch[HYENA_NOALLOC_SCRATCH_BYTES];

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
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        hyena::record_cuda_error(e, "cudaGetDevice");
        return HYENA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return HYENA_ERR_UNSUPPORTED;
    void *scratch = scratch_for_device(dev, &e);
    if (scratch == nullptr) {
        hyena::record_cuda_error(e, "allocation-free modal conv: scratch address");
        return HYENA_ERR_CUDA;
    }
    if (L > 0) {
        // The ticket, finished-CTA and error words must start at zero; the
        // epoch word after them must be kept (flags of earlier calls carry
        // older epochs).
        e = cudaMemsetAsync(scratch, 0, 3 * sizeof(unsigned int), static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) {
            hyena::record_cuda_error(e, "allocation-free modal conv: clear counters");
            return HYENA_ERR_CUDA;
        }
    }
    return hyena_modal_long_conv(x1, x2, x3, ld_x, log_poles, residues, Dskip, y, ld_y, state_in, state_out, B, L, D,
                                 N, scratch, HYENA_NOALLOC_SCRATCH_BYTES, stream);
}
