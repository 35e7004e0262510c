// modal_synth.cu -- coefficient table of the long modal filter for the scan
// kernels: p = exp(a) (CUDA's expf on the fp32 log-poles), residues, skip,
// p^MT and p^MH per mode slot and channel (complex modes: poles as given, p^k
// by repeated complex squaring), zero in padded slots and channels.
#include "hyena_device.cuh"
#include "hyena_internal.h"

namespace hyena {

namespace {

// Coefficient synthesis: p = exp(a), p^MT and p^MH in fp32 from the fp32
// log-poles (CUDA's expf); residues and skip copied; padded modes and
// channels zero.  NPT padded mode slots per channel.
template <int NPT>
__global__ void modal_synth_kernel(const ModalSynthArgs S)
{
    // a pass launched as this kernel's dependent may start its input loads
    // now; it waits for this grid before it reads the table
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= NPT * S.Dp) return;
    const int n = idx / S.Dp;
    const int c = idx - n * S.Dp;
    const bool valid = c < S.D && n < S.N;
    const float a = valid ? S.log_poles[static_cast<size_t>(c) * S.N + n] : 0.f;
    const size_t row = static_cast<size_t>(S.Dp);
    S.coef[n * row + c] = valid ? expf(a) : 0.f;
    S.coef[(NPT + n) * row + c] = valid ? S.residues[static_cast<size_t>(c) * S.N + n] : 0.f;
    S.coef[(2 * NPT + 1 + n) * row + c] = valid ? expf(a * static_cast<float>(MT)) : 0.f;
    S.coef[(3 * NPT + 1 + n) * row + c] = valid ? expf(a * static_cast<float>(MH)) : 0.f;
    if (n == 0) S.coef[2 * NPT * row + c] = (c < S.D && S.Dskip != nullptr) ? S.Dskip[c] : 0.f;
}

// Complex modes: slot pairs (2m, 2m+1) of mode m.  The pole is copied as
// given; the residue slot pair holds (Re R, -Im R), so that the output sum
// over slots is Re(R s); p^MH and p^MT are formed by six and seven complex
// squarings in fp32, (x + iy)^2 = (x x - y y) + i (2x) y.  Padded slot pairs
// are zero.
template <int NPT>
__global__ void modal_csynth_kernel(const ModalSynthArgs S)
{
    static_assert(MT == 128 && MH == 64, "p^MH and p^MT by squarings");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= NPT * S.Dp) return;
    const int n = idx / S.Dp;
    const int c = idx - n * S.Dp;
    const bool valid = c < S.D && n < S.N;  // S.N counts slots (2 per mode)
    const size_t row = static_cast<size_t>(S.Dp);
    const float *pc = S.log_poles + static_cast<size_t>(c) * S.N;  // complex poles [D][N/2][2]
    float re = 0.f, im = 0.f, r = 0.f, pn = 0.f, hre = 0.f, him = 0.f;
    if (valid) {
        re = pc[n & ~1];
        im = pc[n | 1];
        pn = pc[n];
        r = S.residues[static_cast<size_t>(c) * S.N + n];
        for (int k = 0; k < 7; ++k) {
            const float sq_re = __fmaf_rn(re, re, -__fmul_rn(im, im));
            const float sq_im = __fmul_rn(__fadd_rn(re, re), im);
            re = sq_re;
            im = sq_im;
            if (k == 5) {
                hre = re;
                him = im;
            }
        }
    }
    S.coef[n * row + c] = pn;
    S.coef[(NPT + n) * row + c] = (n & 1) ? -r : r;
    S.coef[(2 * NPT + 1 + n) * row + c] = valid ? ((n & 1) ? im : re) : 0.f;
    S.coef[(3 * NPT + 1 + n) * row + c] = valid ? ((n & 1) ? him : hre) : 0.f;
    if (n == 0) S.coef[2 * NPT * row + c] = (c < S.D && S.Dskip != nullptr) ? S.Dskip[c] : 0.f;
}

}  // namespace

int launch_modal_synth(const ModalSynthArgs &s, int NPT, bool cx, cudaStream_t st)
{
    const int total = NPT * s.Dp;
    const unsigned int grid = static_cast<unsigned int>((total + 255) / 256);
#define HYENA_SYNTH_CASE(K)                                                  \
    case K:                                                                  \
        if (cx)                                                              \
            modal_csynth_kernel<K><<<grid, 256, 0, st>>>(s);                 \
        else                                                                 \
            modal_synth_kernel<K><<<grid, 256, 0, st>>>(s);                  \
        break;
    switch (NPT) {
        HYENA_SYNTH_CASE(4)
        HYENA_SYNTH_CASE(8)
        HYENA_SYNTH_CASE(16)
        HYENA_SYNTH_CASE(32)
        HYENA_SYNTH_CASE(64)
        default: return -1;
    }
#undef HYENA_SYNTH_CASE
    HYENA_TRY(cudaGetLastError(), "modal synth launch");
    return 1;
}

}  // namespace hyena
