// decode.cu -- one generated token: the recurrent step of the long modal filter
// and of the explicit FIR, with the fused Hyena gates, on sm_100a.
//
// Evo2-7B-262K model card, "Custom cache": generation carries the hcl state
// and the hcs/hcm window from token to token.  For one token
//   v = x1 x2;  modal: s_n <- exp(a_n) s_n + v,  conv = sum_n R_n s_n;
//               FIR:   conv = sum_{k<K} taps[c,k] v[t-k], the window then
//                      advances by one token;
//   y = x3 conv + Dskip v.
//
// One thread per (batch row, channel): the step is a few hundred bytes per
// channel (state or window, filter parameters), so it is bound by launch
// latency at small batch and by HBM bandwidth at large batch.  Each thread
// repeats the arithmetic of the prefill kernels for a one-token sequence in
// the same order (same expf, the same two accumulation chains over the modes
// including the zero-padded ones, the same tap order), so a decode step equals
// the corresponding one-token prefill call bit for bit.
#include "hyena_device.cuh"
#include "hyena_internal.h"

namespace hyena {

namespace {

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h)
{
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f)
{
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

template <int NP>
__global__ void __launch_bounds__(256) modal_decode_kernel(const DecodeArgs A)
{
    const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<long long>(A.B) * A.D) return;
    const int b = static_cast<int>(idx / A.D);
    const int c = static_cast<int>(idx - static_cast<long long>(b) * A.D);
    const size_t xi = static_cast<size_t>(b) * A.ld_x + c;
    const float v = __fmul_rn(bf16_bits_to_float(A.x1[xi]), bf16_bits_to_float(A.x2[xi]));
    const float x3 = bf16_bits_to_float(A.x3[xi]);
    const float *a = A.log_poles + static_cast<size_t>(c) * A.N;
    const float *R = A.residues + static_cast<size_t>(c) * A.N;
    float *st = A.state + (static_cast<size_t>(b) * A.D + c) * A.N;

    float s[NP], r[NP];
#pragma unroll
    for (int n = 0; n < NP; ++n) {
        // padded modes: p = R = 0 and a zero state, as in the prefill kernel
        const bool real = n < A.N;
        const float p = real ? expf(a[n]) : 0.f;
        r[n] = real ? R[n] : 0.f;
        s[n] = __fmaf_rn(p, real ? st[n] : 0.f, v);
    }
    float a0 = __fmul_rn(r[0], s[0]);
    float a1 = __fmul_rn(r[1], s[1]);
#pragma unroll
    for (int n = 2; n < NP; n += 2) {
        a0 = __fmaf_rn(r[n], s[n], a0);
        a1 = __fmaf_rn(r[n + 1], s[n + 1], a1);
    }
    const float conv = __fadd_rn(a0, a1);
    const float dsk = A.Dskip != nullptr ? A.Dskip[c] : 0.f;
    A.y[static_cast<size_t>(b) * A.ld_y + c] = float_to_bf16_bits(__fmaf_rn(dsk, v, __fmul_rn(x3, conv)));
#pragma unroll
    for (int n = 0; n < NP; ++n)
        if (n < A.N) st[n] = s[n];
}

// hist [B, K-1, D] in time order: hist[b][K-2][c] is v of the previous token.
__global__ void __launch_bounds__(256) fir_decode_kernel(const DecodeArgs A)
{
    const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<long long>(A.B) * A.D) return;
    const int b = static_cast<int>(idx / A.D);
    const int c = static_cast<int>(idx - static_cast<long long>(b) * A.D);
    const int K = A.K, H = K - 1;
    const size_t xi = static_cast<size_t>(b) * A.ld_x + c;
    const float v = __fmul_rn(bf16_bits_to_float(A.x1[xi]), bf16_bits_to_float(A.x2[xi]));
    const float x3 = bf16_bits_to_float(A.x3[xi]);
    const uint16_t *tp = A.taps + static_cast<size_t>(c) * K;
    float *hist = A.hist + static_cast<size_t>(b) * H * A.D + c;  // element j at hist[j * D]

    // taps in lag order, from an accumulator starting at +0 (as the prefill
    // kernel's register accumulators do)
    float acc = __fmaf_rn(bf16_bits_to_float(tp[0]), v, 0.f);
    for (int k = 1; k < K; ++k) acc = __fmaf_rn(bf16_bits_to_float(tp[k]), hist[static_cast<size_t>(H - k) * A.D], acc);
    const float dsk = A.Dskip != nullptr ? A.Dskip[c] : 0.f;
    A.y[static_cast<size_t>(b) * A.ld_y + c] = float_to_bf16_bits(__fmaf_rn(dsk, v, __fmul_rn(x3, acc)));
    // advance the window: each thread owns its channel's column, read before written
    for (int j = 0; j + 1 < H; ++j) hist[static_cast<size_t>(j) * A.D] = hist[static_cast<size_t>(j + 1) * A.D];
    if (H > 0) hist[static_cast<size_t>(H - 1) * A.D] = v;
}

}  // namespace

int launch_modal_decode(const DecodeArgs &a, cudaStream_t st)
{
    const long long n = static_cast<long long>(a.B) * a.D;
    const unsigned int grid = static_cast<unsigned int>((n + 255) / 256);
    switch (modal_padded_modes(a.N)) {
        case 4: modal_decode_kernel<4><<<grid, 256, 0, st>>>(a); break;
        case 8: modal_decode_kernel<8><<<grid, 256, 0, st>>>(a); break;
        default: modal_decode_kernel<16><<<grid, 256, 0, st>>>(a); break;
    }
    HYENA_TRY(cudaGetLastError(), "modal decode launch");
    return 1;
}

int launch_fir_decode(const DecodeArgs &a, cudaStream_t st)
{
    const long long n = static_cast<long long>(a.B) * a.D;
    fir_decode_kernel<<<static_cast<unsigned int>((n + 255) / 256), 256, 0, st>>>(a);
    HYENA_TRY(cudaGetLastError(), "fir decode launch");
    return 1;
}

}  // namespace hyena
