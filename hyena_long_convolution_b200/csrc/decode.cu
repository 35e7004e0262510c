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

constexpr int kDecodeThreads = 64;  // small blocks: more CTAs (SMs) per call at batch 1

// The NB floats p[i] for slots i of [base, base + NB) that exist (i < N) into
// v[0, NB), zero beyond N; 16-byte loads when the whole block exists and is
// aligned (N a multiple of 4).
template <int NB>
__device__ __forceinline__ void load_block(float (&v)[NB], const float *p, int base, int N)
{
    if (base + NB <= N && (N & 3) == 0) {
#pragma unroll
        for (int i = 0; i < NB; i += 4) {
            const float4 q = __ldg(reinterpret_cast<const float4 *>(p + base + i));
            v[i] = q.x;
            v[i + 1] = q.y;
            v[i + 2] = q.z;
            v[i + 3] = q.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < NB; ++i) v[i] = base + i < N ? p[base + i] : 0.f;
    }
}

// kCx: complex modes, N counts slots (two per mode, as the prefill kernel's
// coefficient table): the pole pair is used as given and the residue pair as
// (Re R, -Im R); the state update is the prefill kernel's complex step.
// NPT padded slots are taken in blocks of NB = min(NPT, 16), the slots one
// lane of the prefill kernel holds: each block's part of the readout is formed
// with the same two accumulation chains, and the parts are added in the
// prefill kernel's butterfly order ((p0 + p1) + (p2 + p3)).
template <int NPT, bool kCx>
__global__ void __launch_bounds__(kDecodeThreads) modal_decode_kernel(const DecodeArgs A)
{
    constexpr int NB = NPT < 16 ? NPT : 16;
    constexpr int NBLK = NPT / NB;
    const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<long long>(A.B) * A.D) return;
    const int b = static_cast<int>(idx / A.D);
    const int c = static_cast<int>(idx - static_cast<long long>(b) * A.D);
    const size_t xi = static_cast<size_t>(b) * A.ld_x + x_col(c, A.group);
    const float v = __fmul_rn(bf16_bits_to_float(A.x1[xi]), bf16_bits_to_float(A.x2[xi]));
    const float x3 = bf16_bits_to_float(A.x3[xi]);
    float *st = A.state + (static_cast<size_t>(b) * A.D + c) * A.N;
    const float *ap = A.log_poles + static_cast<size_t>(c) * A.N;
    const float *rp = A.residues + static_cast<size_t>(c) * A.N;

    float part[NBLK];
#pragma unroll
    for (int bi = 0; bi < NBLK; ++bi) {
        const int base = bi * NB;
        // padded slots (>= N): p = R = 0 and a zero state, as in the prefill kernel
        float a[NB], r[NB], s[NB];
        load_block<NB>(a, ap, base, A.N);
        load_block<NB>(r, rp, base, A.N);
        if (base + NB <= A.N && (A.N & 3) == 0) {
#pragma unroll
            for (int i = 0; i < NB; i += 4) {
                const float4 q = *reinterpret_cast<const float4 *>(st + base + i);
                s[i] = q.x;
                s[i + 1] = q.y;
                s[i + 2] = q.z;
                s[i + 3] = q.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < NB; ++i) s[i] = base + i < A.N ? st[base + i] : 0.f;
        }
        if constexpr (!kCx) {
#pragma unroll
            for (int n = 0; n < NB; ++n) s[n] = __fmaf_rn(base + n < A.N ? expf(a[n]) : 0.f, s[n], v);
        } else {
            // a[] holds the poles (zero in padded slots); residue pairs (Re, -Im)
#pragma unroll
            for (int m = 0; m < NB; m += 2) {
                r[m + 1] = -r[m + 1];
                const float re = s[m], im = s[m + 1];
                s[m] = __fmaf_rn(a[m], re, __fmaf_rn(-a[m + 1], im, v));
                s[m + 1] = __fmaf_rn(a[m], im, __fmul_rn(a[m + 1], re));
            }
        }
        float a0 = __fmul_rn(r[0], s[0]);
        float a1 = __fmul_rn(r[1], s[1]);
#pragma unroll
        for (int n = 2; n < NB; n += 2) {
            a0 = __fmaf_rn(r[n], s[n], a0);
            a1 = __fmaf_rn(r[n + 1], s[n + 1], a1);
        }
        part[bi] = __fadd_rn(a0, a1);
        if (base + NB <= A.N && (A.N & 3) == 0) {
#pragma unroll
            for (int i = 0; i < NB; i += 4)
                *reinterpret_cast<float4 *>(st + base + i) = make_float4(s[i], s[i + 1], s[i + 2], s[i + 3]);
        } else {
#pragma unroll
            for (int n = 0; n < NB; ++n)
                if (base + n < A.N) st[base + n] = s[n];
        }
    }
    // butterfly: neighbours first, then pairs of neighbours
#pragma unroll
    for (int d = 1; d < NBLK; d <<= 1)
#pragma unroll
        for (int bi = 0; bi < NBLK; bi += 2 * d) part[bi] = __fadd_rn(part[bi], part[bi + d]);
    const float conv = part[0];
    const float dsk = A.Dskip != nullptr ? A.Dskip[c] : 0.f;
    A.y[static_cast<size_t>(b) * A.ld_y + c] = float_to_bf16_bits(__fmaf_rn(dsk, v, __fmul_rn(x3, conv)));
}

// hist [B, K-1, D] in time order: hist[b][K-2][c] is v of the previous token.
// One pass from the newest window entry to the oldest: each entry is read
// once, feeds the lag-ordered FMA chain (lag k = K-1-j for entry j) and is
// written one place older, through a carry register, so the window advances
// in place.
__global__ void __launch_bounds__(kDecodeThreads) fir_decode_kernel(const DecodeArgs A)
{
    const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<long long>(A.B) * A.D) return;
    const int b = static_cast<int>(idx / A.D);
    const int c = static_cast<int>(idx - static_cast<long long>(b) * A.D);
    const int K = A.K, H = K - 1;
    const size_t xi = static_cast<size_t>(b) * A.ld_x + x_col(c, A.group);
    const float v = __fmul_rn(bf16_bits_to_float(A.x1[xi]), bf16_bits_to_float(A.x2[xi]));
    const float x3 = bf16_bits_to_float(A.x3[xi]);
    const uint16_t *tp = A.taps + static_cast<size_t>(c) * K;
    const size_t D = static_cast<size_t>(A.D);
    float *hist = A.hist + static_cast<size_t>(b) * H * D + c;  // entry j at hist[j * D]

    // lag 0, from an accumulator starting at +0 (as the prefill kernel's
    // register accumulators do)
    float acc = __fmaf_rn(bf16_bits_to_float(tp[0]), v, 0.f);
    float carry = v;  // the value entry j receives
    // Entries in batches of 32 (lags k0 .. k0+31, entries H-k0 down): all of a
    // batch's loads are issued before its FMAs and stores.
    constexpr int kBatch = 32;
    for (int k0 = 1; k0 < K; k0 += kBatch) {
        float old[kBatch], tap[kBatch];
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
            const int k = k0 + i;
            if (k < K) {
                old[i] = hist[static_cast<size_t>(H - k) * D];
                tap[i] = bf16_bits_to_float(tp[k]);
            }
        }
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
            const int k = k0 + i;
            if (k < K) {
                acc = __fmaf_rn(tap[i], old[i], acc);
                hist[static_cast<size_t>(H - k) * D] = carry;
                carry = old[i];
            }
        }
    }
    const float dsk = A.Dskip != nullptr ? A.Dskip[c] : 0.f;
    A.y[static_cast<size_t>(b) * A.ld_y + c] = float_to_bf16_bits(__fmaf_rn(dsk, v, __fmul_rn(x3, acc)));
}

}  // namespace

int launch_modal_decode(const DecodeArgs &a, bool cx, cudaStream_t st)
{
    const long long n = static_cast<long long>(a.B) * a.D;
    const unsigned int grid = static_cast<unsigned int>((n + kDecodeThreads - 1) / kDecodeThreads);
    const int npt = modal_padded_modes(a.N);
#define HYENA_DECODE_CASE(NPT)                                                                  \
    case NPT:                                                                                    \
        if (cx)                                                                                  \
            modal_decode_kernel<NPT, true><<<grid, kDecodeThreads, 0, st>>>(a);                  \
        else                                                                                     \
            modal_decode_kernel<NPT, false><<<grid, kDecodeThreads, 0, st>>>(a);                 \
        break;
    switch (npt) {
        HYENA_DECODE_CASE(4)
        HYENA_DECODE_CASE(8)
        HYENA_DECODE_CASE(16)
        HYENA_DECODE_CASE(32)
        HYENA_DECODE_CASE(64)
        default: return -1;
    }
#undef HYENA_DECODE_CASE
    HYENA_TRY(cudaGetLastError(), "modal decode launch");
    return 1;
}

int launch_fir_decode(const DecodeArgs &a, cudaStream_t st)
{
    const long long n = static_cast<long long>(a.B) * a.D;
    fir_decode_kernel<<<static_cast<unsigned int>((n + kDecodeThreads - 1) / kDecodeThreads), kDecodeThreads, 0,
                        st>>>(a);
    HYENA_TRY(cudaGetLastError(), "fir decode launch");
    return 1;
}

}  // namespace hyena
