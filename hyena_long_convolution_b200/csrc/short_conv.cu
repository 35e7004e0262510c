// short_conv.cu -- explicit short causal FIR (hcs: 7 taps, hcm: 128 taps)
// with the fused Hyena gates, on sm_100a.
//
// Operator (Evo2-7B-262K model card, §Implementation Notes: "Block dispatch"
// names FIR cascades of inner length 7 and 128; "Custom cache" and the
// Evo1-1.5-7B-8K card's "Cache subclass" carry the FIR window):
//   v[t] = x1[t] x2[t];  conv[t] = sum_{k<K} taps[c,k] v[t-k];
//   y[t] = x3[t] conv[t] + Dskip[c] v[t].
//
// Design.  One CTA owns FCH = 64 channels x FT = 128 output tokens of one
// batch row.  TMA stages x1, x2 for the tile plus a halo of HR >= K-1 earlier
// rows (a second, shorter box) and x3 for the tile.  The bf16 x1 and x2 rows
// land inside the fp32 buffer that then holds v = x1 x2 (two bf16 rows take
// the bytes of one fp32 row), and are converted in place through registers
// (halo rows before t = 0 come from hist_in), which keeps the CTA small
// enough for two per SM even at K = 128.  Warp w computes FRW = 16
// consecutive outputs for the lane's two channels with a register-blocked
// window: per block of 8 taps it issues 8 x 16 packed f32x2 FMAs on the 8 taps
// and 23 window values, 15 of them carried over in registers from the
// previous block (the window slides along the taps).  The gates are applied
// in registers and y is stored as coalesced 128-byte rows.  A second small
// kernel writes hist_out (the last K-1 values of v).
//
// Inputs come as three tensors, as one packed projection buffer whose rows
// hold channel groups [x1 | x2 | x3] (4-D tensor maps address a group's
// column), or as per-channel triples (x1_c, x2_c, x3_c adjacent).  Triples
// load one box of 3 x 64 interleaved values per row; the rows are turned into
// v and x3 in place in row batches (v of a batch only overwrites rows already
// read), and the taps stay bf16 in shared memory, which keeps that layout at
// two CTAs per SM for K = 128 as well.
#include "hyena_device.cuh"
#include "hyena_internal.h"

namespace hyena {

namespace {

constexpr int kMaxHalo = 128;  // HR <= 128 since K <= 128
constexpr int kRowWords = FCH / 2;  // 32-bit words per bf16 row

// Shared-memory layouts of one CTA.
enum FirMode : int {
    kSeparate = 0,  // bf16 x1, x2, x3 rows in buffers of their own, fp32 taps
    kInPlace = 1,   // bf16 x1, x2 rows inside v's buffer (two bf16 rows take
                    // the bytes of one fp32 row), fp32 taps
    kTriples = 2,   // interleaved rows of 96 words; v, then x3, written over
                    // them; bf16 taps
};

struct FirSmemView {
    uint32_t *x1, *x2, *x3;  // bf16 rows [HR + FT][32], [HR + FT][32], [FT][32]
    uint32_t *raw;           // kTriples: interleaved rows [HR + FT][96]
    float2 *v;               // [HR + FT][32]
    float2 *taps;            // [K][32] fp32 pairs
    uint32_t *taps_h;        // kTriples: [K][32] bf16 pairs
    uint64_t *bar;
};

__host__ __device__ inline size_t fir_smem_bytes(int HR, int K, int mode)
{
    const size_t rows = static_cast<size_t>(HR) + FT;
    if (mode == kTriples) return rows * 3 * kRowWords * 4 + static_cast<size_t>(K) * 32 * 4 + 16;
    const size_t raw = mode == kInPlace ? 0 : rows * kRowWords * 4 * 2;
    return raw + rows * 32 * 8 + static_cast<size_t>(FT) * kRowWords * 4 + static_cast<size_t>(K) * 32 * 8 + 16;
}

// The in-place layout is used when the separate one would not let two CTAs
// share an SM (long filters, with their long halos).
__host__ inline bool fir_in_place(int HR, int K) { return fir_smem_bytes(HR, K, kSeparate) > 112u * 1024u; }

template <int kMode>
__device__ inline FirSmemView fir_smem(unsigned char *base, int HR, int K)
{
    FirSmemView s{};
    const int rows = HR + FT;
    if (kMode == kTriples) {
        s.raw = reinterpret_cast<uint32_t *>(base);
        s.v = reinterpret_cast<float2 *>(base);
        s.x3 = reinterpret_cast<uint32_t *>(s.v + rows * 32);
        s.taps_h = s.raw + rows * 3 * kRowWords;
        s.bar = reinterpret_cast<uint64_t *>(s.taps_h + K * 32);
        return s;
    }
    if (kMode == kInPlace) {
        s.v = reinterpret_cast<float2 *>(base);
        s.x1 = reinterpret_cast<uint32_t *>(base);  // first half of v's bytes
        s.x2 = s.x1 + rows * kRowWords;               // second half
        s.x3 = reinterpret_cast<uint32_t *>(s.v + rows * 32);
        s.taps = reinterpret_cast<float2 *>(s.x3 + FT * kRowWords);
    } else {
        s.x1 = reinterpret_cast<uint32_t *>(base);
        s.x2 = s.x1 + rows * kRowWords;
        s.x3 = s.x2 + rows * kRowWords;
        s.v = reinterpret_cast<float2 *>(s.x3 + FT * kRowWords);
        s.taps = s.v + rows * 32;
    }
    s.bar = reinterpret_cast<uint64_t *>(s.taps + K * 32);
    return s;
}

// Tap k of this lane's channel pair, from fp32 pairs or (exactly) from bf16
// pairs.
struct TapsF32 {
    const float2 *t;
    __device__ __forceinline__ float2 operator()(int k, int lane) const { return t[k * 32 + lane]; }
};
struct TapsBF16 {
    const uint32_t *t;
    __device__ __forceinline__ float2 operator()(int k, int lane) const
    {
        return bf16x2_to_float2(t[k * 32 + lane]);
    }
};

// Accumulates taps [kb, kb + nq) into acc for this warp's FRW outputs.
template <int NQ, class Taps>
__device__ __forceinline__ void fir_block(float2 (&acc)[FRW], const float2 *vbase, const Taps &taps, int kb,
                                          int lane)
{
    // vbase points at v row (first output row - kb - (NQ-1)), this lane.
    float2 tq[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) tq[q] = taps(kb + q, lane);
    float2 w[FRW + NQ - 1];
#pragma unroll
    for (int j = 0; j < FRW + NQ - 1; ++j) w[j] = vbase[j * 32 + lane];
#pragma unroll
    for (int q = 0; q < NQ; ++q)
#pragma unroll
        for (int i = 0; i < FRW; ++i) acc[i] = __ffma2_rn(tq[q], w[i - q + NQ - 1], acc[i]);
}

// Taps [0, 8*nblk) in blocks of 8 with the window sliding along the taps in
// registers: block kb uses v rows [row0 - kb - 7, row0 - kb + 15]; the next
// block reuses 15 of those 23 values and loads 8, which halves the
// shared-memory traffic per FMA.  NBLK > 0: the block count is a compile-time
// constant and the window shift is register renaming; NBLK == 0: runtime
// count, the shift is register moves.
template <int NBLK, class Taps>
__device__ __forceinline__ void fir_sliding8(float2 (&acc)[FRW], const float2 *v, const Taps &taps, int row0,
                                             int nblk, int lane)
{
    constexpr int NW = FRW + 7;
    if (NBLK > 0) nblk = NBLK;
    float2 w[NW];
#pragma unroll
    for (int j = 0; j < NW; ++j) w[j] = v[(row0 - 7 + j) * 32 + lane];
#pragma unroll(NBLK > 0 ? NBLK : 1)
    for (int bk = 0; bk < nblk; ++bk) {
        const int kb = bk * 8;
        float2 tq[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) tq[q] = taps(kb + q, lane);
#pragma unroll
        for (int q = 0; q < 8; ++q)
#pragma unroll
            for (int i = 0; i < FRW; ++i) acc[i] = __ffma2_rn(tq[q], w[i - q + 7], acc[i]);
        if (bk + 1 < nblk) {
#pragma unroll
            for (int j = NW - 1; j >= 8; --j) w[j] = w[j - 8];
#pragma unroll
            for (int j = 0; j < 8; ++j) w[j] = v[(row0 - kb - 15 + j) * 32 + lane];
        }
    }
}

template <int kMode>
__global__ void __launch_bounds__(FW * 32)
    fir_kernel(const __grid_constant__ CUtensorMap tm1, const __grid_constant__ CUtensorMap tm2,
               const __grid_constant__ CUtensorMap tm3, const __grid_constant__ CUtensorMap th1,
               const __grid_constant__ CUtensorMap th2, const FirArgs A)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const int HR = A.HR;
    const int K = A.K;
    FirSmemView sm = fir_smem<kMode>(smem_raw, HR, K);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cb = blockIdx.x;
    const int t0 = blockIdx.y * FT;
    const int b = blockIdx.z;
    const int c0 = cb * FCH + 2 * lane;
    const bool ch_ok = c0 < A.D;

    if (tid == 0) {
        mbar_init(sm.bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        const int ch = cb * FCH;
        if constexpr (kMode == kTriples) {
            mbar_arrive_expect_tx(sm.bar, static_cast<uint32_t>((HR + FT) * 3 * kRowWords * 4));
            if (HR > 0) tma_load_4d(sm.raw, &th1, sm.bar, 3 * ch, 0, t0 - HR, b);
            tma_load_4d(sm.raw + HR * 3 * kRowWords, &tm1, sm.bar, 3 * ch, 0, t0, b);
        } else {
            const int cx = ch % A.group, cg = ch / A.group;
            mbar_arrive_expect_tx(sm.bar, static_cast<uint32_t>((2 * (HR + FT) + FT) * kRowWords * 4));
            if (HR > 0) {
                tma_load_4d(sm.x1, &th1, sm.bar, cx, cg, t0 - HR, b);
                tma_load_4d(sm.x2, &th2, sm.bar, cx, cg, t0 - HR, b);
            }
            tma_load_4d(sm.x1 + HR * kRowWords, &tm1, sm.bar, cx, cg, t0, b);
            tma_load_4d(sm.x2 + HR * kRowWords, &tm2, sm.bar, cx, cg, t0, b);
            tma_load_4d(sm.x3, &tm3, sm.bar, cx, cg, t0, b);
        }
    }
    // taps -> [K][lane] pairs (fp32, or bf16 for kTriples) while the tiles
    // are in flight
    if ((K & 7) == 0) {
        // 8 consecutive taps of one channel per 16-byte load
        for (int idx = tid; idx < (K / 8) * 32; idx += FW * 32) {
            const int l = idx & 31, kb = (idx >> 5) * 8;
            const int c = cb * FCH + 2 * l;
            uint4 ta = make_uint4(0u, 0u, 0u, 0u), tb = ta;
            if (c < A.D) {
                ta = __ldg(reinterpret_cast<const uint4 *>(A.taps + static_cast<size_t>(c) * K + kb));
                tb = __ldg(reinterpret_cast<const uint4 *>(A.taps + static_cast<size_t>(c + 1) * K + kb));
            }
            const uint32_t wa[4] = {ta.x, ta.y, ta.z, ta.w}, wb[4] = {tb.x, tb.y, tb.z, tb.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if constexpr (kMode == kTriples) {
                    sm.taps_h[(kb + 2 * i) * 32 + l] = __byte_perm(wa[i], wb[i], 0x5410);
                    sm.taps_h[(kb + 2 * i + 1) * 32 + l] = __byte_perm(wa[i], wb[i], 0x7632);
                } else {
                    const float2 lo = make_float2(__uint_as_float(wa[i] << 16), __uint_as_float(wb[i] << 16));
                    const float2 hi =
                        make_float2(__uint_as_float(wa[i] & 0xffff0000u), __uint_as_float(wb[i] & 0xffff0000u));
                    sm.taps[(kb + 2 * i) * 32 + l] = lo;
                    sm.taps[(kb + 2 * i + 1) * 32 + l] = hi;
                }
            }
        }
    } else {
        for (int idx = tid; idx < K * 32; idx += FW * 32) {
            const int k = idx >> 5, l = idx & 31;
            const int c = cb * FCH + 2 * l;
            uint32_t ha = 0u, hb = 0u;
            if (c < A.D) {
                ha = A.taps[static_cast<size_t>(c) * K + k];
                hb = A.taps[static_cast<size_t>(c + 1) * K + k];
            }
            if constexpr (kMode == kTriples)
                sm.taps_h[idx] = ha | (hb << 16);
            else
                sm.taps[idx] = make_float2(__uint_as_float(ha << 16), __uint_as_float(hb << 16));
        }
    }
    const bool ok = mbar_wait_bounded(sm.bar, 0);
    if (__syncthreads_or(!ok)) {
        (void)mbar_wait_bounded(sm.bar, 0);
        return;  // tiles never arrived; output left unwritten
    }

    // v = x1 * x2 for the halo and the tile; rows before t = 0 from hist_in.
    const int H = K - 1;
    const int rows = HR + FT;
    auto v_of = [&](int r, float2 x1, float2 x2) {
        const int t = t0 - HR + r;
        if (t >= 0) return __fmul2_rn(x1, x2);
        if (t >= -H && A.hist_in != nullptr && ch_ok)
            return *reinterpret_cast<const float2 *>(A.hist_in + (static_cast<size_t>(b) * H + (H + t)) * A.D + c0);
        return make_float2(0.f, 0.f);
    };
    if constexpr (kMode == kTriples) {
        // x3 of this warp's output rows first (those interleaved rows are
        // overwritten by v below), then v in batches of 32 rows: all reads of a
        // batch precede its writes, and v rows [32p, 32p + 32) occupy the bytes
        // of interleaved rows below 32p * 2/3 + 22, all read by then.  The x3
        // words are stored after every interleaved row has been read.
        uint32_t x3w[FRW];
#pragma unroll
        for (int i = 0; i < FRW; ++i) {
            const uint32_t *rw = sm.raw + (HR + warp * FRW + i) * 3 * kRowWords + 3 * lane;
            x3w[i] = __byte_perm(rw[1], rw[2], 0x7610);
        }
        for (int p0 = 0; p0 < rows; p0 += 32) {
            float2 vv[32 / FW];
#pragma unroll
            for (int j = 0; j < 32 / FW; ++j) {
                const int r = p0 + warp + j * FW;
                if (r < rows) {
                    const uint32_t *rw = sm.raw + r * 3 * kRowWords + 3 * lane;
                    const uint32_t w0 = rw[0], w1 = rw[1], w2 = rw[2];
                    vv[j] = v_of(r, tri_x1(w0, w1), tri_x2(w0, w2));
                }
            }
            __syncthreads();
#pragma unroll
            for (int j = 0; j < 32 / FW; ++j) {
                const int r = p0 + warp + j * FW;
                if (r < rows) sm.v[r * 32 + lane] = vv[j];
            }
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < FRW; ++i) sm.x3[(warp * FRW + i) * kRowWords + lane] = x3w[i];
    } else if constexpr (kMode == kInPlace) {
        // every thread first reads the bf16 words of its rows and then, after
        // the barrier, writes their fp32 products over them
        constexpr int kMaxRowsPerWarp = (kMaxHalo + FT) / FW;
        uint32_t w1[kMaxRowsPerWarp], w2[kMaxRowsPerWarp];
#pragma unroll
        for (int i = 0; i < kMaxRowsPerWarp; ++i) {
            const int r = warp + i * FW;
            if (r < rows) {
                w1[i] = sm.x1[r * kRowWords + lane];
                w2[i] = sm.x2[r * kRowWords + lane];
            }
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kMaxRowsPerWarp; ++i) {
            const int r = warp + i * FW;
            if (r < rows) sm.v[r * 32 + lane] = v_of(r, bf16x2_to_float2(w1[i]), bf16x2_to_float2(w2[i]));
        }
    } else {
        for (int r = warp; r < rows; r += FW)
            sm.v[r * 32 + lane] =
                v_of(r, bf16x2_to_float2(sm.x1[r * kRowWords + lane]), bf16x2_to_float2(sm.x2[r * kRowWords + lane]));
    }
    __syncthreads();

    float2 acc[FRW];
#pragma unroll
    for (int i = 0; i < FRW; ++i) acc[i] = make_float2(0.f, 0.f);
    const int row0 = HR + warp * FRW;  // v row of this warp's first output
    const int nblk = K / 8;
    auto conv = [&](const auto &taps) {
        if (nblk == HYENA_MAX_TAPS / 8)
            fir_sliding8<HYENA_MAX_TAPS / 8>(acc, sm.v, taps, row0, nblk, lane);
        else if (nblk > 0)
            fir_sliding8<0>(acc, sm.v, taps, row0, nblk, lane);
        const int kb = nblk * 8;
        switch (K - kb) {
            case 7: fir_block<7>(acc, sm.v + (row0 - kb - 6) * 32, taps, kb, lane); break;
            case 6: fir_block<6>(acc, sm.v + (row0 - kb - 5) * 32, taps, kb, lane); break;
            case 5: fir_block<5>(acc, sm.v + (row0 - kb - 4) * 32, taps, kb, lane); break;
            case 4: fir_block<4>(acc, sm.v + (row0 - kb - 3) * 32, taps, kb, lane); break;
            case 3: fir_block<3>(acc, sm.v + (row0 - kb - 2) * 32, taps, kb, lane); break;
            case 2: fir_block<2>(acc, sm.v + (row0 - kb - 1) * 32, taps, kb, lane); break;
            case 1: fir_block<1>(acc, sm.v + (row0 - kb) * 32, taps, kb, lane); break;
            default: break;
        }
    };
    if constexpr (kMode == kTriples)
        conv(TapsBF16{sm.taps_h});
    else
        conv(TapsF32{sm.taps});

    const float2 dsk = (A.Dskip != nullptr && ch_ok)
                           ? make_float2(A.Dskip[c0], A.Dskip[c0 + 1])
                           : make_float2(0.f, 0.f);
    const int tw0 = t0 + warp * FRW;
    const int nvalid = min(FRW, A.L - tw0);
    uint32_t *yrow = reinterpret_cast<uint32_t *>(A.y + (static_cast<size_t>(b) * A.L + tw0) * A.ld_y + c0);
    const size_t ystride = static_cast<size_t>(A.ld_y) / 2;
#pragma unroll
    for (int i = 0; i < FRW; ++i) {
        if (i < nvalid && ch_ok) {
            const float2 x3 = bf16x2_to_float2(sm.x3[(warp * FRW + i) * kRowWords + lane]);
            const float2 v = sm.v[(row0 + i) * 32 + lane];
            yrow[i * ystride] = float2_to_bf16x2(__ffma2_rn(dsk, v, __fmul2_rn(x3, acc[i])));
        }
    }
}

// Short filters (K <= 8, halo of at most 8 rows): the window values are formed
// from the bf16 x1, x2 rows as they are used instead of from an fp32 v buffer,
// and each warp computes its 16 outputs in two halves of 8.  That keeps the CTA
// at 53 KB of shared memory and at most 64 registers, four CTAs per SM
// instead of two, for this HBM-bound case.  kTri: the rows are the interleaved
// per-channel triples (96 words per row), read the same way.  The FMA order per
// output is the general kernel's (taps in lag order from a zero accumulator),
// so results are bit-identical to it.
constexpr int kSmallMaxK = 8;
constexpr int kSmallHalf = 8;  // outputs per pass

__host__ __device__ inline size_t fir_small_smem_bytes(int HR, int K, bool tri)
{
    const size_t rows = static_cast<size_t>(HR) + FT;
    const size_t x = tri ? rows * 3 * kRowWords * 4 : rows * kRowWords * 4 * 2 + static_cast<size_t>(FT) * kRowWords * 4;
    return x + static_cast<size_t>(K) * 32 * 8 + 16;
}

template <bool kTri>
__global__ void __launch_bounds__(FW * 32, 4)
    fir_small_kernel(const __grid_constant__ CUtensorMap tm1, const __grid_constant__ CUtensorMap tm2,
                     const __grid_constant__ CUtensorMap tm3, const __grid_constant__ CUtensorMap th1,
                     const __grid_constant__ CUtensorMap th2, const FirArgs A)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const int HR = A.HR, K = A.K, H = K - 1;
    const int rows = HR + FT;
    uint32_t *x1 = reinterpret_cast<uint32_t *>(smem_raw);  // kTri: the interleaved rows
    uint32_t *x2 = x1 + rows * kRowWords;
    uint32_t *x3 = x2 + rows * kRowWords;
    float2 *taps = reinterpret_cast<float2 *>(kTri ? x1 + rows * 3 * kRowWords : x3 + FT * kRowWords);
    uint64_t *bar = reinterpret_cast<uint64_t *>(taps + K * 32);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cb = blockIdx.x;
    const int t0 = blockIdx.y * FT;
    const int b = blockIdx.z;
    const int c0 = cb * FCH + 2 * lane;
    const bool ch_ok = c0 < A.D;

    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        const int ch = cb * FCH;
        if constexpr (kTri) {
            mbar_arrive_expect_tx(bar, static_cast<uint32_t>(rows * 3 * kRowWords * 4));
            if (HR > 0) tma_load_4d(x1, &th1, bar, 3 * ch, 0, t0 - HR, b);
            tma_load_4d(x1 + HR * 3 * kRowWords, &tm1, bar, 3 * ch, 0, t0, b);
        } else {
            const int cx = ch % A.group, cg = ch / A.group;
            mbar_arrive_expect_tx(bar, static_cast<uint32_t>((2 * rows + FT) * kRowWords * 4));
            if (HR > 0) {
                tma_load_4d(x1, &th1, bar, cx, cg, t0 - HR, b);
                tma_load_4d(x2, &th2, bar, cx, cg, t0 - HR, b);
            }
            tma_load_4d(x1 + HR * kRowWords, &tm1, bar, cx, cg, t0, b);
            tma_load_4d(x2 + HR * kRowWords, &tm2, bar, cx, cg, t0, b);
            tma_load_4d(x3, &tm3, bar, cx, cg, t0, b);
        }
    }
    for (int idx = tid; idx < K * 32; idx += FW * 32) {
        const int k = idx >> 5, l = idx & 31;
        const int c = cb * FCH + 2 * l;
        float2 t = make_float2(0.f, 0.f);
        if (c < A.D) {
            t.x = __uint_as_float(static_cast<uint32_t>(A.taps[static_cast<size_t>(c) * K + k]) << 16);
            t.y = __uint_as_float(static_cast<uint32_t>(A.taps[static_cast<size_t>(c + 1) * K + k]) << 16);
        }
        taps[idx] = t;
    }
    const bool ok = mbar_wait_bounded(bar, 0);
    if (__syncthreads_or(!ok)) {
        (void)mbar_wait_bounded(bar, 0);
        return;  // tiles never arrived; output left unwritten
    }

    // v of row r (rows before t = 0 from hist_in, or zero)
    auto vrow = [&](int r) {
        const int t = t0 - HR + r;
        if (t >= 0) {
            if constexpr (kTri) {
                const uint32_t *rw = x1 + r * 3 * kRowWords + 3 * lane;
                const uint32_t w0 = rw[0], w1 = rw[1], w2 = rw[2];
                return __fmul2_rn(tri_x1(w0, w1), tri_x2(w0, w2));
            } else {
                return __fmul2_rn(bf16x2_to_float2(x1[r * kRowWords + lane]),
                                  bf16x2_to_float2(x2[r * kRowWords + lane]));
            }
        }
        if (t >= -H && A.hist_in != nullptr && ch_ok)
            return *reinterpret_cast<const float2 *>(A.hist_in + (static_cast<size_t>(b) * H + (H + t)) * A.D + c0);
        return make_float2(0.f, 0.f);
    };
    const float2 dsk = (A.Dskip != nullptr && ch_ok) ? make_float2(A.Dskip[c0], A.Dskip[c0 + 1])
                                                     : make_float2(0.f, 0.f);
    const size_t ystride = static_cast<size_t>(A.ld_y) / 2;
#pragma unroll 1
    for (int h = 0; h < FRW / kSmallHalf; ++h) {
        const int orow = warp * FRW + h * kSmallHalf;  // first output row of this pass (tile-relative)
        const int row0 = HR + orow;                    // its v row
        float2 acc[kSmallHalf];
#pragma unroll
        for (int i = 0; i < kSmallHalf; ++i) acc[i] = make_float2(0.f, 0.f);
        // window rows row0 - (kSmallMaxK - 1) .. row0 + kSmallHalf - 1 (only the last K - 1 + 8 are used)
        float2 w[kSmallHalf + kSmallMaxK - 1];
#pragma unroll
        for (int j = 0; j < kSmallHalf + kSmallMaxK - 1; ++j) {
            const int r = row0 - (kSmallMaxK - 1) + j;
            w[j] = r >= 0 ? vrow(r) : make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int q = 0; q < kSmallMaxK; ++q) {
            if (q < K) {
                const float2 tq = taps[q * 32 + lane];
#pragma unroll
                for (int i = 0; i < kSmallHalf; ++i) acc[i] = __ffma2_rn(tq, w[i - q + kSmallMaxK - 1], acc[i]);
            }
        }
        const int tw0 = t0 + orow;
        const int nvalid = min(kSmallHalf, A.L - tw0);
        uint32_t *yrow = reinterpret_cast<uint32_t *>(A.y + (static_cast<size_t>(b) * A.L + tw0) * A.ld_y + c0);
#pragma unroll
        for (int i = 0; i < kSmallHalf; ++i) {
            if (i < nvalid && ch_ok) {
                float2 x3v;
                if constexpr (kTri) {
                    const uint32_t *rw = x1 + (HR + orow + i) * 3 * kRowWords + 3 * lane;
                    x3v = tri_x3(rw[1], rw[2]);
                } else {
                    x3v = bf16x2_to_float2(x3[(orow + i) * kRowWords + lane]);
                }
                yrow[i * ystride] = float2_to_bf16x2(__ffma2_rn(dsk, w[i + kSmallMaxK - 1], __fmul2_rn(x3v, acc[i])));
            }
        }
    }
}

// hist_out[b][j][c] = v[L-H+j] (from hist_in when that index is negative).
// One thread per (batch row, channel pair) walks j upward, so reading
// hist_in[j + L] before writing hist_out[j + L] keeps in-place use safe.
// hist_out row j = v[L - H + j]: from x (t >= 0), from hist_in (t < 0), or
// zero.  One thread per (batch row, history row, channel pair): every output
// element is independent, so the launch is as wide as the history.  Used
// unless hist_out aliases hist_in and 0 < L < H (then rows move within the
// buffer and the ordered kernel below runs instead).
__global__ void fir_history_rows_kernel(const FirArgs A)
{
    const int pairs = A.D / 2;
    const int H = A.K - 1;
    const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<long long>(A.B) * H * pairs) return;
    const int b = static_cast<int>(idx / (static_cast<long long>(H) * pairs));
    const int rem = static_cast<int>(idx - static_cast<long long>(b) * H * pairs);
    const int j = rem / pairs;
    const int c = (rem - j * pairs) * 2;
    const int t = A.L - H + j;
    float2 v;
    if (t >= 0) {
        const size_t row = (static_cast<size_t>(b) * A.L + t) * A.ld_x;
        const size_t i0 = row + x_col(c, A.group), i1 = row + x_col(c + 1, A.group);
        const float2 x1 = make_float2(__uint_as_float(static_cast<uint32_t>(A.x1[i0]) << 16),
                                      __uint_as_float(static_cast<uint32_t>(A.x1[i1]) << 16));
        const float2 x2 = make_float2(__uint_as_float(static_cast<uint32_t>(A.x2[i0]) << 16),
                                      __uint_as_float(static_cast<uint32_t>(A.x2[i1]) << 16));
        v = __fmul2_rn(x1, x2);
    } else if (A.hist_in != nullptr) {
        v = *reinterpret_cast<const float2 *>(A.hist_in + (static_cast<size_t>(b) * H + (H + t)) * A.D + c);
    } else {
        v = make_float2(0.f, 0.f);
    }
    *reinterpret_cast<float2 *>(A.hist_out + (static_cast<size_t>(b) * H + j) * A.D + c) = v;
}

// The same values, one thread per (batch row, channel pair) walking the rows
// forward: hist_out row j is written only after row L + j, its source in the
// aliased buffer, has been read.
__global__ void fir_history_kernel(const FirArgs A)
{
    const int pairs = A.D / 2;
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= A.B * pairs) return;
    const int b = idx / pairs;
    const int c = (idx - b * pairs) * 2;
    const int H = A.K - 1;
    for (int j = 0; j < H; ++j) {
        const int t = A.L - H + j;
        float2 v;
        if (t >= 0) {
            const size_t row = (static_cast<size_t>(b) * A.L + t) * A.ld_x;
            const size_t i0 = row + x_col(c, A.group), i1 = row + x_col(c + 1, A.group);
            const float2 x1 = make_float2(__uint_as_float(static_cast<uint32_t>(A.x1[i0]) << 16),
                                          __uint_as_float(static_cast<uint32_t>(A.x1[i1]) << 16));
            const float2 x2 = make_float2(__uint_as_float(static_cast<uint32_t>(A.x2[i0]) << 16),
                                          __uint_as_float(static_cast<uint32_t>(A.x2[i1]) << 16));
            v = __fmul2_rn(x1, x2);
        } else if (A.hist_in != nullptr) {
            v = *reinterpret_cast<const float2 *>(A.hist_in + (static_cast<size_t>(b) * H + (H + t)) * A.D + c);
        } else {
            v = make_float2(0.f, 0.f);
        }
        *reinterpret_cast<float2 *>(A.hist_out + (static_cast<size_t>(b) * H + j) * A.D + c) = v;
    }
}

}  // namespace

int launch_fir(const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &m3,
               const CUtensorMap &h1, const CUtensorMap &h2, const FirArgs &a, bool triples, cudaStream_t st)
{
    int launches = 0;
    if (a.L > 0) {
        const bool small = a.K <= kSmallMaxK;
        const int mode = triples ? kTriples : (fir_in_place(a.HR, a.K) ? kInPlace : kSeparate);
        const size_t smem = small ? fir_small_smem_bytes(a.HR, a.K, triples) : fir_smem_bytes(a.HR, a.K, mode);
        static int configured_device = -1;
        int dev = 0;
        HYENA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
        if (configured_device != dev) {
            // the largest request of each layout (halos up to kMaxHalo rows)
            HYENA_TRY(cudaFuncSetAttribute(fir_kernel<kSeparate>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(fir_smem_bytes(kMaxHalo, HYENA_MAX_TAPS, kSeparate))),
                      "fir: set max dynamic shared memory");
            HYENA_TRY(cudaFuncSetAttribute(fir_kernel<kInPlace>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(fir_smem_bytes(kMaxHalo, HYENA_MAX_TAPS, kInPlace))),
                      "fir: set max dynamic shared memory");
            HYENA_TRY(cudaFuncSetAttribute(fir_kernel<kTriples>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(fir_smem_bytes(kMaxHalo, HYENA_MAX_TAPS, kTriples))),
                      "fir: set max dynamic shared memory");
            HYENA_TRY(cudaFuncSetAttribute(fir_small_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(fir_small_smem_bytes(fir_halo_rows(kSmallMaxK),
                                                                                 kSmallMaxK, false))),
                      "fir: set max dynamic shared memory");
            HYENA_TRY(cudaFuncSetAttribute(fir_small_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(fir_small_smem_bytes(fir_halo_rows(kSmallMaxK),
                                                                                 kSmallMaxK, true))),
                      "fir: set max dynamic shared memory");
            configured_device = dev;
        }
        const dim3 grid((a.D + FCH - 1) / FCH, (a.L + FT - 1) / FT, a.B);
        if (small && triples)
            fir_small_kernel<true><<<grid, FW * 32, smem, st>>>(m1, m2, m3, h1, h2, a);
        else if (small)
            fir_small_kernel<false><<<grid, FW * 32, smem, st>>>(m1, m2, m3, h1, h2, a);
        else if (mode == kTriples)
            fir_kernel<kTriples><<<grid, FW * 32, smem, st>>>(m1, m2, m3, h1, h2, a);
        else if (mode == kInPlace)
            fir_kernel<kInPlace><<<grid, FW * 32, smem, st>>>(m1, m2, m3, h1, h2, a);
        else
            fir_kernel<kSeparate><<<grid, FW * 32, smem, st>>>(m1, m2, m3, h1, h2, a);
        HYENA_TRY(cudaGetLastError(), "fir launch");
        ++launches;
    }
    if (a.hist_out != nullptr && a.K > 1) {
        const int H = a.K - 1;
        if (a.hist_in == a.hist_out && a.L > 0 && a.L < H) {
            const int threads = a.B * (a.D / 2);
            fir_history_kernel<<<(threads + 255) / 256, 256, 0, st>>>(a);
        } else {
            const long long threads = static_cast<long long>(a.B) * H * (a.D / 2);
            fir_history_rows_kernel<<<static_cast<unsigned int>((threads + 255) / 256), 256, 0, st>>>(a);
        }
        HYENA_TRY(cudaGetLastError(), "fir history launch");
        ++launches;
    }
    return launches;
}

}  // namespace hyena
