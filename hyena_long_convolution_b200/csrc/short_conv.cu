// short_conv.cu -- explicit short causal FIR (hcs: 7 taps, hcm: 128 taps)
// with the fused Hyena gates, on sm_100a.
//
// Operator (Evo2-7B-262K model card, §Implementation Notes: "Block dispatch"
// names FIR cascades of inner length 7 and 128; "Custom cache" and the
// Evo1-1.5-7B-8K card's "Cache subclass" carry the FIR window):
//   v[t] = x1[t] x2[t];  conv[t] = sum_{k<K} taps[c,k] v[t-k];
//   y[t] = x3[t] conv[t] + Dskip[c] v[t].
//
// Filters longer than 8 taps (hcm) are bound by their FP32 arithmetic (K
// FMAs per channel-token against 8 bytes), so their kernel is built to keep
// the FMA pipe busy: a persistent grid, one CTA per SM, in which each CTA
// walks a contiguous range of tiles of FCH = 64 channels x FT = 128 tokens in
// (batch row, channel group, time) order.  v = x1 x2 lives in a ring of two
// tiles of fp32 rows, so a tile's window history is the previous tile's v,
// converted once; the taps are converted to fp32 once per channel group; and
// TMA requests the x1/x2/x3 rows of the tile after next while the current one
// computes.  Warp w computes FRW = 16 consecutive outputs for the lane's two
// channels with a register-blocked window: per block of 8 taps it issues
// 8 x 16 packed f32x2 FMAs on the 8 taps and 23 window values, 15 of them
// carried over in registers from the previous block.  The gates are applied
// in registers and y is stored as coalesced 128-byte rows.  Every output's
// FMAs run in lag order from a zero accumulator, in every kernel of this
// file, so results do not depend on tiling, chunking or the kernel chosen.
// A second small kernel writes hist_out (the last K-1 values of v).
//
// Inputs come as three tensors, as one packed projection buffer whose rows
// hold channel groups [x1 | x2 | x3] (4-D tensor maps address a group's
// column), or as per-channel triples (x1_c, x2_c, x3_c adjacent; one box of
// 3 x 64 interleaved values per row).
#include "hyena_device.cuh"
#include "hyena_internal.h"

namespace hyena {

namespace {

constexpr int kRowWords = FCH / 2;  // 32-bit words per bf16 row

// Tap k of this lane's channel pair (fp32 pairs [K][32] in shared memory).
struct TapsF32 {
    const float2 *t;
    __device__ __forceinline__ float2 operator()(int k, int lane) const { return t[k * 32 + lane]; }
};

// v rows of the persistent kernel, relative to the current tile's first row:
// the window history (the previous tile) always sits directly before it, so
// every row of a warp's window is a fixed offset from one base address.
struct TileRows {
    const float2 *cur;
    __device__ __forceinline__ float2 operator()(int r, int lane) const { return cur[r * 32 + lane]; }
};

// Accumulates taps [kb, kb + NQ) into acc for this warp's FRW outputs, whose
// first output is token row0.
template <int NQ, class Rows, class Taps>
__device__ __forceinline__ void fir_block(float2 (&acc)[FRW], const Rows &vr, const Taps &taps, int row0, int kb,
                                          int lane)
{
    float2 tq[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) tq[q] = taps(kb + q, lane);
    float2 w[FRW + NQ - 1];  // tokens row0 - kb - (NQ-1) ..
#pragma unroll
    for (int j = 0; j < FRW + NQ - 1; ++j) w[j] = vr(row0 - kb - (NQ - 1) + j, lane);
#pragma unroll
    for (int q = 0; q < NQ; ++q)
#pragma unroll
        for (int i = 0; i < FRW; ++i) acc[i] = __ffma2_rn(tq[q], w[i - q + NQ - 1], acc[i]);
}

// Taps [0, 8*nblk) in blocks of 8 with the window sliding along the taps in
// registers: block kb uses tokens [row0 - kb - 7, row0 - kb + 15]; the next
// block reuses 15 of those 23 values and loads 8, which halves the
// shared-memory traffic per FMA.  NBLK > 0: the block count is a compile-time
// constant and the window shift is register renaming; NBLK == 0: runtime
// count, the shift is register moves.
template <int NBLK, class Rows, class Taps>
__device__ __forceinline__ void fir_sliding8(float2 (&acc)[FRW], const Rows &vr, const Taps &taps, int row0,
                                             int nblk, int lane)
{
    constexpr int NW = FRW + 7;
    if (NBLK > 0) nblk = NBLK;
    float2 w[NW];
#pragma unroll
    for (int j = 0; j < NW; ++j) w[j] = vr(row0 - 7 + j, lane);
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
            for (int j = 0; j < 8; ++j) w[j] = vr(row0 - kb - 15 + j, lane);
        }
    }
}

// conv for this warp's FRW outputs (first output token row0), all K taps in
// lag order.
template <class Rows, class Taps>
__device__ __forceinline__ void fir_conv(float2 (&acc)[FRW], const Rows &vr, const Taps &taps, int row0, int K,
                                         int lane)
{
    const int nblk = K / 8;
    if (nblk == HYENA_MAX_TAPS / 8)
        fir_sliding8<HYENA_MAX_TAPS / 8>(acc, vr, taps, row0, nblk, lane);
    else if (nblk > 0)
        fir_sliding8<0>(acc, vr, taps, row0, nblk, lane);
    const int kb = nblk * 8;
    switch (K - kb) {
        case 7: fir_block<7>(acc, vr, taps, row0, kb, lane); break;
        case 6: fir_block<6>(acc, vr, taps, row0, kb, lane); break;
        case 5: fir_block<5>(acc, vr, taps, row0, kb, lane); break;
        case 4: fir_block<4>(acc, vr, taps, row0, kb, lane); break;
        case 3: fir_block<3>(acc, vr, taps, row0, kb, lane); break;
        case 2: fir_block<2>(acc, vr, taps, row0, kb, lane); break;
        case 1: fir_block<1>(acc, vr, taps, row0, kb, lane); break;
        default: break;
    }
}

// Shared memory of the persistent kernel: four areas of FT v rows; the x1/x2
// rows of the next tile to convert (two [FT][32] word blocks, then the first
// x3 slot; triples: FT interleaved rows of 96 words holding x3 as well); a
// block of [FT][32] words (the second x3 slot; triples: the x3 words of the
// tile being finished); the taps as fp32 pairs; three barriers.
constexpr int kVAreas = 4;
constexpr int kX12Words = 3 * FT * kRowWords;  // sized for the interleaved rows
constexpr int kX3Words = FT * kRowWords;

__host__ __device__ inline size_t fir_stream_smem_bytes(int K)
{
    return static_cast<size_t>(kVAreas * FT) * 32 * sizeof(float2) +
           static_cast<size_t>(kX12Words + kX3Words) * 4 + static_cast<size_t>(K) * 32 * sizeof(float2) +
           3 * sizeof(uint64_t);
}

// taps[c, 0..K) of this CTA's 64 channels -> fp32 pairs [K][32].
__device__ __forceinline__ void fir_load_taps(float2 *taps, const FirArgs &A, int cb)
{
    const int K = A.K;
    if ((K & 7) == 0) {
        // 8 consecutive taps of one channel per 16-byte load
        for (int idx = threadIdx.x; idx < (K / 8) * 32; idx += blockDim.x) {
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
                taps[(kb + 2 * i) * 32 + l] =
                    make_float2(__uint_as_float(wa[i] << 16), __uint_as_float(wb[i] << 16));
                taps[(kb + 2 * i + 1) * 32 + l] =
                    make_float2(__uint_as_float(wa[i] & 0xffff0000u), __uint_as_float(wb[i] & 0xffff0000u));
            }
        }
    } else {
        for (int idx = threadIdx.x; idx < K * 32; idx += blockDim.x) {
            const int k = idx >> 5, l = idx & 31;
            const int c = cb * FCH + 2 * l;
            uint32_t ha = 0u, hb = 0u;
            if (c < A.D) {
                ha = A.taps[static_cast<size_t>(c) * K + k];
                hb = A.taps[static_cast<size_t>(c + 1) * K + k];
            }
            taps[idx] = make_float2(__uint_as_float(ha << 16), __uint_as_float(hb << 16));
        }
    }
}

// v[t] for channels c0, c0 + 1 of batch row b read from global memory: x1 x2
// for t >= 0, hist_in for -H <= t < 0, zero before that.
__device__ __forceinline__ float2 fir_v_global(const FirArgs &A, int b, int t, int c0)
{
    const int H = A.K - 1;
    if (t >= 0) {
        const size_t row = (static_cast<size_t>(b) * A.L + t) * A.ld_x;
        const size_t i0 = row + x_col(c0, A.group), i1 = row + x_col(c0 + 1, A.group);
        const float2 x1 = make_float2(__uint_as_float(static_cast<uint32_t>(A.x1[i0]) << 16),
                                      __uint_as_float(static_cast<uint32_t>(A.x1[i1]) << 16));
        const float2 x2 = make_float2(__uint_as_float(static_cast<uint32_t>(A.x2[i0]) << 16),
                                      __uint_as_float(static_cast<uint32_t>(A.x2[i1]) << 16));
        return __fmul2_rn(x1, x2);
    }
    if (t >= -H && A.hist_in != nullptr)
        return *reinterpret_cast<const float2 *>(A.hist_in + (static_cast<size_t>(b) * H + (H + t)) * A.D + c0);
    return make_float2(0.f, 0.f);
}

// Position of a tile: batch row b, channel group cb, time tile j.  Tiles are
// ordered (b, cb, j) with j fastest.
struct FirTile {
    int b, cb, j;
    __device__ __forceinline__ void advance(int NT, int nCB)
    {
        if (++j == NT) {
            j = 0;
            if (++cb == nCB) {
                cb = 0;
                ++b;
            }
        }
    }
};

// Persistent kernel for K > 8 (see the top of the file).  Of the
// T = B * ceil(D/64) * ceil(L/FT) tiles, CTA g takes [g T / G, (g+1) T / G).
//
// v rows live in four areas of FT rows, P0..P3; a tile reads its history and
// its own rows from two adjacent areas, at phase 0 from (P0, P1), at phase 1
// from (P1, P2), at phase 2 from (P2, P3).  While a tile is computed nobody
// reads the area that the next tile's rows go to: phase 0 writes them to P2,
// phase 1 to P3 and to P0 (the history of a phase-0 tile), phase 2 to P1.
// So each warp converts the next tile's rows right after its own outputs,
// and one barrier per tile separates a tile from the next.  A new sequence
// starts at phase 0 with its history from global memory in P0.
//
// TMA requests (thread 0, after the barrier that ends a tile): the x1/x2 rows
// (separate or packed inputs; the interleaved rows for triples) of the next
// tile to convert go to one slot, requested once the tile before it in that
// slot has been converted.  Separate or packed inputs: the x3 rows of the
// m-th tile, requested once the outputs of tile m - 1 are stored (one slot),
// or for filters of at most 32 taps once those of tile m - 2 are (two slots,
// slot m & 1; kTwoX3).  Triples: the conversion copies a tile's x3 words to a
// buffer of their own.
template <bool kTri, bool kTwoX3>
__global__ void __launch_bounds__(FW * 32, 1)
    fir_stream_kernel(const __grid_constant__ CUtensorMap tm1, const __grid_constant__ CUtensorMap tm2,
                      const __grid_constant__ CUtensorMap tm3, const FirArgs A)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    float2 *v = reinterpret_cast<float2 *>(smem_raw);                    // [kVAreas FT][32]
    uint32_t *x12 = reinterpret_cast<uint32_t *>(v + kVAreas * FT * 32);  // [kX12Words]
    uint32_t *x3s = x12 + kX12Words;                                      // [FT][32]
    float2 *taps = reinterpret_cast<float2 *>(x3s + kX3Words);            // [K][32]
    uint64_t *bar12 = reinterpret_cast<uint64_t *>(taps + A.K * 32);
    uint64_t *bar3 = bar12 + 1;  // [2], one per x3 slot
    // x3 rows of the m-th tile of the range.  Separate or packed inputs with
    // short filters: two slots, so that a tile's x3 is requested a whole tile
    // ahead (their tiles compute too quickly to cover the request otherwise);
    // measured slower for long filters, which keep one slot.
    static_assert(!(kTri && kTwoX3), "triples keep their x3 words in one buffer");
    auto x3slot = [&](int m) { return (kTwoX3 && !(m & 1)) ? x12 + 2 * FT * kRowWords : x3s; };
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nCB = (A.D + FCH - 1) / FCH;
    const int NT = (A.L + FT - 1) / FT;
    const long long T = static_cast<long long>(A.B) * nCB * NT;
    const long long u0 = T * blockIdx.x / gridDim.x;
    const int n = static_cast<int>(T * (blockIdx.x + 1) / gridDim.x - u0);
    if (n <= 0) return;
    FirTile first;
    {
        const long long seq = u0 / NT;
        first.j = static_cast<int>(u0 - seq * NT);
        first.b = static_cast<int>(seq / nCB);
        first.cb = static_cast<int>(seq - static_cast<long long>(first.b) * nCB);
    }

    // thread 0 only: requests, in tile order
    FirTile next12 = first, next3 = first;  // the next tile whose x1/x2 (x3) rows to request
    int issued12 = 0, issued3 = 0;         // requests made so far
    auto issue12 = [&]() {
        const int ch = next12.cb * FCH, t0 = next12.j * FT;
        if constexpr (kTri) {
            mbar_arrive_expect_tx(bar12, static_cast<uint32_t>(FT * 3 * kRowWords * 4));
            tma_load_4d(x12, &tm1, bar12, 3 * ch, 0, t0, next12.b);
        } else {
            const int cx = ch % A.group, cg = ch / A.group;
            mbar_arrive_expect_tx(bar12, static_cast<uint32_t>(2 * FT * kRowWords * 4));
            tma_load_4d(x12, &tm1, bar12, cx, cg, t0, next12.b);
            tma_load_4d(x12 + FT * kRowWords, &tm2, bar12, cx, cg, t0, next12.b);
        }
        next12.advance(NT, nCB);
        ++issued12;
    };
    auto issue3 = [&]() {
        if constexpr (!kTri) {
            const int ch = next3.cb * FCH, cx = ch % A.group, cg = ch / A.group;
            uint64_t *bar = kTwoX3 ? bar3 + (issued3 & 1) : bar3;
            mbar_arrive_expect_tx(bar, static_cast<uint32_t>(FT * kRowWords * 4));
            tma_load_4d(x3slot(issued3), &tm3, bar, cx, cg, next3.j * FT, next3.b);
            next3.advance(NT, nCB);
            ++issued3;
        }
    };
    if (tid == 0) {
        mbar_init(bar12, 1);
        mbar_init(bar3, 1);
        mbar_init(bar3 + 1, 1);
        fence_mbar_init();
        issue12();
        issue3();
        if (kTwoX3 && n > 1) issue3();
    }
    __syncthreads();

    int waited12 = 0;  // waits completed (every thread, in the same order)
    // v of a tile's FT rows from the x1/x2 slot into area `dst` (and into P0
    // with `copy`); triples also move the x3 words to their slot.  Rows past
    // L and channels past D are the tensor maps' zero fill.
    auto convert = [&](float2 *dst, bool copy) {
        const bool ok = mbar_wait_bounded(bar12, waited12 & 1);
        ++waited12;
        float2 cv[FRW];
#pragma unroll
        for (int i = 0; i < FRW; ++i) {
            const int r = warp * FRW + i;
            if constexpr (kTri) {
                const uint32_t *rw = x12 + r * 3 * kRowWords + 3 * lane;
                const uint32_t w0 = rw[0], w1 = rw[1], w2 = rw[2];
                cv[i] = __fmul2_rn(tri_x1(w0, w1), tri_x2(w0, w2));
                x3s[r * kRowWords + lane] = __byte_perm(w1, w2, 0x7610);
            } else {
                cv[i] = __fmul2_rn(bf16x2_to_float2(x12[r * kRowWords + lane]),
                                   bf16x2_to_float2(x12[(FT + r) * kRowWords + lane]));
            }
        }
#pragma unroll
        for (int i = 0; i < FRW; ++i) dst[(warp * FRW + i) * 32 + lane] = cv[i];
        if (copy) {
#pragma unroll
            for (int i = 0; i < FRW; ++i) v[(warp * FRW + i) * 32 + lane] = cv[i];
        }
        return ok;
    };

    FirTile q = first;
    int phase = 0;
    float2 dsk = make_float2(0.f, 0.f);
    bool ok = true;
    for (int k = 0; k < n; ++k) {
        const int t0 = q.j * FT;
        const int c0 = q.cb * FCH + 2 * lane;
        const bool ch_ok = c0 < A.D;
        if (k == 0 || q.j == 0) {
            // A new sequence: its taps and Dskip, the FT tokens before t0 (the
            // window history) from global memory into P0, its first tile's
            // rows into P1.
            fir_load_taps(taps, A, q.cb);
            dsk = (A.Dskip != nullptr && ch_ok) ? make_float2(A.Dskip[c0], A.Dskip[c0 + 1]) : make_float2(0.f, 0.f);
            const int th = t0 - FT + warp * FRW;  // this warp's first history token
            float2 hv[FRW];
            if (th >= 0 && ch_ok) {
                // all rows from x1, x2: every load issued before the first use
                const size_t row = (static_cast<size_t>(q.b) * A.L + th) * A.ld_x;
                const long long i0 = x_col(c0, A.group), i1 = x_col(c0 + 1, A.group);
                uint32_t h1[FRW], h2[FRW];
#pragma unroll
                for (int i = 0; i < FRW; ++i) {
                    const size_t ri = row + static_cast<size_t>(i) * A.ld_x;
                    h1[i] = static_cast<uint32_t>(A.x1[ri + i0]) | (static_cast<uint32_t>(A.x1[ri + i1]) << 16);
                    h2[i] = static_cast<uint32_t>(A.x2[ri + i0]) | (static_cast<uint32_t>(A.x2[ri + i1]) << 16);
                }
#pragma unroll
                for (int i = 0; i < FRW; ++i) hv[i] = __fmul2_rn(bf16x2_to_float2(h1[i]), bf16x2_to_float2(h2[i]));
            } else {
#pragma unroll
                for (int i = 0; i < FRW; ++i)
                    hv[i] = ch_ok ? fir_v_global(A, q.b, th + i, c0) : make_float2(0.f, 0.f);
            }
#pragma unroll
            for (int i = 0; i < FRW; ++i) v[(warp * FRW + i) * 32 + lane] = hv[i];
            ok = convert(v + FT * 32, false) && ok;
            phase = 0;
            if (__syncthreads_or(!ok)) break;
            if (tid == 0 && issued12 < n) {  // the x1/x2 slot is free again
                fence_proxy_async_smem();
                issue12();
            }
        }
        float2 *cur = v + (1 + phase) * FT * 32;

        float2 acc[FRW];
#pragma unroll
        for (int i = 0; i < FRW; ++i) acc[i] = make_float2(0.f, 0.f);
        const TileRows vr{cur};
        fir_conv(acc, vr, TapsF32{taps}, warp * FRW, A.K, lane);

        // outputs: y = x3 conv + Dskip v
        if constexpr (!kTri) {
            ok = (kTwoX3 ? mbar_wait_bounded(bar3 + (k & 1), (k >> 1) & 1) : mbar_wait_bounded(bar3, k & 1)) && ok;
        }
        const int row0 = t0 + warp * FRW;  // this warp's first output token
        const int nvalid = min(FRW, A.L - row0);
        uint32_t *yrow = reinterpret_cast<uint32_t *>(A.y + (static_cast<size_t>(q.b) * A.L + row0) * A.ld_y + c0);
        const size_t ystride = static_cast<size_t>(A.ld_y) / 2;
        auto y_of = [&](int i) {
            const int r = warp * FRW + i;
            const float2 x3 = bf16x2_to_float2(x3slot(k)[r * kRowWords + lane]);
            return float2_to_bf16x2(__ffma2_rn(dsk, vr(r, lane), __fmul2_rn(x3, acc[i])));
        };
        if (ok) {
            if (nvalid == FRW && ch_ok) {
                uint32_t yw[FRW];
#pragma unroll
                for (int i = 0; i < FRW; ++i) yw[i] = y_of(i);
#pragma unroll
                for (int i = 0; i < FRW; ++i) yrow[i * ystride] = yw[i];
            } else if (ch_ok) {
#pragma unroll
                for (int i = 0; i < FRW; ++i)
                    if (i < nvalid) yrow[i * ystride] = y_of(i);
            }
        }

        // the next tile's rows, when it continues this sequence
        FirTile nq = q;
        nq.advance(NT, nCB);
        const bool chained = k + 1 < n && nq.j != 0;
        if (chained) {
            float2 *dst = v + (phase == 0 ? 2 : phase == 1 ? 3 : 1) * FT * 32;
            ok = convert(dst, phase == 1) && ok;
        }
        // every read of this tile's areas and of both slots is done
        if (__syncthreads_or(!ok)) break;
        if (tid == 0) {
            fence_proxy_async_smem();
            if (chained && issued12 < n) issue12();
            if (issued3 < n) issue3();
        }
        phase = chained ? (phase == 2 ? 0 : phase + 1) : 0;
        q = nq;
    }
    if (!ok && tid == 0) {
        // rows never arrived: wait (bounded) for the last request on each
        // barrier (every earlier one was consumed before a later one went
        // out); the outputs of this tile and of the rest of the range stay
        // unwritten
        if (issued12 > 0) (void)mbar_wait_bounded(bar12, (issued12 - 1) & 1);
        if (kTwoX3) {
            for (int m = issued3 > 2 ? issued3 - 2 : 0; m < issued3; ++m)
                (void)mbar_wait_bounded(bar3 + (m & 1), (m >> 1) & 1);
        } else if (issued3 > 0) {
            (void)mbar_wait_bounded(bar3, (issued3 - 1) & 1);
        }
    }
}

// Short filters (K <= 8, halo of at most 8 rows; hcs) are bound by HBM, not
// by arithmetic: one CTA per tile of 64 channels x FT tokens, many CTAs per
// SM.  The window values are formed from the bf16 x1, x2 rows as they are used
// instead of from an fp32 v buffer, and each warp computes its 16 outputs in
// two halves of 8.  That keeps the CTA at 53 KB of shared memory and at most
// 64 registers, four CTAs per SM.  kTri: the rows are the interleaved
// per-channel triples (96 words per row), read the same way.  The FMA order per
// output is the persistent kernel's (taps in lag order from a zero
// accumulator).
constexpr int kSmallMaxK = 8;
static_assert(kSmallMaxK == 8, "fir_persistent() routes filters of more than 8 taps away");
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
        static int configured_device = -1;
        static int sm_count = 0;
        int dev = 0;
        HYENA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
        if (configured_device != dev) {
            HYENA_TRY(cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, dev), "SM count");
            const int smax = static_cast<int>(fir_stream_smem_bytes(HYENA_MAX_TAPS));
            HYENA_TRY(cudaFuncSetAttribute(fir_stream_kernel<false, false>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smax),
                      "fir: set max dynamic shared memory");
            HYENA_TRY(cudaFuncSetAttribute(fir_stream_kernel<false, true>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smax),
                      "fir: set max dynamic shared memory");
            HYENA_TRY(cudaFuncSetAttribute(fir_stream_kernel<true, false>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smax),
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
        if (!fir_persistent(a.K)) {
            const size_t smem = fir_small_smem_bytes(a.HR, a.K, triples);
            const dim3 grid((a.D + FCH - 1) / FCH, (a.L + FT - 1) / FT, a.B);
            if (triples)
                fir_small_kernel<true><<<grid, FW * 32, smem, st>>>(m1, m2, m3, h1, h2, a);
            else
                fir_small_kernel<false><<<grid, FW * 32, smem, st>>>(m1, m2, m3, h1, h2, a);
        } else {
            // one CTA per SM over all tiles (fewer when there are fewer tiles)
            const long long tiles = static_cast<long long>(a.B) * ((a.D + FCH - 1) / FCH) * ((a.L + FT - 1) / FT);
            const unsigned int grid = static_cast<unsigned int>(tiles < sm_count ? tiles : sm_count);
            const size_t smem = fir_stream_smem_bytes(a.K);
            if (triples)
                fir_stream_kernel<true, false><<<grid, FW * 32, smem, st>>>(m1, m2, m3, a);
            else if (a.K <= 32)
                fir_stream_kernel<false, true><<<grid, FW * 32, smem, st>>>(m1, m2, m3, a);
            else
                fir_stream_kernel<false, false><<<grid, FW * 32, smem, st>>>(m1, m2, m3, a);
        }
        HYENA_TRY(cudaGetLastError(), "fir launch");
        ++launches;
    }
    const int nh = launch_fir_history(a, st);
    if (nh < 0) return -1;
    return launches + nh;
}

int launch_fir_history(const FirArgs &a, cudaStream_t st)
{
    if (a.hist_out == nullptr || a.K <= 1) return 0;
    const int H = a.K - 1;
    if (a.hist_in == a.hist_out && a.L > 0 && a.L < H) {
        const int threads = a.B * (a.D / 2);
        fir_history_kernel<<<(threads + 255) / 256, 256, 0, st>>>(a);
    } else {
        const long long threads = static_cast<long long>(a.B) * H * (a.D / 2);
        fir_history_rows_kernel<<<static_cast<unsigned int>((threads + 255) / 256), 256, 0, st>>>(a);
    }
    HYENA_TRY(cudaGetLastError(), "fir history launch");
    return 1;
}

}  // namespace hyena
