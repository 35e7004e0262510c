// fir_dft.cu -- the explicit FIR (hcs / hcm, K <= 128 taps) as DFT-as-GEMM on
// the sm_100a tensor cores: a second implementation of the operator of
// short_conv.cu, for comparison with its FP32 SIMT kernels.
//
// Operator (Evo2-7B-262K model card, §Implementation Notes: "Block dispatch",
// FIR cascades of inner length 7 and 128, and hcl evaluated "via FFT"):
//   v[t] = x1[t] x2[t];  conv[t] = sum_{k<K} taps[c,k] v[t-k];
//   y[t] = x3[t] conv[t] + Dskip[c] v[t].
//
// Overlap-save with a P = 256-point real DFT.  For an output block of 128
// tokens starting at t0 and one channel, the window u[j] = v[t0 - 128 + j],
// j < 256, holds the block and the 128 tokens before it, so the circular
// convolution of u with the zero-padded taps equals the linear one at the
// circular indices n = 128 .. 255.  With a shared real DFT matrix F
// (256 x 256: rows r < 128 give Re U_r = sum_j u_j cos(2 pi r j / 256),
// row 128 the Nyquist term sum_j u_j (-1)^j, rows 128 + r, 0 < r < 128, give
// Im U_r = -sum_j u_j sin(2 pi r j / 256)) and the matching inverse G
// (128 outputs x 256 spectral values), a CTA of 64 channels x 128 tokens does
//   GEMM 0:  Hs = F[:, 0:128] . taps^T      (M = 2 x 128, N = 64, K = 128)
//   GEMM 1:  Us = F . u^T                   (M = 2 x 128, N = 64, K = 256)
//   Z      = Us (x) Hs, bin by bin, on the CUDA cores (complex product)
//   GEMM 2:  conv^T = G . Z^T               (M = 128, N = 64, K = 256)
// with tcgen05.mma kind::tf32 (fp32 accumulators in tensor memory): channels
// are the N dimension, so F and G are shared by every CTA.  Operands are
// rounded to tf32 (11 significant bits) on the way in; the taps (bf16) are
// exact in tf32.  The accumulators in TMEM: Us at columns 0 (Re) and 64 (Im),
// Hs at 128 and 192, conv at 256.  F and G live in global memory in the
// tensor cores' shared-memory layout and stream through a ring of four
// 16 KB slots by bulk copy; one thread issues the copies and the MMAs.
//
// Unlike the SIMT kernels, a result depends on where the 128-token blocks
// start, so chunked calls agree with the single pass to rounding, not bit
// for bit.  Inputs: three tensors or packed channel groups (no triples).
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "hyena_device.cuh"
#include "hyena_internal.h"

namespace hyena {

namespace {

constexpr int kDftP = 256;        // DFT length (window)
constexpr int kDftOut = 128;      // outputs per block
constexpr int kDftCh = 64;        // channels per CTA (the MMA's N)
constexpr int kDftWarps = 4;      // one per TMEM lane quarter
constexpr int kSlotBytes = 16384;
constexpr int kSlots = 4;
constexpr int kFChunks = 16;      // F: 32 K-steps of 8 KB, two per chunk
constexpr int kGChunks = 8;       // G: 32 K-steps of 4 KB, four per chunk
constexpr int kChunks = kFChunks + kGChunks;
constexpr uint32_t kTmemCols = 512;

// F and G in the layout of a K-major tf32 operand without swizzle: for each
// K-step of 8 values, core matrices of 8 rows x 16 bytes, the rows of a
// 128-row half 16 bytes apart (SBO = 128) and the two 4-value columns of the
// K-step 2 KB apart (LBO = 2048).  F: [K-step][half][column][row][4];
// G: [K-step][column][row][4].
__device__ uint32_t g_dft_f[kDftP * kDftP];
__device__ uint32_t g_dft_g[kDftOut * kDftP];

// Shared memory of one CTA (bytes).
constexpr int kOffU = 0;                        // u^T, then Z^T: [32 K-steps][2][64 rows][16 B] = 64 KB
constexpr int kOffT = kOffU + 65536;            // taps^T [16 K-steps][2][64][16 B] = 32 KB
constexpr int kOffRaw = kOffT + 32768;          // x1, x2 window [256 rows][64 ch] bf16, then x3 = 64 KB
constexpr int kOffRing = kOffRaw + 65536;       // four 16 KB slots
constexpr int kOffBar = kOffRing + kSlots * kSlotBytes;
constexpr int kDftSmem = kOffBar + 128;

__device__ __forceinline__ uint32_t to_tf32(float f)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(f));
    return r;
}

// Byte offset of element (row, k) of a K-major tf32 operand with `rows` rows.
__host__ __device__ __forceinline__ uint32_t kmajor_off(int row, int k, int rows)
{
    return static_cast<uint32_t>((k >> 2) * rows * 16 + row * 16 + (k & 3) * 4);
}

__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo)
{
    return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);  // version 1, no swizzle
}

// D (tmem) (+)= A (smem desc) x B (smem desc), kind::tf32, one thread.
__device__ __forceinline__ void mma_tf32(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, bool acc)
{
    const uint32_t z = 0, en = acc ? 1u : 0u;
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(en), "r"(z), "r"(z), "r"(z), "r"(z));
}

__device__ __forceinline__ void mma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 16 consecutive fp32 columns of this warp's 32 TMEM lanes (one lane per thread).
__device__ __forceinline__ void tmem_ld16(uint32_t addr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(addr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// The issuing thread's view of the ring: chunk i sits in slot i % kSlots;
// it is the (i / kSlots)-th fill of that slot (full barrier phase) and the
// (i / kSlots)-th commit of the MMAs that read it (empty barrier phase).
struct DftRing {
    uint64_t *full, *empty;
    unsigned char *slots;
    int fills[kSlots];  // copies requested per slot
    __device__ void fill(int i)
    {
        const int s = i % kSlots;
        const unsigned char *src = i < kFChunks
                                       ? reinterpret_cast<const unsigned char *>(g_dft_f) + i * kSlotBytes
                                       : reinterpret_cast<const unsigned char *>(g_dft_g) + (i - kFChunks) * kSlotBytes;
        mbar_arrive_expect_tx(full + s, kSlotBytes);
        bulk_load(slots + s * kSlotBytes, src, kSlotBytes, full + s);
        ++fills[s];
    }
};

// One CTA: channels [64 cb, 64 cb + 64) of batch row b, outputs [128 j, 128 j + 128).
__global__ void __launch_bounds__(kDftWarps * 32, 1)
    fir_dft_kernel(const __grid_constant__ CUtensorMap tm1, const __grid_constant__ CUtensorMap tm2,
                   const __grid_constant__ CUtensorMap tm3, const FirArgs A)
{
    extern __shared__ __align__(1024) unsigned char sm[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kOffBar);
    uint64_t *full = bars;                  // [kSlots] ring slot loaded
    uint64_t *empty = bars + kSlots;        // [kSlots] the MMAs reading the slot are done
    uint64_t *xin = bars + 2 * kSlots;      // x1/x2 window arrived
    uint64_t *x3in = xin + 1;               // x3 arrived
    uint64_t *g1 = xin + 2;                 // GEMMs 0 and 1 done
    uint64_t *g2 = xin + 3;                 // GEMM 2 done
    uint64_t *gall = xin + 4;               // every MMA done (error path)
    uint32_t *tslot = reinterpret_cast<uint32_t *>(xin + 5);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cb = blockIdx.x, t0 = blockIdx.y * kDftOut, b = blockIdx.z;
    const int ch = cb * kDftCh;
    const int cx = ch % A.group, cg = ch / A.group;
    const uint32_t *rawp = reinterpret_cast<const uint32_t *>(sm + kOffRaw);  // [256 rows x 32 words] x1, then x2

    DftRing ring{full, empty, sm + kOffRing, {0, 0, 0, 0}};
    bool x3_req = false, mma_issued = false;
    if (tid == 0) {
        for (int i = 0; i < kSlots; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, 1);
        }
        for (int i = 0; i < 5; ++i) mbar_init(xin + i, 1);
        fence_mbar_init();
    }
    __syncthreads();  // every barrier is initialised before anyone waits on it
    if (tid == 0) {
        // the x1, x2 window: rows t0 - 128 .. t0 + 127 (rows before 0 read as zeros)
        mbar_arrive_expect_tx(xin, 4 * 128 * 128);
        tma_load_4d(sm + kOffRaw, &tm1, xin, cx, cg, t0 - 128, b);
        tma_load_4d(sm + kOffRaw + 128 * 128, &tm1, xin, cx, cg, t0, b);
        tma_load_4d(sm + kOffRaw + 256 * 128, &tm2, xin, cx, cg, t0 - 128, b);
        tma_load_4d(sm + kOffRaw + 384 * 128, &tm2, xin, cx, cg, t0, b);
        for (int i = 0; i < kSlots; ++i) ring.fill(i);
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    // taps^T: element (c, k) = taps[ch + c][k] for k < K, else 0 (exact in tf32)
    {
        uint32_t *T = reinterpret_cast<uint32_t *>(sm + kOffT);
        for (int i = tid; i < kDftCh * 128; i += kDftWarps * 32) {
            const int c = i >> 7, k = i & 127;
            float h = 0.f;
            if (k < A.K && ch + c < A.D)
                h = __uint_as_float(static_cast<uint32_t>(A.taps[static_cast<size_t>(ch + c) * A.K + k]) << 16);
            T[kmajor_off(c, k, kDftCh) >> 2] = __float_as_uint(h);
        }
    }
    const bool xin_ok = mbar_wait_bounded(xin, 0);
    bool ok = xin_ok;
    // u^T: element (c, j) = v[t0 - 128 + j] of channel ch + c; before t = 0 the
    // history (hist_in, or zeros).  Tokens more than K - 1 before t0 reach no
    // output (their terms cancel in exact arithmetic) and are set to zero, so
    // that a block's operands are the same whether its history comes from the
    // inputs or from a carried window.
    {
        uint32_t *U = reinterpret_cast<uint32_t *>(sm + kOffU);
        const int H = A.K - 1;
        const int c = 2 * lane;
        for (int j = warp; j < kDftP; j += kDftWarps) {
            const int t = t0 - 128 + j;
            float2 v = make_float2(0.f, 0.f);
            if (t < t0 - H) {
                // outside every window of the block's outputs
            } else if (t >= 0) {
                v = __fmul2_rn(bf16x2_to_float2(rawp[j * 32 + lane]), bf16x2_to_float2(rawp[(256 + j) * 32 + lane]));
            } else if (t >= -H && A.hist_in != nullptr && ch + c < A.D) {
                v = *reinterpret_cast<const float2 *>(A.hist_in + (static_cast<size_t>(b) * H + (H + t)) * A.D + ch + c);
            }
            U[kmajor_off(c, j, kDftCh) >> 2] = to_tf32(v.x);
            U[kmajor_off(c + 1, j, kDftCh) >> 2] = to_tf32(v.y);
        }
    }
    // the tensor cores read u^T and taps^T: make the stores visible to them
    fence_proxy_async_smem();
    tc_fence_before();
    ok = !__syncthreads_or(!ok);
    tc_fence_after();
    const uint32_t tmem = *tslot;
    const uint32_t idesc = (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(kDftCh >> 3) << 17) |
                           (static_cast<uint32_t>(128 >> 4) << 24);
    const uint32_t uaddr = smem_u32(sm + kOffU), taddr = smem_u32(sm + kOffT);
    const uint32_t ring_addr = smem_u32(sm + kOffRing);

    // Thread 0 issues the MMAs of chunks [i0, i1) and refills each slot with
    // chunk i + kSlots once the MMAs of chunk i are done (checked one chunk
    // later, so that the tensor pipe is not drained in between).
    auto issue_chunks = [&](int i0, int i1) {
        for (int i = i0; i < i1; ++i) {
            const int s = i % kSlots;
            if (!mbar_wait_bounded(full + s, (i / kSlots) & 1)) return false;
            tc_fence_after();
            const uint32_t base = ring_addr + s * kSlotBytes;
            if (i < kFChunks) {
                for (int kk = 0; kk < 2; ++kk) {
                    const int ks = 2 * i + kk;  // K-step: samples 8 ks .. 8 ks + 7
                    const uint64_t bu = smem_desc(uaddr + ks * 2048, 1024, 128);
                    for (int h = 0; h < 2; ++h) {
                        const uint64_t af = smem_desc(base + kk * 8192 + h * 4096, 2048, 128);
                        mma_tf32(tmem + 64 * h, af, bu, idesc, ks > 0);
                        if (ks < 16)
                            mma_tf32(tmem + 128 + 64 * h, af, smem_desc(taddr + ks * 2048, 1024, 128), idesc, ks > 0);
                    }
                }
            } else {
                for (int kk = 0; kk < 4; ++kk) {
                    const int ks = 4 * (i - kFChunks) + kk;  // spectral values 8 ks .. 8 ks + 7
                    mma_tf32(tmem + 256, smem_desc(base + kk * 4096, 2048, 128),
                             smem_desc(uaddr + ks * 2048, 1024, 128), idesc, ks > 0);
                }
            }
            mma_issued = true;
            mma_commit(empty + s);
            if (i > i0 && i - 1 + kSlots < kChunks) {
                const int p = i - 1;
                if (!mbar_wait_bounded(empty + p % kSlots, (p / kSlots) & 1)) return false;
                ring.fill(p + kSlots);
            }
        }
        const int p = i1 - 1;
        if (p + kSlots < kChunks) {
            if (!mbar_wait_bounded(empty + p % kSlots, (p / kSlots) & 1)) return false;
            ring.fill(p + kSlots);
        }
        return true;
    };

    if (tid == 0 && ok) {
        // x3 over the history rows of x1 (read by the conversion above)
        mbar_arrive_expect_tx(x3in, 128 * 128);
        tma_load_4d(sm + kOffRaw, &tm3, x3in, cx, cg, t0, b);
        x3_req = true;
        const bool issued = issue_chunks(0, kFChunks);
        if (mma_issued) mma_commit(g1);  // GEMMs 0 and 1 (g1 fires when they are done)
        ok = issued;
    }
    // ---------------- Z = Us (x) Hs, bin by bin; thread = TMEM lane = bin
    const int bin = warp * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    ok = !__syncthreads_or(!ok);  // thread 0 reports whether the first phase was issued
    if (ok) {
        ok = mbar_wait_bounded(g1, 0);
        tc_fence_after();
    }
    if (ok) {
        uint32_t *Z = reinterpret_cast<uint32_t *>(sm + kOffU);  // replaces u^T (GEMM 1 is done)
        for (int c0 = 0; c0 < kDftCh; c0 += 16) {
            float ur[16], ui[16], hr[16], hi[16];
            __syncwarp();  // the TMEM loads are warp-wide
            tmem_ld16(lane_addr + c0, ur);
            tmem_ld16(lane_addr + 64 + c0, ui);
            tmem_ld16(lane_addr + 128 + c0, hr);
            tmem_ld16(lane_addr + 192 + c0, hi);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float zr, zi;
                if (bin == 0) {  // bin 0 and the Nyquist bin are real
                    zr = ur[i] * hr[i];
                    zi = ui[i] * hi[i];
                } else {
                    zr = fmaf(ur[i], hr[i], -ui[i] * hi[i]);
                    zi = fmaf(ur[i], hi[i], ui[i] * hr[i]);
                }
                Z[kmajor_off(c0 + i, bin, kDftCh) >> 2] = to_tf32(zr);
                Z[kmajor_off(c0 + i, 128 + bin, kDftCh) >> 2] = to_tf32(zi);
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    ok = !__syncthreads_or(!ok);
    tc_fence_after();
    if (tid == 0 && ok) {
        ok = issue_chunks(kFChunks, kChunks);  // GEMM 2
        mma_commit(g2);
    }
    ok = !__syncthreads_or(!ok);
    if (ok) {
        ok = mbar_wait_bounded(g2, 0) && mbar_wait_bounded(x3in, 0);
        tc_fence_after();
    }

    // ---------------- y = x3 conv + Dskip v; thread = TMEM lane = output row.
    // The TMEM loads are warp-wide (.sync.aligned): every lane takes part,
    // lanes past L only skip their stores.
    const int r = warp * 32 + lane;  // output t0 + r
    const int t = t0 + r;
    if (ok) {
        const uint32_t *x3w = rawp + r * 32;
        const uint32_t *x1w = rawp + (128 + r) * 32, *x2w = rawp + (256 + 128 + r) * 32;
        uint32_t *yrow = reinterpret_cast<uint32_t *>(A.y + (static_cast<size_t>(b) * A.L + t) * A.ld_y + ch);
        for (int c0 = 0; c0 < kDftCh; c0 += 16) {
            float cv[16];
            __syncwarp();
            tmem_ld16(lane_addr + 256 + c0, cv);
            if (t >= A.L) continue;
            uint32_t out[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int c = c0 + 2 * i;
                const float2 x3 = bf16x2_to_float2(x3w[c / 2]);
                const float2 v = __fmul2_rn(bf16x2_to_float2(x1w[c / 2]), bf16x2_to_float2(x2w[c / 2]));
                float2 d = make_float2(0.f, 0.f);
                if (A.Dskip != nullptr && ch + c < A.D) d = make_float2(A.Dskip[ch + c], A.Dskip[ch + c + 1]);
                out[i] = float2_to_bf16x2(__ffma2_rn(d, v, __fmul2_rn(x3, make_float2(cv[2 * i], cv[2 * i + 1]))));
            }
#pragma unroll
            for (int i = 0; i < 8; i += 4) {
                // D is a multiple of 8: a group of 8 channels is inside D or past it
                if (ch + c0 + 2 * i < A.D)
                    *reinterpret_cast<uint4 *>(yrow + c0 / 2 + i) = make_uint4(out[i], out[i + 1], out[i + 2], out[i + 3]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && !ok) {
        // a wait ran out: every MMA and copy still in flight lands before the
        // tensor memory is freed and the CTA leaves
        if (mma_issued) {
            mma_commit(gall);
            (void)mbar_wait_bounded(gall, 0);
        }
        for (int s = 0; s < kSlots; ++s)
            if (ring.fills[s] > 0) (void)mbar_wait_bounded(full + s, (ring.fills[s] - 1) & 1);
        if (!xin_ok) (void)mbar_wait_bounded(xin, 0);
        if (x3_req) (void)mbar_wait_bounded(x3in, 0);
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

// The F and G tables in double precision, rounded to tf32 (nearest, ties away)
// and laid out as above.
uint32_t host_tf32(double x)
{
    float f = static_cast<float>(x);
    uint32_t u;
    std::memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) != 0x7f800000u) u = (u + 0x1000u) & 0xffffe000u;
    return u;
}

void build_tables(std::vector<uint32_t> &F, std::vector<uint32_t> &G)
{
    const double tau = 2.0 * 3.14159265358979323846;
    F.assign(kDftP * kDftP, 0u);
    G.assign(kDftOut * kDftP, 0u);
    // F row (spectral index) q, column (sample) j
    for (int q = 0; q < kDftP; ++q) {
        for (int j = 0; j < kDftP; ++j) {
            double f;
            if (q < 128)
                f = std::cos(tau * q * j / kDftP);
            else if (q == 128)
                f = (j & 1) ? -1.0 : 1.0;
            else
                f = -std::sin(tau * (q - 128) * j / kDftP);
            const int ks = j >> 3, col = (j >> 2) & 1, half = q >> 7, row = q & 127;
            F[((((ks * 2 + half) * 2 + col) * 128 + row) * 4) + (j & 3)] = host_tf32(f);
        }
    }
    // G row (output o: circular index n = 128 + o), column (spectral index) q
    for (int o = 0; o < kDftOut; ++o) {
        const int n = 128 + o;
        for (int q = 0; q < kDftP; ++q) {
            double g;
            if (q == 0)
                g = 1.0 / kDftP;
            else if (q < 128)
                g = 2.0 * std::cos(tau * q * n / kDftP) / kDftP;
            else if (q == 128)
                g = ((n & 1) ? -1.0 : 1.0) / kDftP;
            else
                g = -2.0 * std::sin(tau * (q - 128) * n / kDftP) / kDftP;
            const int ks = q >> 3, col = (q >> 2) & 1;
            G[(((ks * 2 + col) * 128 + o) * 4) + (q & 3)] = host_tf32(g);
        }
    }
}

}  // namespace

int launch_fir_dft(const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &m3, const FirArgs &a,
                   cudaStream_t st)
{
    int launches = 0;
    if (a.L > 0) {
        // the tables and the kernel attribute, once per device
        static std::mutex mu;
        static std::vector<int> ready;
        int dev = 0;
        HYENA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
        {
            std::lock_guard<std::mutex> lock(mu);
            if (static_cast<int>(ready.size()) <= dev) ready.resize(dev + 1, 0);
            if (!ready[dev]) {
                std::vector<uint32_t> F, G;
                build_tables(F, G);
                HYENA_TRY(cudaMemcpyToSymbol(g_dft_f, F.data(), F.size() * 4), "dft tables");
                HYENA_TRY(cudaMemcpyToSymbol(g_dft_g, G.data(), G.size() * 4), "dft tables");
                HYENA_TRY(cudaFuncSetAttribute(fir_dft_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDftSmem),
                          "fir dft: set max dynamic shared memory");
                ready[dev] = 1;
            }
        }
        const dim3 grid((a.D + kDftCh - 1) / kDftCh, (a.L + kDftOut - 1) / kDftOut, a.B);
        fir_dft_kernel<<<grid, kDftWarps * 32, kDftSmem, st>>>(m1, m2, m3, a);
        HYENA_TRY(cudaGetLastError(), "fir dft launch");
        ++launches;
    }
    const int nh = launch_fir_history(a, st);
    if (nh < 0) return -1;
    return launches + nh;
}

}  // namespace hyena
