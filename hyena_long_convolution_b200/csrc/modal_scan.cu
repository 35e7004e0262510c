// modal_scan.cu -- the long modal-form filter (hcl) as a single-pass,
// decoupled look-back scan over time, on sm_100a.
//
// Operator (Evo2-7B-262K model card, §Architecture and §Implementation Notes:
// an IIR in modal form with fp32 log-poles a and residues R; Evo2-7B-262K
// "Custom cache" and the turboquant-evo2-int4 card's chunked-prefill sections
// for the carried state):
//   v[t] = x1[t] x2[t];  s_n[t] = p_n s_n[t-1] + v[t] with p_n = exp(a_n);
//   y[t] = x3[t] * sum_n R_n s_n[t] + Dskip * v[t].
//
// Design.  The time axis is cut into units of MT tokens; a unit covers MCH
// channels of one batch row.  Units are handed out by an atomic ticket in
// time-major order, so every unit's predecessor (same channels, previous time
// segment) holds a smaller ticket and is running or finished: forward
// progress never depends on scheduling.  Per unit a CTA
//   1. stages x1, x2, x3 tiles [MT x MCH] bf16 with three TMA loads;
//   2. phase A: each warp runs the N recurrences from a zero state over its
//      MS tokens (registers, packed f32x2 FMAs: lane = two channels), leaving
//      its end state Z_w; a short Horner pass over the warps turns the Z_w into
//      per-warp exclusive prefixes E_w and the unit aggregate A;
//   3. publishes A (ring slot, flag AGG), then warp 0 looks back along the
//      chain: predecessors' aggregates are folded in with the decay p^MT until
//      an inclusive prefix (flag INCL) is found; the carry-in C of this unit
//      follows, and INCL = p^MT C + A is published;
//   4. phase C: warp w restarts its recurrences from S_w = p^(MS w) C + E_w and
//      emits y for its tokens straight from registers (coalesced 128-byte rows),
//      writing state_out after the last token of the sequence.
// The state stays fp32 throughout; the carry scan is exact up to fp32
// rounding (no truncation of the decays).
//
// Ring: each chain owns MRING slots; unit g writes slot g % MRING.  Look-back
// never goes deeper than MLB units (it waits for an INCL at depth MLB), and
// before writing, unit g checks that units g-MRING .. g-MLB are finished, so a
// slot is never overwritten while someone may still read it.  Flags are
// 64-bit: (epoch << 32) | (unit << 1) | is_inclusive.  The epoch lives in the
// workspace and advances at the end of every launch, so stale flags from
// earlier launches never match and a captured CUDA graph can be replayed.  Every wait is bounded
// (about one second of %globaltimer) and records an error bit instead of
// hanging; once an error bit is set all other waits give up at once.
#include "hyena_device.cuh"
#include "hyena_internal.h"

namespace hyena {

namespace {

constexpr int kTileWords = MT * MCH / 2;  // 32-bit words per bf16 tile
constexpr int kTileBytes = MT * MCH * 2;

template <int NP>
struct ModalSmem {
    uint32_t x1[kTileWords];
    uint32_t x2[kTileWords];
    uint32_t x3[kTileWords];
    float2 z[MW * NP * 32];  // per-warp end states, then exclusive prefixes
    float2 agg[NP * 32];     // unit aggregate
    float2 carry[NP * 32];   // carry into the unit
    uint64_t bar;
    unsigned int ticket;
    int abort;
};

__device__ __forceinline__ unsigned long long flag_word(unsigned int epoch, unsigned int unit,
                                                        bool incl)
{
    return (static_cast<unsigned long long>(epoch) << 32) |
           (static_cast<unsigned long long>(unit) << 1) | (incl ? 1ull : 0ull);
}

// Spins on a flag until pred(flag) holds.  Returns false if the wait timed out
// or another wait already failed (error bit set).
template <class Pred>
__device__ __forceinline__ bool spin_flag(const unsigned long long *f, unsigned int *hdr,
                                          unsigned int errbit, unsigned long long &val,
                                          Pred pred)
{
    val = ld_acquire_u64(f);
    if (pred(val)) return true;
    const unsigned long long t0 = global_timer_ns();
    unsigned int it = 0;
    for (;;) {
        __nanosleep(32);
        val = ld_acquire_u64(f);
        if (pred(val)) return true;
        if ((++it & 63u) == 0u) {
            if (ld_volatile_u32(hdr + 2) != 0u) return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                atomicOr(hdr + 2, errbit);
                return false;
            }
        }
    }
}

template <int NP>
__global__ void __launch_bounds__(MW * 32, 2)
    modal_scan_kernel(const __grid_constant__ CUtensorMap tm1,
                      const __grid_constant__ CUtensorMap tm2,
                      const __grid_constant__ CUtensorMap tm3, const ModalArgs A)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    ModalSmem<NP> &sm = *reinterpret_cast<ModalSmem<NP> *>(smem_raw);

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    // Flags carry the launch's epoch: the workspace keeps a counter that the
    // last CTA of every launch advances, so flags left by earlier launches
    // (including replays of a captured graph) never match.
    const unsigned int epoch = ld_volatile_u32(A.hdr + 3) + 1u;
    const unsigned int chains = static_cast<unsigned int>(A.B) * A.nCB;

    if (tid == 0) {
        mbar_init(&sm.bar, 1);
        fence_mbar_init();
        sm.abort = 0;
    }
    __syncthreads();

    uint32_t parity = 0;
    for (;;) {
        if (tid == 0) {
            unsigned int t = atomicAdd(A.hdr, 1u);
            if (ld_volatile_u32(A.hdr + 2) != 0u) t = A.nUnits;  // an error: stop early
            sm.ticket = t;
        }
        __syncthreads();
        const unsigned int u = sm.ticket;
        if (u >= A.nUnits) break;

        const int cb = static_cast<int>(u % A.nCB);
        const int b = static_cast<int>((u / A.nCB) % A.B);
        const unsigned int g = u / chains;
        const int t0 = static_cast<int>(g) * MT;
        const unsigned int chain = static_cast<unsigned int>(b) * A.nCB + cb;
        unsigned long long *chain_flags = A.flags + static_cast<size_t>(chain) * MRING;
        float *chain_slots = A.slots + static_cast<size_t>(chain) * MRING * 2 * NP * MCH;

        if (tid == 0) {
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&sm.bar, 3 * kTileBytes);
            tma_load_3d(sm.x1, &tm1, &sm.bar, cb * MCH, t0, b);
            tma_load_3d(sm.x2, &tm2, &sm.bar, cb * MCH, t0, b);
            tma_load_3d(sm.x3, &tm3, &sm.bar, cb * MCH, t0, b);
        }

        // Ring guard: units g-MRING .. g-MLB of this chain must be finished
        // before this unit writes slot g % MRING.
        if (warp == 0 && g >= static_cast<unsigned int>(MLB)) {
            bool ok = true;
            if (lane <= MRING - MLB) {
                const long long j = static_cast<long long>(g) - MRING + lane;
                if (j >= 0) {
                    const unsigned long long need = flag_word(epoch, static_cast<unsigned int>(j), true);
                    unsigned long long f;
                    ok = spin_flag(chain_flags + (j % MRING), A.hdr, kErrRingTimeout, f,
                                   [&](unsigned long long x) {
                                       return (x >> 32) == epoch && (x & 0xffffffffull) >= (need & 0xffffffffull);
                                   });
                }
            }
            (void)ok;  // on failure the error bit is set and the output is invalid
        }

        // This lane's two channels.
        const int c0 = cb * MCH + 2 * lane;

        const bool tiles_ok = mbar_wait_bounded(&sm.bar, parity);
        if (__syncthreads_or(!tiles_ok)) {
            if (tid == 0) atomicOr(A.hdr + 2, kErrTmaTimeout);
            // Let any copy still in flight land before the CTA leaves.
            (void)mbar_wait_bounded(&sm.bar, parity);
            break;
        }
        parity ^= 1u;

        // ---------------- phase A: end state of each warp's sub-segment
        {
            float2 p[NP], s[NP];
#pragma unroll
            for (int n = 0; n < NP; ++n) {
                p[n] = ldg_f2_fresh(A.cP + static_cast<size_t>(n) * A.Dp + c0);
                s[n] = make_float2(0.f, 0.f);
            }
            const uint32_t *r1 = sm.x1 + warp * MS * 32 + lane;
            const uint32_t *r2 = sm.x2 + warp * MS * 32 + lane;
#pragma unroll
            for (int k = 0; k < MS; ++k) {
                const float2 v = __fmul2_rn(bf16x2_to_float2(r1[k * 32]), bf16x2_to_float2(r2[k * 32]));
#pragma unroll
                for (int n = 0; n < NP; ++n) s[n] = __ffma2_rn(p[n], s[n], v);
            }
#pragma unroll
            for (int n = 0; n < NP; ++n) sm.z[(warp * NP + n) * 32 + lane] = s[n];
        }
        __syncthreads();

        // ---------------- combine: exclusive prefixes E_w, aggregate A
#pragma unroll
        for (int j = 0; j < (NP + MW - 1) / MW; ++j) {
            const int n = warp + j * MW;
            if (n < NP) {
                const float2 ps = ldg_f2(A.cPw + (static_cast<size_t>(1) * NP + n) * A.Dp + c0);
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int w = 0; w < MW; ++w) {
                    float2 *zp = &sm.z[(w * NP + n) * 32 + lane];
                    const float2 z = *zp;
                    *zp = acc;
                    acc = __ffma2_rn(ps, acc, z);
                }
                sm.agg[n * 32 + lane] = acc;
                if (g > 0u) {
                    float *dst = chain_slots + (static_cast<size_t>(g % MRING) * 2 + 0) * NP * MCH;
                    *reinterpret_cast<float2 *>(dst + n * MCH + 2 * lane) = acc;
                }
            }
        }
        if (g > 0u) __threadfence();
        __syncthreads();
        if (g > 0u && tid == 0)
            st_release_u64(chain_flags + (g % MRING), flag_word(epoch, g, false));

        // ---------------- look-back (warp 0)
        if (warp == 0) {
            float2 cin[NP];
            if (g == 0u) {
#pragma unroll
                for (int n = 0; n < NP; ++n) {
                    float2 v = make_float2(0.f, 0.f);
                    if (A.state_in != nullptr && n < A.N && c0 < A.D) {
                        v.x = A.state_in[(static_cast<size_t>(b) * A.D + c0) * A.N + n];
                        v.y = A.state_in[(static_cast<size_t>(b) * A.D + c0 + 1) * A.N + n];
                    }
                    cin[n] = v;
                }
            } else {
                // Walk back to the nearest inclusive prefix (never deeper than
                // MLB units), then rebuild the carry forward with exactly the
                // operations the chain itself would perform:
                //   C_{j+1} = p^MT C_j + A_j  (C_j = carry into unit j).
                // The result does not depend on how far the walk went, so the
                // output is bitwise deterministic.
                const unsigned int floor_unit = g > static_cast<unsigned int>(MLB) ? g - MLB : 0u;
                unsigned int j = g - 1u;
                bool ok = true;
                for (;;) {
                    const bool need_incl = (j == floor_unit);
                    unsigned long long f;
                    ok = spin_flag(chain_flags + (j % MRING), A.hdr, kErrLookbackTimeout, f,
                                   [&](unsigned long long x) {
                                       if ((x >> 32) != epoch) return false;
                                       const unsigned long long lo = x & 0xffffffffull;
                                       if ((lo >> 1) != j) return false;
                                       return !need_incl || (lo & 1ull);
                                   });
                    if (!ok || (f & 1ull) != 0ull) break;
                    --j;
                }
                const float *inc_src = chain_slots + (static_cast<size_t>(j % MRING) * 2 + 1) * NP * MCH + 2 * lane;
#pragma unroll
                for (int n = 0; n < NP; ++n)
                    cin[n] = ok ? *reinterpret_cast<const float2 *>(inc_src + n * MCH) : make_float2(0.f, 0.f);
                for (unsigned int jj = j + 1u; ok && jj < g; ++jj) {
                    const float *agg_src = chain_slots + (static_cast<size_t>(jj % MRING) * 2) * NP * MCH + 2 * lane;
#pragma unroll
                    for (int n = 0; n < NP; ++n) {
                        const float2 pT = ldg_f2(A.cPw + (static_cast<size_t>(MW) * NP + n) * A.Dp + c0);
                        cin[n] = __ffma2_rn(pT, cin[n], *reinterpret_cast<const float2 *>(agg_src + n * MCH));
                    }
                }
            }
            // inclusive prefix of this unit: the carry into unit g + 1
            {
                float *dst = chain_slots + (static_cast<size_t>(g % MRING) * 2 + 1) * NP * MCH + 2 * lane;
                // A sequence that ends exactly on a unit boundary takes its
                // final state from this same expression, so that feeding the
                // sequence in chunks of whole units reproduces the single-pass
                // output bit for bit.
                const bool last_full = (g + 1u) * static_cast<unsigned int>(MT) == static_cast<unsigned int>(A.L);
                const bool write_state = last_full && A.state_out != nullptr && c0 < A.D;
#pragma unroll
                for (int n = 0; n < NP; ++n) {
                    const float2 pT = ldg_f2(A.cPw + (static_cast<size_t>(MW) * NP + n) * A.Dp + c0);
                    const float2 inc = __ffma2_rn(pT, cin[n], sm.agg[n * 32 + lane]);
                    *reinterpret_cast<float2 *>(dst + n * MCH) = inc;
                    sm.carry[n * 32 + lane] = cin[n];
                    if (write_state && n < A.N) {
                        A.state_out[(static_cast<size_t>(b) * A.D + c0) * A.N + n] = inc.x;
                        A.state_out[(static_cast<size_t>(b) * A.D + c0 + 1) * A.N + n] = inc.y;
                    }
                }
                __threadfence();
                __syncwarp();
                if (lane == 0) st_release_u64(chain_flags + (g % MRING), flag_word(epoch, g, true));
            }
        }
        __syncthreads();

        // ---------------- phase C: outputs
        {
            float2 p[NP], R[NP], s[NP];
#pragma unroll
            for (int n = 0; n < NP; ++n) {
                const float2 pw = ldg_f2(A.cPw + (static_cast<size_t>(warp) * NP + n) * A.Dp + c0);
                s[n] = __ffma2_rn(pw, sm.carry[n * 32 + lane], sm.z[(warp * NP + n) * 32 + lane]);
                p[n] = ldg_f2_fresh(A.cP + static_cast<size_t>(n) * A.Dp + c0);
                R[n] = ldg_f2_fresh(A.cR + static_cast<size_t>(n) * A.Dp + c0);
            }
            const float2 dsk = ldg_f2_fresh(A.cDs + c0);
            const int tw0 = t0 + warp * MS;
            const int nvalid = min(MS, A.L - tw0);
            const uint32_t *r1 = sm.x1 + warp * MS * 32 + lane;
            const uint32_t *r2 = sm.x2 + warp * MS * 32 + lane;
            const uint32_t *r3 = sm.x3 + warp * MS * 32 + lane;
            const bool ch_ok = c0 < A.D;
            uint32_t *yrow = reinterpret_cast<uint32_t *>(
                A.y + (static_cast<size_t>(b) * A.L + tw0) * A.ld_y + c0);
            const size_t ystride = static_cast<size_t>(A.ld_y) / 2;  // in 32-bit words
#pragma unroll 2
            for (int k = 0; k < MS; ++k) {
                if (k < nvalid) {
                    const float2 v = __fmul2_rn(bf16x2_to_float2(r1[k * 32]), bf16x2_to_float2(r2[k * 32]));
                    float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0, acc2 = acc0, acc3 = acc0;
#pragma unroll
                    for (int n = 0; n < NP; n += 4) {
                        s[n] = __ffma2_rn(p[n], s[n], v);
                        acc0 = __ffma2_rn(R[n], s[n], acc0);
                        s[n + 1] = __ffma2_rn(p[n + 1], s[n + 1], v);
                        acc1 = __ffma2_rn(R[n + 1], s[n + 1], acc1);
                        s[n + 2] = __ffma2_rn(p[n + 2], s[n + 2], v);
                        acc2 = __ffma2_rn(R[n + 2], s[n + 2], acc2);
                        s[n + 3] = __ffma2_rn(p[n + 3], s[n + 3], v);
                        acc3 = __ffma2_rn(R[n + 3], s[n + 3], acc3);
                    }
                    const float2 conv = __fadd2_rn(__fadd2_rn(acc0, acc1), __fadd2_rn(acc2, acc3));
                    const float2 x3 = bf16x2_to_float2(r3[k * 32]);
                    const float2 yv = __ffma2_rn(dsk, v, __fmul2_rn(x3, conv));
                    if (ch_ok) yrow[k * ystride] = float2_to_bf16x2(yv);
                }
            }
            // A ragged last unit: the final state is the recurrence state
            // after token L-1 (the unit's aggregate covers padded rows).
            if (A.state_out != nullptr && ch_ok && (A.L % MT) != 0 && tw0 <= A.L - 1 && A.L - 1 < tw0 + MS) {
#pragma unroll
                for (int n = 0; n < NP; ++n) {
                    if (n < A.N) {
                        A.state_out[(static_cast<size_t>(b) * A.D + c0) * A.N + n] = s[n].x;
                        A.state_out[(static_cast<size_t>(b) * A.D + c0 + 1) * A.N + n] = s[n].y;
                    }
                }
            }
        }
        __syncthreads();
    }

    // The last CTA to leave resets the ticket and advances the epoch so the
    // workspace is ready for the next launch without a memset.
    if (tid == 0) {
        __threadfence();
        const unsigned int done = atomicAdd(A.hdr + 1, 1u);
        if (done == gridDim.x - 1) {
            atomicExch(A.hdr + 0, 0u);
            atomicExch(A.hdr + 1, 0u);
            atomicExch(A.hdr + 3, epoch);
            __threadfence();
        }
    }
}

template <int NP>
__global__ void modal_synth_kernel(const ModalSynthArgs S)
{
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= NP * S.Dp) return;
    const int n = idx / S.Dp;
    const int c = idx - n * S.Dp;
    const bool valid = c < S.D && n < S.N;
    const float a = valid ? S.log_poles[static_cast<size_t>(c) * S.N + n] : 0.f;
    S.cP[idx] = valid ? expf(a) : 0.f;
    S.cR[idx] = valid ? S.residues[static_cast<size_t>(c) * S.N + n] : 0.f;
#pragma unroll
    for (int w = 0; w <= MW; ++w)
        S.cPw[(static_cast<size_t>(w) * NP + n) * S.Dp + c] = valid ? expf(a * static_cast<float>(MS * w)) : 0.f;
    if (n == 0) S.cDs[c] = (c < S.D && S.Dskip != nullptr) ? S.Dskip[c] : 0.f;
}

template <int NP>
int launch_modal_np(const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &m3,
                    const ModalArgs &a, const ModalSynthArgs &s, cudaStream_t st)
{
    static int configured_device = -1;
    static int sms = 0, per_sm = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    const int smem = static_cast<int>(sizeof(ModalSmem<NP>));
    if (configured_device != dev) {
        if (cudaFuncSetAttribute(modal_scan_kernel<NP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem) != cudaSuccess)
            return -1;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, modal_scan_kernel<NP>, MW * 32,
                                                          smem) != cudaSuccess)
            return -1;
        if (per_sm < 1) per_sm = 1;
        configured_device = dev;
    }
    const int total = NP * s.Dp;
    modal_synth_kernel<NP><<<(total + 255) / 256, 256, 0, st>>>(s);
    if (cudaGetLastError() != cudaSuccess) return -1;
    const unsigned int grid = static_cast<unsigned int>(
        a.nUnits < static_cast<unsigned int>(sms * per_sm) ? a.nUnits : static_cast<unsigned int>(sms * per_sm));
    modal_scan_kernel<NP><<<grid, MW * 32, smem, st>>>(m1, m2, m3, a);
    if (cudaGetLastError() != cudaSuccess) return -1;
    return 2;
}

}  // namespace

int launch_modal(const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &m3,
                 const ModalArgs &a, const ModalSynthArgs &s, int NP, cudaStream_t st)
{
    switch (NP) {
        case 4: return launch_modal_np<4>(m1, m2, m3, a, s, st);
        case 8: return launch_modal_np<8>(m1, m2, m3, a, s, st);
        case 16: return launch_modal_np<16>(m1, m2, m3, a, s, st);
        default: return -1;
    }
}

}  // namespace hyena
