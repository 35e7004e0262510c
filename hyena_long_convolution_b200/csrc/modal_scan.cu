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
// Work decomposition.  The time axis is cut into units of MT tokens; a unit
// covers MCH channels of one batch row (a "chain" is the sequence of units of
// one batch row and channel block).  Units are handed out by an atomic ticket
// in time-major order, so every unit's predecessor in its chain holds a
// smaller ticket and is running or finished: forward progress never depends
// on scheduling.  Inside a unit, warp w owns tokens [w*MS, (w+1)*MS) and lane
// l the channel pair (2l, 2l+1) (packed f32x2 arithmetic).
//
// Per unit:
//   phase A  each warp runs the N recurrences from a zero state over its MS
//            tokens, leaving its end state Z_w, and writes v = x1 x2 back over
//            the x1/x2 words it read (v.x over x1, v.y over x2);
//   combine  a Horner pass over the warps' end states gives the unit
//            aggregate A (A = sum_w p^(MS (MW-1-w)) Z_w);
//   look-back  A is published (ring slot, flag AGG); predecessors' flags are
//            read back to the nearest inclusive prefix, and the carry C into
//            the unit is rebuilt forward with exactly the operations the chain
//            itself performs (C_{j+1} = p^MT C_j + A_j), so the result does not
//            depend on timing: the kernel is bitwise deterministic.
//            INCL = p^MT C + A is published; the warps' start states follow
//            from a second Horner pass over the Z_w seeded with C
//            (S_0 = C, S_{w+1} = p^MS S_w + Z_w);
//   phase C  each warp reruns its recurrences from S_w and emits
//            y = x3 * sum_n R_n s_n + Dskip v straight from registers
//            (coalesced 128-byte rows); the final state goes to state_out.
//
// Pipeline (one persistent CTA per SM: 8 compute warps, a control warp and a
// publisher warp).  The control warp takes tickets, keeps a 3-stage ring of
// TMA-staged x1/x2 tiles and coefficient blocks full and performs the
// look-backs; the publisher warp releases every aggregate as soon as it is
// written; the compute warps run phase A of unit k, then phase C of unit k-1
// whose carry the control warp produced meanwhile.  x3 is needed only in
// phase C and is read straight from global memory, prefetched into registers
// one phase ahead.  Neither the loads nor the look-back sit on the compute
// warps' critical path.
//
// Ring: each chain owns MRING slots; unit g writes slot g % MRING.  The
// look-back never goes deeper than MLB units (it waits for an INCL at depth
// MLB), and before writing, unit g checks that units g-MRING .. g-MLB are
// finished, so a slot is never overwritten while someone may still read it.
// Flags are 64-bit: (epoch << 32) | (unit << 1) | is_inclusive.  The epoch
// lives in the workspace and advances at the end of every launch, so stale
// flags from earlier launches never match and a captured CUDA graph can be
// replayed.  Every wait is bounded (about one second of %globaltimer) and
// records an error bit instead of hanging; once an error bit is set all other
// waits give up at once.
#include "hyena_device.cuh"
#include "hyena_internal.h"

namespace hyena {

namespace {

constexpr int kTileWords = MT * MCH / 2;  // 32-bit words per bf16 tile
constexpr int kTileBytes = MT * MCH * 2;
constexpr int kStages = 3;
constexpr int kCompute = MW * 32;         // compute threads
constexpr int kThreads = kCompute + 64;   // + control warp + publisher warp
constexpr int kCtrlWarp = MW;
constexpr int kPubWarp = MW + 1;

template <int NP>
struct ModalSmem {
    uint32_t x12[kStages][2][kTileWords];    // x1 (then v.x), x2 (then v.y)
    float coef[kStages][3 * NP + 1][MCH];    // p, R, p^MS, Dskip of the unit's channels
    float2 z[2][MW * NP * 32];               // Z_w, then start states S_w
    float2 agg[2][NP * 32];                  // unit aggregate
    float2 carry[2][NP * 32];                // carry into the unit
    uint64_t full[kStages];                  // stage landed (TMA transaction bytes)
    uint64_t empty[kStages];                 // compute warps done with a stage
    uint64_t idrdy[kStages];                 // unit id of a stage is known
    uint64_t aggrdy[2];                      // aggregate written (compute -> control, publisher)
    uint64_t srdy[2];                        // carry written (control -> compute)
    uint64_t slotok[2];                      // ring slot may be written (publisher -> compute)
    uint64_t aggpub[2];                      // aggregate flag released (publisher -> control)
    int unit[kStages];
};

template <int NP>
__host__ __device__ constexpr uint32_t stage_tx_bytes()
{
    return 2u * kTileBytes + static_cast<uint32_t>((3 * NP + 1) * MCH * 4);
}

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

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Bounded wait for TMA completion; records an error bit on timeout.  It does
// not give up early on other errors: the copies land whatever else happens,
// and the CTA must not leave while they are in flight.
__device__ __forceinline__ bool mbar_wait_tiles(uint64_t *bar, uint32_t parity, unsigned int *hdr)
{
    if (mbar_wait_bounded(bar, parity)) return true;
    atomicOr(hdr + 2, kErrTmaTimeout);
    return false;
}

// Bounded wait on a hand-off between the CTA's own warps; gives up at once if
// an error has already been recorded anywhere, so a failure ends the launch
// quickly instead of timing out wait after wait.
__device__ __forceinline__ bool mbar_wait_or_flag(uint64_t *bar, uint32_t parity, unsigned int *hdr)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_timer_ns();
    for (unsigned int it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0u) {
            if (ld_volatile_u32(hdr + 2) != 0u) return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                atomicOr(hdr + 2, kErrTmaTimeout);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void compute_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kCompute) : "memory"); }

// Store of one bf16x2 word, predicated without a branch.
__device__ __forceinline__ void st_pred_u32(uint32_t *p, uint32_t v, bool pred)
{
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q st.global.b32 [%0], %1;\n\t}" ::"l"(p),
        "r"(v), "r"(pred ? 1u : 0u)
        : "memory");
}

// Read-only 32-bit load, predicated (returns 0 when pred is false).
__device__ __forceinline__ uint32_t ld_pred_nc_u32(const void *p, bool pred)
{
    uint32_t v;
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\tmov.u32 %0, 0;\n\t@q ld.global.nc.b32 %0, [%1];\n\t}"
        : "=r"(v)
        : "l"(p), "r"(pred ? 1u : 0u));
    return v;
}

struct UnitPos {
    int cb, b;
    unsigned int g;
};

__device__ __forceinline__ UnitPos unit_pos(unsigned int u, const ModalArgs &A)
{
    UnitPos q;
    q.cb = static_cast<int>(u % static_cast<unsigned int>(A.nCB));
    q.b = static_cast<int>((u / static_cast<unsigned int>(A.nCB)) % static_cast<unsigned int>(A.B));
    q.g = u / (static_cast<unsigned int>(A.B) * A.nCB);
    return q;
}

template <int NP>
__device__ __forceinline__ float2 coef2(const ModalSmem<NP> &sm, int st, int row, int lane)
{
    return *reinterpret_cast<const float2 *>(&sm.coef[st][row][2 * lane]);
}

// ------------------------------------------------------------------ control warp
// Fills the stage of pipeline iteration `it` with the next ticket's x1/x2
// tiles and coefficient block, or with an end marker once the tickets are
// exhausted (control warp, all lanes).
template <int NP>
__device__ __forceinline__ void issue_stage(ModalSmem<NP> &sm, const CUtensorMap *tm1,
                                            const CUtensorMap *tm2, const CUtensorMap *tmc,
                                            const ModalArgs &A, int it, bool &ended)
{
    const int st = it % kStages;
    if ((threadIdx.x & 31) == 0) {
        unsigned int t = A.nUnits;
        if (!ended) {
            t = atomicAdd(A.hdr, 1u);
            if (ld_volatile_u32(A.hdr + 2) != 0u) t = A.nUnits;  // an error: stop early
        }
        if (t >= A.nUnits) {
            ended = true;
            sm.unit[st] = -1;
            mbar_arrive(&sm.idrdy[st]);
            mbar_arrive(&sm.full[st]);
        } else {
            sm.unit[st] = static_cast<int>(t);
            mbar_arrive(&sm.idrdy[st]);
            const UnitPos q = unit_pos(t, A);
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&sm.full[st], stage_tx_bytes<NP>());
            tma_load_3d(sm.x12[st][0], tm1, &sm.full[st], q.cb * MCH, static_cast<int>(q.g) * MT, q.b);
            tma_load_3d(sm.x12[st][1], tm2, &sm.full[st], q.cb * MCH, static_cast<int>(q.g) * MT, q.b);
            tma_load_2d(&sm.coef[st][0][0], tmc, &sm.full[st], q.cb * MCH, 0);
        }
    }
    ended = __shfl_sync(0xffffffffu, ended ? 1 : 0, 0) != 0;
}

template <int NP>
__device__ void control_warp(ModalSmem<NP> &sm, const CUtensorMap *tm1, const CUtensorMap *tm2,
                             const CUtensorMap *tmc, const ModalArgs &A, unsigned int epoch)
{
    const int lane = threadIdx.x & 31;
    bool ended = false;
    issue_stage<NP>(sm, tm1, tm2, tmc, A, 0, ended);
    issue_stage<NP>(sm, tm1, tm2, tmc, A, 1, ended);
    issue_stage<NP>(sm, tm1, tm2, tmc, A, 2, ended);
    for (int k = 0;; ++k) {
        const int st = k % kStages;
        __syncwarp();
        const int us = sm.unit[st];  // written by lane 0 of this warp
        if (us < 0) break;
        const unsigned int u = static_cast<unsigned int>(us);
        const UnitPos q = unit_pos(u, A);
        const unsigned int g = q.g;
        const int b = q.b;
        const int c0 = q.cb * MCH + 2 * lane;
        const unsigned int chain = static_cast<unsigned int>(b) * A.nCB + q.cb;
        unsigned long long *chain_flags = A.flags + static_cast<size_t>(chain) * MRING;
        float *chain_slots = A.slots + static_cast<size_t>(chain) * MRING * 2 * NP * MCH;
        float2 pT[NP];
#pragma unroll
        for (int n = 0; n < NP; ++n) pT[n] = ldg_f2(A.cPT + static_cast<size_t>(n) * A.Dp + c0);

        // ---------------- look-back: carry C into this unit
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
            const unsigned int floor_unit = g > static_cast<unsigned int>(MLB) ? g - MLB : 0u;
            const unsigned int depth = g - floor_unit;  // 1 .. MLB
            // Lane i watches unit g-1-i.  Wait until the nearest inclusive
            // prefix is visible and every unit after it has an aggregate.
            const unsigned long long t0 = global_timer_ns();
            unsigned int jincl = 0;
            bool ok = true;
            for (unsigned int it = 0;; ++it) {
                bool avail = false, incl = false;
                if (static_cast<unsigned int>(lane) < depth) {
                    const unsigned int j = g - 1u - lane;
                    const unsigned long long f = ld_acquire_u64(chain_flags + (j % MRING));
                    avail = (f >> 32) == epoch && ((f & 0xffffffffull) >> 1) == j;
                    incl = avail && (f & 1ull);
                }
                const unsigned int mi = __ballot_sync(0xffffffffu, incl);
                const unsigned int ma = __ballot_sync(0xffffffffu, avail);
                if (mi != 0u) {
                    const int first = __ffs(mi) - 1;  // nearest inclusive prefix
                    const unsigned int need = first == 0 ? 0u : ((1u << first) - 1u);
                    if ((ma & need) == need) {
                        jincl = g - 1u - static_cast<unsigned int>(first);
                        break;
                    }
                }
                __nanosleep(64);
                if ((it & 63u) == 63u) {
                    // warp-uniform decision: every lane leaves the loop together
                    const bool stop = __any_sync(0xffffffffu, ld_volatile_u32(A.hdr + 2) != 0u ||
                                                                  global_timer_ns() - t0 > kWaitLimitNs);
                    if (stop) {
                        if (lane == 0) atomicOr(A.hdr + 2, kErrLookbackTimeout);
                        ok = false;
                        break;
                    }
                }
            }
            // The flags were acquired by several lanes; the warp barrier
            // orders those acquires before every lane's slot reads, which go
            // to L2 (never a stale L1 line of an earlier use of the slot).
            __syncwarp();
            const float *inc_src = chain_slots + (static_cast<size_t>(jincl % MRING) * 2 + 1) * NP * MCH + 2 * lane;
#pragma unroll
            for (int n = 0; n < NP; ++n)
                cin[n] = ok ? __ldcg(reinterpret_cast<const float2 *>(inc_src + n * MCH)) : make_float2(0.f, 0.f);
            // Forward pass over the aggregates after the inclusive prefix; the
            // next slot's values are loaded while the current one is folded.
            if (ok && jincl + 1u < g) {
                float2 nxt[NP];
                const float *src = chain_slots + static_cast<size_t>((jincl + 1u) % MRING) * 2 * NP * MCH + 2 * lane;
#pragma unroll
                for (int n = 0; n < NP; ++n) nxt[n] = __ldcg(reinterpret_cast<const float2 *>(src + n * MCH));
                for (unsigned int jj = jincl + 1u; jj < g; ++jj) {
                    const bool more = jj + 1u < g;
                    const float *s2 = chain_slots + static_cast<size_t>((jj + 1u) % MRING) * 2 * NP * MCH + 2 * lane;
#pragma unroll
                    for (int n = 0; n < NP; ++n) {
                        cin[n] = __ffma2_rn(pT[n], cin[n], nxt[n]);
                        if (more) nxt[n] = __ldcg(reinterpret_cast<const float2 *>(s2 + n * MCH));
                    }
                }
            }
        }

        // The carry goes to the compute warps first; the inclusive prefix is
        // published after.
#pragma unroll
        for (int n = 0; n < NP; ++n) sm.carry[k & 1][n * 32 + lane] = cin[n];
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.srdy[k & 1]);

        // ---------------- inclusive prefix (the carry into unit g + 1)
        // A sequence that ends exactly on a unit boundary takes its final
        // state from this same expression, so chunks made of whole units
        // reproduce the single pass bit for bit.
        (void)mbar_wait_or_flag(&sm.aggrdy[k & 1], (k >> 1) & 1, A.hdr);
        {
            float *slot = chain_slots + static_cast<size_t>(g % MRING) * 2 * NP * MCH + 2 * lane;
            const bool last_full = (g + 1u) * static_cast<unsigned int>(MT) == static_cast<unsigned int>(A.L);
            const bool write_state = last_full && A.state_out != nullptr && c0 < A.D;
#pragma unroll
            for (int n = 0; n < NP; ++n) {
                const float2 inc = __ffma2_rn(pT[n], cin[n], sm.agg[k & 1][n * 32 + lane]);
                *reinterpret_cast<float2 *>(slot + NP * MCH + n * MCH) = inc;
                if (write_state && n < A.N) {
                    A.state_out[(static_cast<size_t>(b) * A.D + c0) * A.N + n] = inc.x;
                    A.state_out[(static_cast<size_t>(b) * A.D + c0 + 1) * A.N + n] = inc.y;
                }
            }
            // The inclusive flag must land after the publisher's aggregate
            // flag on the same word.
            (void)mbar_wait_or_flag(&sm.aggpub[k & 1], (k >> 1) & 1, A.hdr);
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release_u64(chain_flags + (g % MRING), flag_word(epoch, g, true));
        }

        // Refill the stage that phase C of the previous unit is releasing.
        if (k >= 1) {
            (void)mbar_wait_or_flag(&sm.empty[(k - 1) % kStages], ((k - 1) / kStages) & 1, A.hdr);
            issue_stage<NP>(sm, tm1, tm2, tmc, A, k + 2, ended);
        }
    }
}

// ------------------------------------------------------------------ publisher warp
// Releases every unit's aggregate as soon as the compute warps have written it,
// independently of any look-back, so successors in the chain can skip over a
// unit long before its inclusive prefix is known.  It also guards the ring:
// before the compute warps may write slot g % MRING, units g-MRING .. g-MLB of
// the chain must be finished.
template <int NP>
__device__ void publisher_warp(ModalSmem<NP> &sm, const ModalArgs &A, unsigned int epoch)
{
    const int lane = threadIdx.x & 31;
    for (int k = 0;; ++k) {
        const int st = k % kStages;
        (void)mbar_wait_or_flag(&sm.idrdy[st], (k / kStages) & 1, A.hdr);
        const int us = sm.unit[st];
        if (us < 0) break;
        const UnitPos q = unit_pos(static_cast<unsigned int>(us), A);
        const unsigned int g = q.g;
        const unsigned int chain = static_cast<unsigned int>(q.b) * A.nCB + q.cb;
        unsigned long long *chain_flags = A.flags + static_cast<size_t>(chain) * MRING;
        if (g >= static_cast<unsigned int>(MLB) && lane <= MRING - MLB) {
            const long long j = static_cast<long long>(g) - MRING + lane;
            if (j >= 0) {
                const unsigned long long need = flag_word(epoch, static_cast<unsigned int>(j), true);
                unsigned long long f;
                (void)spin_flag(chain_flags + (j % MRING), A.hdr, kErrRingTimeout, f,
                                [&](unsigned long long x) {
                                    return (x >> 32) == epoch && (x & 0xffffffffull) >= (need & 0xffffffffull);
                                });
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.slotok[k & 1]);
        (void)mbar_wait_or_flag(&sm.aggrdy[k & 1], (k >> 1) & 1, A.hdr);
        if (g > 0u) {
            // The compute warps' slot writes happen-before this point (mbarrier
            // release/acquire); the fence and release store order them before
            // the flag for any reader that acquires it.
            __threadfence();
            if (lane == 0) st_release_u64(chain_flags + (g % MRING), flag_word(epoch, g, false));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.aggpub[k & 1]);
    }
}

// ------------------------------------------------------------------ compute warps
// One token of phase C for this lane's channel pair: advance the N states,
// form conv = sum_n R_n s_n with four independent accumulation chains (all
// state updates first, so the chains find their inputs ready), apply the
// gates and store y.
template <int NP>
__device__ __forceinline__ void phase_c_token(float2 (&s)[NP], const float2 (&p)[NP], const float2 (&R)[NP],
                                              float2 dsk, const uint32_t *r1, const uint32_t *r2,
                                              uint32_t x3w, uint32_t *yrow, size_t ystride, int i, bool ch_ok)
{
    const float2 v = make_float2(__uint_as_float(r1[i * 32]), __uint_as_float(r2[i * 32]));
    const float2 x3 = bf16x2_to_float2(x3w);
#pragma unroll
    for (int n = 0; n < NP; ++n) s[n] = __ffma2_rn(p[n], s[n], v);
    float2 a0 = __fmul2_rn(R[0], s[0]);
    float2 a1 = __fmul2_rn(R[1], s[1]);
    float2 a2 = __fmul2_rn(R[2], s[2]);
    float2 a3 = __fmul2_rn(R[3], s[3]);
#pragma unroll
    for (int n = 4; n < NP; n += 4) {
        a0 = __ffma2_rn(R[n], s[n], a0);
        a1 = __ffma2_rn(R[n + 1], s[n + 1], a1);
        a2 = __ffma2_rn(R[n + 2], s[n + 2], a2);
        a3 = __ffma2_rn(R[n + 3], s[n + 3], a3);
    }
    const float2 conv = __fadd2_rn(__fadd2_rn(a0, a1), __fadd2_rn(a2, a3));
    const float2 yv = __ffma2_rn(dsk, v, __fmul2_rn(x3, conv));
    st_pred_u32(yrow + i * ystride, float2_to_bf16x2(yv), ch_ok);
}

template <int NP>
__device__ void compute_warps(ModalSmem<NP> &sm, const ModalArgs &A)
{
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    constexpr int kModesPerWarp = (NP + MW - 1) / MW;
    int prev = -1;  // unit of the previous iteration

    for (int k = 0;; ++k) {
        const int st = k % kStages;

        // x3 of the previous unit (its phase C runs later in this iteration),
        // prefetched into registers.
        uint32_t x3r[MS];
        int ptw0 = 0, pnvalid = 0, pc0 = 0, pb = 0;
        bool pch_ok = false;
        if (prev >= 0) {
            const UnitPos q = unit_pos(static_cast<unsigned int>(prev), A);
            pc0 = q.cb * MCH + 2 * lane;
            pb = q.b;
            ptw0 = static_cast<int>(q.g) * MT + warp * MS;
            pnvalid = min(MS, A.L - ptw0);
            pch_ok = pc0 < A.D;
            const uint16_t *x3p = A.x3 + (static_cast<size_t>(pb) * A.L + ptw0) * A.ld_x + pc0;
#pragma unroll
            for (int i = 0; i < MS; ++i) x3r[i] = ld_pred_nc_u32(x3p + i * A.ld_x, pch_ok && i < pnvalid);
        }

        (void)mbar_wait_tiles(&sm.full[st], (k / kStages) & 1, A.hdr);
        const int u = sm.unit[st];

        if (u >= 0) {
            // ---------------- phase A: end state of each warp's sub-segment
            float2 p[NP], sA[NP];
#pragma unroll
            for (int n = 0; n < NP; ++n) {
                p[n] = coef2(sm, st, n, lane);
                sA[n] = make_float2(0.f, 0.f);
            }
            uint32_t *r1 = sm.x12[st][0] + warp * MS * 32 + lane;
            uint32_t *r2 = sm.x12[st][1] + warp * MS * 32 + lane;
#pragma unroll 4
            for (int i = 0; i < MS; ++i) {
                const float2 v = __fmul2_rn(bf16x2_to_float2(r1[i * 32]), bf16x2_to_float2(r2[i * 32]));
                r1[i * 32] = __float_as_uint(v.x);
                r2[i * 32] = __float_as_uint(v.y);
#pragma unroll
                for (int n = 0; n < NP; ++n) sA[n] = __ffma2_rn(p[n], sA[n], v);
            }
            float2 *zk = sm.z[k & 1];
#pragma unroll
            for (int n = 0; n < NP; ++n) zk[(warp * NP + n) * 32 + lane] = sA[n];
            compute_bar();

            // ---------------- combine: aggregate A of the unit
            float2 accs[kModesPerWarp];
#pragma unroll
            for (int j = 0; j < kModesPerWarp; ++j) {
                const int n = warp + j * MW;
                float2 acc = make_float2(0.f, 0.f);
                if (n < NP) {
                    const float2 ps = coef2(sm, st, 2 * NP + n, lane);
#pragma unroll
                    for (int w = 0; w < MW; ++w) acc = __ffma2_rn(ps, acc, zk[(w * NP + n) * 32 + lane]);
                    sm.agg[k & 1][n * 32 + lane] = acc;
                }
                accs[j] = acc;
            }
            // The aggregate also goes to this unit's ring slot (once the
            // publisher warp has found the slot free); the publisher releases
            // the flag as soon as every warp has written its part.
            {
                const UnitPos q = unit_pos(static_cast<unsigned int>(u), A);
                const unsigned int chain = static_cast<unsigned int>(q.b) * A.nCB + q.cb;
                float *slot = A.slots + (static_cast<size_t>(chain) * MRING + q.g % MRING) * 2 * NP * MCH + 2 * lane;
                (void)mbar_wait_or_flag(&sm.slotok[k & 1], (k >> 1) & 1, A.hdr);
#pragma unroll
                for (int j = 0; j < kModesPerWarp; ++j) {
                    const int n = warp + j * MW;
                    if (n < NP) *reinterpret_cast<float2 *>(slot + n * MCH) = accs[j];
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.aggrdy[k & 1]);
        }

        // ---------------- phase C of the previous unit
        if (prev >= 0) {
            const int kp = k - 1;
            const int sp = kp % kStages;
            (void)mbar_wait_or_flag(&sm.srdy[kp & 1], (kp >> 1) & 1, A.hdr);
            // Start states: S_0 = C, S_{w+1} = p^MS S_w + Z_w (in place over Z).
            float2 *zp = sm.z[kp & 1];
#pragma unroll
            for (int j = 0; j < kModesPerWarp; ++j) {
                const int n = warp + j * MW;
                if (n < NP) {
                    const float2 ps = coef2(sm, sp, 2 * NP + n, lane);
                    float2 S = sm.carry[kp & 1][n * 32 + lane];
#pragma unroll
                    for (int w = 0; w < MW; ++w) {
                        float2 *q = &zp[(w * NP + n) * 32 + lane];
                        const float2 zv = *q;
                        *q = S;
                        S = __ffma2_rn(ps, S, zv);
                    }
                }
            }
            compute_bar();
            float2 p[NP], R[NP], s[NP];
#pragma unroll
            for (int n = 0; n < NP; ++n) {
                s[n] = zp[(warp * NP + n) * 32 + lane];
                p[n] = coef2(sm, sp, n, lane);
                R[n] = coef2(sm, sp, NP + n, lane);
            }
            const float2 dsk = coef2(sm, sp, 3 * NP, lane);
            const uint32_t *r1 = sm.x12[sp][0] + warp * MS * 32 + lane;
            const uint32_t *r2 = sm.x12[sp][1] + warp * MS * 32 + lane;
            uint32_t *yrow = reinterpret_cast<uint32_t *>(A.y + (static_cast<size_t>(pb) * A.L + ptw0) * A.ld_y + pc0);
            const size_t ystride = static_cast<size_t>(A.ld_y) / 2;  // in 32-bit words
            if (pnvalid == MS) {
                // whole sub-segment: branch-free so consecutive tokens interleave
#pragma unroll
                for (int i = 0; i < MS; ++i)
                    phase_c_token<NP>(s, p, R, dsk, r1, r2, x3r[i], yrow, ystride, i, pch_ok);
            } else {
#pragma unroll
                for (int i = 0; i < MS; ++i)
                    if (i < pnvalid) phase_c_token<NP>(s, p, R, dsk, r1, r2, x3r[i], yrow, ystride, i, pch_ok);
            }
            // A ragged last unit: the final state is the recurrence state
            // after token L-1 (the unit's aggregate covers padded rows).
            if (A.state_out != nullptr && pch_ok && (A.L % MT) != 0 && ptw0 <= A.L - 1 && A.L - 1 < ptw0 + MS) {
#pragma unroll
                for (int n = 0; n < NP; ++n) {
                    if (n < A.N) {
                        A.state_out[(static_cast<size_t>(pb) * A.D + pc0) * A.N + n] = s[n].x;
                        A.state_out[(static_cast<size_t>(pb) * A.D + pc0 + 1) * A.N + n] = s[n].y;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[sp]);
        }
        if (u < 0) break;
        prev = u;
        compute_bar();
    }
}

template <int NP>
__global__ void __launch_bounds__(kThreads, 1)
    modal_scan_kernel(const __grid_constant__ CUtensorMap tm1,
                      const __grid_constant__ CUtensorMap tm2,
                      const __grid_constant__ CUtensorMap tmc, const ModalArgs A)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    ModalSmem<NP> &sm = *reinterpret_cast<ModalSmem<NP> *>(smem_raw);
    // Flags carry the launch's epoch: the workspace keeps a counter that the
    // last CTA of every launch advances, so flags left by earlier launches
    // (including replays of a captured graph) never match.
    const unsigned int epoch = ld_volatile_u32(A.hdr + 3) + 1u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], MW);
            mbar_init(&sm.idrdy[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.aggrdy[s], MW);
            mbar_init(&sm.srdy[s], 1);
            mbar_init(&sm.slotok[s], 1);
            mbar_init(&sm.aggpub[s], 1);
        }
        fence_mbar_init();
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5;
    if (warp == kCtrlWarp)
        control_warp<NP>(sm, &tm1, &tm2, &tmc, A, epoch);
    else if (warp == kPubWarp)
        publisher_warp<NP>(sm, A, epoch);
    else
        compute_warps<NP>(sm, A);

    // Every TMA this CTA issued has been waited on by the compute warps.
    __syncthreads();
    // The last CTA to leave resets the ticket and advances the epoch so the
    // workspace is ready for the next launch without a memset.
    if (threadIdx.x == 0) {
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

// Coefficient synthesis: p = exp(a), p^MS, p^MT in fp32 from the fp32 log-poles
// (CUDA's expf), residues and skip copied, padded modes and channels zero.
template <int NP>
__global__ void modal_synth_kernel(const ModalSynthArgs S)
{
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= NP * S.Dp) return;
    const int n = idx / S.Dp;
    const int c = idx - n * S.Dp;
    const bool valid = c < S.D && n < S.N;
    const float a = valid ? S.log_poles[static_cast<size_t>(c) * S.N + n] : 0.f;
    const size_t row = static_cast<size_t>(S.Dp);
    S.coef[n * row + c] = valid ? expf(a) : 0.f;
    S.coef[(NP + n) * row + c] = valid ? S.residues[static_cast<size_t>(c) * S.N + n] : 0.f;
    S.coef[(2 * NP + n) * row + c] = valid ? expf(a * static_cast<float>(MS)) : 0.f;
    S.cPT[n * row + c] = valid ? expf(a * static_cast<float>(MT)) : 0.f;
    if (n == 0) S.coef[3 * NP * row + c] = (c < S.D && S.Dskip != nullptr) ? S.Dskip[c] : 0.f;
}

template <int NP>
int launch_modal_np(const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &mc,
                    const ModalArgs &a, const ModalSynthArgs &s, cudaStream_t st)
{
    static int configured_device = -1;
    static int sms = 0, per_sm = 0;
    int dev = 0;
    HYENA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
    const int smem = static_cast<int>(sizeof(ModalSmem<NP>));
    if (configured_device != dev) {
        HYENA_TRY(cudaFuncSetAttribute(modal_scan_kernel<NP>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
                  "modal scan: set max dynamic shared memory");
        HYENA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "multiprocessor count");
        HYENA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, modal_scan_kernel<NP>, kThreads, smem),
                  "modal scan: occupancy");
        if (per_sm < 1) per_sm = 1;
        configured_device = dev;
    }
    const int total = NP * s.Dp;
    modal_synth_kernel<NP><<<(total + 255) / 256, 256, 0, st>>>(s);
    HYENA_TRY(cudaGetLastError(), "modal synth launch");
    const unsigned int grid = static_cast<unsigned int>(
        a.nUnits < static_cast<unsigned int>(sms * per_sm) ? a.nUnits : static_cast<unsigned int>(sms * per_sm));
    modal_scan_kernel<NP><<<grid, kThreads, smem, st>>>(m1, m2, mc, a);
    HYENA_TRY(cudaGetLastError(), "modal scan launch");
    return 2;
}

}  // namespace

int launch_modal(const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &mc,
                 const ModalArgs &a, const ModalSynthArgs &s, int NP, cudaStream_t st)
{
    switch (NP) {
        case 4: return launch_modal_np<4>(m1, m2, mc, a, s, st);
        case 8: return launch_modal_np<8>(m1, m2, mc, a, s, st);
        case 16: return launch_modal_np<16>(m1, m2, mc, a, s, st);
        default: return -1;
    }
}

}  // namespace hyena
