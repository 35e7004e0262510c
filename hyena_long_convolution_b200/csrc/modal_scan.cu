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
// Decomposition.  A chain (MCH channels of one batch row) is cut into units
// of MT tokens.  The carry into unit j of a chain follows one canonical
// recurrence, C_0 = state_in, C_{j+1} = p^MT C_j + A_j, where the unit
// aggregate A_j = sum_t p^(MT-1-t) v[t] is the unit's end state from a zero
// start.  Every carry the kernel forms is evaluated by exactly this sequence
// of fp32 operations, whoever evaluates it and however far a look-back
// reaches, so the output is bitwise deterministic and feeding a sequence in
// chunks of whole units reproduces the single pass bit for bit.
//
// Work.  G consecutive units of a chain form a group, handed out by an atomic
// ticket in time-major order (a group's predecessor holds a smaller ticket
// and is running or finished: forward progress never depends on scheduling).
// A CTA has G compute warps and one control warp.  Compute warp w owns unit
// j = s G + w of group s, lane l its channel pair (packed f32x2 arithmetic):
//   A sweep  the warp streams its unit's x1/x2 rows and runs the N
//            recurrences from zero: the aggregate A_j (N FMAs per token);
//   control  the control warp publishes the group's aggregates (ring slot,
//            flag AGG), looks back along the chain to the nearest inclusive
//            prefix, folds the aggregates forward into the group's carry,
//            derives the carry of every unit of the group, hands them to the
//            compute warps and publishes the group's carry-out (flag INCL);
//   C sweep  the warp streams its unit's x1/x2/x3 rows again (x1/x2 come back
//            from L2) and reruns the recurrences from C_j, emitting
//            y = x3 * sum_n R_n s_n + Dskip v as coalesced 128-byte rows
//            (2N FMAs per token).
// Each compute warp streams its rows through its own ring of chunk buffers,
// filled several chunks ahead by the CTA's producer warp with TMA; the compute
// warps publish their own aggregates (the control warp only raises the flag),
// and several CTAs share an SM, so one CTA's look-back overlaps the others'
// sweeps.
//
// Ring of slots: each chain owns MRING group slots; group s writes slot
// s % MRING.  The look-back never goes deeper than MLB groups (it waits for an
// inclusive prefix at depth MLB), and before writing, group s checks that
// groups s-MRING .. s-MLB are finished, so a slot is never overwritten while
// someone may still read it.  Flags are 64-bit: (epoch << 32) | (group << 1) |
// is_inclusive.  The epoch lives in the workspace and advances at the end of
// every launch, so stale flags from earlier launches never match and a
// captured CUDA graph can be replayed.  Every wait is bounded (about one
// second of %globaltimer) and records an error bit instead of hanging; once
// an error bit is set all other waits give up at once.
#include "hyena_device.cuh"
#include "hyena_internal.h"

namespace hyena {

namespace {

constexpr int kChunkWords = MCK * MCH / 2;  // 32-bit words per bf16 chunk of one tensor
constexpr int kChunkBytes = MCK * MCH * 2;
constexpr int kChunksPerSweep = MT / MCK;   // 8
constexpr int kChunksPerGroup = 2 * kChunksPerSweep;

template <int G>
struct GroupTraits {
    static constexpr int kRing = G >= 4 ? 4 : 5;  // chunk buffers per compute warp
    static constexpr int kThreads = 32 * (G + 2);  // compute warps, control warp, producer warp
    static constexpr int kCtasPerSm = G >= 4 ? 2 : 3;
};

template <int NP, int G>
struct GroupSmem {
    uint32_t ring[G][GroupTraits<G>::kRing][3][kChunkWords];  // x1, x2, x3 chunks per compute warp
    float2 ac[G][NP * 32];       // unit aggregate A_j, then (in place) the carry C_j
    uint64_t full[G][GroupTraits<G>::kRing];   // chunk landed (producer TMA -> compute)
    uint64_t empty[G][GroupTraits<G>::kRing];  // chunk consumed (compute -> producer)
    uint64_t gready[2];          // group id known (control -> compute, producer)
    uint64_t slotok[2];          // ring slot may be written (control -> compute)
    uint64_t adone[2];           // aggregates written (compute -> control)
    uint64_t cdone[2];           // carries written (control -> compute)
    int gid[2];
};

__device__ __forceinline__ unsigned long long flag_word(unsigned int epoch, unsigned int group,
                                                        bool incl)
{
    return (static_cast<unsigned long long>(epoch) << 32) |
           (static_cast<unsigned long long>(group) << 1) | (incl ? 1ull : 0ull);
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

// Spins on a flag until pred(flag) holds.  Returns false if the wait timed out
// or another wait already failed (error bit set).
template <class Pred>
__device__ __forceinline__ bool spin_flag(const unsigned long long *f, unsigned int *hdr,
                                          unsigned int errbit, Pred pred)
{
    if (pred(ld_acquire_u64(f))) return true;
    const unsigned long long t0 = global_timer_ns();
    unsigned int it = 0;
    for (;;) {
        __nanosleep(64);
        if (pred(ld_acquire_u64(f))) return true;
        if ((++it & 63u) == 0u) {
            if (ld_volatile_u32(hdr + 2) != 0u) return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                atomicOr(hdr + 2, errbit);
                return false;
            }
        }
    }
}

// Store of one bf16x2 word, predicated without a branch.
__device__ __forceinline__ void st_pred_u32(uint32_t *p, uint32_t v, bool pred)
{
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q st.global.b32 [%0], %1;\n\t}" ::"l"(p),
        "r"(v), "r"(pred ? 1u : 0u)
        : "memory");
}

struct GroupPos {
    int cb, b;
    unsigned int s;  // group index within the chain
};

__device__ __forceinline__ GroupPos group_pos(unsigned int t, const ModalArgs &A)
{
    GroupPos q;
    const unsigned int chains = static_cast<unsigned int>(A.B) * A.nCB;
    const unsigned int chain = t % chains;
    q.s = t / chains;
    q.b = static_cast<int>(chain / static_cast<unsigned int>(A.nCB));
    q.cb = static_cast<int>(chain % static_cast<unsigned int>(A.nCB));
    return q;
}

template <int NP>
__device__ __forceinline__ void load_rows(float2 (&dst)[NP], const float *table, int row0, int Dp, int c0)
{
#pragma unroll
    for (int n = 0; n < NP; ++n) dst[n] = ldg_f2(table + static_cast<size_t>(row0 + n) * Dp + c0);
}

// ------------------------------------------------------------------ control warp
// Takes the next ticket for group iteration k and announces it (lane 0).
template <int NP, int G>
__device__ __forceinline__ void announce_group(GroupSmem<NP, G> &sm, const ModalArgs &A, int k)
{
    if ((threadIdx.x & 31) == 0) {
        unsigned int t = atomicAdd(A.hdr, 1u);
        if (ld_volatile_u32(A.hdr + 2) != 0u) t = A.nGroups;  // an error: stop early
        sm.gid[k & 1] = t < A.nGroups ? static_cast<int>(t) : -1;
        mbar_arrive(&sm.gready[k & 1]);
    }
}

template <int NP, int G, bool kCx>
__device__ void control_warp(GroupSmem<NP, G> &sm, const ModalArgs &A, unsigned int epoch)
{
    const int lane = threadIdx.x & 31;
    const int groups_per_chain = (A.units + G - 1) / G;
    const size_t slot_floats = static_cast<size_t>(MGMAX + 1) * NP * MCH;
    const size_t incl_off = static_cast<size_t>(MGMAX) * NP * MCH;

    // A CTA takes its next ticket when it has formed the carries of its
    // current group: early enough for the producer to prefetch the next
    // group's rows during the current output sweep, late enough that groups
    // start in about ticket order (a look-back then rarely waits on a group
    // that started late) and that short sequences spread over all CTAs.
    constexpr int ahead = 1;
    announce_group<NP, G>(sm, A, 0);
    for (int k = 0;; ++k) {
        __syncwarp();
        const int gi = sm.gid[k & 1];  // written by lane 0 of this warp
        if (gi < 0) break;
        const GroupPos q = group_pos(static_cast<unsigned int>(gi), A);
        const unsigned int s = q.s;
        const int c0 = q.cb * MCH + 2 * lane;
        const unsigned int chain = static_cast<unsigned int>(q.b) * A.nCB + q.cb;
        unsigned long long *chain_flags = A.flags + static_cast<size_t>(chain) * MRING;
        float *chain_slots = A.slots + static_cast<size_t>(chain) * MRING * slot_floats;
        float *slot = chain_slots + static_cast<size_t>(s % MRING) * slot_floats + 2 * lane;
        const int j0 = static_cast<int>(s) * G;              // first unit of the group
        const int nvalid_units = min(G, A.units - j0);       // units of the group inside L
        const bool has_successor = static_cast<int>(s) + 1 < groups_per_chain;
        float2 pT[NP];
        load_rows<NP>(pT, A.coef, 2 * NP + 1, A.Dp, c0);

        // Ring guard: groups s-MRING .. s-MLB must be finished before this
        // group's slot s % MRING is written.
        if (s >= static_cast<unsigned int>(MRING) && lane <= MRING - MLB) {
            const unsigned int jg = s - MRING + lane;
            const unsigned long long need = flag_word(epoch, jg, true) & 0xffffffffull;
            (void)spin_flag(chain_flags + (jg % MRING), A.hdr, kErrRingTimeout, [&](unsigned long long x) {
                return (x >> 32) == epoch && (x & 0xffffffffull) >= need;
            });
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.slotok[k & 1]);

        // ---------------- publish the group's unit aggregates (flag AGG)
        // Each compute warp wrote its unit's aggregate to the slot and fenced
        // before arriving; the release store orders all of them before the
        // flag for any reader that acquires it.
        (void)mbar_wait_or_flag(&sm.adone[k & 1], (k >> 1) & 1, A.hdr);
        if (s > 0u && has_successor && lane == 0)
            st_release_u64(chain_flags + (s % MRING), flag_word(epoch, s, false));

        // ---------------- look-back: the carry into the group's first unit
        float2 C[NP];
        if (s == 0u) {
#pragma unroll
            for (int n = 0; n < NP; ++n) {
                float2 v = make_float2(0.f, 0.f);
                if (A.state_in != nullptr && n < A.N && c0 < A.D) {
                    v.x = A.state_in[(static_cast<size_t>(q.b) * A.D + c0) * A.N + n];
                    v.y = A.state_in[(static_cast<size_t>(q.b) * A.D + c0 + 1) * A.N + n];
                }
                C[n] = v;
            }
        } else {
            const unsigned int floor_g = s > static_cast<unsigned int>(MLB) ? s - MLB : 0u;
            const unsigned int depth = s - floor_g;  // 1 .. MLB
            // Lane i watches group s-1-i: wait until the nearest inclusive
            // prefix is visible and every group after it has its aggregates.
            const unsigned long long t0 = global_timer_ns();
            unsigned int jincl = 0;
            bool ok = true;
            for (unsigned int it = 0;; ++it) {
                bool avail = false, incl = false;
                if (static_cast<unsigned int>(lane) < depth) {
                    const unsigned int jg = s - 1u - lane;
                    const unsigned long long f = ld_acquire_u64(chain_flags + (jg % MRING));
                    avail = (f >> 32) == epoch && ((f & 0xffffffffull) >> 1) == jg;
                    incl = avail && (f & 1ull);
                }
                const unsigned int mi = __ballot_sync(0xffffffffu, incl);
                const unsigned int ma = __ballot_sync(0xffffffffu, avail);
                if (mi != 0u) {
                    const int first = __ffs(mi) - 1;  // nearest inclusive prefix
                    const unsigned int need = first == 0 ? 0u : ((1u << first) - 1u);
                    if ((ma & need) == need) {
                        jincl = s - 1u - static_cast<unsigned int>(first);
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
            const float *inc = chain_slots + static_cast<size_t>(jincl % MRING) * slot_floats + incl_off + 2 * lane;
#pragma unroll
            for (int n = 0; n < NP; ++n)
                C[n] = ok ? __ldcg(reinterpret_cast<const float2 *>(inc + n * MCH)) : make_float2(0.f, 0.f);
            // Fold the skipped groups' unit aggregates forward, unit by unit
            // (the canonical chain).
            for (unsigned int jg = jincl + 1u; ok && jg < s; ++jg) {
                const float *src = chain_slots + static_cast<size_t>(jg % MRING) * slot_floats + 2 * lane;
                for (int w = 0; w < G; w += 2) {
                    // two units' aggregates in flight at once
                    float2 a[NP], b2[NP];
#pragma unroll
                    for (int n = 0; n < NP; ++n) {
                        a[n] = __ldcg(reinterpret_cast<const float2 *>(src + (static_cast<size_t>(w) * NP + n) * MCH));
                        b2[n] = __ldcg(reinterpret_cast<const float2 *>(src + (static_cast<size_t>(w + 1) * NP + n) * MCH));
                    }
                    modes_carry<NP, kCx>(C, pT, a);
                    modes_carry<NP, kCx>(C, pT, b2);
                }
            }
        }

        // ---------------- carries of the group's units (in place over A_j)
        {
            const bool whole_last = (A.L % MT) == 0;
            for (int w = 0; w < nvalid_units; ++w) {
                float2 a[NP];
#pragma unroll
                for (int n = 0; n < NP; ++n) {
                    a[n] = sm.ac[w][n * 32 + lane];
                    sm.ac[w][n * 32 + lane] = C[n];
                }
                modes_carry<NP, kCx>(C, pT, a);
                // A sequence ending on a unit boundary takes its final state
                // from the canonical chain (the expression a later chunk
                // starts from).
                if (whole_last && j0 + w == A.units - 1 && A.state_out != nullptr && c0 < A.D) {
#pragma unroll
                    for (int n = 0; n < NP; ++n) {
                        if (n < A.N) {
                            A.state_out[(static_cast<size_t>(q.b) * A.D + c0) * A.N + n] = C[n].x;
                            A.state_out[(static_cast<size_t>(q.b) * A.D + c0 + 1) * A.N + n] = C[n].y;
                        }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.cdone[k & 1]);

        // ---------------- publish the group's carry-out (flag INCL)
        if (has_successor) {
#pragma unroll
            for (int n = 0; n < NP; ++n) *reinterpret_cast<float2 *>(slot + incl_off + n * MCH) = C[n];
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release_u64(chain_flags + (s % MRING), flag_word(epoch, s, true));
        }

        announce_group<NP, G>(sm, A, k + ahead);
    }
}

// ------------------------------------------------------------------ producer warp
// Streams every compute warp's chunks with TMA: per group iteration, chunks
// 0..7 carry x1/x2 rows of the unit for the A sweep, chunks 8..15 x1/x2/x3
// rows for the C sweep.  Chunk q of warp w goes to buffer q % kRing once the
// warp has released the chunk that used the buffer before.
// Separate or grouped inputs: one box of MCK rows x MCH channels per input
// (x1, x2 for the A sweep, x1, x2, x3 for the C sweep) at 4-D coordinates
// (column in group, group, token, batch row).  Triples: one box of MCK rows x
// 3 MCH interleaved values holds all three inputs, for either sweep.
template <int NP, int G, bool kTri>
__device__ void producer_warp(GroupSmem<NP, G> &sm, const CUtensorMap *tm1, const CUtensorMap *tm2,
                              const CUtensorMap *tm3, const ModalArgs &A)
{
    constexpr int kRing = GroupTraits<G>::kRing;
    const int lane = threadIdx.x & 31;
    int cur_k = -1;
    GroupPos q{};
    int cx = 0, cg = 0;  // box coordinates of the group's channel block
    for (int qn = 0;; ++qn) {
        const int k = qn / kChunksPerGroup;
        const int c = qn % kChunksPerGroup;
        if (k != cur_k) {
            (void)mbar_wait_or_flag(&sm.gready[k & 1], (k >> 1) & 1, A.hdr);
            const int gi = sm.gid[k & 1];
            if (gi < 0) break;
            q = group_pos(static_cast<unsigned int>(gi), A);
            const int ch = q.cb * MCH;
            cx = kTri ? 3 * ch : ch % A.group;
            cg = kTri ? 0 : ch / A.group;
            cur_k = k;
        }
        const int b = qn % kRing;
        const int row_in_unit = (c % kChunksPerSweep) * MCK;
        for (int w = 0; w < G; ++w) {
            if (qn >= kRing) (void)mbar_wait_or_flag(&sm.empty[w][b], ((qn / kRing) - 1) & 1, A.hdr);
            if (lane == 0) {
                const int row = (static_cast<int>(q.s) * G + w) * MT + row_in_unit;
                uint64_t *bar = &sm.full[w][b];
                fence_proxy_async_smem();
                if constexpr (kTri) {
                    mbar_arrive_expect_tx(bar, 3 * kChunkBytes);
                    tma_load_4d(sm.ring[w][b][0], tm1, bar, cx, 0, row, q.b);
                } else {
                    if (c < kChunksPerSweep) {
                        mbar_arrive_expect_tx(bar, 2 * kChunkBytes);
                    } else {
                        mbar_arrive_expect_tx(bar, 3 * kChunkBytes);
                        tma_load_4d(sm.ring[w][b][2], tm3, bar, cx, cg, row, q.b);
                    }
                    tma_load_4d(sm.ring[w][b][0], tm1, bar, cx, cg, row, q.b);
                    tma_load_4d(sm.ring[w][b][1], tm2, bar, cx, cg, row, q.b);
                }
            }
        }
    }
}

// ------------------------------------------------------------------ compute warps
// Separate buffers: lane l reads word l of each 32-word row of x1, x2 (x3).
template <int NP, bool kCx>
__device__ __forceinline__ void sweep_a_chunk(float2 (&s)[NP], const float2 (&p)[NP], const uint32_t *r1,
                                              const uint32_t *r2)
{
#pragma unroll 4
    for (int i = 0; i < MCK; ++i) {
        const float2 v = __fmul2_rn(bf16x2_to_float2(r1[i * 32]), bf16x2_to_float2(r2[i * 32]));
        modes_step<NP, kCx>(s, p, v);
    }
}

// Triples: rows of 96 words, the lane's three words at 3 l (x1/x2/x3 of its
// channel pair interleaved).
template <int NP, bool kCx>
__device__ __forceinline__ void sweep_a_chunk_tri(float2 (&s)[NP], const float2 (&p)[NP], const uint32_t *rw)
{
#pragma unroll 4
    for (int i = 0; i < MCK; ++i) {
        const uint32_t w0 = rw[i * 96], w1 = rw[i * 96 + 1], w2 = rw[i * 96 + 2];
        const float2 v = __fmul2_rn(tri_x1(w0, w1), tri_x2(w0, w2));
        modes_step<NP, kCx>(s, p, v);
    }
}

// One token of the C sweep for this lane's channel pair: advance the N states,
// form conv = sum_n R_n s_n with two independent accumulation chains (all
// state updates first, so the chains find their inputs ready), apply the
// gates and store y.  Complex modes: the table holds (Re R, -Im R) in the
// slot pair, so the same sum is Re sum_m R_m s_m.
template <int NP, bool kCx>
__device__ __forceinline__ void sweep_c_token(float2 (&s)[NP], const float2 (&p)[NP], const float2 (&R)[NP],
                                              float2 dsk, float2 v, float2 x3, uint32_t *yp, bool store)
{
    modes_step<NP, kCx>(s, p, v);
    float2 a0 = __fmul2_rn(R[0], s[0]);
    float2 a1 = __fmul2_rn(R[1], s[1]);
#pragma unroll
    for (int n = 2; n < NP; n += 2) {
        a0 = __ffma2_rn(R[n], s[n], a0);
        a1 = __ffma2_rn(R[n + 1], s[n + 1], a1);
    }
    const float2 conv = __fadd2_rn(a0, a1);
    const float2 yv = __ffma2_rn(dsk, v, __fmul2_rn(x3, conv));
    st_pred_u32(yp, float2_to_bf16x2(yv), store);
}

// v and x3 of row r of a chunk for this lane's channel pair.
template <bool kTri>
__device__ __forceinline__ void chunk_row(const uint32_t (&chunk)[3][kChunkWords], int lane, int r, float2 &v,
                                          float2 &x3)
{
    if constexpr (kTri) {
        const uint32_t *rw = &chunk[0][0] + r * 96 + 3 * lane;
        const uint32_t w0 = rw[0], w1 = rw[1], w2 = rw[2];
        v = __fmul2_rn(tri_x1(w0, w1), tri_x2(w0, w2));
        x3 = tri_x3(w1, w2);
    } else {
        v = __fmul2_rn(bf16x2_to_float2(chunk[0][r * 32 + lane]), bf16x2_to_float2(chunk[1][r * 32 + lane]));
        x3 = bf16x2_to_float2(chunk[2][r * 32 + lane]);
    }
}

template <int NP, int G, bool kTri, bool kCx>
__device__ void compute_warp(GroupSmem<NP, G> &sm, const ModalArgs &A)
{
    constexpr int kRing = GroupTraits<G>::kRing;
    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    const int groups_per_chain = (A.units + G - 1) / G;
    const size_t slot_floats = static_cast<size_t>(MGMAX + 1) * NP * MCH;
    int used = 0;  // next chunk number to consume

    for (int k = 0;; ++k) {
        (void)mbar_wait_or_flag(&sm.gready[k & 1], (k >> 1) & 1, A.hdr);
        const int gi = sm.gid[k & 1];
        if (gi < 0) break;
        const GroupPos q = group_pos(static_cast<unsigned int>(gi), A);
        const int c0 = q.cb * MCH + 2 * lane;
        const bool ch_ok = c0 < A.D;
        const int j = static_cast<int>(q.s) * G + w;
        const int t0 = j * MT;  // first token of this warp's unit

        // ---------------- A sweep: aggregate of the unit from a zero start
        float2 p[NP], s[NP];
        load_rows<NP>(p, A.coef, 0, A.Dp, c0);
#pragma unroll
        for (int n = 0; n < NP; ++n) s[n] = make_float2(0.f, 0.f);
        for (int i = 0; i < kChunksPerSweep; ++i, ++used) {
            const int b = used % kRing;
            (void)mbar_wait_tiles(&sm.full[w][b], (used / kRing) & 1, A.hdr);
            if constexpr (kTri)
                sweep_a_chunk_tri<NP, kCx>(s, p, &sm.ring[w][b][0][0] + 3 * lane);
            else
                sweep_a_chunk<NP, kCx>(s, p, sm.ring[w][b][0] + lane, sm.ring[w][b][1] + lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[w][b]);
        }
#pragma unroll
        for (int n = 0; n < NP; ++n) sm.ac[w][n * 32 + lane] = s[n];
        // The aggregate also goes to the group's ring slot (for successors'
        // look-backs); the fence lets the control warp release the flag
        // without a fence of its own.
        if (q.s > 0u && static_cast<int>(q.s) + 1 < groups_per_chain) {
            const unsigned int chain = static_cast<unsigned int>(q.b) * A.nCB + q.cb;
            float *slot = A.slots + (static_cast<size_t>(chain) * MRING + q.s % MRING) * slot_floats +
                          static_cast<size_t>(w) * NP * MCH + 2 * lane;
            (void)mbar_wait_or_flag(&sm.slotok[k & 1], (k >> 1) & 1, A.hdr);
#pragma unroll
            for (int n = 0; n < NP; ++n) *reinterpret_cast<float2 *>(slot + n * MCH) = s[n];
            __threadfence();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.adone[k & 1]);

        // ---------------- C sweep: outputs from the unit's carry
        float2 R[NP];
        load_rows<NP>(R, A.coef, NP, A.Dp, c0);
        const float2 dsk = ldg_f2(A.coef + static_cast<size_t>(2 * NP) * A.Dp + c0);
        (void)mbar_wait_or_flag(&sm.cdone[k & 1], (k >> 1) & 1, A.hdr);
#pragma unroll
        for (int n = 0; n < NP; ++n) s[n] = sm.ac[w][n * 32 + lane];
        uint32_t *yrow = reinterpret_cast<uint32_t *>(A.y + (static_cast<size_t>(q.b) * A.L + t0) * A.ld_y + c0);
        const size_t ystride = static_cast<size_t>(A.ld_y) / 2;  // in 32-bit words
        const int nvalid = min(MT, A.L - t0);                    // tokens of this unit inside L
        for (int i = 0; i < kChunksPerSweep; ++i, ++used) {
            const int b = used % kRing;
            (void)mbar_wait_tiles(&sm.full[w][b], (used / kRing) & 1, A.hdr);
            const int base = i * MCK;
            uint32_t *yc = yrow + static_cast<size_t>(base) * ystride;
            if (base + MCK <= nvalid) {
#pragma unroll
                for (int r = 0; r < MCK; ++r) {
                    float2 v, x3;
                    chunk_row<kTri>(sm.ring[w][b], lane, r, v, x3);
                    sweep_c_token<NP, kCx>(s, p, R, dsk, v, x3, yc + r * ystride, ch_ok);
                }
            } else {
                for (int r = 0; r < MCK && base + r < nvalid; ++r) {
                    float2 v, x3;
                    chunk_row<kTri>(sm.ring[w][b], lane, r, v, x3);
                    sweep_c_token<NP, kCx>(s, p, R, dsk, v, x3, yc + r * ystride, ch_ok);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[w][b]);
        }
        // A ragged last unit: the final state is the recurrence state after
        // token L-1 (its aggregate covers zero-padded rows).
        if (A.state_out != nullptr && ch_ok && (A.L % MT) != 0 && j == A.units - 1) {
#pragma unroll
            for (int n = 0; n < NP; ++n) {
                if (n < A.N) {
                    A.state_out[(static_cast<size_t>(q.b) * A.D + c0) * A.N + n] = s[n].x;
                    A.state_out[(static_cast<size_t>(q.b) * A.D + c0 + 1) * A.N + n] = s[n].y;
                }
            }
        }
    }
}

template <int NP, int G, bool kTri, bool kCx>
__global__ void __launch_bounds__(GroupTraits<G>::kThreads, GroupTraits<G>::kCtasPerSm)
    modal_scan_kernel(const __grid_constant__ CUtensorMap tm1, const __grid_constant__ CUtensorMap tm2,
                      const __grid_constant__ CUtensorMap tm3, const ModalArgs A)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    GroupSmem<NP, G> &sm = *reinterpret_cast<GroupSmem<NP, G> *>(smem_raw);
    // Flags carry the launch's epoch: the workspace keeps a counter that the
    // last CTA of every launch advances, so flags left by earlier launches
    // (including replays of a captured graph) never match.
    const unsigned int epoch = ld_volatile_u32(A.hdr + 3) + 1u;

    if (threadIdx.x == 0) {
        for (int w = 0; w < G; ++w)
            for (int b = 0; b < GroupTraits<G>::kRing; ++b) {
                mbar_init(&sm.full[w][b], 1);
                mbar_init(&sm.empty[w][b], 1);
            }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.gready[i], 1);
            mbar_init(&sm.slotok[i], 1);
            mbar_init(&sm.adone[i], G);
            mbar_init(&sm.cdone[i], 1);
        }
        fence_mbar_init();
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5;
    if (warp == G)
        control_warp<NP, G, kCx>(sm, A, epoch);
    else if (warp == G + 1)
        producer_warp<NP, G, kTri>(sm, &tm1, &tm2, &tm3, A);
    else
        compute_warp<NP, G, kTri, kCx>(sm, A);

    // Every chunk the producer issued belongs to a group the compute warps
    // consumed in full, so no TMA is in flight here.
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

template <int NP, int G, bool kTri, bool kCx>
int launch_scan(const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &m3, ModalArgs a,
                cudaStream_t st)
{
    static int configured_device = -1;
    static int sms = 0, per_sm = 0;
    int dev = 0;
    HYENA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
    const int smem = static_cast<int>(sizeof(GroupSmem<NP, G>));
    const int threads = GroupTraits<G>::kThreads;
    auto kernel = modal_scan_kernel<NP, G, kTri, kCx>;
    if (configured_device != dev) {
        HYENA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
                  "modal scan: set max dynamic shared memory");
        HYENA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "multiprocessor count");
        HYENA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem),
                  "modal scan: occupancy");
        if (per_sm < 1) per_sm = 1;
        configured_device = dev;
    }
    const unsigned int groups_per_chain = static_cast<unsigned int>((a.units + G - 1) / G);
    a.nGroups = groups_per_chain * static_cast<unsigned int>(a.B) * static_cast<unsigned int>(a.nCB);
    const unsigned int slots = static_cast<unsigned int>(sms * per_sm);
    const unsigned int grid = a.nGroups < slots ? a.nGroups : slots;
    kernel<<<grid, threads, smem, st>>>(m1, m2, m3, a);
    HYENA_TRY(cudaGetLastError(), "modal scan launch");
    return 1;
}

template <int NP, bool kTri, bool kCx>
int launch_narrow_np(const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &m3, const ModalArgs &a,
                     cudaStream_t st)
{
    // Four-unit groups (two CTAs per SM) while that still gives every SM
    // several groups; two-unit groups (three CTAs per SM) for short sequences.
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) (void)cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long chains = static_cast<long long>(a.B) * a.nCB;
    const long long groups4 = chains * ((a.units + 3) / 4);
    return groups4 >= 4ll * sms ? launch_scan<NP, 4, kTri, kCx>(m1, m2, m3, a, st)
                                : launch_scan<NP, 2, kTri, kCx>(m1, m2, m3, a, st);
}

template <bool kTri, bool kCx>
int launch_narrow_layout(const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &m3, const ModalArgs &a,
                         int NP, cudaStream_t st)
{
    switch (NP) {
        case 4: return launch_narrow_np<4, kTri, kCx>(m1, m2, m3, a, st);
        case 8: return launch_narrow_np<8, kTri, kCx>(m1, m2, m3, a, st);
        case 16: return launch_narrow_np<16, kTri, kCx>(m1, m2, m3, a, st);
        default: return -1;
    }
}

// ------------------------------------------------------------------ short sequences
// With few units per chain the look-back kernel leaves most sub-partitions
// idle and its chain of look-backs is most of the launch.  There two plain
// passes over all units at once do better:
//   pass 1  one warp per unit sweeps the unit's aggregate A_j from a zero
//           start into the chain's slot area (the warp of unit 0 also copies
//           state_in there as C_0, so that pass 2 never reads a state_in
//           that aliases state_out);
//   pass 2  one warp per unit forms its carry C_j by folding C_0 and
//           A_0 .. A_{j-1} forward in order and sweeps the unit's outputs;
//           x1/x2 come back from L2.
// Every value is formed by the look-back kernel's operations in the same
// order (aggregate sweep, canonical carry chain, output sweep), so the two
// paths give the same bits and a chunked sequence may mix them.
//
// Each warp requests all of its unit's rows with TMA at once (one barrier per
// chunk of MCK rows), so a launch keeps every unit's bytes in flight.  The
// coefficient kernel and the two passes are chained by programmatic dependent
// launch: a pass issues its row loads (inputs no kernel of the call writes)
// before it waits for the previous kernel's results.
constexpr int kShortWarps = 2;          // units per CTA
constexpr int kShortChunks = MT / MCK;  // chunks of MCK rows per unit
static_assert(MSHORT_UNITS + 1 <= MRING * (MGMAX + 1), "a chain's slot area holds C_0 and every unit's aggregate");

template <int kTensors>
struct ShortSmem {
    uint32_t chunk[kShortWarps][kShortChunks][kTensors][kChunkWords];
    uint64_t full[kShortWarps][kShortChunks];
};
static_assert(sizeof(uint32_t) * 2 * kChunkWords % 128 == 0, "TMA destinations stay 128-byte aligned");

__device__ __forceinline__ void pdl_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

struct ShortPos {
    int chain, b, cb, j, c0, t0, nvalid;
    bool ch_ok;
};

// Position of this warp's unit; false past the last unit.
__device__ __forceinline__ bool short_pos(const ModalArgs &A, ShortPos &q)
{
    const long long u = static_cast<long long>(blockIdx.x) * kShortWarps + (threadIdx.x >> 5);
    const long long chains = static_cast<long long>(A.B) * A.nCB;
    if (u >= chains * A.units) return false;
    q.chain = static_cast<int>(u / A.units);
    q.j = static_cast<int>(u - static_cast<long long>(q.chain) * A.units);
    q.b = q.chain / A.nCB;
    q.cb = q.chain % A.nCB;
    q.c0 = q.cb * MCH + 2 * (threadIdx.x & 31);
    q.ch_ok = q.c0 < A.D;
    q.t0 = q.j * MT;
    q.nvalid = min(MT, A.L - q.t0);
    return true;
}

// Lane 0 requests chunks 0 .. nchunks-1 of the warp's unit: x1/x2 (and x3
// with kX3), or the triples box, one barrier per chunk.  Rows past L and
// channels past D land as zeros, as in the look-back kernel.  The warp waits
// for every chunk it requested before it leaves.
template <int kTensors, bool kTri, bool kX3>
__device__ __forceinline__ void short_issue(ShortSmem<kTensors> &sm, int w, int nchunks, const ShortPos &q,
                                            const ModalArgs &A, const CUtensorMap *tm1, const CUtensorMap *tm2,
                                            const CUtensorMap *tm3)
{
    if ((threadIdx.x & 31) == 0) {
#pragma unroll
        for (int i = 0; i < kShortChunks; ++i) mbar_init(&sm.full[w][i], 1);
        fence_mbar_init();
        const int ch = q.cb * MCH;
        const int cx = kTri ? 3 * ch : ch % A.group;
        const int cg = kTri ? 0 : ch / A.group;
#pragma unroll 1
        for (int i = 0; i < nchunks; ++i) {
            uint64_t *bar = &sm.full[w][i];
            const int row = q.t0 + i * MCK;
            if constexpr (kTri) {
                mbar_arrive_expect_tx(bar, 3 * kChunkBytes);
                tma_load_4d(sm.chunk[w][i][0], tm1, bar, cx, 0, row, q.b);
            } else {
                mbar_arrive_expect_tx(bar, (kX3 ? 3 : 2) * kChunkBytes);
                tma_load_4d(sm.chunk[w][i][0], tm1, bar, cx, cg, row, q.b);
                tma_load_4d(sm.chunk[w][i][1], tm2, bar, cx, cg, row, q.b);
                if constexpr (kX3) tma_load_4d(sm.chunk[w][i][2], tm3, bar, cx, cg, row, q.b);
            }
        }
    }
    __syncwarp();
}

// Slot of unit j's aggregate (j == units: C_0), this lane's channel pair.
template <int NP>
__device__ __forceinline__ float *short_unit_slot(const ModalArgs &A, int chain, int j)
{
    const size_t slot_floats = static_cast<size_t>(MGMAX + 1) * NP * MCH;
    return A.slots + static_cast<size_t>(chain) * MRING * slot_floats + static_cast<size_t>(j) * NP * MCH +
           2 * (threadIdx.x & 31);
}

template <int NP, bool kTri, bool kCx>
__global__ void __launch_bounds__(32 * kShortWarps) modal_short_agg_kernel(const __grid_constant__ CUtensorMap tm1,
                                                                          const __grid_constant__ CUtensorMap tm2,
                                                                          const ModalArgs A)
{
    constexpr int kT = kTri ? 3 : 2;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    ShortSmem<kT> &sm = *reinterpret_cast<ShortSmem<kT> *>(smem_raw);
    pdl_launch_dependents();
    ShortPos q;
    if (!short_pos(A, q)) return;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // all chunks: the aggregate runs over the zero rows past L as well
    short_issue<kT, kTri, false>(sm, w, kShortChunks, q, A, &tm1, &tm2, nullptr);
    pdl_wait();  // the coefficient table, and the slot area a previous call read
    if (q.j == 0) {
        float *c0slot = short_unit_slot<NP>(A, q.chain, A.units);
#pragma unroll
        for (int n = 0; n < NP; ++n) {
            float2 v = make_float2(0.f, 0.f);
            if (A.state_in != nullptr && n < A.N && q.ch_ok) {
                v.x = A.state_in[(static_cast<size_t>(q.b) * A.D + q.c0) * A.N + n];
                v.y = A.state_in[(static_cast<size_t>(q.b) * A.D + q.c0 + 1) * A.N + n];
            }
            *reinterpret_cast<float2 *>(c0slot + n * MCH) = v;
        }
    }
    float2 p[NP], s[NP];
    load_rows<NP>(p, A.coef, 0, A.Dp, q.c0);
#pragma unroll
    for (int n = 0; n < NP; ++n) s[n] = make_float2(0.f, 0.f);
    for (int i = 0; i < kShortChunks; ++i) {
        (void)mbar_wait_tiles(&sm.full[w][i], 0, A.hdr);
        if constexpr (kTri)
            sweep_a_chunk_tri<NP, kCx>(s, p, &sm.chunk[w][i][0][0] + 3 * lane);
        else
            sweep_a_chunk<NP, kCx>(s, p, sm.chunk[w][i][0] + lane, sm.chunk[w][i][1] + lane);
    }
    float *slot = short_unit_slot<NP>(A, q.chain, q.j);
#pragma unroll
    for (int n = 0; n < NP; ++n) *reinterpret_cast<float2 *>(slot + n * MCH) = s[n];
}

template <int NP, bool kTri, bool kCx>
__global__ void __launch_bounds__(32 * kShortWarps) modal_short_out_kernel(const __grid_constant__ CUtensorMap tm1,
                                                                          const __grid_constant__ CUtensorMap tm2,
                                                                          const __grid_constant__ CUtensorMap tm3,
                                                                          const ModalArgs A)
{
    extern __shared__ __align__(128) unsigned char smem_raw[];
    ShortSmem<3> &sm = *reinterpret_cast<ShortSmem<3> *>(smem_raw);
    ShortPos q;
    if (!short_pos(A, q)) return;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nchunks = (q.nvalid + MCK - 1) / MCK;  // the chunks holding rows inside L
    short_issue<3, kTri, true>(sm, w, nchunks, q, A, &tm1, &tm2, &tm3);
    pdl_wait();  // the aggregates and C_0 of pass 1
    pdl_launch_dependents();

    // ---------------- the carry into unit j: the canonical chain
    float2 C[NP];
    {
        float2 pT[NP];
        load_rows<NP>(pT, A.coef, 2 * NP + 1, A.Dp, q.c0);
        const float *c0slot = short_unit_slot<NP>(A, q.chain, A.units);
#pragma unroll
        for (int n = 0; n < NP; ++n) C[n] = __ldcg(reinterpret_cast<const float2 *>(c0slot + n * MCH));
        const float *base = short_unit_slot<NP>(A, q.chain, 0);
        int jj = 0;
        for (; jj + 2 <= q.j; jj += 2) {
            // two units' aggregates in flight at once
            float2 a[NP], b2[NP];
#pragma unroll
            for (int n = 0; n < NP; ++n) {
                a[n] = __ldcg(reinterpret_cast<const float2 *>(base + (static_cast<size_t>(jj) * NP + n) * MCH));
                b2[n] = __ldcg(reinterpret_cast<const float2 *>(base + (static_cast<size_t>(jj + 1) * NP + n) * MCH));
            }
            modes_carry<NP, kCx>(C, pT, a);
            modes_carry<NP, kCx>(C, pT, b2);
        }
        if (jj < q.j) {
            float2 a[NP];
#pragma unroll
            for (int n = 0; n < NP; ++n)
                a[n] = __ldcg(reinterpret_cast<const float2 *>(base + (static_cast<size_t>(jj) * NP + n) * MCH));
            modes_carry<NP, kCx>(C, pT, a);
        }
        // A sequence ending on a unit boundary takes its final state from the
        // canonical chain, C_units.
        if ((A.L % MT) == 0 && q.j == A.units - 1 && A.state_out != nullptr && q.ch_ok) {
            float2 a[NP], Cn[NP];
#pragma unroll
            for (int n = 0; n < NP; ++n) {
                a[n] = __ldcg(reinterpret_cast<const float2 *>(base + (static_cast<size_t>(q.j) * NP + n) * MCH));
                Cn[n] = C[n];
            }
            modes_carry<NP, kCx>(Cn, pT, a);
#pragma unroll
            for (int n = 0; n < NP; ++n) {
                if (n < A.N) {
                    A.state_out[(static_cast<size_t>(q.b) * A.D + q.c0) * A.N + n] = Cn[n].x;
                    A.state_out[(static_cast<size_t>(q.b) * A.D + q.c0 + 1) * A.N + n] = Cn[n].y;
                }
            }
        }
    }

    // ---------------- outputs of the unit from its carry
    float2 p[NP], R[NP];
    load_rows<NP>(p, A.coef, 0, A.Dp, q.c0);
    load_rows<NP>(R, A.coef, NP, A.Dp, q.c0);
    const float2 dsk = ldg_f2(A.coef + static_cast<size_t>(2 * NP) * A.Dp + q.c0);
    uint32_t *yrow = reinterpret_cast<uint32_t *>(A.y + (static_cast<size_t>(q.b) * A.L + q.t0) * A.ld_y + q.c0);
    const size_t ystride = static_cast<size_t>(A.ld_y) / 2;  // in 32-bit words
    for (int i = 0; i < nchunks; ++i) {
        (void)mbar_wait_tiles(&sm.full[w][i], 0, A.hdr);
        const int base = i * MCK;
        uint32_t *yc = yrow + static_cast<size_t>(base) * ystride;
        if (base + MCK <= q.nvalid) {
#pragma unroll
            for (int r = 0; r < MCK; ++r) {
                float2 v, x3;
                chunk_row<kTri>(sm.chunk[w][i], lane, r, v, x3);
                sweep_c_token<NP, kCx>(C, p, R, dsk, v, x3, yc + r * ystride, q.ch_ok);
            }
        } else {
            for (int r = 0; r < MCK && base + r < q.nvalid; ++r) {
                float2 v, x3;
                chunk_row<kTri>(sm.chunk[w][i], lane, r, v, x3);
                sweep_c_token<NP, kCx>(C, p, R, dsk, v, x3, yc + r * ystride, q.ch_ok);
            }
        }
    }
    // A ragged last unit: the final state is the recurrence state after token L-1.
    if (A.state_out != nullptr && q.ch_ok && (A.L % MT) != 0 && q.j == A.units - 1) {
#pragma unroll
        for (int n = 0; n < NP; ++n) {
            if (n < A.N) {
                A.state_out[(static_cast<size_t>(q.b) * A.D + q.c0) * A.N + n] = C[n].x;
                A.state_out[(static_cast<size_t>(q.b) * A.D + q.c0 + 1) * A.N + n] = C[n].y;
            }
        }
    }
}

template <class Kernel, class... Args>
cudaError_t launch_dependent(Kernel kernel, unsigned int grid, int threads, size_t smem, cudaStream_t st,
                             Args... args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int NP, bool kTri, bool kCx>
int launch_short_np(const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &m3, const ModalArgs &a,
                    cudaStream_t st)
{
    static int configured_device = -1;
    int dev = 0;
    HYENA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
    constexpr size_t smem_agg = sizeof(ShortSmem<kTri ? 3 : 2>);
    constexpr size_t smem_out = sizeof(ShortSmem<3>);
    auto agg = modal_short_agg_kernel<NP, kTri, kCx>;
    auto out = modal_short_out_kernel<NP, kTri, kCx>;
    if (configured_device != dev) {
        HYENA_TRY(cudaFuncSetAttribute(agg, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_agg)),
                  "modal scan (short): set max dynamic shared memory");
        HYENA_TRY(cudaFuncSetAttribute(out, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_out)),
                  "modal scan (short): set max dynamic shared memory");
        configured_device = dev;
    }
    const long long units = static_cast<long long>(a.B) * a.nCB * a.units;
    const unsigned int grid = static_cast<unsigned int>((units + kShortWarps - 1) / kShortWarps);
    HYENA_TRY(launch_dependent(agg, grid, 32 * kShortWarps, smem_agg, st, m1, m2, a),
              "modal scan (short): aggregate pass launch");
    HYENA_TRY(launch_dependent(out, grid, 32 * kShortWarps, smem_out, st, m1, m2, m3, a),
              "modal scan (short): output pass launch");
    return 2;
}

template <bool kTri, bool kCx>
int launch_short_layout(const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &m3, const ModalArgs &a,
                        int NP, cudaStream_t st)
{
    switch (NP) {
        case 4: return launch_short_np<4, kTri, kCx>(m1, m2, m3, a, st);
        case 8: return launch_short_np<8, kTri, kCx>(m1, m2, m3, a, st);
        case 16: return launch_short_np<16, kTri, kCx>(m1, m2, m3, a, st);
        default: return -1;
    }
}

}  // namespace

int launch_modal_narrow(const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &m3, ModalArgs a, int NP,
                        bool triples, bool cx, cudaStream_t st)
{
    if (triples)
        return cx ? launch_narrow_layout<true, true>(m1, m2, m3, a, NP, st)
                  : launch_narrow_layout<true, false>(m1, m2, m3, a, NP, st);
    return cx ? launch_narrow_layout<false, true>(m1, m2, m3, a, NP, st)
              : launch_narrow_layout<false, false>(m1, m2, m3, a, NP, st);
}

bool modal_short_path(int B, int L, int D, int NP, bool triples)
{
    if (NP > 16 || L < 1) return false;
    const long long units = (static_cast<long long>(L) + MT - 1) / MT;
    const long long bytes = static_cast<long long>(B) * L * D * (triples ? 6 : 4);
    return units <= MSHORT_UNITS && bytes <= MSHORT_L2_BYTES;
}

int launch_modal_short(const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &m3, const ModalArgs &a,
                       int NP, bool triples, bool cx, cudaStream_t st)
{
    if (triples)
        return cx ? launch_short_layout<true, true>(m1, m2, m3, a, NP, st)
                  : launch_short_layout<true, false>(m1, m2, m3, a, NP, st);
    return cx ? launch_short_layout<false, true>(m1, m2, m3, a, NP, st)
              : launch_short_layout<false, false>(m1, m2, m3, a, NP, st);
}

}  // namespace hyena
