// modal_scan_wide.cu -- the long modal-form filter (hcl) with 32 or 64 mode
// slots per channel (17..64 real or 9..32 complex modes) as a single-pass,
// decoupled look-back scan over time, on sm_100a.  Up to 16 slots the
// two-CTAs-per-SM kernel of modal_scan.cu runs instead (the same canonical
// carry chain and token arithmetic).
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
// start.  The carry into the second half of unit j is p^MH C_j + H_j, with H_j
// the end state of the unit's first MH tokens from a zero start.  Every carry
// the kernel forms is evaluated by exactly these fp32 operations, whoever
// evaluates it and however far a look-back reaches, so the output is bitwise
// deterministic and feeding a sequence in chunks of whole units reproduces
// the single pass bit for bit.
//
// Work.  MGMAX consecutive units of a chain form a group, handed out by an
// atomic ticket in time-major order (a group's predecessor holds a smaller
// ticket and is running or finished: forward progress never depends on
// scheduling).  One persistent CTA per SM, warp-specialised; lane l of a
// compute warp owns the channel pair 2l, 2l+1 (packed f32x2 arithmetic):
//   aggregate warps (one per unit of the group)  stream the unit's x1/x2 rows
//       and run the N recurrences from zero: H_j after MH tokens and A_j at the
//       end (N FMAs per token), into the group's context in shared memory and
//       the chain's ring slot in global memory (for later groups' look-backs);
//   control warp  takes the group tickets, publishes the group's aggregates
//       (flag AGG), looks back along the chain to the nearest inclusive
//       prefix, folds the skipped groups' unit aggregates forward, derives the
//       carry of every unit and half unit of the group and publishes the
//       group's carry-out (flag INCL);
//   output warps (one per half unit)  stream the half unit's x1/x2/x3 rows
//       (x1/x2 come back from L2) and rerun the recurrences from the half
//       unit's carry, emitting y = x3 * sum_n R_n s_n + Dskip v as coalesced
//       128-byte rows (2N FMAs per token);
//   producer warp  keeps every compute warp's ring of chunk buffers filled
//       with TMA loads, one lane per ring, without blocking on any one ring.
// Each group has one of two contexts in shared memory (its id, the unit
// aggregates that the control warp overwrites with the carries), so the
// aggregate warps sweep group k+2 while the output warps sweep group k and
// the control warp resolves group k+1: every SM sub-partition keeps one
// aggregate and two output warps busy at all times, which is what the FMA
// pipe needs (the kernel runs 3N FMAs per channel-token).
//
// Ring of slots: each chain owns MRING group slots; group s writes slot
// s % MRING.  The look-back never goes deeper than MLB groups (it waits for an
// inclusive prefix at depth MLB), and before a group is handed to the compute
// warps the control warp checks that groups s-MRING .. s-MLB are finished, so
// a slot is never overwritten while someone may still read it.  Flags are
// 64-bit: (epoch << 32) | (group << 1) | is_inclusive.  The epoch lives in the
// workspace and advances at the end of every launch, so stale flags from
// earlier launches never match and a captured CUDA graph can be replayed.
// Waits on other CTAs are bounded (about one second of %globaltimer) and
// record an error bit instead of hanging; once an error bit is set they give
// up at once.  Hand-offs between a CTA's own warps are bounded too (four
// seconds) but never give up early: every group that was handed out is
// swept to the end, so no TMA copy is in flight when the CTA exits.
#include "hyena_device.cuh"
#include "hyena_internal.h"

namespace hyena {

namespace {

constexpr int kAW = MGMAX;                 // aggregate warps: warp w sweeps unit w of the group
constexpr int kCW = 2 * MGMAX;             // output warps: warp 2w + h sweeps half h of unit w
constexpr int kCtrlWarp = kAW + kCW;       // tickets, look-back, carries
constexpr int kProdWarp = kCtrlWarp + 1;   // TMA issue for every ring
constexpr int kThreads = 32 * (kProdWarp + 3);  // four whole warpgroups (two warps of the last idle)
// Registers per thread: the block is launched with 65536 / kThreads = 128 and
// rebalanced per warpgroup (setmaxnreg): the output warps need their modes'
// states, poles and residues in registers, the others less.  The split must
// add up to the launch total: 4 RA + 8 RC + 4 RX = 4 * 128 * 4.
constexpr int kRegsAgg = 96, kRegsOut = 152, kRegsAux = 112;
static_assert(4 * kRegsAgg + 8 * kRegsOut + 4 * kRegsAux <= 4 * 4 * 128, "register split");
constexpr int kAChunks = MT / MA_ROWS;     // chunks per unit (aggregate sweep)
constexpr int kCChunks = MH / MC_ROWS;     // chunks per half unit (output sweep)
constexpr int kProdCLane = 8;              // producer lanes kProdCLane.. serve the output warps
constexpr int kProdKLane = 16;             // producer lane that stages each group's coefficients
constexpr unsigned long long kLocalWaitNs = 4ull * kWaitLimitNs;
constexpr unsigned int kProdSleepNs = 128;  // producer back-off when no ring needs a chunk

static_assert(MA_ROWS * kAChunks == MT && MC_ROWS * kCChunks == MH, "chunking");
static_assert(kProdCLane >= kAW && kProdCLane + kCW <= kProdKLane && kProdKLane < 32, "producer lanes");

// A chain of kWidth = MCH / LPC channels: rows of kRowWords 32-bit words
// (bf16 channel pairs) per input.
template <int LPC>
struct ChainTraits {
    static constexpr int kWidth = MCH / LPC;
    static constexpr int kRowWords = 32 / LPC;
};

template <bool kTri, int LPC>
struct RingTraits {
    static constexpr int kADepth = kTri ? 2 : 3;  // chunk buffers per aggregate warp
    static constexpr int kCDepth = 2;             // chunk buffers per output warp
    static constexpr int kRW = ChainTraits<LPC>::kRowWords;
    // separate inputs: x1 (and x2, x3) boxes one after the other, kRW words
    // per row; triples: one box of interleaved rows, 3 kRW words per row
    static constexpr int kAWords = kTri ? MA_ROWS * 3 * kRW : 2 * MA_ROWS * kRW;
    static constexpr int kCWords = kTri ? MC_ROWS * 3 * kRW : 3 * MC_ROWS * kRW;
    static constexpr uint32_t kABytes = kAWords * 4;
    static constexpr uint32_t kCBytes = kCWords * 4;
};

// Where lane l works: the channel pair l / LPC of its chain (first channel c0)
// and the mode slots [mo, mo + NP) of the NP * LPC padded slots.
template <int NP, int LPC>
struct LanePos {
    int pair, mo, c0;
    __device__ __forceinline__ LanePos(int lane, int cb)
        : pair(lane / LPC), mo((lane % LPC) * NP), c0(cb * ChainTraits<LPC>::kWidth + 2 * (lane / LPC))
    {
    }
};

template <int NP, int LPC, bool kTri>
struct ScanSmem {
    using T = RingTraits<kTri, LPC>;
    static constexpr int kW = ChainTraits<LPC>::kWidth;
    static constexpr int kCoefRows = 2 * NP * LPC + 1;                   // p, residues, Dskip of the chain
    static constexpr uint32_t kCoefBytes = kCoefRows * kW * 4;          // one TMA box
    static constexpr int kCoefFloats = ((kCoefRows * kW + 31) / 32) * 32;  // padded to 128 bytes
    // Every TMA destination below starts on a 128-byte boundary: the arrays
    // are multiples of 128 bytes long and so are the boxes within a chunk.
    static_assert((T::kAWords * 4) % 128 == 0 && (MA_ROWS * T::kRW * 4) % 128 == 0, "aggregate chunk alignment");
    static_assert((T::kCWords * 4) % 128 == 0 && (MC_ROWS * T::kRW * 4) % 128 == 0, "output chunk alignment");
    static_assert((kCoefFloats * 4) % 128 == 0, "coefficient box alignment");
    uint32_t aring[kAW][T::kADepth][T::kAWords];
    uint32_t cring[kCW][T::kCDepth][T::kCWords];
    float coef[2][kCoefFloats];  // per group context: rows of kW floats
    // per group context: slot 2w holds A_w, then (control warp) the carry C_w;
    // slot 2w+1 holds H_w
    float2 ctx[2][kCW][NP * 32];
    uint64_t afull[kAW][T::kADepth], aempty[kAW][T::kADepth];
    uint64_t cfull[kCW][T::kCDepth], cempty[kCW][T::kCDepth];
    uint64_t gready[2];  // group id of the context known (control -> all)
    uint64_t adone[2];   // aggregates written (aggregate warps -> control)
    uint64_t cdone[2];   // carries written (control -> output warps)
    uint64_t cfree[2];   // carries read (output warps -> control)
    uint64_t coefbar[2]; // the group's coefficients landed (producer TMA -> compute)
    int gid[2];
};

__device__ __forceinline__ unsigned long long flag_word(unsigned int epoch, unsigned int group, bool incl)
{
    return (static_cast<unsigned long long>(epoch) << 32) | (static_cast<unsigned long long>(group) << 1) |
           (incl ? 1ull : 0ull);
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Bounded wait on a hand-off between the CTA's own warps.  It never gives up
// because of an error elsewhere (the pipeline must drain), only after
// kLocalWaitNs, recording an error bit.
__device__ __forceinline__ void wait_local(uint64_t *bar, uint32_t parity, unsigned int *hdr)
{
    if (mbar_try_wait(bar, parity)) return;
    const unsigned long long t0 = global_timer_ns();
    for (unsigned int it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return;
        if ((it & 63u) == 0u && global_timer_ns() - t0 > kLocalWaitNs) {
            atomicOr(hdr + 2, kErrLocalTimeout);
            return;
        }
    }
}

// Spins on a flag written by another CTA until pred(flag) holds.  Returns
// false if the wait timed out or another wait already failed (error bit set).
template <class Pred>
__device__ __forceinline__ bool spin_flag(const unsigned long long *f, unsigned int *hdr, unsigned int errbit,
                                          Pred pred)
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

// Rows [row0, row0 + NP) of a group's staged coefficients (rows of W
// floats), this lane's pair.
template <int NP, int W>
__device__ __forceinline__ void coef_rows(float2 (&dst)[NP], const float *coef, int row0, int pair)
{
#pragma unroll
    for (int n = 0; n < NP; ++n) dst[n] = *reinterpret_cast<const float2 *>(coef + (row0 + n) * W + 2 * pair);
}

template <int NP>
__device__ __forceinline__ void load_rows(float2 (&dst)[NP], const float *table, int row0, int Dp, int c0)
{
#pragma unroll
    for (int n = 0; n < NP; ++n) dst[n] = ldg_f2(table + static_cast<size_t>(row0 + n) * Dp + c0);
}

// ------------------------------------------------------------------ control warp
// Hands group iteration k of this CTA a ticket: once the output warps have read
// the carries of group k-2 (the context's previous user), take the next
// ticket, check the ring guard of the group's slot and announce the group id.
template <int NP, int LPC, bool kTri>
__device__ void announce(ScanSmem<NP, LPC, kTri> &sm, const ModalArgs &A, int k, unsigned int epoch)
{
    const int lane = threadIdx.x & 31;
    const int c = k & 1;
    if (k >= 2) wait_local(&sm.cfree[c], ((k - 2) >> 1) & 1, A.hdr);
    unsigned int t = 0;
    if (lane == 0) {
        t = atomicAdd(A.hdr, 1u);
        if (ld_volatile_u32(A.hdr + 2) != 0u) t = A.nGroups;  // an error: hand out no more groups
    }
    t = __shfl_sync(0xffffffffu, t, 0);
    const int gi = t < A.nGroups ? static_cast<int>(t) : -1;
    if (gi >= 0) {
        // Ring guard: groups s-MRING .. s-MLB must be finished before this
        // group's slot s % MRING is written (by the aggregate warps).
        const GroupPos q = group_pos(static_cast<unsigned int>(gi), A);
        const unsigned int chain = static_cast<unsigned int>(q.b) * A.nCB + q.cb;
        const unsigned long long *chain_flags = A.flags + static_cast<size_t>(chain) * MRING;
        if (q.s >= static_cast<unsigned int>(MRING) && lane <= MRING - MLB) {
            const unsigned int jg = q.s - MRING + lane;
            const unsigned long long need = flag_word(epoch, jg, true) & 0xffffffffull;
            (void)spin_flag(chain_flags + (jg % MRING), A.hdr, kErrRingTimeout, [&](unsigned long long x) {
                return (x >> 32) == epoch && (x & 0xffffffffull) >= need;
            });
        }
        __syncwarp();
    }
    if (lane == 0) {
        sm.gid[c] = gi;
        mbar_arrive(&sm.gready[c]);
    }
    __syncwarp();
}

// Look-back, carries and publication of group iteration k (id gi).
template <int NP, int LPC, bool kTri, bool kCx>
__device__ void process_group(ScanSmem<NP, LPC, kTri> &sm, const ModalArgs &A, int k, int gi, unsigned int epoch)
{
    constexpr int NPT = NP * LPC;
    constexpr int W = ChainTraits<LPC>::kWidth;
    const int lane = threadIdx.x & 31;
    const int c = k & 1;
    const int groups_per_chain = (A.units + MGMAX - 1) / MGMAX;
    const size_t slot_floats = static_cast<size_t>(MGMAX + 1) * NPT * W;
    const size_t incl_off = static_cast<size_t>(MGMAX) * NPT * W;
    const GroupPos q = group_pos(static_cast<unsigned int>(gi), A);
    const unsigned int s = q.s;
    const LanePos<NP, LPC> lp(lane, q.cb);
    const int c0 = lp.c0;
    const unsigned int chain = static_cast<unsigned int>(q.b) * A.nCB + q.cb;
    unsigned long long *chain_flags = A.flags + static_cast<size_t>(chain) * MRING;
    float *chain_slots = A.slots + static_cast<size_t>(chain) * MRING * slot_floats;
    // this lane's first mode slot of a unit's block in a ring slot
    const size_t lane_off = static_cast<size_t>(lp.mo) * W + 2 * lp.pair;
    float *slot = chain_slots + static_cast<size_t>(s % MRING) * slot_floats + lane_off;
    const int j0 = static_cast<int>(s) * MGMAX;         // first unit of the group
    const int nvalid_units = min(MGMAX, A.units - j0);  // units of the group inside L
    const bool has_successor = static_cast<int>(s) + 1 < groups_per_chain;
    float2 pT[NP];
    load_rows<NP>(pT, A.coef, 2 * NPT + 1 + lp.mo, A.Dp, c0);

    // ---------------- publish the group's unit aggregates (flag AGG)
    // Each aggregate warp wrote its unit's aggregate to the slot and fenced
    // before arriving; the release store orders all of them before the flag
    // for any reader that acquires it.
    wait_local(&sm.adone[c], (k >> 1) & 1, A.hdr);
    if (s > 0u && has_successor && lane == 0) st_release_u64(chain_flags + (s % MRING), flag_word(epoch, s, false));

    // ---------------- look-back: the carry into the group's first unit
    float2 C[NP];
    if (s == 0u) {
#pragma unroll
        for (int n = 0; n < NP; ++n) {
            float2 v = make_float2(0.f, 0.f);
            const int m = lp.mo + n;
            if (A.state_in != nullptr && m < A.N && c0 < A.D) {
                v.x = A.state_in[(static_cast<size_t>(q.b) * A.D + c0) * A.N + m];
                v.y = A.state_in[(static_cast<size_t>(q.b) * A.D + c0 + 1) * A.N + m];
            }
            C[n] = v;
        }
    } else {
        const unsigned int floor_g = s > static_cast<unsigned int>(MLB) ? s - MLB : 0u;
        const unsigned int depth = s - floor_g;  // 1 .. MLB
        // Lane i watches group s-1-i: wait until the nearest inclusive prefix
        // is visible and every group after it has its aggregates.
        const unsigned long long t0 = global_timer_ns();
        unsigned int jincl = 0;
        // after an error: zero carries, no waiting (a warp-uniform decision)
        bool ok = __all_sync(0xffffffffu, ld_volatile_u32(A.hdr + 2) == 0u);
        for (unsigned int it = 0; ok; ++it) {
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
                }
            }
        }
        // The flags were acquired by several lanes; the warp barrier orders
        // those acquires before every lane's slot reads, which go to L2 (never
        // a stale L1 line of an earlier use of the slot).
        __syncwarp();
        const float *inc = chain_slots + static_cast<size_t>(jincl % MRING) * slot_floats + incl_off + lane_off;
#pragma unroll
        for (int n = 0; n < NP; ++n)
            C[n] = ok ? __ldcg(reinterpret_cast<const float2 *>(inc + n * W)) : make_float2(0.f, 0.f);
        // Fold the skipped groups' unit aggregates forward, unit by unit (the
        // canonical chain).
        for (unsigned int jg = jincl + 1u; ok && jg < s; ++jg) {
            const float *src = chain_slots + static_cast<size_t>(jg % MRING) * slot_floats + lane_off;
            for (int w = 0; w < MGMAX; ++w) {
#pragma unroll
                for (int n = 0; n < NP; n += 2) {
                    const float *u = src + (static_cast<size_t>(w) * NPT + n) * W;
                    carry_pair<kCx>(C[n], C[n + 1], pT[n], pT[n + 1], __ldcg(reinterpret_cast<const float2 *>(u)),
                                    __ldcg(reinterpret_cast<const float2 *>(u + W)));
                }
            }
        }
    }

    // ---------------- carries of the group's units (in place over A_j); the
    // output warp of a unit's second half forms its own carry from C_j and H_j
    {
        const bool whole_last = (A.L % MT) == 0;
        for (int w = 0; w < nvalid_units; ++w) {
            float2 *full = sm.ctx[c][2 * w] + lane;
#pragma unroll
            for (int n = 0; n < NP; n += 2) {
                const float2 a0 = full[n * 32], a1 = full[(n + 1) * 32];
                full[n * 32] = C[n];
                full[(n + 1) * 32] = C[n + 1];
                carry_pair<kCx>(C[n], C[n + 1], pT[n], pT[n + 1], a0, a1);
            }
            // A sequence ending on a unit boundary takes its final state from
            // the canonical chain (the expression a later chunk starts from).
            if (whole_last && j0 + w == A.units - 1 && A.state_out != nullptr && c0 < A.D) {
#pragma unroll
                for (int n = 0; n < NP; ++n) {
                    const int m = lp.mo + n;
                    if (m < A.N) {
                        A.state_out[(static_cast<size_t>(q.b) * A.D + c0) * A.N + m] = C[n].x;
                        A.state_out[(static_cast<size_t>(q.b) * A.D + c0 + 1) * A.N + m] = C[n].y;
                    }
                }
            }
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.cdone[c]);

    // ---------------- publish the group's carry-out (flag INCL)
    if (has_successor) {
#pragma unroll
        for (int n = 0; n < NP; ++n) *reinterpret_cast<float2 *>(slot + incl_off + n * W) = C[n];
        __threadfence();
        __syncwarp();
        if (lane == 0) st_release_u64(chain_flags + (s % MRING), flag_word(epoch, s, true));
    }
}

template <int NP, int LPC, bool kTri, bool kCx>
__device__ void control_warp(ScanSmem<NP, LPC, kTri> &sm, const ModalArgs &A, unsigned int epoch)
{
    announce<NP, LPC, kTri>(sm, A, 0, epoch);
    // With no more groups than CTAs every CTA takes exactly one: a second
    // early ticket would only take a group from a CTA that has none.
    if (sm.gid[0] >= 0 && A.nGroups > gridDim.x) {
        announce<NP, LPC, kTri>(sm, A, 1, epoch);
    } else if ((threadIdx.x & 31) == 0) {
        sm.gid[1] = -1;
        mbar_arrive(&sm.gready[1]);
    }
    __syncwarp();
    for (int k = 0;; ++k) {
        const int gi = sm.gid[k & 1];  // written by lane 0 of this warp before a __syncwarp
        if (gi < 0) break;
        process_group<NP, LPC, kTri, kCx>(sm, A, k, gi, epoch);
        if (sm.gid[(k + 1) & 1] < 0) break;
        announce<NP, LPC, kTri>(sm, A, k + 2, epoch);
    }
}

// ------------------------------------------------------------------ producer warp
// Lane w < kAW keeps aggregate warp w's ring filled, lane kProdCLane + w output
// warp w's; the loop is warp-uniform and polls without blocking, so one slow
// consumer never delays the others' refills.  Chunk q of a ring belongs to the
// consumer's group iteration q / (chunks per group); it goes to buffer
// q % depth once the consumer has released the chunk that used it before.
// Separate or grouped inputs: one box per input at 4-D coordinates (column in
// group, group, token, batch row); triples: one box of interleaved rows holds
// all three inputs.
template <int NP, int LPC, bool kTri>
__device__ void producer_warp(ScanSmem<NP, LPC, kTri> &sm, const ModalMaps &maps, const ModalArgs &A)
{
    using T = RingTraits<kTri, LPC>;
    const int lane = threadIdx.x & 31;
    const bool isA = lane < kAW;
    const bool isC = lane >= kProdCLane && lane < kProdCLane + kCW;
    const bool isK = lane == kProdKLane;  // one coefficient box per group, no ring
    const int w = isA ? lane : lane - kProdCLane;
    const int depth = isA ? T::kADepth : T::kCDepth;
    const int chunks = isA ? kAChunks : (isC ? kCChunks : 1);
    constexpr uint32_t kCoefBytes = ScanSmem<NP, LPC, kTri>::kCoefBytes;
    bool done = !(isA || isC || isK);
    int q = 0, cur_k = -1;
    int cx = 0, cg = 0, brow = 0, row0 = 0;
    unsigned long long t_last = global_timer_ns();
    for (unsigned int it = 0;; ++it) {
        bool progress = false;
        if (!done) {
            const int k = q / chunks;
            const int ci = q - k * chunks;
            if (k != cur_k && mbar_test_wait(&sm.gready[k & 1], (k >> 1) & 1)) {
                const int gi = sm.gid[k & 1];
                progress = true;
                if (gi < 0) {
                    done = true;
                } else {
                    const GroupPos g = group_pos(static_cast<unsigned int>(gi), A);
                    const int ch = g.cb * ChainTraits<LPC>::kWidth;
                    cx = isK ? ch : (kTri ? 3 * ch : ch % A.group);
                    cg = kTri ? 0 : ch / A.group;
                    brow = g.b;
                    const int unit = static_cast<int>(g.s) * MGMAX + (isA ? w : (w >> 1));
                    row0 = unit * MT + (isA ? 0 : (w & 1) * MH);
                    cur_k = k;
                }
            }
            if (!done && cur_k == k && isK) {
                // The context's coefficient area is free once the group is
                // announced: its previous group's warps read it before the
                // context was handed on.
                uint64_t *bar = &sm.coefbar[k & 1];
                mbar_arrive_expect_tx(bar, kCoefBytes);
                tma_load_2d(&sm.coef[k & 1][0], &maps.coef, bar, cx, 0);
                ++q;
                progress = true;
            } else if (!done && cur_k == k) {
                const int b = q % depth;
                const uint32_t par = static_cast<uint32_t>((q / depth) - 1) & 1u;
                const bool free = q < depth || mbar_test_wait(isA ? &sm.aempty[w][b] : &sm.cempty[w][b], par);
                if (free) {
                    fence_proxy_async_smem();
                    if (isA) {
                        uint64_t *bar = &sm.afull[w][b];
                        const int row = row0 + ci * MA_ROWS;
                        mbar_arrive_expect_tx(bar, T::kABytes);
                        tma_load_4d(&sm.aring[w][b][0], &maps.a1, bar, cx, cg, row, brow);
                        if constexpr (!kTri)
                            tma_load_4d(&sm.aring[w][b][MA_ROWS * T::kRW], &maps.a2, bar, cx, cg, row, brow);
                    } else {
                        uint64_t *bar = &sm.cfull[w][b];
                        const int row = row0 + ci * MC_ROWS;
                        mbar_arrive_expect_tx(bar, T::kCBytes);
                        tma_load_4d(&sm.cring[w][b][0], &maps.c1, bar, cx, cg, row, brow);
                        if constexpr (!kTri) {
                            tma_load_4d(&sm.cring[w][b][MC_ROWS * T::kRW], &maps.c2, bar, cx, cg, row, brow);
                            tma_load_4d(&sm.cring[w][b][2 * MC_ROWS * T::kRW], &maps.c3, bar, cx, cg, row, brow);
                        }
                    }
                    ++q;
                    progress = true;
                }
            }
        }
        if (__all_sync(0xffffffffu, done)) break;
        if (__any_sync(0xffffffffu, progress)) {
            t_last = global_timer_ns();
        } else {
            // nothing to issue: step aside for the compute warps of this SM
            // sub-partition instead of spinning on their issue slots
            __nanosleep(kProdSleepNs);
        }
        if ((it & 63u) == 0u) {
            // lane 0's clock decides for the whole warp
            if (__shfl_sync(0xffffffffu, global_timer_ns() - t_last > kLocalWaitNs, 0)) {
                if (lane == 0) atomicOr(A.hdr + 2, kErrLocalTimeout);
                break;
            }
        }
    }
}

// ------------------------------------------------------------------ compute warps
// Aggregate sweep over one chunk.  Separate buffers: lane l reads word
// l / LPC of each row of x1 and x2 (rows of RW words).
template <int NP, bool kCx, int RW>
__device__ __forceinline__ void sweep_a_chunk(float2 (&s)[NP], const float2 (&p)[NP], const uint32_t *r1,
                                              const uint32_t *r2)
{
#pragma unroll 4
    for (int i = 0; i < MA_ROWS; ++i) {
        const float2 v = __fmul2_rn(bf16x2_to_float2(r1[i * RW]), bf16x2_to_float2(r2[i * RW]));
        modes_step<NP, kCx>(s, p, v);
    }
}

// Triples: rows of 3 RW words, the lane's three words at 3 (l / LPC) (x1/x2/x3
// of its channel pair interleaved).
template <int NP, bool kCx, int RW>
__device__ __forceinline__ void sweep_a_chunk_tri(float2 (&s)[NP], const float2 (&p)[NP], const uint32_t *rw)
{
#pragma unroll 4
    for (int i = 0; i < MA_ROWS; ++i) {
        const uint32_t w0 = rw[i * 3 * RW], w1 = rw[i * 3 * RW + 1], w2 = rw[i * 3 * RW + 2];
        const float2 v = __fmul2_rn(tri_x1(w0, w1), tri_x2(w0, w2));
        modes_step<NP, kCx>(s, p, v);
    }
}

// One token of the output sweep for this lane's channel pair: advance the NP
// states, form the lane's part of conv = sum_n R_n s_n with two independent
// accumulation chains (all state updates first, so the chains find their
// inputs ready), add the LPC lanes' parts of the channel pair (butterfly:
// lane pairs first, then pairs of pairs), apply the gates and store y.
// Complex modes: the table holds (Re R, -Im R) in the slot pair, so the same
// sum is Re sum_m R_m s_m.
template <int NP, int LPC, bool kCx>
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
    float2 conv = __fadd2_rn(a0, a1);
#pragma unroll
    for (int d = 1; d < LPC; d <<= 1) {
        const float2 o = make_float2(__shfl_xor_sync(0xffffffffu, conv.x, d), __shfl_xor_sync(0xffffffffu, conv.y, d));
        conv = __fadd2_rn(conv, o);
    }
    const float2 yv = __ffma2_rn(dsk, v, __fmul2_rn(x3, conv));
    if (store) *yp = float2_to_bf16x2(yv);
}

// v and x3 of row r of an output chunk for the channel pair `pair`.
template <bool kTri, int RW>
__device__ __forceinline__ void chunk_row(const uint32_t *chunk, int pair, int r, float2 &v, float2 &x3)
{
    if constexpr (kTri) {
        const uint32_t *rw = chunk + r * 3 * RW + 3 * pair;
        const uint32_t w0 = rw[0], w1 = rw[1], w2 = rw[2];
        v = __fmul2_rn(tri_x1(w0, w1), tri_x2(w0, w2));
        x3 = tri_x3(w1, w2);
    } else {
        v = __fmul2_rn(bf16x2_to_float2(chunk[r * RW + pair]), bf16x2_to_float2(chunk[(MC_ROWS + r) * RW + pair]));
        x3 = bf16x2_to_float2(chunk[(2 * MC_ROWS + r) * RW + pair]);
    }
}

template <int NP, int LPC, bool kTri, bool kCx>
__device__ void agg_warp(ScanSmem<NP, LPC, kTri> &sm, const ModalArgs &A)
{
    using T = RingTraits<kTri, LPC>;
    constexpr int NPT = NP * LPC;
    constexpr int W = ChainTraits<LPC>::kWidth;
    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    const int groups_per_chain = (A.units + MGMAX - 1) / MGMAX;
    const size_t slot_floats = static_cast<size_t>(MGMAX + 1) * NPT * W;
    int used = 0;  // next chunk number to consume
    for (int k = 0;; ++k) {
        const int c = k & 1;
        wait_local(&sm.gready[c], (k >> 1) & 1, A.hdr);
        const int gi = sm.gid[c];
        if (gi < 0) break;
        const GroupPos q = group_pos(static_cast<unsigned int>(gi), A);
        const LanePos<NP, LPC> lp(lane, q.cb);
        float2 p[NP], s[NP];
        wait_local(&sm.coefbar[c], (k >> 1) & 1, A.hdr);
        coef_rows<NP, ChainTraits<LPC>::kWidth>(p, sm.coef[c], lp.mo, lp.pair);
#pragma unroll
        for (int n = 0; n < NP; ++n) s[n] = make_float2(0.f, 0.f);
        for (int i = 0; i < kAChunks; ++i, ++used) {
            const int b = used % T::kADepth;
            wait_local(&sm.afull[w][b], static_cast<uint32_t>(used / T::kADepth) & 1u, A.hdr);
            if constexpr (kTri)
                sweep_a_chunk_tri<NP, kCx, T::kRW>(s, p, &sm.aring[w][b][0] + 3 * lp.pair);
            else
                sweep_a_chunk<NP, kCx, T::kRW>(s, p, &sm.aring[w][b][0] + lp.pair,
                                               &sm.aring[w][b][MA_ROWS * T::kRW] + lp.pair);
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.aempty[w][b]);
            if (i == kAChunks / 2 - 1) {
#pragma unroll
                for (int n = 0; n < NP; ++n) sm.ctx[c][2 * w + 1][n * 32 + lane] = s[n];
            }
        }
#pragma unroll
        for (int n = 0; n < NP; ++n) sm.ctx[c][2 * w][n * 32 + lane] = s[n];
        // The aggregate also goes to the group's ring slot (for successors'
        // look-backs); the fence lets the control warp release the flag
        // without a fence of its own.
        if (q.s > 0u && static_cast<int>(q.s) + 1 < groups_per_chain) {
            const unsigned int chain = static_cast<unsigned int>(q.b) * A.nCB + q.cb;
            float *slot = A.slots + (static_cast<size_t>(chain) * MRING + q.s % MRING) * slot_floats +
                          (static_cast<size_t>(w) * NPT + lp.mo) * W + 2 * lp.pair;
#pragma unroll
            for (int n = 0; n < NP; ++n) *reinterpret_cast<float2 *>(slot + n * W) = s[n];
            __threadfence();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.adone[c]);
    }
}

template <int NP, int LPC, bool kTri, bool kCx>
__device__ void out_warp(ScanSmem<NP, LPC, kTri> &sm, const ModalArgs &A)
{
    using T = RingTraits<kTri, LPC>;
    constexpr int NPT = NP * LPC;
    const int lane = threadIdx.x & 31;
    const int cw = (threadIdx.x >> 5) - kAW;
    const int w = cw >> 1, h = cw & 1;
    const size_t ystride = static_cast<size_t>(A.ld_y) / 2;  // in 32-bit words
    int used = 0;                                              // next chunk number to consume
    for (int k = 0;; ++k) {
        const int c = k & 1;
        const uint32_t ph = static_cast<uint32_t>(k >> 1) & 1u;
        wait_local(&sm.gready[c], ph, A.hdr);
        const int gi = sm.gid[c];
        if (gi < 0) break;
        const GroupPos q = group_pos(static_cast<unsigned int>(gi), A);
        const LanePos<NP, LPC> lp(lane, q.cb);
        const int c0 = lp.c0;
        const bool ch_ok = c0 < A.D;
        const bool writer = ch_ok && lp.mo == 0;  // one lane per channel pair stores y
        const int j = static_cast<int>(q.s) * MGMAX + w;
        const int t0 = j * MT + h * MH;  // first token of this warp's half unit
        // the second half's p^MH from global first: its loads overlap the waits
        float2 p[NP], R[NP], s[NP];
        if (h == 1) load_rows<NP>(R, A.coef, 3 * NPT + 1 + lp.mo, A.Dp, c0);
        wait_local(&sm.cdone[c], ph, A.hdr);
#pragma unroll
        for (int n = 0; n < NP; ++n) s[n] = sm.ctx[c][2 * w][n * 32 + lane];  // C_j
        if (h == 1) {
            // carry into the second half: p^MH C_j + H_j
#pragma unroll
            for (int n = 0; n < NP; n += 2)
                carry_pair<kCx>(s[n], s[n + 1], R[n], R[n + 1], sm.ctx[c][2 * w + 1][n * 32 + lane],
                                sm.ctx[c][2 * w + 1][(n + 1) * 32 + lane]);
        }
        wait_local(&sm.coefbar[c], ph, A.hdr);
        constexpr int W = ChainTraits<LPC>::kWidth;
        coef_rows<NP, W>(p, sm.coef[c], lp.mo, lp.pair);
        coef_rows<NP, W>(R, sm.coef[c], NPT + lp.mo, lp.pair);
        const float2 dsk = *reinterpret_cast<const float2 *>(sm.coef[c] + 2 * NPT * W + 2 * lp.pair);
        // Release the context only once this group's first chunk has landed:
        // the producer reads the group's id from the context before issuing it.
        wait_local(&sm.cfull[cw][used % T::kCDepth], static_cast<uint32_t>(used / T::kCDepth) & 1u, A.hdr);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.cfree[c]);
        const int nvalid = min(MH, A.L - t0);  // tokens of this half unit inside L (may be <= 0)
        for (int i = 0; i < kCChunks; ++i, ++used) {
            const int b = used % T::kCDepth;
            if (i > 0) wait_local(&sm.cfull[cw][b], static_cast<uint32_t>(used / T::kCDepth) & 1u, A.hdr);
            const int base = i * MC_ROWS;
            const uint32_t *chunk = &sm.cring[cw][b][0];
            if (base < nvalid) {
                uint32_t *yc = reinterpret_cast<uint32_t *>(A.y + (static_cast<size_t>(q.b) * A.L + t0 + base) * A.ld_y +
                                                            c0);
                if (base + MC_ROWS <= nvalid) {
#pragma unroll
                    for (int r = 0; r < MC_ROWS; ++r) {
                        float2 v, x3;
                        chunk_row<kTri, T::kRW>(chunk, lp.pair, r, v, x3);
                        sweep_c_token<NP, LPC, kCx>(s, p, R, dsk, v, x3, yc + r * ystride, writer);
                    }
                } else {
                    for (int r = 0; r < MC_ROWS && base + r < nvalid; ++r) {
                        float2 v, x3;
                        chunk_row<kTri, T::kRW>(chunk, lp.pair, r, v, x3);
                        sweep_c_token<NP, LPC, kCx>(s, p, R, dsk, v, x3, yc + r * ystride, writer);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.cempty[cw][b]);
        }
        // A ragged last unit: the final state is the recurrence state after
        // token L-1, taken by the output warp whose half unit holds it.
        if (A.state_out != nullptr && ch_ok && (A.L % MT) != 0 && nvalid > 0 && t0 + nvalid == A.L) {
#pragma unroll
            for (int n = 0; n < NP; ++n) {
                const int m = lp.mo + n;
                if (m < A.N) {
                    A.state_out[(static_cast<size_t>(q.b) * A.D + c0) * A.N + m] = s[n].x;
                    A.state_out[(static_cast<size_t>(q.b) * A.D + c0 + 1) * A.N + m] = s[n].y;
                }
            }
        }
    }
}

static_assert(sizeof(ScanSmem<16, 2, false>) <= 227 * 1024 && sizeof(ScanSmem<16, 2, true>) <= 227 * 1024 &&
                  sizeof(ScanSmem<16, 4, false>) <= 227 * 1024 && sizeof(ScanSmem<16, 4, true>) <= 227 * 1024,
              "one CTA per SM must fit the shared memory of an SM");

template <int NP, int LPC, bool kTri, bool kCx>
__global__ void __launch_bounds__(kThreads, 1)
    modal_scan_kernel(const __grid_constant__ ModalMaps maps, const ModalArgs A)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    using T = RingTraits<kTri, LPC>;
    ScanSmem<NP, LPC, kTri> &sm = *reinterpret_cast<ScanSmem<NP, LPC, kTri> *>(smem_raw);
    // Flags carry the launch's epoch: the workspace keeps a counter that the
    // last CTA of every launch advances, so flags left by earlier launches
    // (including replays of a captured graph) never match.
    const unsigned int epoch = ld_volatile_u32(A.hdr + 3) + 1u;

    if (threadIdx.x == 0) {
        for (int w = 0; w < kAW; ++w)
            for (int b = 0; b < T::kADepth; ++b) {
                mbar_init(&sm.afull[w][b], 1);
                mbar_init(&sm.aempty[w][b], 1);
            }
        for (int w = 0; w < kCW; ++w)
            for (int b = 0; b < T::kCDepth; ++b) {
                mbar_init(&sm.cfull[w][b], 1);
                mbar_init(&sm.cempty[w][b], 1);
            }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.gready[i], 1);
            mbar_init(&sm.adone[i], kAW);
            mbar_init(&sm.cdone[i], 1);
            mbar_init(&sm.cfree[i], kCW);
            mbar_init(&sm.coefbar[i], 1);
        }
        fence_mbar_init();
    }
    __syncthreads();

    // Warp w runs on SM sub-partition w % 4: each sub-partition gets one
    // aggregate warp, two output warps and one auxiliary warp.
    const int warp = threadIdx.x >> 5;
    if (warp < kAW) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsAgg));
        agg_warp<NP, LPC, kTri, kCx>(sm, A);
    } else if (warp < kAW + kCW) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsOut));
        out_warp<NP, LPC, kTri, kCx>(sm, A);
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsAux));
        if (warp == kCtrlWarp)
            control_warp<NP, LPC, kTri, kCx>(sm, A, epoch);
        else if (warp == kProdWarp)
            producer_warp<NP, LPC, kTri>(sm, maps, A);
    }

    // Every chunk the producer issued belongs to a group the compute warps
    // swept in full, so no TMA is in flight here.
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

template <int NP, int LPC, bool kTri, bool kCx>
int launch_scan(const ModalMaps &maps, ModalArgs a, cudaStream_t st)
{
    static int configured_device = -1;
    static int sms = 0;
    int dev = 0;
    HYENA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
    const int smem = static_cast<int>(sizeof(ScanSmem<NP, LPC, kTri>));
    auto kernel = modal_scan_kernel<NP, LPC, kTri, kCx>;
    if (configured_device != dev) {
        HYENA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
                  "modal scan: set max dynamic shared memory");
        HYENA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "multiprocessor count");
        configured_device = dev;
    }
    const unsigned int groups_per_chain = static_cast<unsigned int>((a.units + MGMAX - 1) / MGMAX);
    a.nGroups = groups_per_chain * static_cast<unsigned int>(a.B) * static_cast<unsigned int>(a.nCB);
    const unsigned int slots = static_cast<unsigned int>(sms);  // one CTA per SM
    const unsigned int grid = a.nGroups < slots ? a.nGroups : slots;
    kernel<<<grid, kThreads, smem, st>>>(maps, a);
    HYENA_TRY(cudaGetLastError(), "modal scan launch");
    return 1;
}

// NPT padded slots beyond 16: NPT / 16 lanes per channel pair, 16 slots each.
template <bool kTri, bool kCx>
int launch_wide_layout(const ModalMaps &maps, const ModalArgs &a, int NPT, cudaStream_t st)
{
    switch (NPT) {
        case 32: return launch_scan<MSLOTS_LANE, 2, kTri, kCx>(maps, a, st);
        case 64: return launch_scan<MSLOTS_LANE, 4, kTri, kCx>(maps, a, st);
        default: return -1;
    }
}

}  // namespace

int launch_modal_wide(const ModalMaps &maps, ModalArgs a, int NPT, bool triples, bool cx, cudaStream_t st)
{
    if (triples)
        return cx ? launch_wide_layout<true, true>(maps, a, NPT, st) : launch_wide_layout<true, false>(maps, a, NPT, st);
    return cx ? launch_wide_layout<false, true>(maps, a, NPT, st) : launch_wide_layout<false, false>(maps, a, NPT, st);
}

}  // namespace hyena
