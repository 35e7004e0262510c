// hyena_internal.h -- host-side declarations shared by the entry points and
// the kernel launchers (not part of the public interface).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/hyena.h"

namespace hyena {

// Remembers the most recent failing CUDA call of this thread (reported by
// hyena_last_error_message).
void record_cuda_error(cudaError_t e, const char *where);
void record_message(const char *msg);
// Adds to the launch count that hyena_last_launch_count reports for the
// calling thread's most recent call.
void add_launches(int n);
void set_last_launches(int n);  // the launch count hyena_last_launch_count reports

#define HYENA_TRY(call, where)                       \
    do {                                             \
        const cudaError_t e_ = (call);               \
        if (e_ != cudaSuccess) {                     \
            ::hyena::record_cuda_error(e_, where);   \
            return -1;                               \
        }                                            \
    } while (0)

// ---------------------------------------------------------------- inputs
// Where x1, x2 and x3 live.  Channels come in groups of `group`; the row of
// token t holds, for group g, the group's x1 values, then its x2 values, then
// its x3 values, and x[k] points at element 0 of x_{k+1}.  Channel c of x_{k+1}
// is therefore at column x_col(c, group) of x[k]:
//   separate tensors  group = D, x[k] = the tensor (column c);
//   packed, group G   x[k] = xp + k G (column 3G (c / G) + c % G);
//   triples           group = 1, x[k] = xp + k (column 3c): the per-channel
//                     interleave (x1_c, x2_c, x3_c adjacent).
__host__ __device__ __forceinline__ long long x_col(int c, int group)
{
    return 3ll * group * (c / group) + c % group;
}

// ---------------------------------------------------------------- modal scan
// A chain is the sequence of MCH channels of one batch row over time.  A unit
// is MT consecutive tokens of a chain: the carry from one unit to the next
// follows one canonical fp32 recurrence, so feeding a sequence in chunks of
// whole units reproduces the single pass bit for bit.  A group is up to MGMAX
// consecutive units of a chain, the work item one CTA takes at a time.
// Up to 16 mode slots per lane: lane l of a warp owns the channel pair 2l,
// 2l+1 of a 64-channel chain and all its (padded) mode slots.  With 32 or 64
// slots, LPC = 2 or 4 lanes share a channel pair, each owning 16 consecutive
// slots, and a chain is 64 / LPC channels wide.
constexpr int MCH = 64;
constexpr int MT = 128;
constexpr int MH = MT / 2;
constexpr int MRING = 16;  // group slots per chain
constexpr int MLB = 8;     // deepest look-back, in groups
constexpr int MGMAX = 4;   // units per group (slots are sized for it)

constexpr int MSLOTS_LANE = 16;  // most mode slots one lane holds

// Padded mode slots per channel (NPT): 4, 8, 16, 32 or 64.
inline int modal_padded_modes(int N) { return N <= 4 ? 4 : (N <= 8 ? 8 : (N <= 16 ? 16 : (N <= 32 ? 32 : 64))); }
// Lanes per channel pair (LPC) and slots per lane for NPT padded slots.
inline int modal_lanes_per_pair(int NPT) { return NPT <= MSLOTS_LANE ? 1 : NPT / MSLOTS_LANE; }
inline int modal_lane_slots(int NPT) { return NPT <= MSLOTS_LANE ? NPT : MSLOTS_LANE; }

// Coefficient table [4NPT+1][Dp]: rows [0, NPT) p = exp(a), [NPT, 2NPT)
// residues, row 2NPT Dskip, rows [2NPT+1, 3NPT+1) p^MT, rows [3NPT+1, 4NPT+1)
// p^MH.
inline int modal_coef_rows(int NPT) { return 4 * NPT + 1; }

struct ModalLayout {
    int NP = 0;    // padded mode slots per channel (NPT)
    int LPC = 1;   // lanes per channel pair
    int nCB = 0;   // chains per batch row (chain width MCH / LPC)
    int Dp = 0;
    size_t off_hdr = 0, off_coef = 0, off_flags = 0, off_slots = 0, total = 0;
};

ModalLayout modal_layout(int B, int D, int N);

struct ModalArgs {
    const uint16_t *x1, *x2, *x3;  // x[0..2] of the input source (see x_col)
    long long ld_x;
    int group;                  // channel group of the inputs (see x_col)
    uint16_t *y;
    long long ld_y;
    const float *state_in;
    float *state_out;
    int B, L, D, N;
    int nCB, Dp;                // chains per batch row (MCH / LPC channels each), nCB * chain width
    int units;                  // units per chain, ceil(L / MT)
    unsigned int nGroups;       // groups over all chains
    const float *coef;          // [4NPT+1][Dp]
    unsigned long long *flags;  // [B*nCB][MRING]
    float *slots;               // [B*nCB][MRING][MGMAX+1][NPT][chain width]
    unsigned int *hdr;          // [0] ticket, [1] finished CTAs, [2] error bits, [3] epoch
};

// Real modes: log_poles [D][N], residues [D][N].  Complex modes: log_poles
// holds the poles and residues the residues as [D][N/2][2] (N counts slots,
// two per complex mode).
struct ModalSynthArgs {
    const float *log_poles, *residues, *Dskip;
    int D, N, Dp;
    float *coef;
};

// Up to 16 mode slots (the common case) the scan runs as the look-back kernel
// of modal_scan.cu (two or three CTAs per SM): each compute warp sweeps its
// unit's aggregate and then its outputs, streaming chunks of MCK rows x MCH
// channels of x1/x2 (and x3); short sequences take that file's two-pass path
// (below).  With 32 or 64 slots the scan runs as the warp-specialised kernel of
// modal_scan_wide.cu (chains of MCH / LPC channels; aggregate warps read
// chunks of MA_ROWS rows, output warps chunks of MC_ROWS rows).
constexpr int MCK = 16;
constexpr int MA_ROWS = 16;
constexpr int MC_ROWS = 16;

// Launches the coefficient-synthesis kernel for NPT padded slots; returns the
// number of launches enqueued or a negative value on a CUDA error.  With `cx`
// the N of the arguments counts mode slots, two per complex mode.
int launch_modal_synth(const ModalSynthArgs &s, int NPT, bool cx, cudaStream_t st);

// The scan for NP <= 16 padded slots: three 4-D tensor maps [B][L][groups][group]
// over x1, x2, x3 with boxes of MCK rows x MCH channels; with `triples` the
// first map alone covers the interleaved rows (boxes of MCK rows x 3 MCH
// elements) and the other two are unused.  With `cx` the N of the arguments
// counts mode slots, two per complex mode (state [B][D][N/2][2] = [B][D][N]).
// Returns the number of launches or a negative value on a CUDA error.
int launch_modal_narrow(const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &m3, ModalArgs a, int NP,
                        bool triples, bool cx, cudaStream_t st);

// The scan for NPT = 32 or 64 padded slots.  Maps over x1, x2 (a1, a2: boxes
// of MA_ROWS rows x chain width) and x1, x2, x3 (c1..c3: boxes of MC_ROWS
// rows); with `triples` a1 and c1 alone cover the interleaved rows.  coef: a
// 2-D map over the coefficient table [4NPT+1][Dp] fp32, box of one chain's
// columns x rows [0, 2NPT+1) (p, residues, Dskip).
struct ModalMaps {
    CUtensorMap a1, a2, c1, c2, c3, coef;
};

// Short sequences: up to 16 slots, at most MSHORT_UNITS units per chain whose
// x1/x2 rows (B L D 4 bytes, 6 for triples) fit in MSHORT_L2_BYTES of L2.
// There the scan runs as two plain passes over all units at once (aggregates,
// then carries and outputs) with the look-back kernel's arithmetic.
constexpr int MSHORT_UNITS = 24;
constexpr long long MSHORT_L2_BYTES = 48ll << 20;
bool modal_short_path(int B, int L, int D, int NP, bool triples);
int launch_modal_short(const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &m3, const ModalArgs &a,
                       int NP, bool triples, bool cx, cudaStream_t st);

int launch_modal_wide(const ModalMaps &maps, ModalArgs a, int NPT, bool triples, bool cx, cudaStream_t st);

// ---------------------------------------------------------------- short FIR
constexpr int FCH = 64;   // channels per CTA
constexpr int FT = 128;   // output tokens per CTA
constexpr int FW = 8;     // warps per CTA
constexpr int FRW = FT / FW;  // output rows per warp

inline int fir_halo_rows(int K) { return K <= 1 ? 0 : ((K - 1 + 7) / 8) * 8; }

// Filters longer than 8 taps run the persistent kernel (one CTA per SM walking
// tile ranges); shorter ones one CTA per tile.
inline bool fir_persistent(int K) { return K > 8; }

struct FirArgs {
    const uint16_t *taps;
    const float *Dskip;
    uint16_t *y;
    long long ld_y;
    const float *hist_in;
    int B, L, D, K, HR;
    const uint16_t *x1, *x2;  // for the history kernel
    long long ld_x;
    int group;                // channel group of the inputs (see x_col)
    float *hist_out;
};

// One-token decode step (modal state or FIR window advanced in place).
struct DecodeArgs {
    const uint16_t *x1, *x2, *x3;
    long long ld_x;
    int group;                          // channel group of the inputs (see x_col)
    const float *log_poles, *residues;  // modal
    const uint16_t *taps;               // FIR
    const float *Dskip;
    uint16_t *y;
    long long ld_y;
    float *state;  // modal [B, D, N]
    float *hist;   // FIR [B, K-1, D]
    int B, D, N, K;
};

int launch_modal_decode(const DecodeArgs &a, bool cx, cudaStream_t st);
int launch_fir_decode(const DecodeArgs &a, cudaStream_t st);

// Tile maps m1..m3 (FT rows) and halo maps h1, h2 (HR rows) over x1, x2, x3,
// as for the modal scan; with `triples`, m1 and h1 alone cover the
// interleaved rows.
int launch_fir(const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &m3,
               const CUtensorMap &h1, const CUtensorMap &h2, const FirArgs &a,
               bool triples, cudaStream_t st);

// hist_out (the last K-1 values of v), when requested: 0 or 1 launches, or -1.
int launch_fir_history(const FirArgs &a, cudaStream_t st);

// The FIR as overlap-save DFT-as-GEMM on the tensor cores (fir_dft.cu): tile
// maps m1..m3 of FT rows over separate or packed inputs (no triples), then the
// history as launch_fir_history.
int launch_fir_dft(const CUtensorMap &m1, const CUtensorMap &m2, const CUtensorMap &m3, const FirArgs &a,
                   cudaStream_t st);

}  // namespace hyena
