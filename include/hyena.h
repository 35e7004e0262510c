/*
 * hyena.h -- C ABI of libhyena_b200.so: the gated Hyena cascade operator of
 * StripedHyena 2 / Evo 2 on NVIDIA B200 (sm_100a).
 *
 *   v[t]    = x1[t] * x2[t]
 *   conv[t] = (h_c * v)[t]               causal, depthwise (one filter per channel)
 *   y[t]    = x3[t] * conv[t] + Dskip[c] * v[t]
 *
 * x1, x2, x3 are the three slices of the Hyena input projection and y is the
 * gated filter output that feeds out_proj (evo2_flash README, hook table rows
 * "blocks.N.projections" and "blocks.N.filter").  The filter h_c is either
 * explicit and short (hcs: 7 taps, hcm: 128 taps) or the long modal-form hcl
 * filter h_c[t] = sum_n R[c,n] exp(a[c,n] t) with fp32 log-poles a and
 * residues R (Evo2-7B-262K model card, §Architecture and §Implementation
 * Notes).  Long sequences can be fed in chunks: the modal state (hcl) or the
 * FIR window (hcs/hcm) is carried from one call to the next, and every
 * position of every chunk is produced (Evo2-7B-262K model card, "Custom
 * cache"; turboquant-evo2-int4 model card, §"Important: a correctness fix
 * comes with this" and §"Chunk size").  The long filter is also offered with
 * complex modes, the modal form of Evo 1 (h_c[t] = Re sum_n R p^t), and every
 * operation can read x1, x2, x3 straight from one packed in_proj output
 * (*_packed entry points).
 *
 * Conventions shared by every entry point
 *   - Tensors are bf16 (passed as hyena_bf16_t bit patterns), layout
 *     [B, L, D], channel-contiguous: element (b, t, c) sits at
 *     (b * L + t) * ld + c.  ld >= D is a row stride in elements, so x1, x2,
 *     x3 may be three views of one [B, L, 3D] projection output (ld = 3D).
 *   - Every device pointer is a device address owned by the caller; no
 *     entry point allocates device memory (the modal conv takes a caller
 *     workspace; its allocation-free variant uses a fixed array of the
 *     library's module).  Pointers must be 16-byte aligned, D and ld must be
 *     multiples of 8.
 *   - Arithmetic is fp32 (v is exact in fp32); y is rounded once to bf16
 *     (round to nearest even).  NaN and Inf propagate.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Argument checks run on the host before any launch;
 *     on failure nothing is launched and a non-zero status is returned.
 *     No C++ exception crosses this interface.
 *   - y must not overlap x1, x2, x3.  state_in may equal state_out and
 *     hist_in may equal hist_out (in-place chunking).
 */
#ifndef HYENA_B200_H
#define HYENA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t hyena_bf16_t; /* bf16 bit pattern */

typedef enum {
    HYENA_OK = 0,
    HYENA_ERR_INVALID_ARG = 1, /* null pointer, bad size or shape            */
    HYENA_ERR_ALIGNMENT = 2,   /* pointer / D / ld not aligned as required   */
    HYENA_ERR_UNSUPPORTED = 3, /* N or K outside the supported range         */
    HYENA_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed       */
    HYENA_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out         */
    HYENA_ERR_WORKSPACE = 6    /* workspace missing or too small             */
} hyena_status_t;

/* Human-readable name of a status code (static string, never NULL). */
const char *hyena_status_string(hyena_status_t s);

/* Version of this interface (major * 100 + minor). */
int hyena_abi_version(void);

/* Largest supported number of modes N (real; complex) and of FIR taps K. */
#define HYENA_MAX_MODES 64
#define HYENA_MAX_COMPLEX_MODES 32
#define HYENA_MAX_TAPS 128

/*
 * Explicit short causal FIR (hcs, K = 7; hcm, K = 128): Evo2-7B-262K model
 * card, §Implementation Notes ("Block dispatch": FIR cascades with inner
 * lengths 7 and 128; "Custom cache": the FIR window carried between steps).
 *
 *   conv[t] = sum_{k<K} taps[c*K + k] * v[t-k]     (lag order)
 *
 * taps      [D, K] bf16, device.  1 <= K <= HYENA_MAX_TAPS.
 * Dskip     [D] fp32, device, or NULL (no skip term).
 * hist_in   [B, K-1, D] fp32, device, or NULL: the K-1 values of v that
 *           precede t = 0, oldest first (hist_in[b][K-1-j][c] = v[-j]).
 *           NULL means zeros.
 * hist_out  [B, K-1, D] fp32, device, or NULL: receives the last K-1
 *           values of v of the sequence continued by this call, in the same
 *           layout, ready to be passed as the next call's hist_in.
 * L == 0 is valid: y is untouched and hist_out receives hist_in (or zeros).
 */
hyena_status_t hyena_short_conv(const hyena_bf16_t *x1, const hyena_bf16_t *x2,
                                const hyena_bf16_t *x3, int64_t ld_x,
                                const hyena_bf16_t *taps, const float *Dskip,
                                hyena_bf16_t *y, int64_t ld_y,
                                const float *hist_in, float *hist_out,
                                int B, int L, int D, int K, void *stream);

/*
 * The same operator as hyena_short_conv, computed on the tensor cores as
 * overlap-save DFT-as-GEMM: the FFT route of the Evo2-7B-262K model card,
 * §Implementation Notes (hcl "via FFT", "Block dispatch" for the FIR
 * cascades), restated as GEMMs with a shared real DFT matrix of 256 points
 * so that channels are the MMA's N dimension (tcgen05 kind::tf32, fp32
 * accumulation).  A second implementation for comparison with the FP32 SIMT
 * kernels of hyena_short_conv; the arguments, layouts, ownership and error
 * behaviour are those of hyena_short_conv.  Differences:
 *  - v, the DFT matrices and the spectrum product are rounded to tf32 (11
 *    significant bits) before each product; results agree with
 *    hyena_short_conv to that rounding, not bit for bit;
 *  - each output depends on where its 128-token block starts, so feeding a
 *    sequence in chunks reproduces the single pass to rounding, not bit for
 *    bit (use hyena_short_conv where chunked results must match exactly);
 *  - hist_in values are rounded to tf32 like v (v = x1 x2 of bf16 inputs
 *    is exact only in fp32).
 * The first call on a device copies the DFT tables (384 KB of the library's
 * device memory) with a synchronous copy: make it before any stream capture.
 */
hyena_status_t hyena_short_conv_dft(const hyena_bf16_t *x1, const hyena_bf16_t *x2,
                                    const hyena_bf16_t *x3, int64_t ld_x,
                                    const hyena_bf16_t *taps, const float *Dskip,
                                    hyena_bf16_t *y, int64_t ld_y,
                                    const float *hist_in, float *hist_out,
                                    int B, int L, int D, int K, void *stream);

/*
 * Bytes of device workspace hyena_modal_long_conv needs for B, D, N
 * (independent of L).  Returns 0 for invalid sizes.
 */
size_t hyena_modal_long_conv_workspace_size(int B, int D, int N);

/*
 * Zero-fills a workspace (asynchronously on `stream`).  A workspace must be
 * zero-filled once before its first use; afterwards it can be reused by any
 * number of calls whose workspace size fits, on one stream at a time.
 */
hyena_status_t hyena_modal_workspace_init(void *workspace, size_t workspace_bytes,
                                          void *stream);

/*
 * Long modal-form filter (hcl): Evo2-7B-262K model card, §Architecture
 * (log_poles / residues kept in fp32) and §Implementation Notes (hcl as a
 * modal-form IIR; "Custom cache" for the carried IIR state).
 *
 *   h_c[t] = sum_{n<N} residues[c*N+n] * exp(log_poles[c*N+n] * t),  t >= 0
 *
 * log_poles, residues  [D, N] fp32, device.  1 <= N <= HYENA_MAX_MODES.
 *           Any real log-pole is accepted; the pages' filters have a < 0.
 * Dskip     [D] fp32, device, or NULL (no skip term).
 * state_in  [B, D, N] fp32, device, or NULL (zeros): the per-mode state
 *           s_n = sum_{s<=t} exp(a_n (t-s)) v[s] after the last token of
 *           the previous chunk.  It contributes
 *           sum_n R_n exp(a_n (t+1)) state_in[n] to conv[t].
 * state_out [B, D, N] fp32, device, or NULL: the state after token L-1.
 * workspace device memory of at least
 *           hyena_modal_long_conv_workspace_size(B, D, N) bytes, zero-filled
 *           once by hyena_modal_workspace_init.  Calls sharing a workspace
 *           must not overlap in time (same stream or synchronised).
 * L == 0 is valid: y is untouched and state_out receives state_in (or zeros).
 * Device-side waits are bounded; if one runs out the call's output is
 * invalid and hyena_workspace_check reports HYENA_ERR_TIMEOUT.
 */
hyena_status_t hyena_modal_long_conv(const hyena_bf16_t *x1, const hyena_bf16_t *x2,
                                     const hyena_bf16_t *x3, int64_t ld_x,
                                     const float *log_poles, const float *residues,
                                     const float *Dskip,
                                     hyena_bf16_t *y, int64_t ld_y,
                                     const float *state_in, float *state_out,
                                     int B, int L, int D, int N,
                                     void *workspace, size_t workspace_bytes,
                                     void *stream);

/*
 * Chunked prefill with the filter synthesised once (turboquant-evo2-int4
 * model card, §"Chunk size": a long prompt is fed in chunks through the same
 * layer; the filter is the same for every chunk).
 *
 * hyena_modal_prepare forms the coefficient table of the real-mode filter
 * (p = exp(a) with CUDA's expf, residues, skip, p^64, p^128) in `workspace`,
 * as the first step of every hyena_modal_long_conv call does; arguments and
 * errors as there (the workspace sized for B, D, N).
 * hyena_modal_long_conv_prepared is hyena_modal_long_conv without that step:
 * it uses the table the last hyena_modal_prepare on this workspace left, and
 * gives the same bits as hyena_modal_long_conv with those parameters.  Any
 * other modal call on the workspace (hyena_modal_long_conv and its variants)
 * replaces the table with its own parameters' table; prepare again after it.
 * Real modes only (complex modes: hyena_modal_long_conv_complex).
 */
hyena_status_t hyena_modal_prepare(const float *log_poles, const float *residues, const float *Dskip,
                                   int B, int D, int N, void *workspace, size_t workspace_bytes,
                                   void *stream);

hyena_status_t hyena_modal_long_conv_prepared(const hyena_bf16_t *x1, const hyena_bf16_t *x2,
                                              const hyena_bf16_t *x3, int64_t ld_x,
                                              hyena_bf16_t *y, int64_t ld_y,
                                              const float *state_in, float *state_out,
                                              int B, int L, int D, int N,
                                              void *workspace, size_t workspace_bytes,
                                              void *stream);

/*
 * hyena_modal_long_conv over inputs and outputs in HOST memory (no
 * counterpart on the pages: the chunked prefill of the Evo2-7B-262K model
 * card's "Custom cache" and the turboquant-evo2-int4 card's §"Chunk size",
 * applied to a sequence that is not resident on the device).
 *
 * x1, x2, x3 [B, L, ld_x] and y [B, L, ld_y] are host pointers (bf16); page-
 * locked memory (cudaHostAlloc / cudaHostRegister) lets the copies overlap,
 * pageable memory works but serialises them.  log_poles, residues, Dskip,
 * state_in and state_out are device pointers as in hyena_modal_long_conv.
 * The sequence is streamed through the device in chunks of `chunk` tokens
 * (a positive multiple of 128): while chunk i is scanned on `stream`, chunk
 * i+1 is copied host->device and chunk i-1's output device->host on two copy
 * streams the library owns (one pair per device), so the host link carries
 * both directions at once.  The modal state is carried from chunk to chunk,
 * and because every chunk boundary is a unit boundary y and state_out equal
 * the single pass bit for bit.
 * workspace  device, >= hyena_modal_host_workspace_size(B, D, N, chunk)
 *            bytes, 256-byte aligned, zero-filled once by
 *            hyena_modal_workspace_init: the scan's workspace, two staging
 *            slots of x1/x2/x3/y for `chunk` tokens and the carried state.
 * On return the work is enqueued; `stream` is ordered after the last copy to
 * the host, so synchronising `stream` makes y valid.  Not capturable into a
 * CUDA graph (it orders the library's copy streams with events); calls on
 * one device are enqueued one at a time (a lock), and calls sharing a
 * workspace must not overlap in time.  Errors as hyena_modal_long_conv, plus
 * HYENA_ERR_INVALID_ARG for a chunk that is not a positive multiple of 128.
 */
size_t hyena_modal_host_workspace_size(int B, int D, int N, int chunk);

hyena_status_t hyena_modal_long_conv_host(const hyena_bf16_t *x1, const hyena_bf16_t *x2,
                                          const hyena_bf16_t *x3, int64_t ld_x,
                                          const float *log_poles, const float *residues,
                                          const float *Dskip,
                                          hyena_bf16_t *y, int64_t ld_y,
                                          const float *state_in, float *state_out,
                                          int B, int L, int D, int N, int chunk,
                                          void *workspace, size_t workspace_bytes,
                                          void *stream);

/*
 * hyena_short_conv over inputs and outputs in HOST memory, streamed like
 * hyena_modal_long_conv_host with the FIR window carried from chunk to chunk
 * (Evo1-1.5-7B-8K model card, "Cache subclass": the FIR window).  Any chunk
 * >= 1 gives y and hist_out equal to the single pass bit for bit.  taps,
 * Dskip, hist_in and hist_out are device pointers as in hyena_short_conv.
 * workspace  device, >= hyena_short_host_workspace_size(B, D, K, chunk)
 *            bytes, 256-byte aligned (no initialisation needed): two staging
 *            slots of x1/x2/x3/y for `chunk` tokens and the carried window.
 * Ordering, locking and graph capture as hyena_modal_long_conv_host.
 */
size_t hyena_short_host_workspace_size(int B, int D, int K, int chunk);

hyena_status_t hyena_short_conv_host(const hyena_bf16_t *x1, const hyena_bf16_t *x2,
                                     const hyena_bf16_t *x3, int64_t ld_x,
                                     const hyena_bf16_t *taps, const float *Dskip,
                                     hyena_bf16_t *y, int64_t ld_y,
                                     const float *hist_in, float *hist_out,
                                     int B, int L, int D, int K, int chunk,
                                     void *workspace, size_t workspace_bytes,
                                     void *stream);

/*
 * Allocation-free variant of hyena_modal_long_conv (no counterpart on the
 * pages: it exists for callers of this library that must not allocate device
 * memory).  Some callers cannot call cudaMalloc or take memory from an
 * allocator: a plugin that runs inside a host framework which owns all device
 * memory and accounts for it, or code on a latency-critical path where an
 * allocation could synchronise the device.  This entry point takes the same
 * inputs and outputs as hyena_modal_long_conv but no workspace: its scratch
 * is a fixed array of HYENA_NOALLOC_SCRATCH_BYTES in device memory that the
 * library owns (every GPU that loads that part of the library holds it until
 * the process exits).  It calls no allocating routine.
 *
 * Limit: B, D, N must satisfy
 *   hyena_modal_long_conv_workspace_size(B, D, N) <= HYENA_NOALLOC_SCRATCH_BYTES
 * (at N = 16: B * ceil(D / 64) <= 73 channel blocks, e.g. B = 1 and D up to
 * 4672); larger sizes return HYENA_ERR_WORKSPACE and launch nothing.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  All calls share the one array: calls that overlap on the GPU (on
 * different streams, or from different threads without ordering) race and
 * produce wrong results.  Before its scan, each call enqueues one small
 * kernel that moves the previous call's device-side error bits aside and
 * zeroes the look-back flags of its own (B, D, N) layout.  A bounded device
 * wait that runs out invalidates that call's output; the call itself returns
 * before the GPU runs, so it cannot report it: hyena_modal_noalloc_check does.
 * The cached device address is valid for the device's current context only:
 * do not use this entry point across a device reset.
 */
#define HYENA_NOALLOC_SCRATCH_BYTES (24u << 20)

hyena_status_t hyena_modal_long_conv_noalloc(const hyena_bf16_t *x1, const hyena_bf16_t *x2,
                                             const hyena_bf16_t *x3, int64_t ld_x,
                                             const float *log_poles, const float *residues,
                                             const float *Dskip,
                                             hyena_bf16_t *y, int64_t ld_y,
                                             const float *state_in, float *state_out,
                                             int B, int L, int D, int N, void *stream);

/*
 * Reports device-side failures of hyena_modal_long_conv_noalloc calls on the
 * current device (no counterpart on the pages; the allocation-free
 * counterpart of hyena_workspace_check).  Synchronises `stream`, then returns
 * HYENA_ERR_TIMEOUT if a bounded wait ran out in any call since the previous
 * check (that call's y and state_out are invalid; later calls are not
 * affected) and clears the record; HYENA_OK otherwise.  Allocates nothing.
 */
hyena_status_t hyena_modal_noalloc_check(void *stream);

/*
 * The device address and size of the fixed scratch array that
 * hyena_modal_long_conv_noalloc uses on the current device (no counterpart on
 * the pages), for callers that account for device memory or that want to
 * inspect it.  The array's header holds, as 32-bit words: [0] the next group
 * ticket, [1] finished CTAs, [2] error bits of the running call, [3] the
 * launch epoch, [4] error bits not yet reported by hyena_modal_noalloc_check.
 * Writing to the array while a call runs corrupts that call.  The first use
 * on a device performs the address look-up (make it before any stream
 * capture).
 */
hyena_status_t hyena_modal_noalloc_scratch(void **device_ptr, size_t *bytes);

/*
 * One generated token through the long modal filter: the recurrent form of
 * hcl (Evo2-7B-262K model card, §Implementation Notes and "Custom cache":
 * generation carries the IIR state from token to token).
 *
 *   v = x1 * x2;  s_n <- exp(log_poles[c,n]) * s_n + v;
 *   y = x3 * sum_n residues[c,n] * s_n + Dskip[c] * v
 *
 * x1, x2, x3, y  one token per batch row: element (b, c) at b * ld + c.
 * state  [B, D, N] fp32, device, read and updated in place: the state after
 *        the previous token (zeros before the first one).  Required.
 * log_poles, residues [D, N], Dskip [D] or NULL: as hyena_modal_long_conv.
 * The result equals hyena_modal_long_conv with L = 1 and
 * state_in = state_out = state bit for bit.  No workspace; one launch.
 */
hyena_status_t hyena_modal_decode(const hyena_bf16_t *x1, const hyena_bf16_t *x2,
                                  const hyena_bf16_t *x3, int64_t ld_x,
                                  const float *log_poles, const float *residues,
                                  const float *Dskip,
                                  hyena_bf16_t *y, int64_t ld_y,
                                  float *state, int B, int D, int N, void *stream);

/*
 * One generated token through an explicit FIR (hcs/hcm): conv = sum_{k<K}
 * taps[c,k] v[t-k] with v[t-k], k >= 1, from the window, which then advances
 * by one token in place (Evo2-7B-262K model card, "Custom cache"; the FIR
 * window of Evo1-1.5-7B-8K model card, "Cache subclass").
 *
 * hist   [B, K-1, D] fp32, device, in time order (hist[b, K-2, c] is v of the
 *        previous token; zeros before the first one); read and updated in
 *        place.  Required when K > 1, ignored when K = 1.
 * taps   [D, K] bf16 in lag order, Dskip [D] or NULL: as hyena_short_conv.
 * The result equals hyena_short_conv with L = 1 and hist_in = hist_out = hist
 * bit for bit.  One launch.
 */
hyena_status_t hyena_short_decode(const hyena_bf16_t *x1, const hyena_bf16_t *x2,
                                  const hyena_bf16_t *x3, int64_t ld_x,
                                  const hyena_bf16_t *taps, const float *Dskip,
                                  hyena_bf16_t *y, int64_t ld_y,
                                  float *hist, int B, int D, int K, void *stream);

/*
 * Long modal filter with complex modes: the modal form of Evo1-1.5-7B-8K
 * (model card, §Architecture: modal-form "poles" / "residues" kept in fp32,
 * Hyena state size 8).  Mode n of channel c has a complex pole p and residue
 * R, and the filter is the real part of the modal sum:
 *
 *   h_c[t] = Re sum_{n<N} R[c,n] p[c,n]^t,  t >= 0
 *
 * (a conjugate pair (p, R), (conj p, conj R) is one mode with residue 2R).
 * poles, residues  [D, N, 2] fp32, device: (real, imaginary) of each mode.
 *           1 <= N <= HYENA_MAX_COMPLEX_MODES.
 * state_in, state_out  [B, D, N, 2] fp32, device, or NULL: the complex state
 *           s_n = sum_{s<=t} p_n^(t-s) v[s] after the last token of the
 *           previous chunk (as hyena_modal_long_conv, with complex p).
 * workspace at least hyena_modal_long_conv_workspace_size(B, D, 2N) bytes,
 *           zero-filled once by hyena_modal_workspace_init.
 * Everything else, the chunking guarantees (bit-exact for chunks of whole
 * 128-token units) and the errors are those of hyena_modal_long_conv.
 */
hyena_status_t hyena_modal_long_conv_complex(const hyena_bf16_t *x1, const hyena_bf16_t *x2,
                                             const hyena_bf16_t *x3, int64_t ld_x,
                                             const float *poles, const float *residues,
                                             const float *Dskip,
                                             hyena_bf16_t *y, int64_t ld_y,
                                             const float *state_in, float *state_out,
                                             int B, int L, int D, int N,
                                             void *workspace, size_t workspace_bytes,
                                             void *stream);

/*
 * One generated token through the complex-mode filter: s_n <- p_n s_n + v,
 * y = x3 Re(sum_n R_n s_n) + Dskip v, with state [B, D, N, 2] fp32 updated in
 * place.  Equals hyena_modal_long_conv_complex with L = 1 and
 * state_in = state_out = state bit for bit.
 */
hyena_status_t hyena_modal_decode_complex(const hyena_bf16_t *x1, const hyena_bf16_t *x2,
                                          const hyena_bf16_t *x3, int64_t ld_x,
                                          const float *poles, const float *residues,
                                          const float *Dskip,
                                          hyena_bf16_t *y, int64_t ld_y,
                                          float *state, int B, int D, int N, void *stream);

/*
 * Packed projection inputs.  The Hyena input projection writes one
 * [B, L, 3D] output per block (evo2_flash README, hook table row
 * "blocks.N.projections", the in_proj output of width 3H), and its Hyena
 * channels are interleaved per triple (same README, §Limitations).  The
 * *_packed entry points read x1, x2, x3 straight from such a buffer:
 *
 * xp     [B, L, ld_x] bf16, device, 16-byte aligned; ld_x >= 3D, ld_x % 8 == 0.
 *        For decode, L = 1: row b at b * ld_x.
 * group  channels per group.  Row (b, t) holds, for each group g of `group`
 *        channels, the group's x1 values, then its x2 values, then its x3
 *        values:
 *          x_k[b, t, c] = xp[(b*L + t)*ld_x + 3*group*(c / group)
 *                            + (k-1)*group + c % group],   k = 1, 2, 3.
 *        group = 1 is the per-channel triple interleave (x1_c, x2_c, x3_c
 *        adjacent); group = D is three [x1 | x2 | x3] blocks (the same as
 *        passing the three views to the plain entry points).
 *        Supported: group = 1, group = D, or group a multiple of 8 that
 *        divides D and either divides 64 or is a multiple of 64.  group < 1
 *        or D % group != 0 gives HYENA_ERR_INVALID_ARG, any other group
 *        HYENA_ERR_UNSUPPORTED.
 * Every other argument, the result (bit for bit) and the error behaviour are
 * those of the plain entry point with the same name minus "_packed"; y must
 * not overlap xp.
 */
hyena_status_t hyena_modal_long_conv_packed(const hyena_bf16_t *xp, int64_t ld_x, int group,
                                            const float *log_poles, const float *residues,
                                            const float *Dskip,
                                            hyena_bf16_t *y, int64_t ld_y,
                                            const float *state_in, float *state_out,
                                            int B, int L, int D, int N,
                                            void *workspace, size_t workspace_bytes,
                                            void *stream);

hyena_status_t hyena_short_conv_packed(const hyena_bf16_t *xp, int64_t ld_x, int group,
                                       const hyena_bf16_t *taps, const float *Dskip,
                                       hyena_bf16_t *y, int64_t ld_y,
                                       const float *hist_in, float *hist_out,
                                       int B, int L, int D, int K, void *stream);

hyena_status_t hyena_modal_decode_packed(const hyena_bf16_t *xp, int64_t ld_x, int group,
                                         const float *log_poles, const float *residues,
                                         const float *Dskip,
                                         hyena_bf16_t *y, int64_t ld_y,
                                         float *state, int B, int D, int N, void *stream);

hyena_status_t hyena_short_decode_packed(const hyena_bf16_t *xp, int64_t ld_x, int group,
                                         const hyena_bf16_t *taps, const float *Dskip,
                                         hyena_bf16_t *y, int64_t ld_y,
                                         float *hist, int B, int D, int K, void *stream);

/* The complex-mode filter (hyena_modal_long_conv_complex, hyena_modal_decode_complex)
 * with packed projection inputs, as above. */
hyena_status_t hyena_modal_long_conv_complex_packed(const hyena_bf16_t *xp, int64_t ld_x, int group,
                                                    const float *poles, const float *residues,
                                                    const float *Dskip,
                                                    hyena_bf16_t *y, int64_t ld_y,
                                                    const float *state_in, float *state_out,
                                                    int B, int L, int D, int N,
                                                    void *workspace, size_t workspace_bytes,
                                                    void *stream);

hyena_status_t hyena_modal_decode_complex_packed(const hyena_bf16_t *xp, int64_t ld_x, int group,
                                                 const float *poles, const float *residues,
                                                 const float *Dskip,
                                                 hyena_bf16_t *y, int64_t ld_y,
                                                 float *state, int B, int D, int N, void *stream);

/*
 * Zero-fills a modal state [B, D, N] fp32 (the state before the first token
 * of a sequence): the start of chunked prefill.  The carried IIR state is the
 * cache that the Evo2-7B-262K model card's §Implementation Notes ("Custom
 * cache") keeps for hcl between calls; the turboquant-evo2-int4 model card,
 * §"Important: a correctness fix comes with this" and §"Chunk size", requires
 * every chunk of a prefill to continue from the previous chunk's state, and a
 * new sequence starts from the empty one.  N >= 1 counts the state's floats
 * per channel (pass 2N for N complex modes).  Asynchronous on `stream`.
 */
hyena_status_t hyena_modal_state_init(float *state, int B, int D, int N, void *stream);

/*
 * Synchronises `stream`, then reports (and clears) a device-side error that
 * calls using this workspace recorded: HYENA_ERR_TIMEOUT if a bounded wait
 * ran out, HYENA_OK otherwise.
 */
hyena_status_t hyena_workspace_check(void *workspace, void *stream);

/*
 * Number of kernels (and memset/copy nodes) the most recent successful call
 * of each entry point on this thread enqueued; used by benchmarks to report
 * launch counts.
 */
int hyena_last_launch_count(void);

/*
 * Text describing the most recent failing CUDA runtime call made by an entry
 * point on this thread (the cause behind HYENA_ERR_CUDA); a static,
 * thread-local string, never NULL.
 */
const char *hyena_last_error_message(void);

#ifdef __cplusplus
}
#endif

#endif /* HYENA_B200_H */
