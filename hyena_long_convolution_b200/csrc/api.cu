// api.cu -- the extern "C" entry points of libhyena_b200.so: argument checks,
// TMA descriptor encoding, workspace layout and dispatch to the sm_100a
// kernels.  Nothing here computes any part of the operator.
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>

#include "hyena_internal.h"

namespace hyena {

namespace {

thread_local int g_last_launches = 0;
thread_local char g_last_error[256] = "no error";

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

void resolve_encode()
{
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Where x1, x2, x3 are read from (see x_col): three tensors (group = D), a
// packed projection buffer in channel groups, or per-channel triples.
struct XSource {
    const hyena_bf16_t *x[3];
    long long ld;
    int group;
    bool triples;
};

XSource separate_source(const hyena_bf16_t *x1, const hyena_bf16_t *x2, const hyena_bf16_t *x3, long long ld, int D)
{
    return XSource{{x1, x2, x3}, ld, D, false};
}

XSource packed_source(const hyena_bf16_t *xp, long long ld, int group)
{
    if (xp == nullptr) return XSource{{nullptr, nullptr, nullptr}, ld, group, group == 1};
    return XSource{{xp, xp + group, xp + 2 * static_cast<long long>(group)}, ld, group, group == 1};
}

// 4-D bf16 tensor map [B][L][groups][group] over input k (0..2), box of `rows`
// tokens x `width` channels (64, or 32 / 16 for the modal scan's narrower
// chains): dims {group, D / group, L, B}, the group stride 3 group elements
// (unused for a single group).  Triples: one map over the interleaved rows,
// dims {3D, 1, L, B}, box of `rows` tokens x 3 width values (width channels'
// triples).  `promo`: how far L2 widens each row request; 256 bytes suits
// grids whose concurrent CTAs read neighbouring channel groups (the widened
// half is theirs), 128 bytes a persistent grid whose CTAs are far apart.
bool encode_x_map(CUtensorMap *m, const XSource &xs, int k, int B, int L, int D, int rows, int width = 64,
                  CUtensorMapL2promotion promo = CU_TENSOR_MAP_L2_PROMOTION_L2_256B)
{
    std::call_once(g_encode_once, resolve_encode);
    if (g_encode == nullptr) return false;
    const cuuint64_t row_bytes = static_cast<cuuint64_t>(xs.ld) * 2;
    cuuint64_t dims[4], strides[3];
    cuuint32_t box[4];
    if (xs.triples) {
        dims[0] = 3ull * static_cast<cuuint64_t>(D);
        dims[1] = 1;
        strides[0] = row_bytes;
        box[0] = 3u * static_cast<cuuint32_t>(width);
        box[1] = 1u;
    } else {
        const int groups = D / xs.group;
        dims[0] = static_cast<cuuint64_t>(xs.group);
        dims[1] = static_cast<cuuint64_t>(groups);
        strides[0] = groups > 1 ? 6ull * static_cast<cuuint64_t>(xs.group) : row_bytes;
        // `width` channels per box: one run of width within a group (a single
        // group reads past its end as zeros), or width / group whole groups of
        // fewer channels (group divides width)
        const bool runs = groups == 1 || xs.group >= width;
        box[0] = static_cast<cuuint32_t>(runs ? width : xs.group);
        box[1] = static_cast<cuuint32_t>(runs ? 1 : width / xs.group);
    }
    dims[2] = static_cast<cuuint64_t>(L);
    dims[3] = static_cast<cuuint64_t>(B);
    strides[1] = row_bytes;
    strides[2] = row_bytes * static_cast<cuuint64_t>(L);
    box[2] = static_cast<cuuint32_t>(rows);
    box[3] = 1u;
    cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<hyena_bf16_t *>(xs.x[k]), dims,
                                strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                CU_TENSOR_MAP_SWIZZLE_NONE, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D fp32 tensor map over the modal coefficient table [4 NPT + 1][Dp]: box
// of `width` columns (one chain) x rows [0, 2 NPT + 1) (p, residues, Dskip).
bool encode_coef_map(CUtensorMap *m, void *table, int Dp, int NPT, int width)
{
    std::call_once(g_encode_once, resolve_encode);
    if (g_encode == nullptr) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(Dp), static_cast<cuuint64_t>(modal_coef_rows(NPT))};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(Dp) * 4};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(width), static_cast<cuuint32_t>(2 * NPT + 1)};
    cuuint32_t estr[2] = {1u, 1u};
    const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, table, dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

hyena_status_t check_x(const void *x1, const void *x2, const void *x3, long long ld_x, const void *y,
                       long long ld_y, int B, int L, int D)
{
    if (B < 1 || L < 0 || D < 1) return HYENA_ERR_INVALID_ARG;
    if (L > 0) {
        if (!x1 || !x2 || !x3 || !y) return HYENA_ERR_INVALID_ARG;
        if (ld_x < D || ld_y < D) return HYENA_ERR_INVALID_ARG;
        if ((ld_x % 8) || (ld_y % 8)) return HYENA_ERR_ALIGNMENT;
        if (!aligned16(x1) || !aligned16(x2) || !aligned16(x3) || !aligned16(y))
            return HYENA_ERR_ALIGNMENT;
        // element offsets must fit the 32-bit TMA coordinates and 40-bit strides
        if (static_cast<long long>(L) * ld_x * 2 >= (1ll << 40)) return HYENA_ERR_UNSUPPORTED;
    }
    if (D % 8) return HYENA_ERR_ALIGNMENT;
    return HYENA_OK;
}

// Checks of a packed projection buffer (the counterpart of check_x).
hyena_status_t check_packed(const void *xp, long long ld_x, int group, const void *y, long long ld_y, int B, int L,
                            int D)
{
    if (B < 1 || L < 0 || D < 1) return HYENA_ERR_INVALID_ARG;
    if (D % 8) return HYENA_ERR_ALIGNMENT;
    if (group < 1 || D % group) return HYENA_ERR_INVALID_ARG;
    if (!(group == 1 || group == D || (group % 8 == 0 && (64 % group == 0 || group % 64 == 0))))
        return HYENA_ERR_UNSUPPORTED;
    if (L > 0) {
        if (!xp || !y) return HYENA_ERR_INVALID_ARG;
        if (ld_x < 3ll * D || ld_y < D) return HYENA_ERR_INVALID_ARG;
        if ((ld_x % 8) || (ld_y % 8)) return HYENA_ERR_ALIGNMENT;
        if (!aligned16(xp) || !aligned16(y)) return HYENA_ERR_ALIGNMENT;
        if (static_cast<long long>(L) * ld_x * 2 >= (1ll << 40)) return HYENA_ERR_UNSUPPORTED;
    }
    return HYENA_OK;
}

hyena_status_t copy_or_zero(float *dst, const float *src, size_t bytes, cudaStream_t st, int &launches)
{
    if (dst == nullptr) return HYENA_OK;
    if (src == dst) return HYENA_OK;
    const cudaError_t e = src ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st)
                              : cudaMemsetAsync(dst, 0, bytes, st);
    if (e != cudaSuccess) return HYENA_ERR_CUDA;
    ++launches;
    return HYENA_OK;
}

}  // namespace

void record_cuda_error(cudaError_t e, const char *where)
{
    snprintf(g_last_error, sizeof g_last_error, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

void record_message(const char *msg) { snprintf(g_last_error, sizeof g_last_error, "%s", msg); }

void add_launches(int n) { g_last_launches += n; }
void set_last_launches(int n) { g_last_launches = n; }

ModalLayout modal_layout(int B, int D, int N)
{
    ModalLayout L;
    L.NP = modal_padded_modes(N);
    L.LPC = modal_lanes_per_pair(L.NP);
    const int width = MCH / L.LPC;  // channels per chain
    L.nCB = (D + width - 1) / width;
    L.Dp = L.nCB * width;
    const size_t row = static_cast<size_t>(L.Dp) * sizeof(float);
    size_t off = 0;
    L.off_hdr = off;
    off += 256;
    L.off_coef = off;
    off = align256(off + row * modal_coef_rows(L.NP));
    const size_t chains = static_cast<size_t>(B) * L.nCB;
    L.off_flags = off;
    off = align256(off + chains * MRING * sizeof(unsigned long long));
    L.off_slots = off;
    off = align256(off + chains * MRING * (MGMAX + 1) * L.NP * width * sizeof(float));
    L.total = off;
    return L;
}

}  // namespace hyena

using namespace hyena;

namespace {

// dft: the tensor-core DFT-as-GEMM kernel instead of the FP32 SIMT kernels
// (separate or packed inputs only).
hyena_status_t short_conv_impl(const XSource &xs, const hyena_bf16_t *taps, const float *Dskip, hyena_bf16_t *y,
                               int64_t ld_y, const float *hist_in, float *hist_out, int B, int L, int D, int K,
                               void *stream, bool dft = false)
{
    hyena_status_t st = HYENA_OK;
    if (K < 1 || K > HYENA_MAX_TAPS) return K < 1 ? HYENA_ERR_INVALID_ARG : HYENA_ERR_UNSUPPORTED;
    if (taps == nullptr) return HYENA_ERR_INVALID_ARG;
    if ((Dskip && !aligned16(Dskip)) || (hist_in && !aligned16(hist_in)) ||
        (hist_out && !aligned16(hist_out)) || !aligned16(taps))
        return HYENA_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int launches = 0;
    if (L == 0) {
        if (K > 1) {
            st = copy_or_zero(hist_out, hist_in, static_cast<size_t>(B) * (K - 1) * D * sizeof(float), s,
                              launches);
            if (st != HYENA_OK) return st;
        }
        g_last_launches = launches;
        return HYENA_OK;
    }
    FirArgs a{};
    a.taps = taps;
    a.Dskip = Dskip;
    a.y = y;
    a.ld_y = ld_y;
    a.hist_in = hist_in;
    a.B = B;
    a.L = L;
    a.D = D;
    a.K = K;
    a.HR = fir_halo_rows(K);
    a.x1 = xs.x[0];
    a.x2 = xs.x[1];
    a.ld_x = xs.ld;
    a.group = xs.group;
    a.hist_out = hist_out;
    if (dft) {
        if (xs.triples) return HYENA_ERR_UNSUPPORTED;
        CUtensorMap m1, m2, m3;
        if (!encode_x_map(&m1, xs, 0, B, L, D, FT) || !encode_x_map(&m2, xs, 1, B, L, D, FT) ||
            !encode_x_map(&m3, xs, 2, B, L, D, FT))
            return HYENA_ERR_CUDA;
        const int n = launch_fir_dft(m1, m2, m3, a, s);
        if (n < 0) return HYENA_ERR_CUDA;
        g_last_launches = n;
        return HYENA_OK;
    }
    CUtensorMap m1, m2, m3, h1, h2;
    const CUtensorMapL2promotion promo =
        fir_persistent(K) ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B : CU_TENSOR_MAP_L2_PROMOTION_L2_256B;
    if (!encode_x_map(&m1, xs, 0, B, L, D, FT, 64, promo)) return HYENA_ERR_CUDA;
    if (xs.triples) {
        m2 = m3 = m1;
    } else if (!encode_x_map(&m2, xs, 1, B, L, D, FT, 64, promo) ||
               !encode_x_map(&m3, xs, 2, B, L, D, FT, 64, promo)) {
        return HYENA_ERR_CUDA;
    }
    if (a.HR > 0) {
        if (!encode_x_map(&h1, xs, 0, B, L, D, a.HR)) return HYENA_ERR_CUDA;
        if (xs.triples)
            h2 = h1;
        else if (!encode_x_map(&h2, xs, 1, B, L, D, a.HR))
            return HYENA_ERR_CUDA;
    } else {
        h1 = m1;
        h2 = m2;
    }
    const int n = launch_fir(m1, m2, m3, h1, h2, a, xs.triples, s);
    if (n < 0) return HYENA_ERR_CUDA;
    g_last_launches = n;
    return HYENA_OK;
}

// cx: complex modes; the N of the caller counts modes, the kernels count
// slots (two per complex mode).
// With `synth` false the coefficient table is the one hyena_modal_prepare left
// in the workspace and the filter parameters are not used.
hyena_status_t modal_long_conv_impl(const XSource &xs, const float *log_poles, const float *residues,
                                   const float *Dskip, hyena_bf16_t *y, int64_t ld_y, const float *state_in,
                                   float *state_out, int B, int L, int D, int N, void *workspace,
                                   size_t workspace_bytes, void *stream, bool cx = false, bool synth = true)
{
    hyena_status_t st = HYENA_OK;
    if (N < 1) return HYENA_ERR_INVALID_ARG;
    if (N > (cx ? HYENA_MAX_COMPLEX_MODES : HYENA_MAX_MODES)) return HYENA_ERR_UNSUPPORTED;
    if (cx) N *= 2;
    if (synth && (!log_poles || !residues)) return HYENA_ERR_INVALID_ARG;
    if (!aligned16(log_poles) || !aligned16(residues) || (Dskip && !aligned16(Dskip)) ||
        (state_in && !aligned16(state_in)) || (state_out && !aligned16(state_out)))
        return HYENA_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int launches = 0;
    if (L == 0) {
        st = copy_or_zero(state_out, state_in, static_cast<size_t>(B) * D * N * sizeof(float), s, launches);
        if (st != HYENA_OK) return st;
        g_last_launches = launches;
        return HYENA_OK;
    }
    const ModalLayout lay = modal_layout(B, D, N);
    if (workspace == nullptr || workspace_bytes < lay.total) return HYENA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return HYENA_ERR_ALIGNMENT;
    const long long nseg = (static_cast<long long>(L) + MT - 1) / MT;
    if (nseg * B * lay.nCB >= (1ll << 31)) return HYENA_ERR_UNSUPPORTED;

    unsigned char *ws = static_cast<unsigned char *>(workspace);
    ModalArgs a{};
    a.x1 = xs.x[0];
    a.x2 = xs.x[1];
    a.x3 = xs.x[2];
    a.ld_x = xs.ld;
    a.group = xs.group;
    a.y = y;
    a.ld_y = ld_y;
    a.state_in = state_in;
    a.state_out = state_out;
    a.B = B;
    a.L = L;
    a.D = D;
    a.N = N;
    a.nCB = lay.nCB;
    a.Dp = lay.Dp;
    a.units = static_cast<int>(nseg);
    a.coef = reinterpret_cast<const float *>(ws + lay.off_coef);
    a.flags = reinterpret_cast<unsigned long long *>(ws + lay.off_flags);
    a.slots = reinterpret_cast<float *>(ws + lay.off_slots);
    a.hdr = reinterpret_cast<unsigned int *>(ws + lay.off_hdr);

    ModalSynthArgs sy{};
    sy.log_poles = log_poles;
    sy.residues = residues;
    sy.Dskip = Dskip;
    sy.D = D;
    sy.N = N;
    sy.Dp = lay.Dp;
    sy.coef = reinterpret_cast<float *>(ws + lay.off_coef);

    const int ns = synth ? launch_modal_synth(sy, lay.NP, cx, s) : 0;
    if (ns < 0) return HYENA_ERR_CUDA;
    int n = -1;
    if (lay.LPC == 1) {
        CUtensorMap m1, m2, m3;
        if (!encode_x_map(&m1, xs, 0, B, L, D, MCK)) return HYENA_ERR_CUDA;
        if (xs.triples)
            m2 = m3 = m1;
        else if (!encode_x_map(&m2, xs, 1, B, L, D, MCK) || !encode_x_map(&m3, xs, 2, B, L, D, MCK))
            return HYENA_ERR_CUDA;
        n = modal_short_path(B, L, D, lay.NP, xs.triples)
                ? launch_modal_short(m1, m2, m3, a, lay.NP, xs.triples, cx, s)
                : launch_modal_narrow(m1, m2, m3, a, lay.NP, xs.triples, cx, s);
    } else {
        ModalMaps maps;
        const int width = MCH / lay.LPC;  // channels per chain
        if (!encode_x_map(&maps.a1, xs, 0, B, L, D, MA_ROWS, width) ||
            !encode_x_map(&maps.c1, xs, 0, B, L, D, MC_ROWS, width))
            return HYENA_ERR_CUDA;
        if (xs.triples) {
            maps.a2 = maps.a1;
            maps.c2 = maps.c3 = maps.c1;
        } else if (!encode_x_map(&maps.a2, xs, 1, B, L, D, MA_ROWS, width) ||
                   !encode_x_map(&maps.c2, xs, 1, B, L, D, MC_ROWS, width) ||
                   !encode_x_map(&maps.c3, xs, 2, B, L, D, MC_ROWS, width)) {
            return HYENA_ERR_CUDA;
        }
        if (!encode_coef_map(&maps.coef, ws + lay.off_coef, lay.Dp, lay.NP, width)) return HYENA_ERR_CUDA;
        n = launch_modal_wide(maps, a, lay.NP, xs.triples, cx, s);
    }
    if (n >= 0) n += ns;
    if (n < 0) return HYENA_ERR_CUDA;
    g_last_launches = n;
    return HYENA_OK;
}

hyena_status_t modal_decode_impl(const XSource &xs, const float *log_poles, const float *residues,
                                 const float *Dskip, hyena_bf16_t *y, int64_t ld_y, float *state, int B, int D, int N,
                                 void *stream, bool cx = false)
{
    const int nmax = cx ? HYENA_MAX_COMPLEX_MODES : HYENA_MAX_MODES;
    if (N < 1 || N > nmax) return N < 1 ? HYENA_ERR_INVALID_ARG : HYENA_ERR_UNSUPPORTED;
    if (cx) N *= 2;
    if (!log_poles || !residues || !state) return HYENA_ERR_INVALID_ARG;
    if (!aligned16(log_poles) || !aligned16(residues) || !aligned16(state) || (Dskip && !aligned16(Dskip)))
        return HYENA_ERR_ALIGNMENT;
    DecodeArgs a{};
    a.x1 = xs.x[0];
    a.x2 = xs.x[1];
    a.x3 = xs.x[2];
    a.ld_x = xs.ld;
    a.group = xs.group;
    a.log_poles = log_poles;
    a.residues = residues;
    a.Dskip = Dskip;
    a.y = y;
    a.ld_y = ld_y;
    a.state = state;
    a.B = B;
    a.D = D;
    a.N = N;
    const int n = launch_modal_decode(a, cx, static_cast<cudaStream_t>(stream));
    if (n < 0) return HYENA_ERR_CUDA;
    g_last_launches = n;
    return HYENA_OK;
}

hyena_status_t short_decode_impl(const XSource &xs, const hyena_bf16_t *taps, const float *Dskip, hyena_bf16_t *y,
                                 int64_t ld_y, float *hist, int B, int D, int K, void *stream)
{
    if (K < 1 || K > HYENA_MAX_TAPS) return K < 1 ? HYENA_ERR_INVALID_ARG : HYENA_ERR_UNSUPPORTED;
    if (taps == nullptr || (K > 1 && hist == nullptr)) return HYENA_ERR_INVALID_ARG;
    if (!aligned16(taps) || (Dskip && !aligned16(Dskip)) || (K > 1 && !aligned16(hist))) return HYENA_ERR_ALIGNMENT;
    DecodeArgs a{};
    a.x1 = xs.x[0];
    a.x2 = xs.x[1];
    a.x3 = xs.x[2];
    a.ld_x = xs.ld;
    a.group = xs.group;
    a.taps = taps;
    a.Dskip = Dskip;
    a.y = y;
    a.ld_y = ld_y;
    a.hist = K > 1 ? hist : nullptr;
    a.B = B;
    a.D = D;
    a.K = K;
    const int n = launch_fir_decode(a, static_cast<cudaStream_t>(stream));
    if (n < 0) return HYENA_ERR_CUDA;
    g_last_launches = n;
    return HYENA_OK;
}

}  // namespace

extern "C" {

const char *hyena_status_string(hyena_status_t s)
{
    switch (s) {
        case HYENA_OK: return "HYENA_OK";
        case HYENA_ERR_INVALID_ARG: return "HYENA_ERR_INVALID_ARG";
        case HYENA_ERR_ALIGNMENT: return "HYENA_ERR_ALIGNMENT";
        case HYENA_ERR_UNSUPPORTED: return "HYENA_ERR_UNSUPPORTED";
        case HYENA_ERR_CUDA: return "HYENA_ERR_CUDA";
        case HYENA_ERR_TIMEOUT: return "HYENA_ERR_TIMEOUT";
        case HYENA_ERR_WORKSPACE: return "HYENA_ERR_WORKSPACE";
        default: return "HYENA_ERR_UNKNOWN";
    }
}

int hyena_abi_version(void) { return 100; }

int hyena_last_launch_count(void) { return g_last_launches; }

const char *hyena_last_error_message(void) { return g_last_error; }

size_t hyena_modal_long_conv_workspace_size(int B, int D, int N)
{
    if (B < 1 || D < 1 || N < 1 || N > HYENA_MAX_MODES) return 0;
    return modal_layout(B, D, N).total;
}

hyena_status_t hyena_modal_workspace_init(void *workspace, size_t workspace_bytes, void *stream)
{
    if (workspace == nullptr || workspace_bytes == 0) return HYENA_ERR_INVALID_ARG;
    if (cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return HYENA_ERR_CUDA;
    g_last_launches = 1;
    return HYENA_OK;
}

hyena_status_t hyena_short_conv(const hyena_bf16_t *x1, const hyena_bf16_t *x2, const hyena_bf16_t *x3,
                                int64_t ld_x, const hyena_bf16_t *taps, const float *Dskip,
                                hyena_bf16_t *y, int64_t ld_y, const float *hist_in, float *hist_out,
                                int B, int L, int D, int K, void *stream)
{
    const hyena_status_t st = check_x(x1, x2, x3, ld_x, y, ld_y, B, L, D);
    if (st != HYENA_OK) return st;
    return short_conv_impl(separate_source(x1, x2, x3, ld_x, D), taps, Dskip, y, ld_y, hist_in, hist_out, B, L, D,
                           K, stream);
}

hyena_status_t hyena_short_conv_dft(const hyena_bf16_t *x1, const hyena_bf16_t *x2, const hyena_bf16_t *x3,
                                    int64_t ld_x, const hyena_bf16_t *taps, const float *Dskip, hyena_bf16_t *y,
                                    int64_t ld_y, const float *hist_in, float *hist_out, int B, int L, int D, int K,
                                    void *stream)
{
    const hyena_status_t st = check_x(x1, x2, x3, ld_x, y, ld_y, B, L, D);
    if (st != HYENA_OK) return st;
    return short_conv_impl(separate_source(x1, x2, x3, ld_x, D), taps, Dskip, y, ld_y, hist_in, hist_out, B, L, D,
                           K, stream, true);
}

hyena_status_t hyena_short_conv_packed(const hyena_bf16_t *xp, int64_t ld_x, int group, const hyena_bf16_t *taps,
                                       const float *Dskip, hyena_bf16_t *y, int64_t ld_y, const float *hist_in,
                                       float *hist_out, int B, int L, int D, int K, void *stream)
{
    const hyena_status_t st = check_packed(xp, ld_x, group, y, ld_y, B, L, D);
    if (st != HYENA_OK) return st;
    return short_conv_impl(packed_source(xp, ld_x, group), taps, Dskip, y, ld_y, hist_in, hist_out, B, L, D, K,
                           stream);
}

hyena_status_t hyena_modal_long_conv(const hyena_bf16_t *x1, const hyena_bf16_t *x2, const hyena_bf16_t *x3,
                                     int64_t ld_x, const float *log_poles, const float *residues,
                                     const float *Dskip, hyena_bf16_t *y, int64_t ld_y,
                                     const float *state_in, float *state_out, int B, int L, int D, int N,
                                     void *workspace, size_t workspace_bytes, void *stream)
{
    const hyena_status_t st = check_x(x1, x2, x3, ld_x, y, ld_y, B, L, D);
    if (st != HYENA_OK) return st;
    return modal_long_conv_impl(separate_source(x1, x2, x3, ld_x, D), log_poles, residues, Dskip, y, ld_y, state_in,
                                state_out, B, L, D, N, workspace, workspace_bytes, stream);
}

hyena_status_t hyena_modal_prepare(const float *log_poles, const float *residues, const float *Dskip, int B, int D,
                                   int N, void *workspace, size_t workspace_bytes, void *stream)
{
    if (B < 1 || D < 1 || N < 1) return HYENA_ERR_INVALID_ARG;
    if (N > HYENA_MAX_MODES) return HYENA_ERR_UNSUPPORTED;
    if (!log_poles || !residues) return HYENA_ERR_INVALID_ARG;
    if (D % 8) return HYENA_ERR_ALIGNMENT;
    if (!aligned16(log_poles) || !aligned16(residues) || (Dskip && !aligned16(Dskip))) return HYENA_ERR_ALIGNMENT;
    const ModalLayout lay = modal_layout(B, D, N);
    if (workspace == nullptr || workspace_bytes < lay.total) return HYENA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return HYENA_ERR_ALIGNMENT;
    ModalSynthArgs sy{};
    sy.log_poles = log_poles;
    sy.residues = residues;
    sy.Dskip = Dskip;
    sy.D = D;
    sy.N = N;
    sy.Dp = lay.Dp;
    sy.coef = reinterpret_cast<float *>(static_cast<unsigned char *>(workspace) + lay.off_coef);
    const int n = launch_modal_synth(sy, lay.NP, false, static_cast<cudaStream_t>(stream));
    if (n < 0) return HYENA_ERR_CUDA;
    g_last_launches = n;
    return HYENA_OK;
}

hyena_status_t hyena_modal_long_conv_prepared(const hyena_bf16_t *x1, const hyena_bf16_t *x2, const hyena_bf16_t *x3,
                                              int64_t ld_x, hyena_bf16_t *y, int64_t ld_y, const float *state_in,
                                              float *state_out, int B, int L, int D, int N, void *workspace,
                                              size_t workspace_bytes, void *stream)
{
    const hyena_status_t st = check_x(x1, x2, x3, ld_x, y, ld_y, B, L, D);
    if (st != HYENA_OK) return st;
    return modal_long_conv_impl(separate_source(x1, x2, x3, ld_x, D), nullptr, nullptr, nullptr, y, ld_y, state_in,
                                state_out, B, L, D, N, workspace, workspace_bytes, stream, false, false);
}

hyena_status_t hyena_modal_long_conv_packed(const hyena_bf16_t *xp, int64_t ld_x, int group, const float *log_poles,
                                            const float *residues, const float *Dskip, hyena_bf16_t *y,
                                            int64_t ld_y, const float *state_in, float *state_out, int B, int L,
                                            int D, int N, void *workspace, size_t workspace_bytes, void *stream)
{
    const hyena_status_t st = check_packed(xp, ld_x, group, y, ld_y, B, L, D);
    if (st != HYENA_OK) return st;
    return modal_long_conv_impl(packed_source(xp, ld_x, group), log_poles, residues, Dskip, y, ld_y, state_in,
                                state_out, B, L, D, N, workspace, workspace_bytes, stream);
}

hyena_status_t hyena_modal_decode(const hyena_bf16_t *x1, const hyena_bf16_t *x2, const hyena_bf16_t *x3,
                                  int64_t ld_x, const float *log_poles, const float *residues, const float *Dskip,
                                  hyena_bf16_t *y, int64_t ld_y, float *state, int B, int D, int N, void *stream)
{
    const hyena_status_t st = check_x(x1, x2, x3, ld_x, y, ld_y, B, 1, D);
    if (st != HYENA_OK) return st;
    return modal_decode_impl(separate_source(x1, x2, x3, ld_x, D), log_poles, residues, Dskip, y, ld_y, state, B, D,
                             N, stream);
}

hyena_status_t hyena_modal_decode_packed(const hyena_bf16_t *xp, int64_t ld_x, int group, const float *log_poles,
                                         const float *residues, const float *Dskip, hyena_bf16_t *y, int64_t ld_y,
                                         float *state, int B, int D, int N, void *stream)
{
    const hyena_status_t st = check_packed(xp, ld_x, group, y, ld_y, B, 1, D);
    if (st != HYENA_OK) return st;
    return modal_decode_impl(packed_source(xp, ld_x, group), log_poles, residues, Dskip, y, ld_y, state, B, D, N,
                             stream);
}

hyena_status_t hyena_modal_long_conv_complex(const hyena_bf16_t *x1, const hyena_bf16_t *x2,
                                             const hyena_bf16_t *x3, int64_t ld_x, const float *poles,
                                             const float *residues, const float *Dskip, hyena_bf16_t *y,
                                             int64_t ld_y, const float *state_in, float *state_out, int B, int L,
                                             int D, int N, void *workspace, size_t workspace_bytes, void *stream)
{
    const hyena_status_t st = check_x(x1, x2, x3, ld_x, y, ld_y, B, L, D);
    if (st != HYENA_OK) return st;
    return modal_long_conv_impl(separate_source(x1, x2, x3, ld_x, D), poles, residues, Dskip, y, ld_y, state_in,
                                state_out, B, L, D, N, workspace, workspace_bytes, stream, true);
}

hyena_status_t hyena_modal_decode_complex(const hyena_bf16_t *x1, const hyena_bf16_t *x2, const hyena_bf16_t *x3,
                                          int64_t ld_x, const float *poles, const float *residues,
                                          const float *Dskip, hyena_bf16_t *y, int64_t ld_y, float *state, int B,
                                          int D, int N, void *stream)
{
    const hyena_status_t st = check_x(x1, x2, x3, ld_x, y, ld_y, B, 1, D);
    if (st != HYENA_OK) return st;
    return modal_decode_impl(separate_source(x1, x2, x3, ld_x, D), poles, residues, Dskip, y, ld_y, state, B, D, N,
                             stream, true);
}

hyena_status_t hyena_modal_long_conv_complex_packed(const hyena_bf16_t *xp, int64_t ld_x, int group,
                                                    const float *poles, const float *residues, const float *Dskip,
                                                    hyena_bf16_t *y, int64_t ld_y, const float *state_in,
                                                    float *state_out, int B, int L, int D, int N, void *workspace,
                                                    size_t workspace_bytes, void *stream)
{
    const hyena_status_t st = check_packed(xp, ld_x, group, y, ld_y, B, L, D);
    if (st != HYENA_OK) return st;
    return modal_long_conv_impl(packed_source(xp, ld_x, group), poles, residues, Dskip, y, ld_y, state_in,
                                state_out, B, L, D, N, workspace, workspace_bytes, stream, true);
}

hyena_status_t hyena_modal_decode_complex_packed(const hyena_bf16_t *xp, int64_t ld_x, int group, const float *poles,
                                                 const float *residues, const float *Dskip, hyena_bf16_t *y,
                                                 int64_t ld_y, float *state, int B, int D, int N, void *stream)
{
    const hyena_status_t st = check_packed(xp, ld_x, group, y, ld_y, B, 1, D);
    if (st != HYENA_OK) return st;
    return modal_decode_impl(packed_source(xp, ld_x, group), poles, residues, Dskip, y, ld_y, state, B, D, N,
                             stream, true);
}

hyena_status_t hyena_short_decode(const hyena_bf16_t *x1, const hyena_bf16_t *x2, const hyena_bf16_t *x3,
                                  int64_t ld_x, const hyena_bf16_t *taps, const float *Dskip, hyena_bf16_t *y,
                                  int64_t ld_y, float *hist, int B, int D, int K, void *stream)
{
    const hyena_status_t st = check_x(x1, x2, x3, ld_x, y, ld_y, B, 1, D);
    if (st != HYENA_OK) return st;
    return short_decode_impl(separate_source(x1, x2, x3, ld_x, D), taps, Dskip, y, ld_y, hist, B, D, K, stream);
}

hyena_status_t hyena_short_decode_packed(const hyena_bf16_t *xp, int64_t ld_x, int group, const hyena_bf16_t *taps,
                                         const float *Dskip, hyena_bf16_t *y, int64_t ld_y, float *hist, int B,
                                         int D, int K, void *stream)
{
    const hyena_status_t st = check_packed(xp, ld_x, group, y, ld_y, B, 1, D);
    if (st != HYENA_OK) return st;
    return short_decode_impl(packed_source(xp, ld_x, group), taps, Dskip, y, ld_y, hist, B, D, K, stream);
}

hyena_status_t hyena_modal_state_init(float *state, int B, int D, int N, void *stream)
{
    if (state == nullptr || B < 1 || D < 1 || N < 1) return HYENA_ERR_INVALID_ARG;
    if (cudaMemsetAsync(state, 0, static_cast<size_t>(B) * D * N * sizeof(float),
                        static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return HYENA_ERR_CUDA;
    g_last_launches = 1;
    return HYENA_OK;
}

hyena_status_t hyena_workspace_check(void *workspace, void *stream)
{
    if (workspace == nullptr) return HYENA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) {
        record_cuda_error(e, "workspace check: stream synchronize");
        return HYENA_ERR_CUDA;
    }
    unsigned int err = 0;
    unsigned int *hdr = static_cast<unsigned int *>(workspace);
    e = cudaMemcpy(&err, hdr + 2, sizeof err, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) {
        record_cuda_error(e, "workspace check: read error word");
        return HYENA_ERR_CUDA;
    }
    if (err != 0u) {
        if (cudaMemset(hdr + 2, 0, sizeof err) != cudaSuccess) return HYENA_ERR_CUDA;
        return HYENA_ERR_TIMEOUT;
    }
    return HYENA_OK;
}

}  // extern "C"
