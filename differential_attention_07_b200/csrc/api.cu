// api.cu -- the C ABI of libdiffattn: argument validation, TMA tensor-map
// encoding, workspace layout and kernel launches.  Nothing here allocates
// device memory or synchronises a stream.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <atomic>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "diffattn.h"
#include "kernels.h"

namespace {

thread_local int32_t g_last_launches = 0;
thread_local char g_last_error[256] = "";

// Map a CUDA error to the ABI status, keeping its text for diffattn_last_error.
diffattn_status cuda_status(cudaError_t e)
{
    if (e == cudaSuccess) return DIFFATTN_OK;
    if (g_last_error[0] == 0)
        std::snprintf(g_last_error, sizeof g_last_error, "%s: %s", cudaGetErrorName(e),
                      cudaGetErrorString(e));
    return DIFFATTN_ERR_CUDA;
}
thread_local da::ProfileEvents g_events;

constexpr uint32_t kDefaultTimeoutMs = 2000;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool stride8(int64_t s) { return s % 8 == 0; }

// cuTensorMapEncodeTiled, fetched once from the driver through the runtime
// (so the library does not link libcuda directly).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 4-D map over a [B, N, heads, inner] tensor (element strides sb, sn, sh;
// inner contiguous), box {64, rows, 1, 1}, 128-byte swizzle, zero fill.
bool make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, int64_t inner,
              int64_t N, int64_t heads, int64_t B, int64_t sb, int64_t sn, int64_t sh,
              uint32_t rows)
{
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)inner, (cuuint64_t)N, (cuuint64_t)heads,
                                (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)(sn * 2), (cuuint64_t)(sh * 2),
                                   (cuuint64_t)(sb * 2)};
    const cuuint32_t box[4] = {64, rows, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, dt, 4, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 4-D map over the backward pass's row statistics, fp32 [B, H, S, n_pad]
// (S = da::kBwdStats): box {64 rows, S arrays}, no swizzle.
bool make_stats_map(CUtensorMap *m, const float *base, int64_t n_pad, int64_t H, int64_t B)
{
    auto fn = encode_fn();
    if (!fn) return false;
    constexpr int64_t S = da::kBwdStats;
    const cuuint64_t dims[4] = {(cuuint64_t)n_pad, (cuuint64_t)S, (cuuint64_t)H, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)(n_pad * 4), (cuuint64_t)(S * n_pad * 4),
                                   (cuuint64_t)(H * S * n_pad * 4)};
    const cuuint32_t box[4] = {64, (cuuint32_t)S, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
bool grouped_pairs(const diffattn_fwd_args *a);
// Tiles of the paired grouped heads: (b, noise head, 128-row query tile).
int64_t noise_tiles(const diffattn_fwd_args *a)
{
    const int64_t HN = a->H_N ? a->H_N : a->H;
    return a->B * HN * ((a->N + 127) / 128);
}
// Normalised noise outputs of paired grouped heads, fp32, per tile a
// tile-transposed 128 x 128 block.
size_t noise_out_bytes(const diffattn_fwd_args *a)
{
    return grouped_pairs(a) && !a->save ? align256((size_t)noise_tiles(a) * 128 * 128 * sizeof(float)) : 0;
}
// ... followed by one int per tile: how many epilogue warps have exported.
size_t noise_bytes(const diffattn_fwd_args *a)
{
    if (!grouped_pairs(a) || a->save) return 0;
    return noise_out_bytes(a) + align256((size_t)noise_tiles(a) * sizeof(int));
}

// Grouped heads that run as (signal, noise) and (signal, signal) pairs: each
// group of g = H / H_N signal heads shares one V head, with g odd and >= 3.
bool grouped_pairs(const diffattn_fwd_args *a)
{
    const int64_t HN = a->H_N ? a->H_N : a->H, HV = a->H_V ? a->H_V : a->H;
    if (HN <= 0 || a->H % HN != 0 || HV != HN) return false;
    const int64_t g = a->H / HN;
    return g >= 3 && g % 2 == 1;
}

// Prefill workspace: [fp16 V, except under a window][256 B work counters][paired grouped heads
// only: noise outputs, one fp32 128 x 128 block per (b, noise head, query
// tile), then one ready count per such tile][rotated Q1, K1, Q2, K2 when
// rope_theta > 0: contiguous [B, N, heads, 64] fp16 each].
size_t v16_bytes(const diffattn_fwd_args *a);
size_t noise_bytes(const diffattn_fwd_args *a);
size_t rope_copy_bytes(const diffattn_fwd_args *a, int t)
{
    const int64_t HN = a->H_N ? a->H_N : a->H;
    return align256((size_t)a->B * a->N * (t < 2 ? a->H : HN) * 64 * 2);
}
size_t rope_offset(const diffattn_fwd_args *a) { return v16_bytes(a) + 256 + noise_bytes(a); }
size_t rope_bytes(const diffattn_fwd_args *a)
{
    if (!(a->rope_theta > 0.0f)) return 0;
    size_t n = 0;
    for (int t = 0; t < 4; ++t) n += rope_copy_bytes(a, t);
    return n;
}

// Bytes of the fp16 V copy at the start of the prefill workspace (none
// under a sliding window, whose kernel reads the caller's V and converts
// each step itself).
size_t v16_bytes(const diffattn_fwd_args *a)
{
    if (a->window > 0) return 0;
    const int64_t HV = a->H_V ? a->H_V : a->H;
    return align256((size_t)a->B * a->N * HV * 128 * 2);
}

// The staging kernel's rotary part: rotate Q1, K1, Q2, K2 (heads H, H, H_N,
// H_N) into contiguous fp16 copies starting at `dst`, and point qk[t] /
// qk_stride[t] (t = Q1, K1, Q2, K2) at them; without rotation qk and
// qk_stride keep the caller's tensors.
void set_rope(da::RopeStage *rope, float theta, int64_t B, int64_t N, int64_t H, int64_t HN,
              char *dst, const void *(&qk)[4], int64_t (&qk_stride)[4][3])
{
    *rope = da::RopeStage{};
    if (!(theta > 0.0f)) return;
    for (int t = 0; t < 4; ++t) {
        const int64_t heads = t < 2 ? H : HN;
        rope->src[t] = qk[t];
        rope->sb[t] = qk_stride[t][0];
        rope->sn[t] = qk_stride[t][1];
        rope->sh[t] = qk_stride[t][2];
        rope->dst[t] = dst;
        rope->heads[t] = (int)heads;
        qk[t] = dst;
        qk_stride[t][0] = N * heads * 64;
        qk_stride[t][1] = heads * 64;
        qk_stride[t][2] = 64;
        dst += align256((size_t)B * N * heads * 64 * 2);
    }
    rope->enabled = 1;
    for (int c = 0; c < 32; ++c)  // turns per token of pair c: theta^(-2c/64) / (2 pi)
        rope->g[c] = std::pow((double)theta, -2.0 * c / 64.0) / 6.283185307179586;
}

diffattn_status validate_fwd(const diffattn_fwd_args *a, int grouped)
{
    if (!a) return DIFFATTN_ERR_INVALID_ARG;
    if (a->B < 0 || a->N < 0 || a->H <= 0) return DIFFATTN_ERR_INVALID_ARG;
    const int64_t HN = a->H_N ? a->H_N : a->H, HV = a->H_V ? a->H_V : a->H;
    if (HN <= 0 || HV <= 0 || a->H_N < 0 || a->H_V < 0) return DIFFATTN_ERR_INVALID_ARG;
    if (!grouped && (HN != a->H || HV != a->H)) return DIFFATTN_ERR_INVALID_ARG;
    if (a->H % HN != 0 || a->H % HV != 0) return DIFFATTN_ERR_INVALID_ARG;
    if (a->d != 64 || a->dv != 128) return DIFFATTN_ERR_UNSUPPORTED;
    if (a->flags & ~(DIFFATTN_FLAG_CAUSAL | DIFFATTN_FLAG_APPLY_NORM | DIFFATTN_FLAG_TEST_WITHHOLD_LOAD))
        return DIFFATTN_ERR_INVALID_ARG;
    if (!(a->scale > 0.0f) || !std::isfinite(a->scale)) return DIFFATTN_ERR_INVALID_ARG;
    if (!(a->eps >= 0.0f) || !std::isfinite(a->eps)) return DIFFATTN_ERR_INVALID_ARG;
    if (a->window < 0 || (a->window > 0 && !(a->flags & DIFFATTN_FLAG_CAUSAL)))
        return DIFFATTN_ERR_INVALID_ARG;
    if (!(a->rope_theta >= 0.0f) || !std::isfinite(a->rope_theta)) return DIFFATTN_ERR_INVALID_ARG;
    // Index arithmetic inside the kernels is 32-bit for counts.
    if (a->N > (1 << 24) || a->B > (1 << 16) || a->H > 4096) return DIFFATTN_ERR_UNSUPPORTED;
    if ((a->B * a->H * ((a->N + 127) / 128)) > INT32_MAX) return DIFFATTN_ERR_UNSUPPORTED;
    if (a->B == 0 || a->N == 0) return DIFFATTN_OK;  // nothing to compute
    const void *ptrs[6] = {a->q1, a->q2, a->k1, a->k2, a->v, a->out};
    for (const void *p : ptrs)
        if (!p) return DIFFATTN_ERR_INVALID_ARG;
    if (!a->lambda && !a->lambda_logits) return DIFFATTN_ERR_INVALID_ARG;
    for (const void *p : ptrs)
        if (!aligned16(p)) return DIFFATTN_ERR_ALIGNMENT;
    if (a->gain && !aligned16(a->gain)) return DIFFATTN_ERR_ALIGNMENT;
    if (a->lambda_logits) {
        if (reinterpret_cast<uintptr_t>(a->lambda_logits) % 4) return DIFFATTN_ERR_ALIGNMENT;
        for (int i = 0; i < 3; ++i)
            if (a->lambda_logits_stride[i] < 0) return DIFFATTN_ERR_INVALID_ARG;
    }
    if (a->gate && !aligned16(a->gate)) return DIFFATTN_ERR_ALIGNMENT;
    const int64_t *strides[7] = {a->q1_stride, a->q2_stride, a->k1_stride, a->k2_stride,
                                 a->v_stride, a->out_stride, a->gate_stride};
    for (int t = 0; t < (a->gate ? 7 : 6); ++t)
        for (int i = 0; i < 3; ++i) {
            if (strides[t][i] < 0) return DIFFATTN_ERR_INVALID_ARG;
            if (!stride8(strides[t][i])) return DIFFATTN_ERR_ALIGNMENT;
        }
    if (a->save && !aligned16(a->save)) return DIFFATTN_ERR_ALIGNMENT;
    return DIFFATTN_OK;
}

// ---------------------------------------------------------------- backward
// Workspace of the backward pass: [fp16 V copy [B, N, H_V, 128]][fp16 dD
// [B, N, H, 128]][row statistics fp32 [B, H, kBwdStats, n_pad]][256 B: the
// staging kernel's counters][rotated Q1, K1, Q2, K2, fp16, when rope_theta >
// 0][fp32 sums: dK2 and dQ2 [B, N, H_N, 64] when H_N < H, dV [B, N, H_V,
// 128] when H_V < H].
int64_t bwd_hn(const diffattn_bwd_args *a) { return a->H_N ? a->H_N : a->H; }
int64_t bwd_hv(const diffattn_bwd_args *a) { return a->H_V ? a->H_V : a->H; }
size_t bwd_v16_bytes(const diffattn_bwd_args *a) { return align256((size_t)a->B * a->N * bwd_hv(a) * 128 * 2); }
size_t bwd_dd_bytes(const diffattn_bwd_args *a) { return align256((size_t)a->B * a->N * a->H * 128 * 2); }
size_t bwd_stats_bytes(const diffattn_bwd_args *a)
{
    return align256((size_t)a->B * a->H * da::kBwdStats * ((a->N + 127) / 128) * 128 * sizeof(float));
}
size_t bwd_rope_bytes(const diffattn_bwd_args *a)
{
    if (!(a->rope_theta > 0.0f)) return 0;
    return 2 * align256((size_t)a->B * a->N * a->H * 64 * 2) + 2 * align256((size_t)a->B * a->N * bwd_hn(a) * 64 * 2);
}
size_t bwd_acc_qk_bytes(const diffattn_bwd_args *a)
{
    return bwd_hn(a) < a->H ? (size_t)a->B * a->N * bwd_hn(a) * 64 * sizeof(float) : 0;
}
size_t bwd_acc_v_bytes(const diffattn_bwd_args *a)
{
    return bwd_hv(a) < a->H ? (size_t)a->B * a->N * bwd_hv(a) * 128 * sizeof(float) : 0;
}
size_t bwd_acc_offset(const diffattn_bwd_args *a)
{
    return bwd_v16_bytes(a) + bwd_dd_bytes(a) + bwd_stats_bytes(a) + 256 + bwd_rope_bytes(a);
}

diffattn_status validate_bwd(const diffattn_bwd_args *a)
{
    if (!a) return DIFFATTN_ERR_INVALID_ARG;
    if (a->B < 0 || a->N < 0 || a->H <= 0) return DIFFATTN_ERR_INVALID_ARG;
    if (a->H_N < 0 || a->H_V < 0) return DIFFATTN_ERR_INVALID_ARG;
    const int64_t HN = bwd_hn(a), HV = bwd_hv(a);
    if (a->H % HN != 0 || a->H % HV != 0) return DIFFATTN_ERR_INVALID_ARG;
    if (a->d != 64 || a->dv != 128) return DIFFATTN_ERR_UNSUPPORTED;
    if (a->flags & ~(DIFFATTN_FLAG_CAUSAL | DIFFATTN_FLAG_APPLY_NORM)) return DIFFATTN_ERR_INVALID_ARG;
    if (!(a->scale > 0.0f) || !std::isfinite(a->scale)) return DIFFATTN_ERR_INVALID_ARG;
    if (!(a->eps >= 0.0f) || !std::isfinite(a->eps)) return DIFFATTN_ERR_INVALID_ARG;
    if (a->window < 0 || (a->window > 0 && !(a->flags & DIFFATTN_FLAG_CAUSAL))) return DIFFATTN_ERR_INVALID_ARG;
    if (!(a->rope_theta >= 0.0f) || !std::isfinite(a->rope_theta)) return DIFFATTN_ERR_INVALID_ARG;
    if (a->N > (1 << 24) || a->B > (1 << 16) || a->H > 4096) return DIFFATTN_ERR_UNSUPPORTED;
    if ((a->B * a->H * ((a->N + 127) / 128)) > INT32_MAX) return DIFFATTN_ERR_UNSUPPORTED;
    if (a->B == 0 || a->N == 0) return DIFFATTN_OK;
    const void *ptrs[12] = {a->q1, a->q2, a->k1, a->k2, a->v, a->dout,
                            a->grad_q1, a->grad_q2, a->grad_k1, a->grad_k2, a->grad_v, a->save};
    for (const void *p : ptrs)
        if (!p) return DIFFATTN_ERR_INVALID_ARG;
    if (!a->lambda && !a->lambda_logits) return DIFFATTN_ERR_INVALID_ARG;
    for (const void *p : ptrs)
        if (!aligned16(p)) return DIFFATTN_ERR_ALIGNMENT;
    if (a->gain && !aligned16(a->gain)) return DIFFATTN_ERR_ALIGNMENT;
    if ((a->grad_lambda && reinterpret_cast<uintptr_t>(a->grad_lambda) % 4) ||
        (a->grad_gain && reinterpret_cast<uintptr_t>(a->grad_gain) % 4) ||
        (a->lambda_logits && reinterpret_cast<uintptr_t>(a->lambda_logits) % 4) ||
        (a->grad_lambda_logits && reinterpret_cast<uintptr_t>(a->grad_lambda_logits) % 4))
        return DIFFATTN_ERR_ALIGNMENT;
    for (int i = 0; i < 3; ++i)
        if ((a->lambda_logits && a->lambda_logits_stride[i] < 0) ||
            (a->grad_lambda_logits && a->grad_lambda_logits_stride[i] < 0))
            return DIFFATTN_ERR_INVALID_ARG;
    if ((a->gate && !aligned16(a->gate)) || (a->grad_gate && !aligned16(a->grad_gate))) return DIFFATTN_ERR_ALIGNMENT;
    if (a->grad_gate && !a->gate) return DIFFATTN_ERR_INVALID_ARG;
    const int64_t *strides[13] = {a->q1_stride, a->q2_stride, a->k1_stride, a->k2_stride,
                                  a->v_stride, a->dout_stride, a->grad_q1_stride,
                                  a->grad_q2_stride, a->grad_k1_stride, a->grad_k2_stride,
                                  a->grad_v_stride, a->gate_stride, a->grad_gate_stride};
    const bool used[13] = {true, true, true, true, true, true, true, true, true, true, true,
                           a->gate != nullptr, a->grad_gate != nullptr};
    for (int t = 0; t < 13; ++t)
        for (int i = 0; i < 3 && used[t]; ++i) {
            if (strides[t][i] < 0) return DIFFATTN_ERR_INVALID_ARG;
            if (!stride8(strides[t][i])) return DIFFATTN_ERR_ALIGNMENT;
        }
    return DIFFATTN_OK;
}

diffattn_status validate_decode(const diffattn_decode_args *a)
{
    if (!a) return DIFFATTN_ERR_INVALID_ARG;
    if (a->B < 0 || a->H <= 0 || a->L <= 0) return DIFFATTN_ERR_INVALID_ARG;
    if (a->d != 64 || a->dv != 128) return DIFFATTN_ERR_UNSUPPORTED;
    if (a->flags & ~(DIFFATTN_FLAG_CAUSAL | DIFFATTN_FLAG_APPLY_NORM)) return DIFFATTN_ERR_INVALID_ARG;
    if (a->num_splits < 0 || a->window < 0) return DIFFATTN_ERR_INVALID_ARG;
    if (!(a->scale > 0.0f) || !std::isfinite(a->scale)) return DIFFATTN_ERR_INVALID_ARG;
    if (!(a->eps >= 0.0f) || !std::isfinite(a->eps)) return DIFFATTN_ERR_INVALID_ARG;
    if (a->L > (1 << 26) || a->B > (1 << 16) || a->H > 4096) return DIFFATTN_ERR_UNSUPPORTED;
    if (a->B == 0) return DIFFATTN_OK;
    const void *ptrs[6] = {a->q1, a->q2, a->k1, a->k2, a->v, a->out};
    for (const void *p : ptrs)
        if (!p) return DIFFATTN_ERR_INVALID_ARG;
    if (!a->lambda && !a->lambda_logits) return DIFFATTN_ERR_INVALID_ARG;
    for (const void *p : ptrs)
        if (!aligned16(p)) return DIFFATTN_ERR_ALIGNMENT;
    if (a->lambda_logits) {
        if (reinterpret_cast<uintptr_t>(a->lambda_logits) % 4) return DIFFATTN_ERR_ALIGNMENT;
        if (a->lambda_logits_stride[0] < 0 || a->lambda_logits_stride[1] < 0)
            return DIFFATTN_ERR_INVALID_ARG;
    }
    if (a->gate) {
        if (a->gate_stride[0] < 0 || a->gate_stride[1] < 0) return DIFFATTN_ERR_INVALID_ARG;
        if (!aligned16(a->gate)) return DIFFATTN_ERR_ALIGNMENT;
    }
    const int64_t s2[4] = {a->q1_stride[0], a->q1_stride[1], a->q2_stride[0], a->q2_stride[1]};
    for (int64_t s : s2) {
        if (s < 0) return DIFFATTN_ERR_INVALID_ARG;
        if (!stride8(s)) return DIFFATTN_ERR_ALIGNMENT;
    }
    const int64_t *s3[3] = {a->k1_stride, a->k2_stride, a->v_stride};
    for (const int64_t *s : s3)
        for (int i = 0; i < 3; ++i) {
            if (s[i] < 0) return DIFFATTN_ERR_INVALID_ARG;
            if (!stride8(s[i])) return DIFFATTN_ERR_ALIGNMENT;
        }
    if (a->out_stride[0] < 0 || a->out_stride[1] < 0) return DIFFATTN_ERR_INVALID_ARG;
    return DIFFATTN_OK;
}

int decode_splits(int64_t B, int64_t H, int64_t L, int32_t requested)
{
    const int64_t min_splits = (L + da::kDecodeMaxChunk - 1) / da::kDecodeMaxChunk;
    int64_t s = requested > 0 ? requested : 0;
    if (s == 0) {
        // Enough CTAs for about four per SM of the current device, chunks of
        // >= 256 keys.
        const int64_t bh = B * H > 0 ? B * H : 1;
        s = (4 * (int64_t)da::device_sm_count() + bh - 1) / bh;
        const int64_t max_by_len = (L + 255) / 256;
        if (s > max_by_len) s = max_by_len;
    }
    if (s < min_splits) s = min_splits;
    if (s > L) s = L;
    if (s < 1) s = 1;
    // Chunk rounded up to 64 keys; drop splits that would be empty.
    const int64_t chunk = ((L + s - 1) / s + 63) / 64 * 64;
    s = (L + chunk - 1) / chunk;
    return (int)s;
}

int decode_chunk(int64_t L, int splits) { return (int)(((L + splits - 1) / splits + 63) / 64 * 64); }

diffattn_status run_fwd(const diffattn_fwd_args *a, void *ws, size_t ws_bytes, void *stream,
                        int grouped)
{
    g_last_launches = 0;
    g_last_error[0] = 0;
    diffattn_status st = validate_fwd(a, grouped);
    if (st != DIFFATTN_OK) return st;
    if (a->B == 0 || a->N == 0) return DIFFATTN_OK;
    const size_t need = diffattn_fwd_workspace_size(a);
    if (!ws || ws_bytes < need) return DIFFATTN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return DIFFATTN_ERR_ALIGNMENT;
    const int64_t HN = a->H_N ? a->H_N : a->H, HV = a->H_V ? a->H_V : a->H;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    // Q/K sources of the tensor maps: the caller's tensors, or with a rotary
    // embedding their rotated copies in the workspace (written by the
    // staging kernel that runs first on the stream).
    const void *qk[4] = {a->q1, a->k1, a->q2, a->k2};
    const int64_t *qks[4] = {a->q1_stride, a->k1_stride, a->q2_stride, a->k2_stride};
    int64_t qk_stride[4][3];
    for (int t = 0; t < 4; ++t)
        for (int i = 0; i < 3; ++i) qk_stride[t][i] = qks[t][i];
    da::RopeStage rope;
    set_rope(&rope, a->rope_theta, a->B, a->N, a->H, HN, static_cast<char *>(ws) + rope_offset(a), qk,
             qk_stride);

    const CUtensorMapDataType qkt =
        a->rope_theta > 0.0f ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUtensorMap mq1, mq2, mk1, mk2, mv, mo;
    const bool ok =
        make_map(&mq1, qkt, qk[0], 64, a->N, a->H, a->B,
                 qk_stride[0][0], qk_stride[0][1], qk_stride[0][2], da::kPrefillQRows) &&
        make_map(&mq2, qkt, qk[2], 64, a->N, HN, a->B,
                 qk_stride[2][0], qk_stride[2][1], qk_stride[2][2], da::kPrefillQRows) &&
        make_map(&mk1, qkt, qk[1], 64, a->N, a->H, a->B,
                 qk_stride[1][0], qk_stride[1][1], qk_stride[1][2], da::kPrefillKeyRows) &&
        make_map(&mk2, qkt, qk[3], 64, a->N, HN, a->B,
                 qk_stride[3][0], qk_stride[3][1], qk_stride[3][2], da::kPrefillKeyRows) &&
        (a->window > 0
             // the window kernel reads the caller's bf16 V and converts each step itself
             ? make_map(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a->v, 128, a->N, HV, a->B, a->v_stride[0],
                        a->v_stride[1], a->v_stride[2], da::kPrefillKeyRows)
             : make_map(&mv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws, 128, a->N, HV, a->B, a->N * HV * 128,
                        HV * 128, 128, da::kPrefillKeyRows)) &&
        make_map(&mo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a->out, 128, a->N, a->H, a->B,
                 a->out_stride[0], a->out_stride[1], a->out_stride[2], da::kPrefillOutRows);
    if (!ok) {
        da::set_internal_error("cuTensorMapEncodeTiled failed");
        return DIFFATTN_ERR_CUDA;
    }

    int launches = 0;
    const int sms = da::device_sm_count();
    char *wsc = static_cast<char *>(ws);
    int *tile_counter = reinterpret_cast<int *>(wsc + v16_bytes(a));
    // A call that saves the backward's state runs one signal head per item
    // (the state is per signal head).
    const bool paired = grouped_pairs(a) && !a->save;
    int *noise_ready = paired ? reinterpret_cast<int *>(wsc + v16_bytes(a) + 256 + noise_out_bytes(a)) : nullptr;
    cudaError_t e = da::launch_v_to_f16(a->v, a->v_stride[0], a->v_stride[1], a->v_stride[2], ws,
                                        (int)a->B, (int)a->N, (int)HV, a->dev_status,
                                        tile_counter, noise_ready, paired ? noise_tiles(a) : 0, rope,
                                        sms, s, &launches, a->window <= 0);
    if (e != cudaSuccess) return cuda_status(e);

    da::PrefillParams p{};
    p.B = (int)a->B;
    p.N = (int)a->N;
    p.H = (int)a->H;
    p.H_N = (int)HN;
    p.H_V = (int)HV;
    p.num_qt = (int)((a->N + 127) / 128);
    p.scale_log2 = a->scale * 1.4426950408889634f;
    p.eps = a->eps;
    p.causal = (a->flags & DIFFATTN_FLAG_CAUSAL) ? 1 : 0;
    p.apply_norm = (a->flags & DIFFATTN_FLAG_APPLY_NORM) ? 1 : 0;
    p.window = a->window;
    p.qk_f16 = a->rope_theta > 0.0f ? 1 : 0;
    p.withhold_load = (a->flags & DIFFATTN_FLAG_TEST_WITHHOLD_LOAD) ? 1 : 0;
    p.lambda = a->lambda;
    p.gain = p.apply_norm ? a->gain : nullptr;  // the gain belongs to the norm
    p.lam_logits = a->lambda_logits;
    p.ll_sb = a->lambda_logits_stride[0];
    p.ll_sn = a->lambda_logits_stride[1];
    p.ll_sh = a->lambda_logits_stride[2];
    p.gate = a->gate;
    p.gate_sb = a->gate_stride[0];
    p.gate_sn = a->gate_stride[1];
    p.gate_sh = a->gate_stride[2];
    p.out = a->out;
    p.out_sb = a->out_stride[0];
    p.out_sn = a->out_stride[1];
    p.out_sh = a->out_stride[2];
    p.dev_status = a->dev_status;
    p.timeout_ns = (uint64_t)(a->timeout_ms ? a->timeout_ms : kDefaultTimeoutMs) * 1000000ull;
    // Grouped heads whose group shares one V head and holds an odd number g
    // >= 3 of signal heads compute each map once, in one launch: per (b,
    // group, query tile) an export item (last signal head, noise head) that
    // also exports the normalised noise output, and (g - 1) / 2 pair items
    // of the remaining signal heads that import it.  Any other layout runs
    // one signal head (and its noise map) per work item.
    const int64_t g = a->H / HN;
    p.mode = paired ? 1 : 0;
    p.units = (int)(paired ? HN : a->H);
    p.pairs = paired ? (int)((g - 1) / 2) : 0;
    // (b, unit) pairs whose tiles run together, sharing their K/V in L2:
    // about four query tiles per SM in flight (measured best at the 4K and
    // 16K shapes: 18 and 4 heads, 36 and 32 MB of K/V; for the grouped pairs,
    // where a tile is two items, the same tile count measured 5 % faster at
    // the grouped workload than counting items).
    int G = (4 * sms) / p.num_qt;
    if (G < 1) G = 1;
    if (G > p.B * p.units) G = p.B * p.units;
    p.heads_per_group = G;
    p.tile_counter = tile_counter;
    if (paired) {
        p.noise_out = reinterpret_cast<float *>(wsc + v16_bytes(a) + 256);
        p.noise_ready = noise_ready;
        // Export items lead their tile's pair items by about one item per SM.
        const int64_t nt = noise_tiles(a);
        p.lag = (int)(nt < sms ? nt : sms);
    } else {
        p.save = static_cast<float *>(a->save);
    }
    if (g_events.start) cudaEventRecord(g_events.start, s);
    e = da::launch_prefill(mq1, mq2, mk1, mk2, mv, mo, p, s, &launches);
    if (g_events.stop) cudaEventRecord(g_events.stop, s);
    if (e != cudaSuccess) return cuda_status(e);
    g_last_launches = launches;
    return DIFFATTN_OK;
}

diffattn_status run_bwd(const diffattn_bwd_args *a, void *ws, size_t ws_bytes, void *stream)
{
    g_last_launches = 0;
    g_last_error[0] = 0;
    diffattn_status st = validate_bwd(a);
    if (st != DIFFATTN_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool empty = a->B == 0 || a->N == 0;
    if (!empty) {  // argument errors return before anything is enqueued
        const size_t need = diffattn_bwd_workspace_size(a);
        if (!ws || ws_bytes < need) return DIFFATTN_ERR_WORKSPACE;
        if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return DIFFATTN_ERR_ALIGNMENT;
    }
    // dlambda and dgain are sums over rows: start them at zero (and leave
    // them there for an empty problem; dlambda stays zero with lambda logits).
    if (a->grad_lambda) {
        cudaError_t e = cudaMemsetAsync(a->grad_lambda, 0, (size_t)a->H * sizeof(float), s);
        if (e != cudaSuccess) return cuda_status(e);
    }
    if (a->grad_gain) {
        cudaError_t e = cudaMemsetAsync(a->grad_gain, 0, (size_t)a->H * 128 * sizeof(float), s);
        if (e != cudaSuccess) return cuda_status(e);
    }
    if (empty) return DIFFATTN_OK;
    const int64_t HN = bwd_hn(a), HV = bwd_hv(a);

    char *w = static_cast<char *>(ws);
    void *v16 = w;
    void *dd = w + bwd_v16_bytes(a);
    float *stats = reinterpret_cast<float *>(w + bwd_v16_bytes(a) + bwd_dd_bytes(a));
    int *counters = reinterpret_cast<int *>(w + bwd_v16_bytes(a) + bwd_dd_bytes(a) + bwd_stats_bytes(a));
    char *rope_dst = w + bwd_v16_bytes(a) + bwd_dd_bytes(a) + bwd_stats_bytes(a) + 256;
    char *acc = w + bwd_acc_offset(a);
    float *acc_qk = bwd_acc_qk_bytes(a) ? reinterpret_cast<float *>(acc) : nullptr;
    float *acc_v = bwd_acc_v_bytes(a) ? reinterpret_cast<float *>(acc + 2 * bwd_acc_qk_bytes(a)) : nullptr;
    const int64_t acc_floats = (int64_t)((2 * bwd_acc_qk_bytes(a) + bwd_acc_v_bytes(a)) / sizeof(float));
    const int64_t num_qt = (a->N + 127) / 128, n_pad = num_qt * 128;

    // Q/K operands: the caller's bf16 tensors, or their rotated fp16 copies.
    const void *qk[4] = {a->q1, a->k1, a->q2, a->k2};
    const int64_t *qks[4] = {a->q1_stride, a->k1_stride, a->q2_stride, a->k2_stride};
    int64_t qs[4][3];
    for (int t = 0; t < 4; ++t)
        for (int i = 0; i < 3; ++i) qs[t][i] = qks[t][i];
    da::RopeStage rope;
    set_rope(&rope, a->rope_theta, a->B, a->N, a->H, HN, rope_dst, qk, qs);

    da::BwdKeyMaps km;
    da::BwdQueryMaps qm;
    const CUtensorMapDataType qkt = a->rope_theta > 0.0f ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                         : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUtensorMapDataType f16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const int64_t hs = a->N * a->H * 128, vs = a->N * HV * 128;  // batch strides of the fp16 copies
    auto qkmap = [&](CUtensorMap *m, int t, uint32_t rows) {
        return make_map(m, qkt, qk[t], 64, a->N, t < 2 ? a->H : HN, a->B, qs[t][0], qs[t][1], qs[t][2], rows);
    };
    const bool ok =
        qkmap(&km.k1, 1, 128) && qkmap(&km.k2, 3, 128) &&
        make_map(&km.v, f16, v16, 128, a->N, HV, a->B, vs, HV * 128, 128, 128) &&
        qkmap(&km.q1, 0, 64) && qkmap(&km.q2, 2, 64) &&
        make_map(&km.dd, f16, dd, 128, a->N, a->H, a->B, hs, a->H * 128, 128, 64) &&
        make_stats_map(&km.stats, stats, n_pad, a->H, a->B) &&
        qkmap(&qm.q1, 0, 128) && qkmap(&qm.q2, 2, 128) &&
        make_map(&qm.dd, f16, dd, 128, a->N, a->H, a->B, hs, a->H * 128, 128, 128) &&
        qkmap(&qm.k1, 1, 64) && qkmap(&qm.k2, 3, 64) &&
        make_map(&qm.v, f16, v16, 128, a->N, HV, a->B, vs, HV * 128, 128, 64);
    if (!ok) {
        da::set_internal_error("cuTensorMapEncodeTiled failed");
        return DIFFATTN_ERR_CUDA;
    }

    int launches = 0;
    // Staging: fp16 V, the rotated Q/K copies, and zeroed fp32 sums.
    cudaError_t e = da::launch_v_to_f16(a->v, a->v_stride[0], a->v_stride[1], a->v_stride[2], v16,
                                        (int)a->B, (int)a->N, (int)HV, a->dev_status, counters,
                                        acc_floats ? reinterpret_cast<int *>(acc) : nullptr, acc_floats,
                                        rope, da::device_sm_count(), s, &launches);
    if (e != cudaSuccess) return cuda_status(e);

    da::BwdParams p{};
    p.tile_counter = counters;
    p.B = (int)a->B;
    p.N = (int)a->N;
    p.H = (int)a->H;
    p.H_N = (int)HN;
    p.H_V = (int)HV;
    p.num_qt = (int)num_qt;
    p.n_pad = (int)n_pad;
    p.scale = a->scale;
    p.scale_log2 = a->scale * 1.4426950408889634f;
    p.eps = a->eps;
    p.causal = (a->flags & DIFFATTN_FLAG_CAUSAL) ? 1 : 0;
    p.apply_norm = (a->flags & DIFFATTN_FLAG_APPLY_NORM) ? 1 : 0;
    p.window = a->window;
    p.save = static_cast<const float *>(a->save);
    p.dout = a->dout;
    p.do_sb = a->dout_stride[0];
    p.do_sn = a->dout_stride[1];
    p.do_sh = a->dout_stride[2];
    p.lambda = a->lambda;
    p.lam_logits = a->lambda_logits;
    p.ll_sb = a->lambda_logits_stride[0];
    p.ll_sn = a->lambda_logits_stride[1];
    p.ll_sh = a->lambda_logits_stride[2];
    p.gate = a->gate;
    p.gate_sb = a->gate_stride[0];
    p.gate_sn = a->gate_stride[1];
    p.gate_sh = a->gate_stride[2];
    p.gain = p.apply_norm ? a->gain : nullptr;  // the gain belongs to the norm
    p.dd = dd;
    p.stats = stats;
    p.dq1 = a->grad_q1;
    p.dq2 = a->grad_q2;
    p.dk1 = a->grad_k1;
    p.dk2 = a->grad_k2;
    p.dv = a->grad_v;
    for (int i = 0; i < 3; ++i) {
        p.dq1_s[i] = a->grad_q1_stride[i];
        p.dq2_s[i] = a->grad_q2_stride[i];
        p.dk1_s[i] = a->grad_k1_stride[i];
        p.dk2_s[i] = a->grad_k2_stride[i];
        p.dv_s[i] = a->grad_v_stride[i];
    }
    p.acc_dk2 = acc_qk;
    p.acc_dq2 = acc_qk ? acc_qk + bwd_acc_qk_bytes(a) / sizeof(float) : nullptr;
    p.acc_dv = acc_v;
    p.dlambda = a->lambda_logits ? nullptr : a->grad_lambda;
    p.dgain = a->grad_gain;
    p.dlam_logits = a->grad_lambda_logits;
    p.dll_sb = a->grad_lambda_logits_stride[0];
    p.dll_sn = a->grad_lambda_logits_stride[1];
    p.dll_sh = a->grad_lambda_logits_stride[2];
    p.dgate = a->grad_gate;
    p.dg_sb = a->grad_gate_stride[0];
    p.dg_sn = a->grad_gate_stride[1];
    p.dg_sh = a->grad_gate_stride[2];
    p.qk_f16 = a->rope_theta > 0.0f ? 1 : 0;
    for (int c = 0; c < 32; ++c) p.rope_g[c] = rope.g[c];
    p.dev_status = a->dev_status;
    p.timeout_ns = (uint64_t)(a->timeout_ms ? a->timeout_ms : kDefaultTimeoutMs) * 1000000ull;
    e = da::launch_bwd(km, qm, p, s, &launches, g_events);
    if (e != cudaSuccess) return cuda_status(e);
    g_last_launches = launches;
    return DIFFATTN_OK;
}

// Fill the decode parameters and launch (arguments already validated; the
// partials buffer holds at least diffattn_decode_workspace_size bytes).
diffattn_status run_decode(const diffattn_decode_args *a, float *partials, void *stream)
{
    da::DecodeParams p{};
    p.B = (int)a->B;
    p.H = (int)a->H;
    p.L = (int)a->L;
    p.splits = decode_splits(a->B, a->H, a->L, a->num_splits);
    p.chunk = decode_chunk(a->L, p.splits);
    p.window = a->window;
    if (a->window > 0 && a->window < a->L) {
        // Only the window's keys are split.  The workspace holds the split
        // count for L, so use no more splits than that.
        const int64_t Lw = a->window;
        int s = decode_splits(a->B, a->H, Lw, a->num_splits);
        if (s > p.splits) s = p.splits;
        p.chunk = decode_chunk(Lw, s);
        p.splits = (int)((Lw + p.chunk - 1) / p.chunk);
    }
    p.scale_log2 = a->scale * 1.4426950408889634f;
    p.eps = a->eps;
    p.apply_norm = (a->flags & DIFFATTN_FLAG_APPLY_NORM) ? 1 : 0;
    p.q1 = a->q1;
    p.q2 = a->q2;
    p.k1 = a->k1;
    p.k2 = a->k2;
    p.v = a->v;
    p.q1_sb = a->q1_stride[0];
    p.q1_sh = a->q1_stride[1];
    p.q2_sb = a->q2_stride[0];
    p.q2_sh = a->q2_stride[1];
    p.k1_sb = a->k1_stride[0];
    p.k1_sh = a->k1_stride[1];
    p.k1_sl = a->k1_stride[2];
    p.k2_sb = a->k2_stride[0];
    p.k2_sh = a->k2_stride[1];
    p.k2_sl = a->k2_stride[2];
    p.v_sb = a->v_stride[0];
    p.v_sh = a->v_stride[1];
    p.v_sl = a->v_stride[2];
    p.out = a->out;
    p.out_sb = a->out_stride[0];
    p.out_sh = a->out_stride[1];
    p.kv_len = a->kv_len;
    p.lambda = a->lambda;
    p.gain = a->gain;
    p.lam_logits = a->lambda_logits;
    p.ll_sb = a->lambda_logits_stride[0];
    p.ll_sh = a->lambda_logits_stride[1];
    p.gate = a->gate;
    p.gate_sb = a->gate_stride[0];
    p.gate_sh = a->gate_stride[1];
    p.partials = partials;
    p.dev_status = a->dev_status;
    int launches = 0;
    cudaError_t e = da::launch_decode(p, static_cast<cudaStream_t>(stream), &launches, g_events);
    if (e != cudaSuccess) return cuda_status(e);
    g_last_launches = launches;
    return DIFFATTN_OK;
}

}  // namespace

void da::set_internal_error(const char *text)
{
    std::snprintf(g_last_error, sizeof g_last_error, "%s", text);
}

int da::device_sm_count()
{
    constexpr int kMaxDevices = 64;
    constexpr int kNoDevice = 148;  // a B200, for size queries on a host without a device
    static std::atomic<int> count[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();  // a failed query leaves no sticky error behind
        return kNoDevice;
    }
    int n = count[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return kNoDevice;
    }
    count[dev].store(n, std::memory_order_relaxed);  // idempotent: every thread stores the same value
    return n;
}

extern "C" {

diffattn_status diffattn_fwd_validate(const diffattn_fwd_args *args, int grouped)
{
    return validate_fwd(args, grouped);
}

size_t diffattn_fwd_workspace_size(const diffattn_fwd_args *a)
{
    if (!a || a->B <= 0 || a->N <= 0 || a->H <= 0) return 0;
    return rope_offset(a) + rope_bytes(a);
}

size_t diffattn_fwd_save_size(const diffattn_fwd_args *a)
{
    if (!a || a->B <= 0 || a->N <= 0 || a->H <= 0) return 0;
    return (size_t)a->B * a->H * ((a->N + 127) / 128) * da::kSaveTileFloats * sizeof(float);
}

size_t diffattn_bwd_workspace_size(const diffattn_bwd_args *a)
{
    if (!a || a->B <= 0 || a->N <= 0 || a->H <= 0) return 0;
    return bwd_acc_offset(a) + 2 * bwd_acc_qk_bytes(a) + bwd_acc_v_bytes(a);
}

// A named NVTX range around each entry point, for timeline profilers (a
// no-op unless one is attached).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

diffattn_status diffattn_fwd(const diffattn_fwd_args *args, void *workspace, size_t ws_bytes,
                             void *stream)
{
    NvtxRange range("diffattn_fwd");
    return run_fwd(args, workspace, ws_bytes, stream, 0);
}

diffattn_status diffattn_grouped_fwd(const diffattn_fwd_args *args, void *workspace,
                                     size_t ws_bytes, void *stream)
{
    NvtxRange range("diffattn_grouped_fwd");
    return run_fwd(args, workspace, ws_bytes, stream, 1);
}

diffattn_status diffattn_bwd(const diffattn_bwd_args *args, void *workspace, size_t ws_bytes,
                             void *stream)
{
    NvtxRange range("diffattn_bwd");
    return run_bwd(args, workspace, ws_bytes, stream);
}

diffattn_status diffattn_decode_validate(const diffattn_decode_args *args)
{
    return validate_decode(args);
}

int32_t diffattn_decode_num_splits(int64_t B, int64_t H, int64_t L, int32_t num_splits)
{
    if (B < 0 || H <= 0 || L <= 0 || num_splits < 0) return 0;
    return decode_splits(B, H, L, num_splits);
}

size_t diffattn_decode_workspace_size(int64_t B, int64_t H, int64_t L, int32_t num_splits)
{
    if (B <= 0 || H <= 0 || L <= 0 || num_splits < 0) return 0;
    const int s = decode_splits(B, H, L, num_splits);
    return align256((size_t)B * H * s * da::kDecodePartialFloats * sizeof(float));
}

diffattn_status diffattn_decode(const diffattn_decode_args *a, void *workspace, size_t ws_bytes,
                                void *stream)
{
    NvtxRange range("diffattn_decode");
    g_last_launches = 0;
    g_last_error[0] = 0;
    diffattn_status st = validate_decode(a);
    if (st != DIFFATTN_OK) return st;
    if (a->B == 0) return DIFFATTN_OK;
    const size_t need = diffattn_decode_workspace_size(a->B, a->H, a->L, a->num_splits);
    if (!workspace || ws_bytes < need) return DIFFATTN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0) return DIFFATTN_ERR_ALIGNMENT;
    return run_decode(a, static_cast<float *>(workspace), stream);
}

diffattn_status diffattn_decode_noalloc(const diffattn_decode_args *a, void *stream)
{
    NvtxRange range("diffattn_decode_noalloc");
    g_last_launches = 0;
    g_last_error[0] = 0;
    diffattn_status st = validate_decode(a);
    if (st != DIFFATTN_OK) return st;
    if (a->B == 0) return DIFFATTN_OK;
    const size_t need = diffattn_decode_workspace_size(a->B, a->H, a->L, a->num_splits);
    if (need > da::kNoAllocScratchBytes) {
        std::snprintf(g_last_error, sizeof g_last_error,
                      "decode partials need %zu bytes; the no-allocation scratch holds %zu",
                      need, da::kNoAllocScratchBytes);
        return DIFFATTN_ERR_WORKSPACE;
    }
    float *scratch = nullptr;
    const cudaError_t e = da::decode_noalloc_scratch(&scratch);
    if (e != cudaSuccess) return cuda_status(e);
    return run_decode(a, scratch, stream);
}

const char *diffattn_status_str(diffattn_status s)
{
    switch (s) {
    case DIFFATTN_OK: return "ok";
    case DIFFATTN_ERR_INVALID_ARG: return "invalid argument";
    case DIFFATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case DIFFATTN_ERR_ALIGNMENT: return "misaligned pointer or stride";
    case DIFFATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case DIFFATTN_ERR_CUDA: return "CUDA error";
    case DIFFATTN_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

int32_t diffattn_last_launch_count(void) { return g_last_launches; }

const char *diffattn_last_error(void) { return g_last_error; }

void diffattn_set_profile_events(void *start, void *stop)
{
    g_events.start = static_cast<cudaEvent_t>(start);
    g_events.stop = static_cast<cudaEvent_t>(stop);
}

}  // extern "C"
