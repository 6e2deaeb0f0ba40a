// kernels.h -- host-side launch interface between the C ABI (api.cu) and the
// kernel translation units.  Internal to libdiffattn.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "diffattn.h"

namespace da {

// Record a library-side failure text for diffattn_last_error() (thread-local).
void set_internal_error(const char *text);

// Events to record around the main kernel of a call (benchmark timing hook);
// both null when unused.
struct ProfileEvents {
    cudaEvent_t start = nullptr, stop = nullptr;
};

// Everything the prefill kernel needs besides its five tensor maps.
struct PrefillParams {
    int B, N, H, H_N, H_V;
    int num_qt;           // query tiles per (b, h): ceil(N / 128)
    int heads_per_group;  // (b, h) pairs scheduled together for L2 reuse of K/V
    float scale_log2;     // softmax scale * log2(e)
    float eps;
    int causal, apply_norm;
    int window;           // sliding window in keys (query i sees i-window < j <= i), 0 = none
    int qk_f16;           // Q/K are fp16 (the rotated copies) rather than bf16
    int withhold_load;    // test hook: skip the first K/V load of the CTA's first tile
    int mode;             // 0: one signal head per item; 1: grouped pairs (see prefill_sm100.cu)
    int units;            // tile units per batch entry: signal heads (mode 0), noise heads (mode 1)
    int pairs;            // mode 1: (signal, signal) pairs per group, (H / H_N - 1) / 2
    int lag;              // mode 1: tiles by which a group's pair items trail its export item
    float *noise_out;     // mode 1: normalised noise outputs, fp32, per (b, noise head,
                          // query tile) 32 float4 chunks x 128 rows (chunk-major)
    int *noise_ready;     // mode 1: per (b, noise head, query tile) count of the 4 epilogue
                          // warps that have exported their part (zeroed by the staging kernel)
    const float *lambda;  // [H], unused when lam_logits is set
    const float *gain;    // [H, 128] or nullptr
    const float *lam_logits;  // token-dependent lambda logits [B, N, H] or nullptr
    int64_t ll_sb, ll_sn, ll_sh;
    const void *gate;     // bf16 output-gate logits [B, N, H, 128] or nullptr
    int64_t gate_sb, gate_sn, gate_sh;
    void *out;            // bf16
    int64_t out_sb, out_sn, out_sh;
    int32_t *dev_status;
    uint64_t timeout_ns;
    int *tile_counter;    // work-item counter in the workspace (zeroed by the V staging kernel)
    float *save;          // mode 0: state saved for the backward pass, or nullptr
};

// The forward's saved state, per (b, h, 128-row query tile): A_1 and A_2 as
// fp32 float4 chunks, chunk c of map t and tile row r at float4 index
// (32 t + c) * 128 + r, then lse_t (log2 of the softmax denominator, in the
// units of scale * log2(e) * score) at float index 2 * 128 * 128 + 128 t + r.
constexpr int kSaveTileFloats = 2 * 128 * 128 + 2 * 128;

// Rows per TMA box: a query tile, and a key step of the prefill kernel.
constexpr unsigned kPrefillQRows = 128;
constexpr unsigned kPrefillKeyRows = 64;
constexpr unsigned kPrefillOutRows = 32;  // rows of an output store box (one warp's rows)

// Tensor maps: Q1/K1 over [B, N, H, 64] bf16, Q2/K2 over [B, N, H_N, 64]
// bf16, V over the fp16 copy [B, N, H_V, 128]; all with 128-byte swizzle and
// {64, rows, 1, 1} boxes (kPrefillQRows for Q, kPrefillKeyRows for K and V).
cudaError_t launch_prefill(const CUtensorMap &q1, const CUtensorMap &q2, const CUtensorMap &k1,
                           const CUtensorMap &k2, const CUtensorMap &v16, const CUtensorMap &out,
                           const PrefillParams &p,
                           cudaStream_t stream, int *launches);

// bf16 V [B, N, H_V, 128] (strided) -> contiguous fp16 copy in `dst`; also
// zeroes the two work-item counters of the prefill launches that follow.
// Rotary-embedding part of the staging kernel: tensors 0..3 are Q1, K1, Q2,
// K2 (heads H, H, H_N, H_N); each 64-wide row at token n is rotated into a
// contiguous [B, N, heads, 64] fp16 copy.  g[c] = theta^(-2c/64) / (2 pi).
struct RopeStage {
    const void *src[4];
    int64_t sb[4], sn[4], sh[4];
    void *dst[4];
    int heads[4];
    double g[32];
    int enabled;
};

// `zero`/`n_zero`: ints the staging kernel also clears (the grouped pairs'
// ready counts), or nullptr / 0.  `sm_count`: SMs of the device (grid size).
// `stage_v` false: no fp16 copy of V (the sliding-window prefill converts
// each V step itself); the counters, `zero` and RoPE are done as usual.
cudaError_t launch_v_to_f16(const void *v, int64_t sb, int64_t sn, int64_t sh, void *dst, int B,
                            int N, int H_V, int32_t *dev_status, int *tile_counter,
                            int *zero, int64_t n_zero, const RopeStage &rope, int sm_count,
                            cudaStream_t stream, int *launches, bool stage_v = true);

// SM count of the current device, looked up once per device (thread-safe);
// 148 (a B200) when no device is visible, for host-only size queries.
int device_sm_count();

// Backward pass (backward_sm100.cu).
struct BwdParams {
    int B, N, H, H_N, H_V;
    int num_qt, n_pad;    // 128-row tiles per (b, h) and n_pad = 128 num_qt
    float scale, scale_log2, eps;
    int causal, apply_norm;
    int window;           // sliding window in keys, 0 = none
    const float *save;    // the forward's saved state (kSaveTileFloats per tile)
    const void *dout;     // bf16 [B, N, H, 128]
    int64_t do_sb, do_sn, do_sh;
    const float *lambda;  // [H], unused with lam_logits
    const float *lam_logits;  // [B, N, H] or nullptr
    int64_t ll_sb, ll_sn, ll_sh;
    const void *gate;     // bf16 gate logits [B, N, H, 128] or nullptr
    int64_t gate_sb, gate_sn, gate_sh;
    const float *gain;    // [H, 128] or nullptr (1)
    void *dd;             // workspace: dD as fp16, contiguous [B, N, H, 128]
    float *stats;         // workspace: [B, H, kBwdStats, n_pad] fp32
    void *dq1, *dq2, *dk1, *dk2, *dv;  // bf16 outputs
    int64_t dq1_s[3], dq2_s[3], dk1_s[3], dk2_s[3], dv_s[3];
    float *acc_dq2, *acc_dk2, *acc_dv;  // fp32 [B, N, heads, dim] sums when heads are shared, else nullptr
    float *dlambda;       // [H] (zeroed before the call) or nullptr
    float *dgain;         // [H, 128] (zeroed before the call) or nullptr
    float *dlam_logits;   // [B, N, H] or nullptr
    int64_t dll_sb, dll_sn, dll_sh;
    void *dgate;          // bf16 [B, N, H, 128] or nullptr
    int64_t dg_sb, dg_sn, dg_sh;
    int qk_f16;           // Q/K operands are the rotated fp16 copies (rotary embedding)
    double rope_g[32];    // turns per token of pair c: theta^(-2c/64) / (2 pi)
    int *tile_counter;    // two work counters (key tiles, query tiles), zeroed by the staging kernel
    int32_t *dev_status;
    uint64_t timeout_ns;
};

// Row statistics of the backward pass, per (b, h): lse_1, lse_2, Delta_1,
// Delta_2 and the row's lambda, each n_pad floats.
constexpr int kBwdStats = 5;

// Tensor maps of the key-tile kernel (dK_1, dK_2, dV): K_1, K_2 and the fp16
// V copy in 128-row boxes; Q_1, Q_2 and dD in 64-row boxes (all 128-byte
// swizzled, {64 columns, rows} boxes); the statistics in {64 rows,
// kBwdStats arrays} boxes of fp32, not swizzled.
struct BwdKeyMaps {
    CUtensorMap k1, k2, v, q1, q2, dd, stats;
};
// Tensor maps of the query-tile kernel (dQ_1, dQ_2): Q_1, Q_2, dD in 128-row
// boxes; K_1, K_2 and the fp16 V copy in 64-row boxes.
struct BwdQueryMaps {
    CUtensorMap q1, q2, dd, k1, k2, v;
};

// Launch the backward kernels after the staging pass: the row preparation
// (dD, statistics, dlambda or the lambda logits' gradient, dgain, the gate's
// gradient), the key-tile kernel, the query-tile kernel and, when heads are
// shared, the conversion of the fp32 sums.
cudaError_t launch_bwd(const BwdKeyMaps &km, const BwdQueryMaps &qm, const BwdParams &p,
                       cudaStream_t stream, int *launches, const ProfileEvents &ev);

struct DecodeParams {
    int B, H, L;
    int splits, chunk;    // keys per split (multiple of 64)
    int window;           // the query sees the `window` most recent keys, 0 = all
    float scale_log2, eps;
    int apply_norm;
    const void *q1, *q2, *k1, *k2, *v;
    int64_t q1_sb, q1_sh, q2_sb, q2_sh;
    int64_t k1_sb, k1_sh, k1_sl, k2_sb, k2_sh, k2_sl, v_sb, v_sh, v_sl;
    void *out;
    int64_t out_sb, out_sh;
    const int32_t *kv_len;
    const float *lambda, *gain;
    const float *lam_logits;  // [B, H] or nullptr
    int64_t ll_sb, ll_sh;
    const void *gate;         // bf16 [B, H, 128] or nullptr
    int64_t gate_sb, gate_sh;
    float *partials;      // [B*H][splits][4 + 2*128] fp32
    int32_t *dev_status;
};

// Floats of one split's partial state: m1, l1, m2, l2, acc1[128], acc2[128].
constexpr int kDecodePartialFloats = 4 + 2 * 128;
constexpr int kDecodeMaxChunk = 2048;

cudaError_t launch_decode(const DecodeParams &p, cudaStream_t stream, int *launches,
                          const ProfileEvents &ev);

// Size of the static device array behind diffattn_decode_noalloc.
constexpr size_t kNoAllocScratchBytes = DIFFATTN_DECODE_NOALLOC_SCRATCH_BYTES;

// Device address of that array on the current device (looked up with
// cudaGetSymbolAddress on the first call per device, then cached).
cudaError_t decode_noalloc_scratch(float **ptr);

}  // namespace da
