// backward_sm100.cu -- the backward pass of the differential-attention
// prefill on B200 (sm_100a).
//
// The pages define the forward pass (Motif 2.6B explainer, section
// "Differential attention", figure 1; Motif 3 summary, section 2.2, for the
// grouped heads, the token-dependent lambda and the output gate, section 2.1
// for sliding-window layers; Motif 2.6B explainer, "The block", for the
// rotary embedding) and train the model with it (Motif 2.6B explainer, "A
// schedule for the data"); the backward pass here is its exact gradient.
// With A_t = P_t V the two map outputs, lambda_i the row's lambda (per head,
// or sigma of the token's logit), D = A_1 - lambda_i A_2,
// r = (mean_c D^2 + eps)^-1/2, Yn = D r gain, Y = sigma(G) Yn:
//
//   dYn = dY sigma(G),  dG = dY Yn sigma'(G)           (gate; else dYn = dY)
//   dgain = sum_i dYn D r,  dD = r (dYn gain) - (r^3/128) D sum_c(dYn gain D)
//   dA_1 = dD, dA_2 = -lambda_i dD,  dlambda_i = -sum_c dD A_2
//   per map t: dP_t = dA_t V^T = (1, -lambda_i) x dP with dP = dD V^T (one product)
//              Delta_t = rowsum(dA_t A_t), dS_t = P_t (dP_t - Delta_t)
//              dQ_t = scale dS_t K_t, dK_t = scale dS_t^T Q_t
//   dV = P_1^T dA_1 + P_2^T dA_2 = (P_1 - lambda P_2)^T dD (one product)
//
// (with the rotary embedding the products run on the rotated Q/K, and dQ,
// dK are rotated back).  After the staging pass (fp16 V, rotated Q/K),
// three or four kernels:
//  1. bwd_prep_kernel, one thread per row: reads the forward's saved A_1, A_2
//     and lse, dY and the gate logits; writes dD (fp16, the tensor-core
//     operand), the row statistics (lse_1, lse_2, Delta_1, Delta_2, lambda),
//     the gate's and the lambda logits' gradients, and adds into dlambda and
//     dgain.
//  2. bwd_key_kernel, one CTA per (b, h, 128-key tile), keys on the 128 TMEM
//     lanes, over the 64-query blocks that see them.  Warp-specialised:
//     warp 0 loads (TMA), warp 1 issues the tcgen05 products, warps 2-9
//     (two warpgroups, 32 queries of each block apiece) run the element-wise
//     step.  Per block: S_1^T = K_1 Q_1^T, S_2^T = K_2 Q_2^T, dP^T = V dD^T
//     into TMEM; the element-wise warps load them to registers and release
//     the TMEM at once, so the next block's products run during this
//     block's element-wise step; they write P_1 - lambda P_2 (fp16) and
//     dS_1, dS_2 to shared memory as the A operands of dV += (P_1 - lambda
//     P_2)^T dD and dK_t += dS_t^T Q_t.
//  3. bwd_query_kernel, the same shape per (b, h, 128-query tile) over
//     64-key blocks: S_1, S_2, dP = dD V^T, the element-wise step, dQ_t +=
//     dS_t K_t.
//  4. bwd_convert_kernel, only when noise or V heads are shared by several
//     signal heads: their gradients are summed in fp32 (vector atomics from
//     the tile kernels) and converted to bf16 here.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>
#include <mutex>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace da {
namespace {

constexpr int BT = 128;   // rows of a tile: MMA M, one per TMEM lane
constexpr int BB = 64;    // rows of a block: MMA N of the score products
constexpr int HD = 64;    // Q/K head dim
constexpr int HDV = 128;  // V head dim
constexpr int NT = 352;   // 11 warps: producer, two MMA issuers, two element-wise warpgroups
constexpr int NEW = 8;    // element-wise warps

// Block stages of the two tile kernels' load rings (as many as fit in
// shared memory: a block's load is issued STAGES - 1 blocks ahead).
constexpr int KSTAGES = 3, QSTAGES = 3, MAXSTAGES = 3;

// Which pairs of exponentials (pair index mod 8) the element-wise step
// computes with the software exp2 (FMA pipe) rather than MUFU ex2: the step
// needs two exponentials per (key, query) pair against 1280 MMA FLOP.
constexpr uint32_t BWD_SOFT_EXP_MASK = 0x02u;  // one pair in eight (measured: none 457, 1/8 462, 2/8 456, 4/8 451 TFLOP/s)

// mbarriers of both tile kernels.
enum : int {
    B_TILE = 0,                     // the tile's operands landed (TMA bytes)
    B_FULL = 1,                     // [stages] a block's operands landed (TMA bytes)
    B_EMPTY = B_FULL + MAXSTAGES,   // [stages] the block's last products have read its stage (commit)
    B_SFULL = B_EMPTY + MAXSTAGES,  // the block's score and dP products are in TMEM (commit)
    B_SFREE,                        // the element-wise warps loaded them (8 arrivals)
    B_AFULL,                        // the element-wise warps wrote the A operands (8 arrivals)
    B_AFREE,                        // the accumulating products have read the A operands (commit)
    B_DONE,                         // every product of the tile has completed (commit)
    B_SDRAIN,                       // the score issuer's products have completed (commit)
    B_AOP,                          // the tile's A operands are in TMEM (8 arrivals)
    B_TILEFREE,                     // key tiles: the tile's score products are done with its K and V (commit)
    B_ACCFREE,                      // the epilogue has read the accumulators (8 arrivals)
    B_ADRAIN,                       // the accumulating issuer's products have completed (commit)
    B_ITEM,                         // [4] a tile index published (1 arrival)
    B_ITEMFREE = B_ITEM + 4,        // [4] the tile index read by all ten reader warps
    NBARS = B_ITEMFREE + 4
};

// ---------------------------------------------------------------- key-tile kernel
// Shared memory: the tile's K_1, K_2 ([128][64]) and fp16 V ([128][128] as
// two [128][64] column halves); KSTAGES block stages of Q_1, Q_2 ([64][64]),
// dD (fp16 [64][128] as two halves) and the statistics [kBwdStats][64]
// fp32; the A operands P_1 - lambda P_2, dS_1, dS_2 ([128 keys][64 queries]).
constexpr uint32_t KT_K1 = 0, KT_K2 = 16384, KT_V = 32768, KT_STAGE0 = 65536;
constexpr uint32_t KB_Q1 = 0, KB_Q2 = 8192, KB_DD = 16384, KB_ST = 32768;
constexpr uint32_t KB_LOAD = KB_ST + kBwdStats * BB * 4;  // bytes a stage receives
constexpr uint32_t KB_BYTES = (KB_LOAD + 1023) & ~1023u;   // stages stay 1 KB aligned
constexpr uint32_t KT_A = KT_STAGE0 + KSTAGES * KB_BYTES;
constexpr uint32_t KA_PV = 0, KA_DS1 = 16384, KA_DS2 = 32768;
constexpr uint32_t KT_BARS = KT_A + 3 * 16384;
constexpr uint32_t KT_SMEM = KT_BARS + 8 * NBARS + 32;  // + TMEM address, abort flag, 4-slot tile ring
// TMEM columns: dV, dK_1, dK_2 accumulators, then S_1^T, S_2^T, dP^T, then
// the tile's K_1 and K_2 (bf16 / fp16 pairs) as the A operand of the score
// products, so that every block's score products read only Q from shared
// memory (the kernel is bound by shared-memory bandwidth).
constexpr uint32_t KM_DV = 0, KM_DK1 = 128, KM_DK2 = 192, KM_S1 = 256, KM_S2 = 320, KM_DP = 384,
                   KM_AK1 = 448, KM_AK2 = 480;

// ---------------------------------------------------------------- query-tile kernel
// Shared memory: the tile's Q_1, Q_2 ([128][64]) and dD (fp16 [128][128] as
// two halves); QSTAGES block stages of K_1, K_2 ([64][64]) and fp16 V
// ([64][128] as two halves).
constexpr uint32_t QT_Q1 = 0, QT_Q2 = 16384, QT_DD = 32768, QT_STAGE0 = 65536;
constexpr uint32_t QB_K1 = 0, QB_K2 = 8192, QB_V = 16384, QB_BYTES = 32768;
constexpr uint32_t QT_BARS = QT_STAGE0 + QSTAGES * QB_BYTES;
constexpr uint32_t QT_SMEM = QT_BARS + 8 * NBARS + 32;  // + TMEM address, abort flag, 4-slot tile ring
// TMEM columns: dQ_1, dQ_2 accumulators, then S_1, S_2, dP, then the tile's
// Q_1, Q_2 and dD (16-bit pairs) as the A operands of the score and dP
// products, so that every block's products read only K and V from shared
// memory (the kernel is bound by shared-memory bandwidth), then the block's
// dS_1, dS_2 (16-bit pairs) as the A operands of the dQ products, written
// by the element-wise warps with TMEM stores.
constexpr uint32_t QM_DQ1 = 0, QM_DQ2 = 64, QM_S1 = 128, QM_S2 = 192, QM_DP = 256, QM_AQ1 = 320,
                   QM_AQ2 = 352, QM_ADD = 384, QM_ADS1 = 448, QM_ADS2 = 480;

static_assert(KT_SMEM <= 232448 && QT_SMEM <= 232448, "shared memory budget");
static_assert(KT_A % 1024 == 0 && QT_STAGE0 % 1024 == 0 && KB_BYTES % 1024 == 0, "SW128 tiles are 1 KB aligned");
static_assert(KT_SMEM > 116 * 1024 && QT_SMEM > 116 * 1024, "one CTA per SM owns the 512 TMEM columns");

// Instruction descriptors (fp32 accumulate).  F16QK: Q/K are the rotated
// fp16 copies (and dS is fp16 to match them in the dQ / dK products).
template <bool F16QK>
struct Ids {
    static constexpr uint32_t S = F16QK ? idesc_f16(0, 0, 0, BT, BB) : idesc_f16(1, 1, 0, BT, BB);
    static constexpr uint32_t DS = F16QK ? idesc_f16(0, 0, 1, BT, HD) : idesc_f16(1, 1, 1, BT, HD);
};
constexpr uint32_t ID_DP = idesc_f16(0, 0, 0, BT, BB);   // fp16 x fp16, both K-major
constexpr uint32_t ID_DV = idesc_f16(0, 0, 1, BT, HDV);  // fp16 A (K-major) x fp16 B (MN-major)

// Descriptor of a 128-byte-swizzled operand tile (rows of 128 bytes, 8-row
// atoms of 1 KB); `lbo` is the byte distance between 64-element column
// halves when the MMA's N spans two of them (MN-major B).
__device__ __forceinline__ uint64_t sw128(uint32_t addr, uint32_t lbo = 16)
{
    return smem_desc_sw128(addr, lbo, 1024);
}

// One elected lane of a fully active warp issues; the warp stays converged.
__device__ __forceinline__ void mma_issue(uint32_t d, uint64_t a, uint64_t b, uint32_t id, bool acc)
{
    if (elect_one()) mma_ss(d, a, b, id, acc ? 1u : 0u);
    __syncwarp();
}
__device__ __forceinline__ void mma_issue_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t id, bool acc)
{
    if (elect_one()) mma_ts(d, a_tmem, b, id, acc ? 1u : 0u);
    __syncwarp();
}
__device__ __forceinline__ void commit_to(uint32_t bar)
{
    if (elect_one()) mma_commit(bar);
    __syncwarp();
}

__device__ __forceinline__ uint32_t pack_ds(float lo, float hi, bool f16)
{
    return f16 ? pack_half2(lo, hi) : pack_bf162(lo, hi);
}

// Row r's 32-column half `half` of a [128 rows][64 columns] 16-bit operand
// tile in the 128-byte swizzle (16-byte chunk c of row r at c ^ (r % 8)).
__device__ __forceinline__ void st_operand_half(uint32_t tile, int r, int half, const uint32_t (&w)[16])
{
    const uint32_t row = tile + 128u * r;
#pragma unroll
    for (int c = 0; c < 4; ++c)
        st_shared_v4(row + ((((4 * half + c) ^ (r & 7)) & 7) << 4), w[4 * c], w[4 * c + 1], w[4 * c + 2],
                     w[4 * c + 3]);
}

// The inverse rotary rotation of one 64-wide row at token position `pos`:
// the pair (x[2c], x[2c+1]) turned back by pos * theta^(-2c/64).  The angle
// is reduced to a fraction of a turn in double precision (pos up to 2^24).
__device__ __forceinline__ void unrotate64(float (&x)[64], int pos, const double *g)
{
#pragma unroll
    for (int c = 0; c < 32; ++c) {
        const double turns = (double)pos * g[c];
        const float frac = (float)(turns - rint(turns));
        float sn, cs;
        __sincosf(6.283185307179586f * frac, &sn, &cs);
        const float a = x[2 * c], b = x[2 * c + 1];
        x[2 * c] = a * cs + b * sn;
        x[2 * c + 1] = b * cs - a * sn;
    }
}

// Copy this thread's row r of a [128 rows][64 columns] 16-bit tile in the
// 128-byte swizzle (16-byte chunk c of row r at c ^ (r % 8)) to 32 TMEM
// columns of its lane: column i holds elements 2i, 2i + 1, the layout of an
// A operand read from TMEM.
__device__ __forceinline__ void tile_row_to_tmem(uint32_t tile, int r, uint32_t taddr)
{
    uint32_t w[32];
    const uint32_t row = tile + 128u * r;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 v = ld_shared_v4(row + (((c ^ (r & 7)) & 7) << 4));
        w[4 * c] = v.x;
        w[4 * c + 1] = v.y;
        w[4 * c + 2] = v.z;
        w[4 * c + 3] = v.w;
    }
    tmem_st32(taddr, w);
}

// Write one row of `cols` values (scaled by s) to a bf16 row (16-byte
// aligned), or add it to an fp32 row of sums with vector atomics.
template <int COLS>
__device__ __forceinline__ void put_row(const float *x, float s, __nv_bfloat16 *dst, float *acc)
{
    if (acc) {
#pragma unroll
        for (int i = 0; i < COLS; i += 4)
            asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(acc + i), "f"(x[i] * s),
                         "f"(x[i + 1] * s), "f"(x[i + 2] * s), "f"(x[i + 3] * s)
                         : "memory");
        return;
    }
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int i = 0; i < COLS / 8; ++i)
        d4[i] = make_uint4(pack_bf162(x[8 * i] * s, x[8 * i + 1] * s), pack_bf162(x[8 * i + 2] * s, x[8 * i + 3] * s),
                           pack_bf162(x[8 * i + 4] * s, x[8 * i + 5] * s), pack_bf162(x[8 * i + 6] * s, x[8 * i + 7] * s));
}

// Load 64 fp32 TMEM columns of this warp's lanes into x.
__device__ __forceinline__ void tmem_row64(uint32_t taddr, float (&x)[64])
{
    uint32_t v[2][32];
    tmem_ld32(taddr, v[0]);
    tmem_ld32(taddr + 32, v[1]);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        x[i] = __uint_as_float(v[0][i]);
        x[32 + i] = __uint_as_float(v[1][i]);
    }
}

// ---------------------------------------------------------------- 1. row preparation
// Four threads per row (thread q of a row takes columns [32 q, 32 q + 32):
// 8 chunks of 4 fp32 of A_1 and of A_2, 32 of dY), 16 rows per CTA: a
// quarter row of A_1, A_2 fits in registers, so both passes (the norm's
// sums, then dD) read the saved state once; the row sums combine the four
// quarters with two shuffles.  In a warp, 8 rows x 4 quarters: each load
// instruction reads 8 consecutive rows of 4 chunks of the chunk-major
// state, four full 128-byte lines.  Small CTAs (eight per SM) keep loads
// of some in flight while others reduce.  Dynamic shared memory [16][129] fp32
// holds the per-row dgain terms when dgain is requested (and the norm
// applied), summed per column.
constexpr int PREP_THREADS = 64, PREP_ROWS = PREP_THREADS / 4;
constexpr int PREP_RED_BYTES = PREP_ROWS * (HDV + 1) * 4;
__global__ void __launch_bounds__(PREP_THREADS, 8)
    bwd_prep_kernel(const BwdParams p)
{
    extern __shared__ float red[];
    __shared__ float warp_sum[PREP_THREADS / 32];
    const int part = blockIdx.x % (BT / PREP_ROWS), t = blockIdx.x / (BT / PREP_ROWS);
    const int qt = t % p.num_qt, h = (t / p.num_qt) % p.H, b = t / (p.num_qt * p.H);
    const int q = threadIdx.x & 3, rr = threadIdx.x >> 2;  // column quarter, row of the CTA
    const int r = PREP_ROWS * part + rr, row = qt * BT + r;   // row of the tile, of the sequence
    const bool valid = row < p.N;
    const int rowc = valid ? row : 0;
    const float *tile = p.save + ((size_t)(b * p.H + h) * p.num_qt + qt) * kSaveTileFloats;
    const float4 *a1p = reinterpret_cast<const float4 *>(tile) + r;   // chunk c at c * 128
    const float4 *a2p = a1p + 32 * BT;
    const float ll = p.lam_logits ? p.lam_logits[b * p.ll_sb + (int64_t)rowc * p.ll_sn + h * p.ll_sh] : 0.0f;
    const float lam = p.lam_logits ? logistic_fast(ll) : p.lambda[h];
    const float4 *g4p = p.gain ? reinterpret_cast<const float4 *>(p.gain + (size_t)h * HDV) : nullptr;
    const __nv_bfloat16 *dy = static_cast<const __nv_bfloat16 *>(p.dout) + (size_t)b * p.do_sb +
                              (size_t)rowc * p.do_sn + (size_t)h * p.do_sh + 32 * q;
    const __nv_bfloat16 *gl = p.gate ? static_cast<const __nv_bfloat16 *>(p.gate) + (size_t)b * p.gate_sb +
                                           (size_t)rowc * p.gate_sn + (size_t)h * p.gate_sh + 32 * q
                                     : nullptr;
    const bool want_dgain = p.apply_norm && p.dgain;

    // This thread's quarter row: A_1, A_2 (8 chunks each) and dY, the gate
    // logits (bf16, packed), all loaded at once.
    float4 a1[8], a2[8];
    uint4 dyu[4], glu[4];
#pragma unroll
    for (int k = 0; k < 8; ++k) a1[k] = a2[k] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 4; ++k) dyu[k] = glu[k] = make_uint4(0u, 0u, 0u, 0u);
    if (valid) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            a1[k] = a1p[(8 * q + k) * BT];
            a2[k] = a2p[(8 * q + k) * BT];
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) dyu[k] = *reinterpret_cast<const uint4 *>(dy + 8 * k);
        if (gl) {
#pragma unroll
            for (int k = 0; k < 4; ++k) glu[k] = *reinterpret_cast<const uint4 *>(gl + 8 * k);
        }
    }
    // Column i (of the quarter) of a packed bf16 quarter row.
    auto col = [](const uint4 (&u)[4], int i) {
        const uint4 x = u[i >> 3];
        const int e = (i >> 1) & 3;
        const uint32_t w = e == 0 ? x.x : e == 1 ? x.y : e == 2 ? x.z : x.w;
        return __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
    };
    // dYn = dY sigma(G) of column i (the gate is the forward's last step), and sigma(G)
    auto dyn = [&](int i, float &sgv) {
        sgv = gl ? logistic_fast(col(glu, i)) : 1.0f;
        return col(dyu, i) * sgv;
    };
    auto gain4 = [&](int c) { return g4p ? __ldg(g4p + c) : make_float4(1.f, 1.f, 1.f, 1.f); };
    // the row's sum of the four quarters' values (lanes 4 i .. 4 i + 3 of a warp)
    auto row_sum = [](float x) {
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        return x + __shfl_xor_sync(0xffffffffu, x, 2);
    };

    // Pass 1: sum of squares of D and sum_c dYn gain D.
    float ss = 0.f, tg = 0.f;
    if (p.apply_norm) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float4 g = gain4(8 * q + k);
            const float av1[4] = {a1[k].x, a1[k].y, a1[k].z, a1[k].w}, av2[4] = {a2[k].x, a2[k].y, a2[k].z, a2[k].w};
            const float gg[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float d = fmaf(-lam, av2[e], av1[e]);
                float sgv;
                const float yv = dyn(4 * k + e, sgv);
                ss = fmaf(d, d, ss);
                tg = fmaf(gg[e] * yv, d, tg);
            }
        }
        ss = row_sum(ss);
        tg = row_sum(tg);
    }
    const float rn = p.apply_norm ? 1.0f / sqrtf(ss * (1.0f / HDV) + p.eps) : 1.0f;
    const float coef = rn * rn * rn * (1.0f / HDV) * tg;

    // Pass 2: dD, Delta_1 = dD . A_1, Delta_2 = -lambda dD . A_2, dlambda =
    // -dD . A_2, the dgain terms, dG.  The Deltas take dD as rounded to
    // fp16, the operand the tile kernels' dP = dD V^T products see: then
    // dS = P (dP - Delta) sums to zero over a row to fp32 rounding, and a
    // row whose softmax is constant (one visible key) gets dS = 0 (exact
    // in the gradient).  dlambda takes dD itself.
    float delta1 = 0.f, dot2 = 0.f, dot2h = 0.f;
    bool bad = false;
    uint32_t ddw[16], dgw[16];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const float4 g = gain4(8 * q + k);
        const float av1[4] = {a1[k].x, a1[k].y, a1[k].z, a1[k].w}, av2[4] = {a2[k].x, a2[k].y, a2[k].z, a2[k].w};
        const float gg[4] = {g.x, g.y, g.z, g.w};
        float dd[4], dgv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int i = 4 * k + e;
            const float d = fmaf(-lam, av2[e], av1[e]);
            float sgv;
            const float yv = dyn(i, sgv);
            dd[e] = p.apply_norm ? fmaf(rn * gg[e], yv, -coef * d) : yv;
            const float ddh = __half2float(__float2half_rn(dd[e]));
            delta1 = fmaf(ddh, av1[e], delta1);
            dot2h = fmaf(ddh, av2[e], dot2h);
            dot2 = fmaf(dd[e], av2[e], dot2);
            if (want_dgain) red[rr * (HDV + 1) + 32 * q + i] = yv * d * rn;
            bad |= !(fabsf(dd[e]) <= 65504.0f);
            // dG = dY Yn sigma'(G) = dYn Yn (1 - sigma(G)), Yn = D r gain (or D)
            const float yn = p.apply_norm ? d * rn * gg[e] : d;
            dgv[e] = yv * yn * (1.0f - sgv);
        }
        ddw[2 * k] = pack_half2(dd[0], dd[1]);
        ddw[2 * k + 1] = pack_half2(dd[2], dd[3]);
        dgw[2 * k] = pack_bf162(dgv[0], dgv[1]);
        dgw[2 * k + 1] = pack_bf162(dgv[2], dgv[3]);
    }
    delta1 = row_sum(delta1);
    dot2h = row_sum(dot2h);
    dot2 = row_sum(dot2);
    if (valid) {
        uint4 *ddrow = reinterpret_cast<uint4 *>(static_cast<__half *>(p.dd) +
                                                 (((size_t)b * p.N + row) * p.H + h) * HDV + 32 * q);
#pragma unroll
        for (int k = 0; k < 4; ++k) ddrow[k] = make_uint4(ddw[4 * k], ddw[4 * k + 1], ddw[4 * k + 2], ddw[4 * k + 3]);
        if (p.dgate) {
            uint4 *dgrow = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.dgate) + (size_t)b * p.dg_sb +
                                                     (size_t)row * p.dg_sn + (size_t)h * p.dg_sh + 32 * q);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                dgrow[k] = make_uint4(dgw[4 * k], dgw[4 * k + 1], dgw[4 * k + 2], dgw[4 * k + 3]);
        }
    }
    if (bad) report_error(p.dev_status, DIFFATTN_ERR_UNSUPPORTED);

    // Row statistics, negated (-lse_1, -lse_2, -Delta_1, -Delta_2, -lambda:
    // the tile kernels add them in packed fused multiply-adds); rows past N
    // get zeros (the tile kernels' products see zero operands there).
    if (q == 0) {
        float *st = p.stats + (size_t)(b * p.H + h) * kBwdStats * p.n_pad + qt * BT + r;
        const float *lse = tile + 2 * BT * HDV;
        st[0] = valid ? -lse[r] : 0.f;
        st[p.n_pad] = valid ? -lse[BT + r] : 0.f;
        st[2 * p.n_pad] = -delta1;
        st[3 * p.n_pad] = lam * dot2h;
        st[4 * p.n_pad] = valid ? -lam : 0.f;
    }

    // dlambda_i = -dD . A_2: per token through sigma' with lambda logits,
    // else summed over the CTA's rows into the head's dlambda.
    if (p.lam_logits) {
        if (p.dlam_logits && valid && q == 0)
            p.dlam_logits[b * p.dll_sb + (int64_t)row * p.dll_sn + h * p.dll_sh] = -dot2 * lam * (1.0f - lam);
    } else if (p.dlambda) {
        float v = q == 0 ? -dot2 : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = v;
    }
    __syncthreads();
    if (!p.lam_logits && p.dlambda && threadIdx.x == 0) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < PREP_THREADS / 32; ++w) v += warp_sum[w];
        atomicAdd(p.dlambda + h, v);
    }
    // dgain[h][c] += the CTA's column sums (rows past N hold zeros).
    if (want_dgain) {
        for (int c = threadIdx.x; c < HDV; c += PREP_THREADS) {
            float v = 0.f;
#pragma unroll 8
            for (int i = 0; i < PREP_ROWS; ++i) v += red[i * (HDV + 1) + c];
            atomicAdd(p.dgain + (size_t)h * HDV + c, v);
        }
    }
}

// Roles shared by both tile kernels.
struct Roles {
    int warp, lane;
    __device__ __forceinline__ bool producer() const { return warp == 0; }
    __device__ __forceinline__ bool score_issuer() const { return warp == 1; }
    __device__ __forceinline__ bool acc_issuer() const { return warp == 2; }
    // element-wise warpgroup (0 or 1) and the TMEM lane / tile row of this
    // thread (warps 3-6 and 7-10: each group covers the four lane quarters)
    __device__ __forceinline__ int wg() const { return (warp - 3) >> 2; }
    __device__ __forceinline__ int row() const { return (warp & 3) * 32 + lane; }
    __device__ __forceinline__ uint32_t lane_off() const { return uint32_t((warp & 3) * 32) << 16; }
};

// Both tile kernels run two MMA issuers, one warp each, so that neither
// kind of product waits behind the other in one warp's program order: the
// score issuer (a block's score and dP products, once its stage has landed
// and the element-wise warps have taken the previous block's products out
// of TMEM, early in their step) and the accumulating issuer (a block's
// accumulating products, once the element-wise warps have written their A
// operands, at the end of their step).  A block's score products are
// complete before its accumulating products are issued (the element-wise
// warps waited for them), so the accumulating issuer's commit after a
// tile's last block covers every product of the tile.  Every wait is
// bounded; each issuer drains what it issued before the CTA tears down.

// ---------------------------------------------------------------- 2. key tiles
// A persistent kernel: one CTA per SM takes key tiles, heaviest first (under
// the causal mask key tile 0 meets every query), from a counter in the
// workspace (zeroed by the staging kernel); the producer publishes each to
// the other roles in a 4-slot ring.  The next tile's operands load, and its K rows go into TMEM,
// while the element-wise warps write out the finished tile's dV and dK; its
// first block's score products run during that epilogue.  Per tile:
//   producer: TILEFREE (previous tile) -> the tile's K_1, K_2, V -> its blocks;
//   score issuer: AOP (tile) -> the blocks' score and dP products -> TILEFREE;
//   accumulating issuer: per block AFULL (block 0 also ACCFREE, previous
//     tile) -> dV, dK_1, dK_2 products -> DONE (tile) after the last block;
//   element-wise warps: TILE -> K rows into TMEM, AOP -> the previous tile's
//     epilogue (DONE, TMEM reads, stores), ACCFREE -> the tile's blocks.
// Block barriers count blocks over the CTA's whole sequence (G below).
template <bool F16QK>
__global__ void __launch_bounds__(NT, 1)
    bwd_key_kernel(const __grid_constant__ BwdKeyMaps m, const BwdParams p)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_addr(smem);
    const Roles R{(int)(threadIdx.x >> 5), (int)(threadIdx.x & 31)};
    if (sbase & 1023u) {  // the 128-byte-swizzled tiles need 1 KB alignment
        if (threadIdx.x == 0) report_error(p.dev_status, DIFFATTN_ERR_UNSUPPORTED);
        return;
    }
    const int BH = p.B * p.H, n_tiles = p.num_qt * BH;
    const int nqb_all = (p.N + BB - 1) / BB;
    struct Tile {
        int b, h, hn, hv, k0, qb0, nit;
    };
    auto tile_of = [&](int t) {
        Tile T;
        const int kt = t / BH, bh = t % BH;
        T.b = bh / p.H;
        T.h = bh % p.H;
        T.hn = T.h / (p.H / p.H_N);
        T.hv = T.h / (p.H / p.H_V);
        T.k0 = kt * BT;
        // Query blocks that see a key of the tile: causal from the block
        // holding k0; under a window of W keys up to the one holding
        // k0 + 127 + W - 1.
        T.qb0 = p.causal ? T.k0 / BB : 0;
        const int qb1 = p.window > 0 ? min(nqb_all, (T.k0 + BT - 1 + p.window - 1) / BB + 1) : nqb_all;
        T.nit = qb1 - T.qb0;  // >= 1: k0 < N
        return T;
    };
    auto bar = [&](int i) { return sbase + KT_BARS + 8 * i; };
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(smem + KT_BARS + 8 * NBARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + KT_BARS + 8 * NBARS + 4);
    int *sItem = reinterpret_cast<int *>(smem + KT_BARS + 8 * NBARS + 16);
    const uint64_t lim = p.timeout_ns;
    // Tile k of this CTA from ring slot k % 4; -1 ends the loop (also when
    // a bounded wait gives up).
    auto read_tile = [&](int k) -> int {
        const int slot = k & 3;
        if (!mbar_wait_warp(bar(B_ITEM + slot), (k >> 2) & 1, abort_flag, lim)) return -1;
        const int t = *reinterpret_cast<volatile int *>(&sItem[slot]);
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(bar(B_ITEMFREE + slot));
        return t;
    };

    if (threadIdx.x == 0) {
        mbar_init(bar(B_TILE), 1);
        for (int i = 0; i < 4; ++i) {
            mbar_init(bar(B_ITEM + i), 1);
            mbar_init(bar(B_ITEMFREE + i), 2 + NEW);  // the two issuers and the element-wise warps
        }
        for (int s = 0; s < MAXSTAGES; ++s) {
            mbar_init(bar(B_FULL + s), 1);
            mbar_init(bar(B_EMPTY + s), 1);
        }
        mbar_init(bar(B_SFULL), 1);
        mbar_init(bar(B_SFREE), NEW);
        mbar_init(bar(B_AFULL), NEW);
        mbar_init(bar(B_AFREE), 1);
        mbar_init(bar(B_DONE), 1);
        mbar_init(bar(B_SDRAIN), 1);
        mbar_init(bar(B_AOP), NEW);
        mbar_init(bar(B_TILEFREE), 1);
        mbar_init(bar(B_ACCFREE), NEW);
        mbar_init(bar(B_ADRAIN), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (R.warp == 0) {
        tmem_alloc(smem_addr(tmem_ptr), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_ptr;

    if (R.producer()) {
        // ------------------------------------------------------------ TMA producer
        int G = 0, ti = 0, tile_loads = 0;
        bool ok = true;
        for (;; ++ti) {
            const int slot = ti & 3;
            if (ti >= 4 && !(ok = mbar_wait_warp(bar(B_ITEMFREE + slot), ((ti >> 2) - 1) & 1, abort_flag, lim)))
                break;
            int t = 0;
            if (R.lane == 0) {
                t = *abort_flag ? n_tiles : atomicAdd(p.tile_counter, 1);
                sItem[slot] = t < n_tiles ? t : -1;
                mbar_arrive(bar(B_ITEM + slot));
            }
            t = __shfl_sync(0xffffffffu, t, 0);
            if (t >= n_tiles) break;
            const Tile T = tile_of(t);
            // The previous tile's score products must be done with its K
            // (in TMEM) and V.
            if (ti > 0 && !(ok = mbar_wait_warp(bar(B_TILEFREE), (ti - 1) & 1, abort_flag, lim))) break;
            if (elect_one()) {
                mbar_arrive_expect_tx(bar(B_TILE), KT_STAGE0);
                tma_load_4d_nohint(sbase + KT_K1, &m.k1, bar(B_TILE), 0, T.k0, T.h, T.b);
                tma_load_4d_nohint(sbase + KT_K2, &m.k2, bar(B_TILE), 0, T.k0, T.hn, T.b);
                tma_load_4d_nohint(sbase + KT_V, &m.v, bar(B_TILE), 0, T.k0, T.hv, T.b);
                tma_load_4d_nohint(sbase + KT_V + 16384, &m.v, bar(B_TILE), 64, T.k0, T.hv, T.b);
            }
            __syncwarp();
            ++tile_loads;
            for (int j = 0; j < T.nit; ++j) {
                const int s = G % KSTAGES;
                if (G >= KSTAGES &&
                    !(ok = mbar_wait_warp(bar(B_EMPTY + s), ((G / KSTAGES) - 1) & 1, abort_flag, lim)))
                    break;
                if (elect_one()) {
                    const uint32_t st = sbase + KT_STAGE0 + s * KB_BYTES, fb = bar(B_FULL + s);
                    const int q0 = (T.qb0 + j) * BB;
                    mbar_arrive_expect_tx(fb, KB_LOAD);
                    tma_load_4d_nohint(st + KB_Q1, &m.q1, fb, 0, q0, T.h, T.b);
                    tma_load_4d_nohint(st + KB_Q2, &m.q2, fb, 0, q0, T.hn, T.b);
                    tma_load_4d_nohint(st + KB_DD, &m.dd, fb, 0, q0, T.h, T.b);
                    tma_load_4d_nohint(st + KB_DD + 8192, &m.dd, fb, 64, q0, T.h, T.b);
                    tma_load_4d_nohint(st + KB_ST, &m.stats, fb, q0, 0, T.h, T.b);
                }
                __syncwarp();
                ++G;
            }
            if (!ok) break;
        }
        // No load of ours may land after the CTA has gone.
        bool drained = true;
        if (tile_loads > 0) drained = mbar_wait_drain(bar(B_TILE), (tile_loads - 1) & 1, lim);
        for (int k = (G > KSTAGES ? G - KSTAGES : 0); k < G; ++k)
            drained &= mbar_wait_drain(bar(B_FULL + k % KSTAGES), (k / KSTAGES) & 1, lim);
        if (!__all_sync(0xffffffffu, drained) && R.lane == 0) *abort_flag = 1;
    } else if (R.score_issuer() || R.acc_issuer()) {
        // ------------------------------------------------------------ MMA issuers
        // Warp 1 issues the score and dP products, warp 2 the accumulating
        // products; neither waits behind the other in one program order.
        auto issue_s = [&](int G) {
            const uint32_t st = sbase + KT_STAGE0 + (G % KSTAGES) * KB_BYTES;
#pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk)
                mma_issue_ts(tbase + KM_S1, tbase + KM_AK1 + 8 * kk, sw128(st + KB_Q1 + 32 * kk), Ids<F16QK>::S,
                             kk > 0);
#pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk)
                mma_issue_ts(tbase + KM_S2, tbase + KM_AK2 + 8 * kk, sw128(st + KB_Q2 + 32 * kk), Ids<F16QK>::S,
                             kk > 0);
#pragma unroll
            for (int kk = 0; kk < HDV / 16; ++kk) {
                const uint32_t o = 32 * (kk & 3);
                mma_issue(tbase + KM_DP, sw128(sbase + KT_V + (kk >> 2) * 16384 + o),
                          sw128(st + KB_DD + (kk >> 2) * 8192 + o), ID_DP, kk > 0);
            }
            commit_to(bar(B_SFULL));
        };
        auto issue_acc = [&](int G, bool first) {
            const uint32_t st = sbase + KT_STAGE0 + (G % KSTAGES) * KB_BYTES;
            // dV += (P_1 - lambda P_2)^T dD; dK_t += dS_t^T Q_t (B MN-major).
#pragma unroll
            for (int kk = 0; kk < BB / 16; ++kk)
                mma_issue(tbase + KM_DV, sw128(sbase + KT_A + KA_PV + 32 * kk), sw128(st + KB_DD + 2048 * kk, 8192),
                          ID_DV, !first || kk > 0);
#pragma unroll
            for (int kk = 0; kk < BB / 16; ++kk)
                mma_issue(tbase + KM_DK1, sw128(sbase + KT_A + KA_DS1 + 32 * kk), sw128(st + KB_Q1 + 2048 * kk, 8192),
                          Ids<F16QK>::DS, !first || kk > 0);
#pragma unroll
            for (int kk = 0; kk < BB / 16; ++kk)
                mma_issue(tbase + KM_DK2, sw128(sbase + KT_A + KA_DS2 + 32 * kk), sw128(st + KB_Q2 + 2048 * kk, 8192),
                          Ids<F16QK>::DS, !first || kk > 0);
            commit_to(bar(B_AFREE));
            commit_to(bar(B_EMPTY + G % KSTAGES));
        };
        int G = 0, ti = 0;
        bool ok = true;
        if (R.score_issuer()) {
            for (;; ++ti) {
                const int t = read_tile(ti);
                if (t < 0) break;
                const Tile T = tile_of(t);
                // the tile's K rows are in TMEM (the A operand of its score products)
                if (!(ok = mbar_wait_warp(bar(B_AOP), ti & 1, abort_flag, lim))) break;
                for (int j = 0; ok && j < T.nit; ++j, ++G) {
                    if (!(ok = mbar_wait_warp(bar(B_FULL + G % KSTAGES), (G / KSTAGES) & 1, abort_flag, lim))) break;
                    if (G > 0 && !(ok = mbar_wait_warp(bar(B_SFREE), (G - 1) & 1, abort_flag, lim))) break;
                    tc_fence_after();
                    issue_s(G);
                }
                if (!ok) break;
                commit_to(bar(B_TILEFREE));  // the tile's K (TMEM) and V may be replaced once these are done
            }
            // Nothing of ours may still run on the tensor cores at teardown.
            commit_to(bar(B_SDRAIN));
            if (!__all_sync(0xffffffffu, mbar_wait_drain(bar(B_SDRAIN), 0, lim)) && R.lane == 0) *abort_flag = 1;
        } else {
            for (;; ++ti) {
                const int t = read_tile(ti);
                if (t < 0) break;
                const Tile T = tile_of(t);
                for (int j = 0; ok && j < T.nit; ++j, ++G) {
                    if (!(ok = mbar_wait_warp(bar(B_AFULL), G & 1, abort_flag, lim))) break;
                    // The tile's first products overwrite the accumulators:
                    // the previous tile's epilogue must have read them.
                    if (j == 0 && ti > 0 && !(ok = mbar_wait_warp(bar(B_ACCFREE), (ti - 1) & 1, abort_flag, lim)))
                        break;
                    tc_fence_after();
                    issue_acc(G, j == 0);
                }
                if (!ok) break;
                // DONE completes once every product of the tile has (its
                // score products completed before its last accumulating
                // products were issued): the epilogue's signal.
                commit_to(bar(B_DONE));
            }
            // Nothing of ours may still run on the tensor cores at teardown.
            commit_to(bar(B_ADRAIN));
            if (!__all_sync(0xffffffffu, mbar_wait_drain(bar(B_ADRAIN), 0, lim)) && R.lane == 0) *abort_flag = 1;
        }
    } else {
        // ------------------------------------------------------------ element-wise + epilogue
        const int wg = R.wg(), r = R.row();
        const uint32_t lo = R.lane_off();
        const float c = p.scale_log2;
        bool ok = true, big = false;
        // The finished tile's dV and dK from TMEM to global memory (after
        // its last products): warpgroup 0 writes dV columns [0, 64) and
        // dK_1, warpgroup 1 dV columns [64, 128) and dK_2; then the
        // accumulators are released to the next tile's products.
        auto epilogue = [&](const Tile &T, int ti) -> bool {
            if (!mbar_wait_warp(bar(B_DONE), ti & 1, abort_flag, lim)) return false;
            const int b = T.b, h = T.h, hn = T.hn, hv = T.hv, kj = T.k0 + r;
            // Warpgroup 0 writes dV columns [0, 64) and dK_1; warpgroup 1 dV
            // columns [64, 128) and dK_2.  Every lane takes part in the TMEM
            // loads (warp-collective); only rows of keys below N are stored.
            tc_fence_after();
            const bool own = kj < p.N;
            const int krow = own ? kj : 0;
            float x[64];
            tmem_row64(tbase + lo + KM_DV + 64 * wg, x);
            if (own) {
                __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.dv) + (size_t)b * p.dv_s[0] +
                                     (size_t)krow * p.dv_s[1] + (size_t)hv * p.dv_s[2] + 64 * wg;
                float *acc = p.acc_dv ? p.acc_dv + (((size_t)b * p.N + krow) * p.H_V + hv) * HDV + 64 * wg : nullptr;
                put_row<64>(x, 1.0f, dst, acc);
            }
            tmem_row64(tbase + lo + (wg ? KM_DK2 : KM_DK1), x);
            if (own) {
                if (F16QK) unrotate64(x, krow, p.rope_g);
                if (wg == 0) {
                    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.dk1) + (size_t)b * p.dk1_s[0] +
                                         (size_t)krow * p.dk1_s[1] + (size_t)h * p.dk1_s[2];
                    put_row<64>(x, p.scale, dst, nullptr);
                } else {
                    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.dk2) + (size_t)b * p.dk2_s[0] +
                                         (size_t)krow * p.dk2_s[1] + (size_t)hn * p.dk2_s[2];
                    float *acc = p.acc_dk2 ? p.acc_dk2 + (((size_t)b * p.N + krow) * p.H_N + hn) * HD : nullptr;
                    put_row<64>(x, p.scale, dst, acc);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (R.lane == 0) mbar_arrive(bar(B_ACCFREE));
            return true;
        };
        int G = 0, ti = 0;
        Tile prev{};
        for (;; ++ti) {
            const int t = read_tile(ti);
            if (t < 0) break;
            const Tile T = tile_of(t);
            const int kj = T.k0 + r;  // this thread's key
            // The tile's K_1 (warpgroup 0) and K_2 (warpgroup 1) rows into
            // TMEM, the A operand of every block's score products (the
            // producer loaded them once the previous tile's score products
            // were done with the old ones).
            if (!(ok = mbar_wait_warp(bar(B_TILE), ti & 1, abort_flag, lim))) break;
            tile_row_to_tmem(sbase + (wg ? KT_K2 : KT_K1), r, tbase + lo + (wg ? KM_AK2 : KM_AK1));
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (R.lane == 0) mbar_arrive(bar(B_AOP));
            // The previous tile's epilogue, while this tile's first score
            // products run.
            if (ti > 0 && !(ok = epilogue(prev, ti - 1))) break;
            for (int j = 0; ok && j < T.nit; ++j, ++G) {
                if (!(ok = mbar_wait_warp(bar(B_SFULL), G & 1, abort_flag, lim))) break;
                tc_fence_after();
                uint32_t s1[32], s2[32], dp[32];
                tmem_ld32(tbase + lo + KM_S1 + 32 * wg, s1);
                tmem_ld32(tbase + lo + KM_S2 + 32 * wg, s2);
                tmem_ld32(tbase + lo + KM_DP + 32 * wg, dp);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (R.lane == 0) mbar_arrive(bar(B_SFREE));
                // This warpgroup's 32 queries of the block, and their statistics.
                const int qb = (T.qb0 + j) * BB + 32 * wg;
                const uint32_t st = sbase + KT_STAGE0 + (G % KSTAGES) * KB_BYTES + KB_ST + 4 * 32 * wg;
                const bool mask = (p.causal && qb < T.k0 + BT - 1) || (p.window > 0 && qb + 31 - T.k0 >= p.window);
                uint32_t pv[16], d1p[16], d2p[16];
                const float2 c2 = make_float2(c, c);
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    // the four queries' statistics, negated: -lse_1, -lse_2,
                    // -Delta_1, -Delta_2, -lambda
                    const uint4 ul1 = ld_shared_v4(st + 4 * i), ul2 = ld_shared_v4(st + 256 + 4 * i);
                    const uint4 ud1 = ld_shared_v4(st + 512 + 4 * i), ud2 = ld_shared_v4(st + 768 + 4 * i);
                    const uint4 ulm = ld_shared_v4(st + 1024 + 4 * i);
                    const uint32_t l1[4] = {ul1.x, ul1.y, ul1.z, ul1.w}, l2[4] = {ul2.x, ul2.y, ul2.z, ul2.w};
                    const uint32_t D1[4] = {ud1.x, ud1.y, ud1.z, ud1.w}, D2[4] = {ud2.x, ud2.y, ud2.z, ud2.w};
                    const uint32_t LM[4] = {ulm.x, ulm.y, ulm.z, ulm.w};
#pragma unroll
                    for (int e = 0; e < 4; e += 2) {  // two queries at a time, in packed arithmetic
                        auto f2 = [](const uint32_t *a, int k) { return make_float2(__uint_as_float(a[k]), __uint_as_float(a[k + 1])); };
                        const float2 x1 = ffma2(f2(s1, i + e), c2, f2(l1, e));
                        const float2 x2 = ffma2(f2(s2, i + e), c2, f2(l2, e));
                        float2 p1, p2;
                        if ((BWD_SOFT_EXP_MASK >> (((i + e) >> 1) & 7)) & 1u) {
                            p1 = exp2_soft2(x1);
                            p2 = exp2_soft2(x2);
                        } else {
                            p1 = make_float2(ex2_approx(x1.x), ex2_approx(x1.y));
                            p2 = make_float2(ex2_approx(x2.x), ex2_approx(x2.y));
                        }
                        if (mask) {
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const int q = qb + i + e + u;
                                const bool vis = (!p.causal || q >= kj) && (p.window <= 0 || q - kj < p.window);
                                if (!vis) {
                                    if (u) p1.y = p2.y = 0.f;
                                    else p1.x = p2.x = 0.f;
                                }
                            }
                        }
                        const float2 g = f2(dp, i + e), nlam = f2(LM, e);
                        const float2 vp = ffma2(nlam, p2, p1);                     // P_1 - lambda P_2
                        const float2 v1 = fmul2(p1, fadd2(g, f2(D1, e)));          // P_1 (dP - Delta_1)
                        const float2 v2 = fmul2(p2, ffma2(nlam, g, f2(D2, e)));    // P_2 (-lambda dP - Delta_2)
                        if (F16QK)
                            big |= !(fabsf(v1.x) <= 65504.0f && fabsf(v1.y) <= 65504.0f && fabsf(v2.x) <= 65504.0f &&
                                     fabsf(v2.y) <= 65504.0f);
                        pv[(i + e) / 2] = pack_half2(vp.x, vp.y);
                        d1p[(i + e) / 2] = pack_ds(v1.x, v1.y, F16QK);
                        d2p[(i + e) / 2] = pack_ds(v2.x, v2.y, F16QK);
                    }
                    // Keep the next four queries' statistics loads below this
                    // point: hoisted all at once they would need 160 registers.
                    asm volatile("" ::: "memory");
                }
                // The previous block's accumulating products (of this tile or the
                // one before) must have read the A operands before they are
                // overwritten.
                if (G > 0 && !(ok = mbar_wait_warp(bar(B_AFREE), (G - 1) & 1, abort_flag, lim))) break;
                st_operand_half(sbase + KT_A + KA_PV, r, wg, pv);
                st_operand_half(sbase + KT_A + KA_DS1, r, wg, d1p);
                st_operand_half(sbase + KT_A + KA_DS2, r, wg, d2p);
                fence_proxy_async_smem();
                __syncwarp();
                if (R.lane == 0) mbar_arrive(bar(B_AFULL));
            }
            if (!ok) break;
            prev = T;
        }
        if (ok && ti > 0) ok = epilogue(prev, ti - 1);
        if (big) report_error(p.dev_status, DIFFATTN_ERR_UNSUPPORTED);
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) report_error(p.dev_status, DIFFATTN_ERR_TIMEOUT);
    if (R.warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

// ---------------------------------------------------------------- 3. query tiles
// Persistent like the key-tile kernel: one CTA per SM takes query tiles,
// heaviest first (under the causal mask the last query tile meets every
// key), from the second workspace counter through a 4-slot ring.  The
// tile's Q_1, Q_2 and dD rows live in TMEM (the A operands of its score and
// dP products), so their shared-memory copy may be replaced once they are
// there.  Per tile:
//   producer: AOP (previous tile) -> the tile's Q_1, Q_2, dD -> its blocks;
//   score issuer: AOP (tile) -> the blocks' score and dP products;
//   accumulating issuer: per block AFULL (block 0 also ACCFREE, previous
//     tile) -> dQ_1, dQ_2 products -> DONE (tile) after the last block;
//   element-wise warps: TILE -> Q and dD rows into TMEM (the previous
//     tile's score products are complete: its last SFULL was seen), AOP ->
//     the previous tile's epilogue (DONE, TMEM reads, stores), ACCFREE ->
//     the tile's blocks.
template <bool F16QK>
__global__ void __launch_bounds__(NT, 1)
    bwd_query_kernel(const __grid_constant__ BwdQueryMaps m, const BwdParams p)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_addr(smem);
    const Roles R{(int)(threadIdx.x >> 5), (int)(threadIdx.x & 31)};
    if (sbase & 1023u) {
        if (threadIdx.x == 0) report_error(p.dev_status, DIFFATTN_ERR_UNSUPPORTED);
        return;
    }
    const int BH = p.B * p.H, n_tiles = p.num_qt * BH;
    const int nkb_all = (p.N + BB - 1) / BB;
    struct Tile {
        int b, h, hn, hv, q0, kb0, nit;
    };
    auto tile_of = [&](int t) {
        Tile T;
        const int qt = p.num_qt - 1 - t / BH, bh = t % BH;
        T.b = bh / p.H;
        T.h = bh % p.H;
        T.hn = T.h / (p.H / p.H_N);
        T.hv = T.h / (p.H / p.H_V);
        T.q0 = qt * BT;
        // Key blocks the tile's queries see: up to the diagonal when causal;
        // under a window of W keys from the block holding key q0 - W + 1.
        T.kb0 = p.window > 0 ? max(0, T.q0 - p.window + 1) / BB : 0;
        const int kb1 = p.causal ? min(nkb_all, (T.q0 + BT - 1) / BB + 1) : nkb_all;
        T.nit = kb1 - T.kb0;  // >= 1
        return T;
    };
    auto bar = [&](int i) { return sbase + QT_BARS + 8 * i; };
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(smem + QT_BARS + 8 * NBARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + QT_BARS + 8 * NBARS + 4);
    int *sItem = reinterpret_cast<int *>(smem + QT_BARS + 8 * NBARS + 16);
    const uint64_t lim = p.timeout_ns;
    auto read_tile = [&](int k) -> int {
        const int slot = k & 3;
        if (!mbar_wait_warp(bar(B_ITEM + slot), (k >> 2) & 1, abort_flag, lim)) return -1;
        const int t = *reinterpret_cast<volatile int *>(&sItem[slot]);
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(bar(B_ITEMFREE + slot));
        return t;
    };

    if (threadIdx.x == 0) {
        mbar_init(bar(B_TILE), 1);
        for (int i = 0; i < 4; ++i) {
            mbar_init(bar(B_ITEM + i), 1);
            mbar_init(bar(B_ITEMFREE + i), 2 + NEW);
        }
        for (int s = 0; s < MAXSTAGES; ++s) {
            mbar_init(bar(B_FULL + s), 1);
            mbar_init(bar(B_EMPTY + s), 1);
        }
        mbar_init(bar(B_SFULL), 1);
        mbar_init(bar(B_SFREE), NEW);
        mbar_init(bar(B_AFULL), NEW);
        mbar_init(bar(B_AFREE), 1);
        mbar_init(bar(B_DONE), 1);
        mbar_init(bar(B_SDRAIN), 1);
        mbar_init(bar(B_AOP), NEW);
        mbar_init(bar(B_ACCFREE), NEW);
        mbar_init(bar(B_ADRAIN), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (R.warp == 0) {
        tmem_alloc(smem_addr(tmem_ptr), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_ptr;

    if (R.producer()) {
        // ------------------------------------------------------------ TMA producer
        int G = 0, ti = 0, tile_loads = 0;
        bool ok = true;
        for (;; ++ti) {
            const int slot = ti & 3;
            if (ti >= 4 && !(ok = mbar_wait_warp(bar(B_ITEMFREE + slot), ((ti >> 2) - 1) & 1, abort_flag, lim)))
                break;
            int t = 0;
            if (R.lane == 0) {
                t = *abort_flag ? n_tiles : atomicAdd(p.tile_counter + 1, 1);
                sItem[slot] = t < n_tiles ? t : -1;
                mbar_arrive(bar(B_ITEM + slot));
            }
            t = __shfl_sync(0xffffffffu, t, 0);
            if (t >= n_tiles) break;
            const Tile T = tile_of(t);
            // The previous tile's rows must be in TMEM before its shared-memory
            // copy is replaced.
            if (ti > 0 && !(ok = mbar_wait_warp(bar(B_AOP), (ti - 1) & 1, abort_flag, lim))) break;
            if (elect_one()) {
                mbar_arrive_expect_tx(bar(B_TILE), QT_STAGE0);
                tma_load_4d_nohint(sbase + QT_Q1, &m.q1, bar(B_TILE), 0, T.q0, T.h, T.b);
                tma_load_4d_nohint(sbase + QT_Q2, &m.q2, bar(B_TILE), 0, T.q0, T.hn, T.b);
                tma_load_4d_nohint(sbase + QT_DD, &m.dd, bar(B_TILE), 0, T.q0, T.h, T.b);
                tma_load_4d_nohint(sbase + QT_DD + 16384, &m.dd, bar(B_TILE), 64, T.q0, T.h, T.b);
            }
            __syncwarp();
            ++tile_loads;
            for (int j = 0; j < T.nit; ++j) {
                const int s = G % QSTAGES;
                if (G >= QSTAGES &&
                    !(ok = mbar_wait_warp(bar(B_EMPTY + s), ((G / QSTAGES) - 1) & 1, abort_flag, lim)))
                    break;
                if (elect_one()) {
                    const uint32_t st = sbase + QT_STAGE0 + s * QB_BYTES, fb = bar(B_FULL + s);
                    const int k0 = (T.kb0 + j) * BB;
                    mbar_arrive_expect_tx(fb, QB_BYTES);
                    tma_load_4d_nohint(st + QB_K1, &m.k1, fb, 0, k0, T.h, T.b);
                    tma_load_4d_nohint(st + QB_K2, &m.k2, fb, 0, k0, T.hn, T.b);
                    tma_load_4d_nohint(st + QB_V, &m.v, fb, 0, k0, T.hv, T.b);
                    tma_load_4d_nohint(st + QB_V + 8192, &m.v, fb, 64, k0, T.hv, T.b);
                }
                __syncwarp();
                ++G;
            }
            if (!ok) break;
        }
        // No load of ours may land after the CTA has gone.
        bool drained = true;
        if (tile_loads > 0) drained = mbar_wait_drain(bar(B_TILE), (tile_loads - 1) & 1, lim);
        for (int k = (G > QSTAGES ? G - QSTAGES : 0); k < G; ++k)
            drained &= mbar_wait_drain(bar(B_FULL + k % QSTAGES), (k / QSTAGES) & 1, lim);
        if (!__all_sync(0xffffffffu, drained) && R.lane == 0) *abort_flag = 1;
    } else if (R.score_issuer() || R.acc_issuer()) {
        // ------------------------------------------------------------ MMA issuers
        auto issue_s = [&](int G) {
            const uint32_t st = sbase + QT_STAGE0 + (G % QSTAGES) * QB_BYTES;
#pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk)
                mma_issue_ts(tbase + QM_S1, tbase + QM_AQ1 + 8 * kk, sw128(st + QB_K1 + 32 * kk), Ids<F16QK>::S,
                             kk > 0);
#pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk)
                mma_issue_ts(tbase + QM_S2, tbase + QM_AQ2 + 8 * kk, sw128(st + QB_K2 + 32 * kk), Ids<F16QK>::S,
                             kk > 0);
#pragma unroll
            for (int kk = 0; kk < HDV / 16; ++kk) {
                const uint32_t o = 32 * (kk & 3);
                mma_issue_ts(tbase + QM_DP, tbase + QM_ADD + 8 * kk, sw128(st + QB_V + (kk >> 2) * 8192 + o), ID_DP,
                             kk > 0);
            }
            commit_to(bar(B_SFULL));
        };
        auto issue_acc = [&](int G, bool first) {
            const uint32_t st = sbase + QT_STAGE0 + (G % QSTAGES) * QB_BYTES;
            // dQ_t += dS_t K_t (A: dS_t in TMEM; B: the K block, MN-major).
#pragma unroll
            for (int kk = 0; kk < BB / 16; ++kk)
                mma_issue_ts(tbase + QM_DQ1, tbase + QM_ADS1 + 8 * kk, sw128(st + QB_K1 + 2048 * kk, 8192),
                             Ids<F16QK>::DS, !first || kk > 0);
#pragma unroll
            for (int kk = 0; kk < BB / 16; ++kk)
                mma_issue_ts(tbase + QM_DQ2, tbase + QM_ADS2 + 8 * kk, sw128(st + QB_K2 + 2048 * kk, 8192),
                             Ids<F16QK>::DS, !first || kk > 0);
            commit_to(bar(B_AFREE));
            commit_to(bar(B_EMPTY + G % QSTAGES));
        };
        int G = 0, ti = 0;
        bool ok = true;
        if (R.score_issuer()) {
            for (;; ++ti) {
                const int t = read_tile(ti);
                if (t < 0) break;
                const Tile T = tile_of(t);
                // the tile's Q and dD rows are in TMEM
                if (!(ok = mbar_wait_warp(bar(B_AOP), ti & 1, abort_flag, lim))) break;
                for (int j = 0; ok && j < T.nit; ++j, ++G) {
                    if (!(ok = mbar_wait_warp(bar(B_FULL + G % QSTAGES), (G / QSTAGES) & 1, abort_flag, lim))) break;
                    if (G > 0 && !(ok = mbar_wait_warp(bar(B_SFREE), (G - 1) & 1, abort_flag, lim))) break;
                    tc_fence_after();
                    issue_s(G);
                }
                if (!ok) break;
            }
            // Nothing of ours may still run on the tensor cores at teardown.
            commit_to(bar(B_SDRAIN));
            if (!__all_sync(0xffffffffu, mbar_wait_drain(bar(B_SDRAIN), 0, lim)) && R.lane == 0) *abort_flag = 1;
        } else {
            for (;; ++ti) {
                const int t = read_tile(ti);
                if (t < 0) break;
                const Tile T = tile_of(t);
                for (int j = 0; ok && j < T.nit; ++j, ++G) {
                    if (!(ok = mbar_wait_warp(bar(B_AFULL), G & 1, abort_flag, lim))) break;
                    // The tile's first products overwrite the accumulators:
                    // the previous tile's epilogue must have read them.
                    if (j == 0 && ti > 0 && !(ok = mbar_wait_warp(bar(B_ACCFREE), (ti - 1) & 1, abort_flag, lim)))
                        break;
                    tc_fence_after();
                    issue_acc(G, j == 0);
                }
                if (!ok) break;
                // DONE completes once every product of the tile has: the
                // epilogue's signal.
                commit_to(bar(B_DONE));
            }
            // Nothing of ours may still run on the tensor cores at teardown.
            commit_to(bar(B_ADRAIN));
            if (!__all_sync(0xffffffffu, mbar_wait_drain(bar(B_ADRAIN), 0, lim)) && R.lane == 0) *abort_flag = 1;
        }
    } else {
        // ------------------------------------------------------------ element-wise + epilogue
        const int wg = R.wg(), r = R.row();
        const uint32_t lo = R.lane_off();
        const float c = p.scale_log2;
        bool ok = true, big = false;
        // The finished tile's dQ from TMEM to global memory (after its last
        // products): warpgroup 0 writes dQ_1, warpgroup 1 dQ_2, rows below N
        // only; then the accumulators are released to the next tile.
        auto epilogue = [&](const Tile &T, int ti) -> bool {
            if (!mbar_wait_warp(bar(B_DONE), ti & 1, abort_flag, lim)) return false;
            tc_fence_after();
            const int qrow = T.q0 + r;
            const bool own = qrow < p.N;
            const int qr = own ? qrow : 0;
            float x[64];
            tmem_row64(tbase + lo + (wg ? QM_DQ2 : QM_DQ1), x);
            if (own) {
                if (F16QK) unrotate64(x, qr, p.rope_g);
                if (wg == 0) {
                    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.dq1) + (size_t)T.b * p.dq1_s[0] +
                                         (size_t)qr * p.dq1_s[1] + (size_t)T.h * p.dq1_s[2];
                    put_row<64>(x, p.scale, dst, nullptr);
                } else {
                    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.dq2) + (size_t)T.b * p.dq2_s[0] +
                                         (size_t)qr * p.dq2_s[1] + (size_t)T.hn * p.dq2_s[2];
                    float *acc = p.acc_dq2 ? p.acc_dq2 + (((size_t)T.b * p.N + qr) * p.H_N + T.hn) * HD : nullptr;
                    put_row<64>(x, p.scale, dst, acc);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (R.lane == 0) mbar_arrive(bar(B_ACCFREE));
            return true;
        };
        int G = 0, ti = 0;
        Tile prev{};
        for (;; ++ti) {
            const int t = read_tile(ti);
            if (t < 0) break;
            const Tile T = tile_of(t);
            const int qrow = T.q0 + r;  // this thread's query
            const float *strow = p.stats + (size_t)(T.b * p.H + T.h) * kBwdStats * p.n_pad + qrow;
            // (stored negated: -lse_1, -lse_2, -Delta_1, -Delta_2, -lambda)
            const float nlse1 = strow[0], nlse2 = strow[p.n_pad], ndel1 = strow[2 * p.n_pad],
                        ndel2 = strow[3 * p.n_pad], nlam = strow[4 * p.n_pad];
            // The tile's Q_1, Q_2 (warpgroup 0) and dD (warpgroup 1) rows into
            // TMEM, the A operands of every block's score and dP products.
            if (!(ok = mbar_wait_warp(bar(B_TILE), ti & 1, abort_flag, lim))) break;
            if (wg == 0) {
                tile_row_to_tmem(sbase + QT_Q1, r, tbase + lo + QM_AQ1);
                tile_row_to_tmem(sbase + QT_Q2, r, tbase + lo + QM_AQ2);
            } else {
                tile_row_to_tmem(sbase + QT_DD, r, tbase + lo + QM_ADD);
                tile_row_to_tmem(sbase + QT_DD + 16384, r, tbase + lo + QM_ADD + 32);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (R.lane == 0) mbar_arrive(bar(B_AOP));
            // The previous tile's epilogue, while this tile's first score
            // products run.
            if (ti > 0 && !(ok = epilogue(prev, ti - 1))) break;
            const float2 c2 = make_float2(c, c), nl1 = make_float2(nlse1, nlse1), nl2 = make_float2(nlse2, nlse2);
            const float2 nd1 = make_float2(ndel1, ndel1), nd2 = make_float2(ndel2, ndel2), nlm = make_float2(nlam, nlam);
            for (int j = 0; ok && j < T.nit; ++j, ++G) {
                if (!(ok = mbar_wait_warp(bar(B_SFULL), G & 1, abort_flag, lim))) break;
                tc_fence_after();
                uint32_t s1[32], s2[32], dp[32];
                tmem_ld32(tbase + lo + QM_S1 + 32 * wg, s1);
                tmem_ld32(tbase + lo + QM_S2 + 32 * wg, s2);
                tmem_ld32(tbase + lo + QM_DP + 32 * wg, dp);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (R.lane == 0) mbar_arrive(bar(B_SFREE));
                const int kb = (T.kb0 + j) * BB + 32 * wg;  // this warpgroup's 32 keys of the block
                const bool mask = (p.causal && kb + 31 > T.q0) || (p.window > 0 && T.q0 + BT - 1 - kb >= p.window);
                uint32_t d1p[16], d2p[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {  // two keys at a time, in packed arithmetic
                    const float2 x1 = ffma2(make_float2(__uint_as_float(s1[i]), __uint_as_float(s1[i + 1])), c2, nl1);
                    const float2 x2 = ffma2(make_float2(__uint_as_float(s2[i]), __uint_as_float(s2[i + 1])), c2, nl2);
                    float2 p1, p2;
                    if ((BWD_SOFT_EXP_MASK >> ((i >> 1) & 7)) & 1u) {
                        p1 = exp2_soft2(x1);
                        p2 = exp2_soft2(x2);
                    } else {
                        p1 = make_float2(ex2_approx(x1.x), ex2_approx(x1.y));
                        p2 = make_float2(ex2_approx(x2.x), ex2_approx(x2.y));
                    }
                    if (mask) {
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int key = kb + i + u;
                            const bool vis = (!p.causal || key <= qrow) && (p.window <= 0 || qrow - key < p.window);
                            if (!vis) {
                                if (u) p1.y = p2.y = 0.f;
                                else p1.x = p2.x = 0.f;
                            }
                        }
                    }
                    const float2 g = make_float2(__uint_as_float(dp[i]), __uint_as_float(dp[i + 1]));
                    const float2 v1 = fmul2(p1, fadd2(g, nd1));        // P_1 (dP - Delta_1)
                    const float2 v2 = fmul2(p2, ffma2(nlm, g, nd2));   // P_2 (-lambda dP - Delta_2)
                    if (F16QK)
                        big |= !(fabsf(v1.x) <= 65504.0f && fabsf(v1.y) <= 65504.0f && fabsf(v2.x) <= 65504.0f &&
                                 fabsf(v2.y) <= 65504.0f);
                    d1p[i / 2] = pack_ds(v1.x, v1.y, F16QK);
                    d2p[i / 2] = pack_ds(v2.x, v2.y, F16QK);
                }
                // The previous block's accumulating products (of this tile or
                // the one before) must have read the A operands.
                if (G > 0 && !(ok = mbar_wait_warp(bar(B_AFREE), (G - 1) & 1, abort_flag, lim))) break;
                // this warpgroup's 32 keys: TMEM columns [16 wg, 16 wg + 16) of each operand
                tmem_st16(tbase + lo + QM_ADS1 + 16 * wg, d1p);
                tmem_st16(tbase + lo + QM_ADS2 + 16 * wg, d2p);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (R.lane == 0) mbar_arrive(bar(B_AFULL));
            }
            if (!ok) break;
            prev = T;
        }
        if (ok && ti > 0) ok = epilogue(prev, ti - 1);
        if (big) report_error(p.dev_status, DIFFATTN_ERR_UNSUPPORTED);
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) report_error(p.dev_status, DIFFATTN_ERR_TIMEOUT);
    if (R.warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

// ---------------------------------------------------------------- 4. conversion of shared-head sums
// The fp32 sums of dK_2, dQ_2 (noise heads) and dV (V heads) that several
// signal heads added into, written as bf16 rows (8 elements per thread).
__global__ void bwd_convert_kernel(const BwdParams p)
{
    const int64_t n_qk = p.acc_dk2 ? (int64_t)p.B * p.N * p.H_N * (HD / 8) : 0;
    const int64_t n_v = p.acc_dv ? (int64_t)p.B * p.N * p.H_V * (HDV / 8) : 0;
    const int64_t total = 2 * n_qk + n_v;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const float *src;
        __nv_bfloat16 *dst;
        int64_t k = i;
        if (k < 2 * n_qk) {
            const bool q = k >= n_qk;
            k -= q ? n_qk : 0;
            const int c8 = int(k % (HD / 8));
            const int64_t rowi = k / (HD / 8);
            const int hn = int(rowi % p.H_N);
            const int64_t bn = rowi / p.H_N;
            const int n = int(bn % p.N), b = int(bn / p.N);
            src = (q ? p.acc_dq2 : p.acc_dk2) + rowi * HD + 8 * c8;
            const int64_t *s = q ? p.dq2_s : p.dk2_s;
            dst = static_cast<__nv_bfloat16 *>(q ? p.dq2 : p.dk2) + b * s[0] + (int64_t)n * s[1] + hn * s[2] + 8 * c8;
        } else {
            k -= 2 * n_qk;
            const int c8 = int(k % (HDV / 8));
            const int64_t rowi = k / (HDV / 8);
            const int hv = int(rowi % p.H_V);
            const int64_t bn = rowi / p.H_V;
            const int n = int(bn % p.N), b = int(bn / p.N);
            src = p.acc_dv + rowi * HDV + 8 * c8;
            dst = static_cast<__nv_bfloat16 *>(p.dv) + b * p.dv_s[0] + (int64_t)n * p.dv_s[1] + hv * p.dv_s[2] + 8 * c8;
        }
        const float4 a = *reinterpret_cast<const float4 *>(src), c = *reinterpret_cast<const float4 *>(src + 4);
        *reinterpret_cast<uint4 *>(dst) =
            make_uint4(pack_bf162(a.x, a.y), pack_bf162(a.z, a.w), pack_bf162(c.x, c.y), pack_bf162(c.z, c.w));
    }
}

}  // namespace

cudaError_t launch_bwd(const BwdKeyMaps &km, const BwdQueryMaps &qm, const BwdParams &p,
                       cudaStream_t stream, int *launches, const ProfileEvents &ev)
{
    constexpr int kMaxDevices = 64;
    static std::atomic<bool> attr_set[kMaxDevices] = {};
    static std::mutex attr_mutex;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) {
        set_internal_error("device ordinal beyond the library's table");
        return cudaErrorInvalidDevice;
    }
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lock(attr_mutex);  // first calls from several host threads
        if (!attr_set[dev].load(std::memory_order_relaxed)) {
            e = cudaFuncSetAttribute(bwd_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PREP_RED_BYTES);
            if (e != cudaSuccess) return e;
            for (const void *k : {(const void *)bwd_key_kernel<false>, (const void *)bwd_key_kernel<true>}) {
                e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)KT_SMEM);
                if (e != cudaSuccess) return e;
            }
            for (const void *k : {(const void *)bwd_query_kernel<false>, (const void *)bwd_query_kernel<true>}) {
                e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)QT_SMEM);
                if (e != cudaSuccess) return e;
            }
            attr_set[dev].store(true, std::memory_order_release);
        }
    }
    if ((int64_t)p.B * p.H * p.num_qt == 0) return cudaSuccess;
    const bool want_dgain = p.apply_norm && p.dgain;
    const int tiles = p.B * p.H * p.num_qt;  // query tiles, and key tiles alike: ceil(N / 128)
    bwd_prep_kernel<<<tiles * (BT / PREP_ROWS), PREP_THREADS, want_dgain ? PREP_RED_BYTES : 0, stream>>>(p);
    ++*launches;
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (ev.start) cudaEventRecord(ev.start, stream);
    // Both tile kernels are persistent: one CTA per SM (or per tile, when
    // there are fewer).
    const int sms = device_sm_count();
    const int key_grid = tiles < sms ? tiles : sms;
    if (p.qk_f16)
        bwd_key_kernel<true><<<key_grid, NT, KT_SMEM, stream>>>(km, p);
    else
        bwd_key_kernel<false><<<key_grid, NT, KT_SMEM, stream>>>(km, p);
    ++*launches;
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (p.qk_f16)
        bwd_query_kernel<true><<<key_grid, NT, QT_SMEM, stream>>>(qm, p);
    else
        bwd_query_kernel<false><<<key_grid, NT, QT_SMEM, stream>>>(qm, p);
    ++*launches;
    if (ev.stop) cudaEventRecord(ev.stop, stream);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (p.acc_dk2 || p.acc_dv) {
        bwd_convert_kernel<<<device_sm_count() * 8, 256, 0, stream>>>(p);
        ++*launches;
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace da
