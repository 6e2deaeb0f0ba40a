// backward_sm100.cu -- the backward pass of the differential-attention
// prefill on B200 (sm_100a).
//
// The pages define the forward pass (Motif 2.6B explainer, section
// "Differential attention", figure 1) and train the model with it (same
// page, "A schedule for the data"); the backward pass here is its exact
// gradient.  With A_t = P_t V the two map
// outputs, D = A_1 - lambda A_2, r = (mean_c D^2 + eps)^-1/2, Y = D r gain:
//
//   dgain = sum_i dY D r                 dD = r (dY gain) - (r^3/128) D sum_c(dY gain D)
//   dA_1 = dD, dA_2 = -lambda dD         dlambda = -sum dD A_2
//   per map t: dP_t = dA_t V^T = (1, -lambda) x dP with dP = dD V^T (one product)
//              Delta_t = rowsum(dA_t A_t), dS_t = P_t (dP_t - Delta_t)
//              dQ_t = scale dS_t K_t, dK_t = scale dS_t^T Q_t
//   dV = P_1^T dA_1 + P_2^T dA_2 = (P_1 - lambda P_2)^T dD (one product)
//
// Three kernels after the fp16 staging of V (the forward's staging kernel):
//  1. bwd_prep_kernel, one thread per row: reads the forward's saved A_1, A_2
//     and lse, and dY; writes dD (fp16, the tensor-core operand), the row
//     statistics (lse_1, lse_2, Delta_1, Delta_2), and adds into dlambda and
//     dgain.
//  2. bwd_key_kernel, one CTA per (b, h, 128-key tile), keys on the 128 TMEM
//     lanes: loops over 64-query blocks; per block three tcgen05 products
//     into TMEM (S_1^T = K_1 Q_1^T, S_2^T = K_2 Q_2^T, dP^T = V dD^T), the
//     element-wise step in registers (P_t from the saved lse, the dV operand
//     P_1 - lambda P_2 in fp16, dS_1, dS_2 in bf16, written back to TMEM),
//     then three accumulating products with A from TMEM (dV += (P_1 -
//     lambda P_2)^T dD, dK_t += dS_t^T Q_t).
//  3. bwd_query_kernel, one CTA per (b, h, 128-query tile), queries on the
//     lanes: loops over 64-key blocks; S_1, S_2, dP = dD V^T, the element-wise
//     step, dQ_t += dS_t K_t.
// Both loops double-buffer their block loads (TMA) against the element-wise
// step; the tensor core and the CUDA cores take turns within a CTA (no warp
// specialisation), so the speed comes from one CTA per SM over many CTAs.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace da {
namespace {

constexpr int BT = 128;   // rows of a tile: MMA M, one per TMEM lane / thread
constexpr int BB = 64;    // rows of a block: MMA N of the score products
constexpr int HD = 64;    // Q/K head dim
constexpr int HDV = 128;  // V head dim
constexpr int NT = 128;   // threads per CTA of the tile kernels
constexpr int NBARS = 5;  // tile, full[2], S, M

// ---------------------------------------------------------------- key-tile kernel
// Shared memory: the tile's K_1, K_2 (bf16 [128][64]) and V (fp16 [128][128]
// as two [128][64] column halves), then two block buffers of Q_1, Q_2 (bf16
// [64][64]), dD (fp16 [64][128] as two halves) and the statistics [4][64].
constexpr uint32_t KT_K1 = 0, KT_K2 = 16384, KT_V = 32768, KT_BUF = 65536;
constexpr uint32_t KB_Q1 = 0, KB_Q2 = 8192, KB_DD = 16384, KB_ST = 32768, KB_BYTES = 33792;
constexpr uint32_t KT_BARS = KT_BUF + 2 * KB_BYTES;
constexpr uint32_t KT_SMEM = KT_BARS + 8 * NBARS + 8;
// TMEM columns: dV accumulator, dK_1, dK_2, then S_1^T, S_2^T, dP^T.  The
// element-wise step writes the dV operand over the first half of S_1^T, dS_1
// over the first half of S_2^T and dS_2 over the first half of dP^T.
constexpr uint32_t KM_DV = 0, KM_DK1 = 128, KM_DK2 = 192, KM_S1 = 256, KM_S2 = 320, KM_DP = 384;

// ---------------------------------------------------------------- query-tile kernel
// Shared memory: the tile's Q_1, Q_2 (bf16 [128][64]) and dD (fp16 [128][128]
// as two halves), then two block buffers of K_1, K_2 (bf16 [64][64]) and V
// (fp16 [64][128] as two halves).
constexpr uint32_t QT_Q1 = 0, QT_Q2 = 16384, QT_DD = 32768, QT_BUF = 65536;
constexpr uint32_t QB_K1 = 0, QB_K2 = 8192, QB_V = 16384, QB_BYTES = 32768;
constexpr uint32_t QT_BARS = QT_BUF + 2 * QB_BYTES;
constexpr uint32_t QT_SMEM = QT_BARS + 8 * NBARS + 8;
// TMEM columns: dQ_1, dQ_2, then S_1, S_2, dP; dS_1 goes over the first half
// of S_1 and dS_2 over the first half of S_2.
constexpr uint32_t QM_DQ1 = 0, QM_DQ2 = 64, QM_S1 = 128, QM_S2 = 192, QM_DP = 256;

// Both tile kernels use more than half an SM's shared memory, so one CTA per
// SM holds the 512 TMEM columns it allocates.
static_assert(KT_SMEM > 116 * 1024 && KT_SMEM <= 227 * 1024, "key-tile kernel: one CTA per SM");
static_assert(QT_SMEM > 116 * 1024 && QT_SMEM <= 227 * 1024, "query-tile kernel: one CTA per SM");

// Instruction descriptors (fp32 accumulate).
constexpr uint32_t ID_S = idesc_f16(1, 1, 0, BT, BB);     // bf16 x bf16, both K-major
constexpr uint32_t ID_DP = idesc_f16(0, 0, 0, BT, BB);    // fp16 x fp16, both K-major
constexpr uint32_t ID_DV = idesc_f16(0, 0, 1, BT, HDV);   // fp16 (TMEM) x fp16, B MN-major
constexpr uint32_t ID_ACC64 = idesc_f16(1, 1, 1, BT, HD); // bf16 (TMEM) x bf16, B MN-major

// Descriptor of a 128-byte-swizzled operand tile (rows of 128 bytes, 8-row
// atoms of 1 KB); `lbo` is the byte distance between 64-element column
// halves when the MMA's N spans two of them (MN-major B).
__device__ __forceinline__ uint64_t sw128(uint32_t addr, uint32_t lbo = 16)
{
    return smem_desc_sw128(addr, lbo, 1024);
}

// One elected lane of a fully active warp issues; the warp stays converged.
struct Issuer {
    __device__ __forceinline__ void ss(uint32_t d, uint64_t a, uint64_t b, uint32_t id, bool acc) const
    {
        if (elect_one()) mma_ss(d, a, b, id, acc ? 1u : 0u);
        __syncwarp();
    }
    __device__ __forceinline__ void ts(uint32_t d, uint32_t a, uint64_t b, uint32_t id, bool acc) const
    {
        if (elect_one()) mma_ts(d, a, b, id, acc ? 1u : 0u);
        __syncwarp();
    }
    __device__ __forceinline__ void commit(uint32_t bar) const
    {
        if (elect_one()) mma_commit(bar);
        __syncwarp();
    }
};

// Store 2 x 32 fp32 values (scaled) of one row as bf16 to `dst` (16-byte aligned).
__device__ __forceinline__ void store_row_bf16(__nv_bfloat16 *dst, const uint32_t (&v)[32], float s)
{
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        d4[i] = make_uint4(pack_bf162(__uint_as_float(v[8 * i]) * s, __uint_as_float(v[8 * i + 1]) * s),
                           pack_bf162(__uint_as_float(v[8 * i + 2]) * s, __uint_as_float(v[8 * i + 3]) * s),
                           pack_bf162(__uint_as_float(v[8 * i + 4]) * s, __uint_as_float(v[8 * i + 5]) * s),
                           pack_bf162(__uint_as_float(v[8 * i + 6]) * s, __uint_as_float(v[8 * i + 7]) * s));
}

// ---------------------------------------------------------------- 1. row preparation
// One CTA per (batch entry, head, 128-row query tile), one thread per row.
// Dynamic shared memory [128][129] fp32 holds the per-row dgain terms when
// dgain is requested (and the norm applied), so that one thread per column
// sums them.
__global__ void __launch_bounds__(128)
    bwd_prep_kernel(const BwdParams p)
{
    extern __shared__ float red[];
    __shared__ float warp_sum[4];
    const int qt = blockIdx.x % p.num_qt, h = (blockIdx.x / p.num_qt) % p.H, b = blockIdx.x / (p.num_qt * p.H);
    const int r = threadIdx.x, row = qt * BT + r;
    const bool valid = row < p.N;
    const float *tile = p.save + ((size_t)(b * p.H + h) * p.num_qt + qt) * kSaveTileFloats;
    const float4 *a1p = reinterpret_cast<const float4 *>(tile) + r;   // chunk c at c * 128
    const float4 *a2p = a1p + 32 * BT;
    const float lam = p.lambda[h];
    const float4 *g4p = p.gain ? reinterpret_cast<const float4 *>(p.gain + (size_t)h * HDV) : nullptr;
    const __nv_bfloat16 *dy = static_cast<const __nv_bfloat16 *>(p.dout) + (size_t)b * p.do_sb +
                              (size_t)(valid ? row : 0) * p.do_sn + (size_t)h * p.do_sh;
    const bool want_dgain = p.apply_norm && p.dgain;

    auto load_dy4 = [&](int c, float (&y)[4]) {
        const uint2 u = *reinterpret_cast<const uint2 *>(dy + 4 * c);
        y[0] = __uint_as_float(u.x << 16);
        y[1] = __uint_as_float(u.x & 0xffff0000u);
        y[2] = __uint_as_float(u.y << 16);
        y[3] = __uint_as_float(u.y & 0xffff0000u);
    };
    auto gain4 = [&](int c) { return g4p ? __ldg(g4p + c) : make_float4(1.f, 1.f, 1.f, 1.f); };

    // Pass 1: sum of squares of D and sum_c dY gain D.
    float ss = 0.f, tg = 0.f;
    if (valid && p.apply_norm) {
#pragma unroll 4
        for (int c = 0; c < 32; ++c) {
            const float4 a1 = a1p[c * BT], a2 = a2p[c * BT], g = gain4(c);
            float y[4];
            load_dy4(c, y);
            const float d[4] = {fmaf(-lam, a2.x, a1.x), fmaf(-lam, a2.y, a1.y), fmaf(-lam, a2.z, a1.z),
                                fmaf(-lam, a2.w, a1.w)};
            const float gg[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                ss = fmaf(d[e], d[e], ss);
                tg = fmaf(gg[e] * y[e], d[e], tg);
            }
        }
    }
    const float rn = p.apply_norm ? 1.0f / sqrtf(ss * (1.0f / HDV) + p.eps) : 1.0f;
    const float coef = rn * rn * rn * (1.0f / HDV) * tg;

    // Pass 2: dD, Delta_1 = dD . A_1, dD . A_2, the dgain terms.
    float delta1 = 0.f, dot2 = 0.f;
    bool bad = false;
    __half *ddrow = static_cast<__half *>(p.dd) + (((size_t)b * p.N + (valid ? row : 0)) * p.H + h) * HDV;
#pragma unroll 4
    for (int c = 0; c < 32; ++c) {
        float dd[4] = {0.f, 0.f, 0.f, 0.f}, gt[4] = {0.f, 0.f, 0.f, 0.f};
        if (valid) {
            const float4 a1 = a1p[c * BT], a2 = a2p[c * BT], g = gain4(c);
            float y[4];
            load_dy4(c, y);
            const float av1[4] = {a1.x, a1.y, a1.z, a1.w}, av2[4] = {a2.x, a2.y, a2.z, a2.w};
            const float gg[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float d = fmaf(-lam, av2[e], av1[e]);
                dd[e] = p.apply_norm ? fmaf(rn * gg[e], y[e], -coef * d) : y[e];
                delta1 = fmaf(dd[e], av1[e], delta1);
                dot2 = fmaf(dd[e], av2[e], dot2);
                gt[e] = y[e] * d * rn;
                bad |= !(fabsf(dd[e]) <= 65504.0f);
            }
            *reinterpret_cast<uint2 *>(ddrow + 4 * c) = make_uint2(pack_half2(dd[0], dd[1]), pack_half2(dd[2], dd[3]));
        }
        if (want_dgain) {
#pragma unroll
            for (int e = 0; e < 4; ++e) red[r * (HDV + 1) + 4 * c + e] = gt[e];
        }
    }
    if (bad) report_error(p.dev_status, DIFFATTN_ERR_UNSUPPORTED);

    // Row statistics; rows past N get zeros (the tile kernels mask them).
    float *st = p.stats + (size_t)(b * p.H + h) * 4 * p.n_pad + row;
    const float *lse = tile + 2 * BT * HDV;
    st[0] = valid ? lse[r] : 0.f;
    st[p.n_pad] = valid ? lse[BT + r] : 0.f;
    st[2 * p.n_pad] = delta1;
    st[3 * p.n_pad] = -lam * dot2;

    // dlambda += -sum dD . A_2 over the tile's rows.
    if (p.dlambda) {
        float v = -dot2;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if ((r & 31) == 0) warp_sum[r >> 5] = v;
    }
    __syncthreads();
    if (p.dlambda && r == 0) atomicAdd(p.dlambda + h, warp_sum[0] + warp_sum[1] + warp_sum[2] + warp_sum[3]);
    // dgain[h][c] += sum over the tile's rows (thread r sums column r).
    if (want_dgain) {
        float v = 0.f;
#pragma unroll 8
        for (int i = 0; i < BT; ++i) v += red[i * (HDV + 1) + r];
        atomicAdd(p.dgain + (size_t)h * HDV + r, v);
    }
}

// ---------------------------------------------------------------- 2. key tiles
__global__ void __launch_bounds__(NT, 1)
    bwd_key_kernel(const __grid_constant__ BwdKeyMaps m, const BwdParams p)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_addr(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (sbase & 1023u) {  // the 128-byte-swizzled tiles need 1 KB alignment
        if (threadIdx.x == 0) report_error(p.dev_status, DIFFATTN_ERR_UNSUPPORTED);
        return;
    }
    // Heavy tiles first: under the causal mask key tile 0 meets every query.
    const int BH = p.B * p.H;
    const int kt = blockIdx.x / BH, bh = blockIdx.x % BH, b = bh / p.H, h = bh % p.H;
    const int k0 = kt * BT;
    const int nqb = (p.N + BB - 1) / BB;
    const int qb0 = p.causal ? k0 / BB : 0;
    const int nit = nqb - qb0;  // >= 1: k0 < N
    auto bar = [&](int i) { return sbase + KT_BARS + 8 * i; };
    enum { B_TILE = 0, B_FULL = 1, B_S = 3, B_M = 4 };
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(smem + KT_BARS + 8 * NBARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + KT_BARS + 8 * NBARS + 4);
    const uint64_t lim = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NBARS; ++i) mbar_init(bar(i), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_ptr), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_ptr;
    const Issuer is;

    auto load_block = [&](int j) {  // query block qb0 + j into buffer j & 1 (elected lane)
        const uint32_t buf = sbase + KT_BUF + (j & 1) * KB_BYTES, fb = bar(B_FULL + (j & 1));
        const int q0 = (qb0 + j) * BB;
        mbar_arrive_expect_tx(fb, KB_BYTES);
        tma_load_4d_nohint(buf + KB_Q1, &m.q1, fb, 0, q0, h, b);
        tma_load_4d_nohint(buf + KB_Q2, &m.q2, fb, 0, q0, h, b);
        tma_load_4d_nohint(buf + KB_DD, &m.dd, fb, 0, q0, h, b);
        tma_load_4d_nohint(buf + KB_DD + 8192, &m.dd, fb, 64, q0, h, b);
        tma_load_4d_nohint(buf + KB_ST, &m.stats, fb, q0, 0, h, b);
    };
    int loads = 0;  // blocks whose loads were issued
    if (warp == 0) {
        if (elect_one()) {
            mbar_arrive_expect_tx(bar(B_TILE), KT_BUF);
            tma_load_4d_nohint(sbase + KT_K1, &m.k1, bar(B_TILE), 0, k0, h, b);
            tma_load_4d_nohint(sbase + KT_K2, &m.k2, bar(B_TILE), 0, k0, h, b);
            tma_load_4d_nohint(sbase + KT_V, &m.v, bar(B_TILE), 0, k0, h, b);
            tma_load_4d_nohint(sbase + KT_V + 16384, &m.v, bar(B_TILE), 64, k0, h, b);
            load_block(0);
        }
        __syncwarp();
    }
    loads = 1;

    const int kj = k0 + warp * 32 + lane;  // this thread's key
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    const float lam = p.lambda[h];
    int consumed = 0, commits_s = 0, commits_m = 0;
    bool tile_waited = false, ok = true;
    for (int j = 0; j < nit; ++j) {
        const uint32_t buf = sbase + KT_BUF + (j & 1) * KB_BYTES;
        bool ok_w = true;
        if (warp == 0) {
            if (!tile_waited) ok_w = tile_waited = mbar_wait_warp(bar(B_TILE), 0, abort_flag, lim);
            ok_w = ok_w && mbar_wait_warp(bar(B_FULL + (j & 1)), (j >> 1) & 1, abort_flag, lim);
            if (ok_w) {
                consumed = j + 1;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    is.ss(tbase + KM_S1, sw128(sbase + KT_K1 + 32 * kk), sw128(buf + KB_Q1 + 32 * kk), ID_S, kk > 0);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    is.ss(tbase + KM_S2, sw128(sbase + KT_K2 + 32 * kk), sw128(buf + KB_Q2 + 32 * kk), ID_S, kk > 0);
#pragma unroll
                for (int kk = 0; kk < HDV / 16; ++kk) {
                    const uint32_t o = 32 * (kk & 3);
                    is.ss(tbase + KM_DP, sw128(sbase + KT_V + (kk >> 2) * 16384 + o),
                          sw128(buf + KB_DD + (kk >> 2) * 8192 + o), ID_DP, kk > 0);
                }
                is.commit(bar(B_S));
                ++commits_s;
            }
        }
        // Everyone: the three products of this block are in TMEM (and, as
        // the commit covers all earlier MMAs, the previous block's
        // accumulations have read their operands).
        bool ok_s = ok_w && mbar_wait_warp(bar(B_S), j & 1, abort_flag, lim);
        if (!__syncthreads_and(ok_s)) {
            ok = false;
            break;
        }
        tc_fence_after();
        if (warp == 0 && j + 1 < nit) {
            if (elect_one()) load_block(j + 1);
            __syncwarp();
            loads = j + 2;
        }

        // Element-wise step for this thread's key against the block's 64
        // queries, 32 at a time.
        const float *st = reinterpret_cast<const float *>(smem + KT_BUF + (j & 1) * KB_BYTES + KB_ST);
        const int q0 = (qb0 + j) * BB;
#pragma unroll 1
        for (int ch = 0; ch < 2; ++ch) {
            uint32_t s1[32], s2[32], dp[32];
            tmem_ld32(tbase + lane_off + KM_S1 + 32 * ch, s1);
            tmem_ld32(tbase + lane_off + KM_S2 + 32 * ch, s2);
            tmem_ld32(tbase + lane_off + KM_DP + 32 * ch, dp);
            tmem_wait_ld();
            uint32_t pc[16], ds1[16], ds2[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                float pv[2], d1[2], d2[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int qi = 32 * ch + i + e, q = q0 + qi;
                    const bool vis = q < p.N && kj < p.N && (!p.causal || q >= kj);
                    const float p1 = vis ? ex2_approx(fmaf(__uint_as_float(s1[i + e]), p.scale_log2, -st[qi])) : 0.f;
                    const float p2 = vis ? ex2_approx(fmaf(__uint_as_float(s2[i + e]), p.scale_log2, -st[BB + qi])) : 0.f;
                    const float g = __uint_as_float(dp[i + e]);
                    pv[e] = fmaf(-lam, p2, p1);
                    d1[e] = p1 * (g - st[2 * BB + qi]);
                    d2[e] = p2 * fmaf(-lam, g, -st[3 * BB + qi]);
                }
                pc[i >> 1] = pack_half2(pv[0], pv[1]);
                ds1[i >> 1] = pack_bf162(d1[0], d1[1]);
                ds2[i >> 1] = pack_bf162(d2[0], d2[1]);
            }
            tmem_st16(tbase + lane_off + KM_S1 + 16 * ch, pc);
            tmem_st16(tbase + lane_off + KM_S2 + 16 * ch, ds1);
            tmem_st16(tbase + lane_off + KM_DP + 16 * ch, ds2);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        if (warp == 0) {
            tc_fence_after();
            // dV += (P_1 - lambda P_2)^T dD; dK_t += dS_t^T Q_t (A from TMEM).
#pragma unroll
            for (int kk = 0; kk < BB / 16; ++kk)
                is.ts(tbase + KM_DV, tbase + KM_S1 + 8 * kk, sw128(buf + KB_DD + 2048 * kk, 8192), ID_DV,
                      j > 0 || kk > 0);
#pragma unroll
            for (int kk = 0; kk < BB / 16; ++kk)
                is.ts(tbase + KM_DK1, tbase + KM_S2 + 8 * kk, sw128(buf + KB_Q1 + 2048 * kk, 8192), ID_ACC64,
                      j > 0 || kk > 0);
#pragma unroll
            for (int kk = 0; kk < BB / 16; ++kk)
                is.ts(tbase + KM_DK2, tbase + KM_DP + 8 * kk, sw128(buf + KB_Q2 + 2048 * kk, 8192), ID_ACC64,
                      j > 0 || kk > 0);
            is.commit(bar(B_M));
            ++commits_m;
        }
    }
    // The last accumulations, then the tile's rows of dV, dK_1, dK_2.
    if (ok) ok = __syncthreads_and(mbar_wait_warp(bar(B_M), (nit - 1) & 1, abort_flag, lim));
    if (ok) {
        // Every lane takes part in the TMEM loads (warp-collective); only
        // rows of keys below N are stored.
        tc_fence_after();
        const bool own = kj < p.N;
        const int krow = own ? kj : 0;
        uint32_t v[32];
        __nv_bfloat16 *dvr = static_cast<__nv_bfloat16 *>(p.dv) + (size_t)b * p.dv_s[0] +
                             (size_t)krow * p.dv_s[1] + (size_t)h * p.dv_s[2];
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            tmem_ld32(tbase + lane_off + KM_DV + 32 * c, v);
            tmem_wait_ld();
            if (own) store_row_bf16(dvr + 32 * c, v, 1.0f);
        }
        __nv_bfloat16 *dk1 = static_cast<__nv_bfloat16 *>(p.dk1) + (size_t)b * p.dk1_s[0] +
                             (size_t)krow * p.dk1_s[1] + (size_t)h * p.dk1_s[2];
        __nv_bfloat16 *dk2 = static_cast<__nv_bfloat16 *>(p.dk2) + (size_t)b * p.dk2_s[0] +
                             (size_t)krow * p.dk2_s[1] + (size_t)h * p.dk2_s[2];
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
            tmem_ld32(tbase + lane_off + KM_DK1 + 32 * c, v);
            tmem_wait_ld();
            if (own) store_row_bf16(dk1 + 32 * c, v, p.scale);
            tmem_ld32(tbase + lane_off + KM_DK2 + 32 * c, v);
            tmem_wait_ld();
            if (own) store_row_bf16(dk2 + 32 * c, v, p.scale);
        }
    } else if (threadIdx.x == 0) {
        report_error(p.dev_status, DIFFATTN_ERR_TIMEOUT);
    }
    // Nothing of ours may be in flight when the CTA frees TMEM and exits.
    if (warp == 0) {
        bool drained = true;
        if (!tile_waited) drained &= mbar_wait_drain(bar(B_TILE), 0, lim);
        for (int jj = consumed; jj < loads; ++jj)
            drained &= mbar_wait_drain(bar(B_FULL + (jj & 1)), (jj >> 1) & 1, lim);
        if (commits_s > 0) drained &= mbar_wait_drain(bar(B_S), (commits_s - 1) & 1, lim);
        if (commits_m > 0) drained &= mbar_wait_drain(bar(B_M), (commits_m - 1) & 1, lim);
        if (!__all_sync(0xffffffffu, drained) && lane == 0) report_error(p.dev_status, DIFFATTN_ERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

// ---------------------------------------------------------------- 3. query tiles
__global__ void __launch_bounds__(NT, 1)
    bwd_query_kernel(const __grid_constant__ BwdQueryMaps m, const BwdParams p)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_addr(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (sbase & 1023u) {
        if (threadIdx.x == 0) report_error(p.dev_status, DIFFATTN_ERR_UNSUPPORTED);
        return;
    }
    // Heavy tiles first: under the causal mask the last query tile meets every key.
    const int BH = p.B * p.H;
    const int qt = p.num_qt - 1 - (int)(blockIdx.x / BH), bh = blockIdx.x % BH, b = bh / p.H, h = bh % p.H;
    const int q0 = qt * BT;
    const int nkb_all = (p.N + BB - 1) / BB;
    const int nit = p.causal ? min(nkb_all, (q0 + BT) / BB) : nkb_all;
    auto bar = [&](int i) { return sbase + QT_BARS + 8 * i; };
    enum { B_TILE = 0, B_FULL = 1, B_S = 3, B_M = 4 };
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(smem + QT_BARS + 8 * NBARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + QT_BARS + 8 * NBARS + 4);
    const uint64_t lim = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NBARS; ++i) mbar_init(bar(i), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_ptr), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_ptr;
    const Issuer is;

    auto load_block = [&](int j) {  // key block j into buffer j & 1 (elected lane)
        const uint32_t buf = sbase + QT_BUF + (j & 1) * QB_BYTES, fb = bar(B_FULL + (j & 1));
        const int kb = j * BB;
        mbar_arrive_expect_tx(fb, QB_BYTES);
        tma_load_4d_nohint(buf + QB_K1, &m.k1, fb, 0, kb, h, b);
        tma_load_4d_nohint(buf + QB_K2, &m.k2, fb, 0, kb, h, b);
        tma_load_4d_nohint(buf + QB_V, &m.v, fb, 0, kb, h, b);
        tma_load_4d_nohint(buf + QB_V + 8192, &m.v, fb, 64, kb, h, b);
    };
    int loads = 0;
    if (warp == 0) {
        if (elect_one()) {
            mbar_arrive_expect_tx(bar(B_TILE), QT_BUF);
            tma_load_4d_nohint(sbase + QT_Q1, &m.q1, bar(B_TILE), 0, q0, h, b);
            tma_load_4d_nohint(sbase + QT_Q2, &m.q2, bar(B_TILE), 0, q0, h, b);
            tma_load_4d_nohint(sbase + QT_DD, &m.dd, bar(B_TILE), 0, q0, h, b);
            tma_load_4d_nohint(sbase + QT_DD + 16384, &m.dd, bar(B_TILE), 64, q0, h, b);
            load_block(0);
        }
        __syncwarp();
    }
    loads = 1;

    const int qrow = q0 + warp * 32 + lane;  // this thread's query
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    const float lam = p.lambda[h];
    const float *strow = p.stats + (size_t)(b * p.H + h) * 4 * p.n_pad + qrow;
    const float lse1 = strow[0], lse2 = strow[p.n_pad], del1 = strow[2 * p.n_pad], del2 = strow[3 * p.n_pad];
    int consumed = 0, commits_s = 0, commits_m = 0;
    bool tile_waited = false, ok = true;
    for (int j = 0; j < nit; ++j) {
        const uint32_t buf = sbase + QT_BUF + (j & 1) * QB_BYTES;
        bool ok_w = true;
        if (warp == 0) {
            if (!tile_waited) ok_w = tile_waited = mbar_wait_warp(bar(B_TILE), 0, abort_flag, lim);
            ok_w = ok_w && mbar_wait_warp(bar(B_FULL + (j & 1)), (j >> 1) & 1, abort_flag, lim);
            if (ok_w) {
                consumed = j + 1;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    is.ss(tbase + QM_S1, sw128(sbase + QT_Q1 + 32 * kk), sw128(buf + QB_K1 + 32 * kk), ID_S, kk > 0);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    is.ss(tbase + QM_S2, sw128(sbase + QT_Q2 + 32 * kk), sw128(buf + QB_K2 + 32 * kk), ID_S, kk > 0);
#pragma unroll
                for (int kk = 0; kk < HDV / 16; ++kk) {
                    const uint32_t o = 32 * (kk & 3);
                    is.ss(tbase + QM_DP, sw128(sbase + QT_DD + (kk >> 2) * 16384 + o),
                          sw128(buf + QB_V + (kk >> 2) * 8192 + o), ID_DP, kk > 0);
                }
                is.commit(bar(B_S));
                ++commits_s;
            }
        }
        bool ok_s = ok_w && mbar_wait_warp(bar(B_S), j & 1, abort_flag, lim);
        if (!__syncthreads_and(ok_s)) {
            ok = false;
            break;
        }
        tc_fence_after();
        if (warp == 0 && j + 1 < nit) {
            if (elect_one()) load_block(j + 1);
            __syncwarp();
            loads = j + 2;
        }

        const int kb = j * BB;
#pragma unroll 1
        for (int ch = 0; ch < 2; ++ch) {
            uint32_t s1[32], s2[32], dp[32];
            tmem_ld32(tbase + lane_off + QM_S1 + 32 * ch, s1);
            tmem_ld32(tbase + lane_off + QM_S2 + 32 * ch, s2);
            tmem_ld32(tbase + lane_off + QM_DP + 32 * ch, dp);
            tmem_wait_ld();
            uint32_t ds1[16], ds2[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                float d1[2], d2[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int key = kb + 32 * ch + i + e;
                    const bool vis = key < p.N && (!p.causal || key <= qrow);
                    const float p1 = vis ? ex2_approx(fmaf(__uint_as_float(s1[i + e]), p.scale_log2, -lse1)) : 0.f;
                    const float p2 = vis ? ex2_approx(fmaf(__uint_as_float(s2[i + e]), p.scale_log2, -lse2)) : 0.f;
                    const float g = __uint_as_float(dp[i + e]);
                    d1[e] = p1 * (g - del1);
                    d2[e] = p2 * fmaf(-lam, g, -del2);
                }
                ds1[i >> 1] = pack_bf162(d1[0], d1[1]);
                ds2[i >> 1] = pack_bf162(d2[0], d2[1]);
            }
            tmem_st16(tbase + lane_off + QM_S1 + 16 * ch, ds1);
            tmem_st16(tbase + lane_off + QM_S2 + 16 * ch, ds2);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        if (warp == 0) {
            tc_fence_after();
            // dQ_t += dS_t K_t (A from TMEM, K block as MN-major B).
#pragma unroll
            for (int kk = 0; kk < BB / 16; ++kk)
                is.ts(tbase + QM_DQ1, tbase + QM_S1 + 8 * kk, sw128(buf + QB_K1 + 2048 * kk, 8192), ID_ACC64,
                      j > 0 || kk > 0);
#pragma unroll
            for (int kk = 0; kk < BB / 16; ++kk)
                is.ts(tbase + QM_DQ2, tbase + QM_S2 + 8 * kk, sw128(buf + QB_K2 + 2048 * kk, 8192), ID_ACC64,
                      j > 0 || kk > 0);
            is.commit(bar(B_M));
            ++commits_m;
        }
    }
    if (ok) ok = __syncthreads_and(mbar_wait_warp(bar(B_M), (nit - 1) & 1, abort_flag, lim));
    if (ok) {
        // Every lane takes part in the TMEM loads; rows below N are stored.
        tc_fence_after();
        const bool own = qrow < p.N;
        const int qr = own ? qrow : 0;
        uint32_t v[32];
        __nv_bfloat16 *dq1 = static_cast<__nv_bfloat16 *>(p.dq1) + (size_t)b * p.dq1_s[0] +
                             (size_t)qr * p.dq1_s[1] + (size_t)h * p.dq1_s[2];
        __nv_bfloat16 *dq2 = static_cast<__nv_bfloat16 *>(p.dq2) + (size_t)b * p.dq2_s[0] +
                             (size_t)qr * p.dq2_s[1] + (size_t)h * p.dq2_s[2];
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
            tmem_ld32(tbase + lane_off + QM_DQ1 + 32 * c, v);
            tmem_wait_ld();
            if (own) store_row_bf16(dq1 + 32 * c, v, p.scale);
            tmem_ld32(tbase + lane_off + QM_DQ2 + 32 * c, v);
            tmem_wait_ld();
            if (own) store_row_bf16(dq2 + 32 * c, v, p.scale);
        }
    } else if (threadIdx.x == 0) {
        report_error(p.dev_status, DIFFATTN_ERR_TIMEOUT);
    }
    if (warp == 0) {
        bool drained = true;
        if (!tile_waited) drained &= mbar_wait_drain(bar(B_TILE), 0, lim);
        for (int jj = consumed; jj < loads; ++jj)
            drained &= mbar_wait_drain(bar(B_FULL + (jj & 1)), (jj >> 1) & 1, lim);
        if (commits_s > 0) drained &= mbar_wait_drain(bar(B_S), (commits_s - 1) & 1, lim);
        if (commits_m > 0) drained &= mbar_wait_drain(bar(B_M), (commits_m - 1) & 1, lim);
        if (!__all_sync(0xffffffffu, drained) && lane == 0) report_error(p.dev_status, DIFFATTN_ERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, 512);
    }
}

}  // namespace

cudaError_t launch_bwd(const BwdKeyMaps &km, const BwdQueryMaps &qm, const BwdParams &p,
                       cudaStream_t stream, int *launches)
{
    constexpr int kMaxDevices = 64;
    static bool attr_set[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) {
        set_internal_error("device ordinal beyond the library's table");
        return cudaErrorInvalidDevice;
    }
    const int red_bytes = BT * (HDV + 1) * (int)sizeof(float);
    if (!attr_set[dev]) {
        e = cudaFuncSetAttribute(bwd_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, red_bytes);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(bwd_key_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)KT_SMEM);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(bwd_query_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)QT_SMEM);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    if ((int64_t)p.B * p.H * p.num_qt == 0) return cudaSuccess;
    const bool want_dgain = p.apply_norm && p.dgain;
    const int tiles = p.B * p.H * p.num_qt;  // query tiles, and key tiles alike: ceil(N / 128)
    bwd_prep_kernel<<<tiles, 128, want_dgain ? red_bytes : 0, stream>>>(p);
    ++*launches;
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bwd_key_kernel<<<tiles, NT, KT_SMEM, stream>>>(km, p);
    ++*launches;
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bwd_query_kernel<<<tiles, NT, QT_SMEM, stream>>>(qm, p);
    ++*launches;
    return cudaGetLastError();
}

}  // namespace da
