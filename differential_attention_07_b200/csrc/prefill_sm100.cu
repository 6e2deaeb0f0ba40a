// prefill_sm100.cu -- causal differential-attention prefill on sm_100a.
//
// Computes, per (b, h) and 128-row query tile, the two softmax maps of
// differential attention (Motif 2.6B explainer, section "Differential
// attention": attn = [softmax(Q1 K1^T) - lambda softmax(Q2 K2^T)] V) with an
// online softmax for each map, and finishes with the subtraction and the norm
// after it (same page, figure 1: GroupNorm after the subtraction, read as a
// per-head RMS norm with gain).
//
// A persistent kernel: one CTA per SM (512 threads, four warpgroups) takes
// work items -- (b, unit, 128-row query tile) -- from a global counter until
// none are left.
//   warp 0        TMA producer: takes the next item, publishes it to the
//                 other roles, loads Q1/Q2 once per item, then K1/K2/V per
//                 64-key step into a 4-stage ring (32 KB per stage).
//   warps 1, 2    MMA issuers, one per map: S_t = Q_t K_t^T (bf16, fp32
//                 accumulate in TMEM), then O_t += P_t V with P read from TMEM
//                 and V (fp16) from the shared-memory tile both maps use.
//   warps 4-7     softmax of map 1 (one thread per query row).
//   warps 8-11    softmax of map 2.  A warp reaches TMEM lanes 32 (warp % 4)
//                 onwards, so each warpgroup covers all 128 rows.  At the end
//                 of a tile the softmax warps hand their row sums to the
//                 epilogue warps and go straight on to the next tile.
//   warps 12-15   epilogue, 32 rows per warp, overlapping the next tile's
//                 softmax: D = (O1 - r O2)/l1 with r = lambda l1/l2, RMS norm
//                 over the row's 128 columns, gain, optional output gate
//                 sigma(G) (lambda optionally sigma of a per-token logit:
//                 Motif 3 summary, section 2.2), bf16, staged in each warp's
//                 shared-memory buffer and written by TMA stores.  O goes
//                 back to the MMA warps as soon as it has been read.
//                 Registers are split 56 / 152 / 152 / 152 between the
//                 warpgroups (setmaxnreg).
// TMEM (512 columns): O1 [0,128) O2 [128,256), and two 64-column S buffers
// per map: S1 [256,320) [320,384), S2 [384,448) [448,512).  P (fp16, two per
// column) overwrites the first 32 columns of its S buffer.
//
// Pipeline.  Key steps alternate between the two S buffers of a map, and the
// MMA warp computes S for step j+2 as soon as P.V of step j has been issued,
// so the softmax of step j+1 need not wait for the tensor cores: the score
// MMAs of the next step run while the current step's softmax runs.  Per map t
// and step j the map's MMA warp does:
//   wait P_t,j; O_t += P_t,j V_j; release stage j; S_t,j+2 -> buffer j%2.
// MMAs from one thread execute in issue order, so S_{j+2} overwrites P_j only
// after P_j.V has read it.  The softmax keeps a stale row maximum until a new
// one exceeds it by more than 2^8 (P stays <= 256, exact enough in fp16); only
// then does it rescale its O row, after waiting for the previous P.V product.
//
// Every wait is bounded (PrefillParams::timeout_ns); on expiry the CTA raises
// an abort flag, reports DIFFATTN_ERR_TIMEOUT, drains its own TMA loads and
// MMAs, frees TMEM and exits without storing.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>
#include <climits>
#include <mutex>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace da {
namespace {

constexpr int BM = 128;   // query rows per tile (MMA M)
constexpr int BN = 64;    // keys per step (MMA N of S, K of P.V)
constexpr int HD = 64;    // Q/K head dim
constexpr int HDV = 128;  // V head dim (MMA N of P.V)
constexpr int STAGES = 4;
constexpr int NTHREADS = 512;

constexpr uint32_t Q_BYTES = BM * HD * 2;           // 16 KB
constexpr uint32_t K_BYTES = BN * HD * 2;           // 8 KB
constexpr uint32_t VHALF_BYTES = BN * 64 * 2;       // 8 KB: 64 of the 128 V columns
constexpr uint32_t V_BYTES = 2 * VHALF_BYTES;       // 16 KB
constexpr uint32_t STAGE_BYTES = 2 * K_BYTES + V_BYTES;

constexpr uint32_t OFF_Q1 = 0;
constexpr uint32_t OFF_Q2 = Q_BYTES;
constexpr uint32_t OFF_STAGE0 = 2 * Q_BYTES;
constexpr uint32_t OFF_BARS = OFF_STAGE0 + STAGES * STAGE_BYTES;
// mbarriers, in this order:
enum : int {
    B_QFULL = 0,                 // Q1/Q2 of the current tile landed (TMA bytes)
    B_QFREE = 1,                 // both maps' last score MMA of the tile done (2 commits)
    B_FULL = 2,                  // [STAGES] K1/K2/V of a step landed (TMA bytes)
    B_EMPTY = B_FULL + STAGES,   // [STAGES] both maps' P.V of the step done (2 commits)
    B_S = B_EMPTY + STAGES,      // [2 maps][2 buffers] S ready (commit)
    B_P = B_S + 4,               // [2 maps][2 buffers] P written (4 softmax warps)
    B_PV = B_P + 4,              // [2 maps] latest P.V into O done (commit)
    B_O = B_PV + 2,              // all MMAs of the tile done (2 commits)
    B_OFREE = B_O + 1,           // epilogue finished reading O (4 epilogue warps)
    B_STAT = B_OFREE + 1,        // [2 tile parities] row sums written (8 softmax warps)
    B_ITEM = B_STAT + 2,         // [ITEM_SLOTS] work item published (1 arrival)
    B_ITEMFREE = B_ITEM + 4,     // [ITEM_SLOTS] work item read by all 10 reader warps
    B_AN = B_ITEMFREE + 4,       // [4 epilogue warps] the warp's A_N rows landed (bulk-copy bytes)
    B_VCVT = B_AN + 4,           // [STAGES] window kernels: the step's V converted to fp16 (1 arrival)
    NBARS = B_VCVT + STAGES
};
// S and P barriers come one per S buffer: a softmax may run two steps ahead
// of its MMA warp's wait, and with one P barrier per map the second arrival
// would complete a phase the MMA warp had not yet waited for.  Per buffer,
// the next use needs the MMA warp's action in between, so no barrier is ever
// more than one phase ahead of its waiter; the same holds for the per-tile
// barriers because each tile's use of one depends on the previous tile's use
// of another.
constexpr uint32_t OFF_TMEM_PTR = OFF_BARS + NBARS * 8;
constexpr uint32_t OFF_ABORT = OFF_TMEM_PTR + 4;
constexpr int ITEM_SLOTS = 4;
constexpr int ITEM_READERS = 14;                         // 2 MMA, 8 softmax and 4 epilogue warps
                                                         // (and the V converter under a window)
constexpr uint32_t ITEM_BYTES = 48;                      // one published work item: three int4
constexpr uint32_t OFF_ITEM = (OFF_ABORT + 4 + 15) & ~15u;  // [ITEM_SLOTS] work-item ring
// float [2 tile parities][l1, l2][128]: the softmax warps' row sums
constexpr uint32_t OFF_STAT = (OFF_ITEM + ITEM_BYTES * ITEM_SLOTS + 15) & ~15u;
// Epilogue buffers: per epilogue warp 16 KB.  A one-head item keeps its 32
// rows of D there in fp32 and then the staged output, two 32 x 64 bf16 TMA
// store boxes of 4 KB with the 128-byte swizzle; a pair item keeps its 32
// rows of the group's noise output A_N (fp32) there.
constexpr uint32_t OUT_HALF_BYTES = 32 * 64 * 2;
constexpr uint32_t EPI_WARP_BYTES = 4 * OUT_HALF_BYTES;
constexpr uint32_t OFF_OUT = (OFF_STAT + 2 * 2 * BM * 4 + 1023) & ~1023u;
constexpr uint32_t SMEM_BYTES = OFF_OUT + 4 * EPI_WARP_BYTES;  // dynamic smem is 1024-byte aligned

constexpr uint32_t TM_O1 = 0, TM_O2 = 128, TM_S1 = 256, TM_S2 = 384;
constexpr uint32_t TMEM_COLS = 512;

// Registers per thread: at launch (the most __launch_bounds__(512, 1) allows:
// four warps per SM sub-partition share its 16K registers), and after the
// split between the producer/MMA warpgroup, the two softmax warpgroups and
// the epilogue warpgroup.  Each sub-partition holds one warp of each.
constexpr int REGS_LAUNCH = 128;
constexpr int REGS_IO = 56;
constexpr int REGS_SOFTMAX = 152;
constexpr int REGS_EPI = 152;
static_assert(REGS_IO + 2 * REGS_SOFTMAX + REGS_EPI == 4 * REGS_LAUNCH, "register split must use the pool exactly");
static_assert(NTHREADS == 512, "four warpgroups");

// The producer warms L2 with the K/V of the step this many steps ahead.
constexpr int L2_PREFETCH_STEPS = 8;

// P.V MMAs read a stale-max P of at most 2^RESCALE_THRESHOLD.
constexpr float RESCALE_THRESHOLD = 8.0f;

static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(OFF_BARS % 8 == 0, "mbarriers are 8-byte aligned");
static_assert(kPrefillQRows == BM && kPrefillKeyRows == BN && kPrefillOutRows == 32,
              "TMA boxes match the tiles");
static_assert(OFF_STAGE0 % 1024 == 0 && STAGE_BYTES % 1024 == 0 && K_BYTES % 1024 == 0,
              "SW128 atoms need 1 KB alignment");

struct Work {
    int b, u, qt;  // batch, unit (see heads_of), query tile
};

// The heads one work item computes.  Map 1 is always signal head a (Q1/K1);
// map 2 is noise head b (Q2/K2) or, for a pair of signal heads, signal head
// b (Q1/K1).  Modes (PrefillParams::mode):
//   0  unit = signal head: map 2 is its noise head h / (H / H_N), V head
//      h / (H / H_V); the tile's output is head a.
//   1  grouped pairs, for groups of g = H / H_N (odd, >= 3) signal heads
//      that share V head n with their noise head n.  Two kinds of unit:
//      u < H_N, the export unit of group u: map 1 is the group's last
//      signal head, map 2 the noise head; the output is that signal head,
//      and the normalised noise output A_N is exported for the group;
//      u = H_N + n P + q (P = (g - 1) / 2 pairs per group), a pair unit:
//      maps 1 and 2 are signal heads n g + 2q and n g + 2q + 1, and each
//      finishes against the exported A_N of its group (own = true).
struct Heads {
    int a, b, vh, n;
    bool b_noise, own;
};
__device__ __forceinline__ Heads heads_of(int u, const PrefillParams &p)
{
    if (p.mode == 0) {
        const int n = u / (p.H / p.H_N);
        return Heads{u, n, u / (p.H / p.H_V), n, true, false};
    }
    const int g = p.H / p.H_N;
    if (u < p.H_N) return Heads{u * g + g - 1, u, u, u, true, false};
    const int up = u - p.H_N, n = up / p.pairs, q = up - n * p.pairs;
    return Heads{n * g + 2 * q, n * g + 2 * q + 1, n, n, false, true};
}

// Map the linear CTA index to (b, h, query tile).  (b, h) pairs are taken in
// groups of heads_per_group so that the CTAs running at the same time share
// K/V tiles in L2; inside a group the longest (latest) query tiles go first.
// Work item idx -> (b, unit, query tile).  Items are handed out in this
// order, and the order does two things:
//  * L2 reuse: (b, unit) pairs are taken G = heads_per_group at a time, so
//    the K/V of the heads running together stay in L2;
//  * balance: under a causal mask a tile's cost grows with its index, so
//    each group runs heaviest first, in two phases.  Every group's heavy
//    half of the tiles comes first, then every group's light half, so the
//    schedule ends on the lightest tiles of all.  (Heaviest first within
//    each group alone left the last group's heaviest tiles at the end: 8 %
//    of the kernel idle, measured.)  The light half re-reads the first half
//    of each head's K/V, which costs little against the kernel's 6 % DRAM
//    use.
__device__ __forceinline__ Work tile_of(int idx, const PrefillParams &p)
{
    const int BH = p.B * p.units, G = p.heads_per_group, nq = p.num_qt;
    const int n_light = p.causal ? nq / 2 : 0, n_heavy = nq - n_light;
    // phase: tiles [top - count + 1, top] of every (b, unit), heaviest first
    int count = n_heavy, top = nq - 1;
    if (idx >= BH * n_heavy) {
        idx -= BH * n_heavy;
        count = n_light;
        top = n_light - 1;
    }
    const int full = BH / G, per_group = G * count;
    int bh, qt;
    if (idx < full * per_group) {
        const int g = idx / per_group, r = idx - g * per_group;
        qt = top - r / G;
        bh = g * G + r % G;
    } else {
        const int r = idx - full * per_group, tail = BH - full * G;
        qt = top - r / tail;
        bh = full * G + r % tail;
    }
    return Work{bh / p.units, bh % p.units, qt};
}

// Work items of one launch.  Mode 0: the tiles above, one item each.  Mode
// 1: the tiles are (b, noise head, query tile) triples T[0..NT); each has an
// export item and P pair items, and a pair item's epilogue needs its tile's
// export.  The export items run D = PrefillParams::lag tiles ahead of the
// pair items of the same tile:
//   T[0] .. T[D-1] export;  then per s in [D, NT): export of T[s], the P
//   pair items of T[s - D];  then the pair items of T[NT-D] .. T[NT-1].
// With D about the number of CTAs, an export item has finished long before
// the pair items of its tile reach their epilogue.  Because every item comes
// after the items it waits for, and each CTA takes its items in that order,
// the earliest unfinished item can always proceed: the launch cannot
// deadlock, whatever the number of resident CTAs.
__device__ __forceinline__ Work work_of(int idx, const PrefillParams &p)
{
    if (p.mode == 0) return tile_of(idx, p);
    const int NT = p.B * p.units * p.num_qt, P = p.pairs, S = P + 1, D = p.lag;
    int s, k;
    if (idx < D) {
        s = idx;
        k = 0;
    } else if (idx < D + (NT - D) * S) {
        const int r = idx - D;
        s = D + r / S;
        k = r - (r / S) * S;
        if (k) s -= D;
    } else {
        const int r = idx - D - (NT - D) * S;
        s = NT - D + r / P;
        k = 1 + r % P;
    }
    Work w = tile_of(s, p);
    if (k) w.u = p.units + w.u * P + (k - 1);
    return w;
}

// Spin (bounded) until *flag >= target; the acquire load orders the caller's
// later reads after the writes the flag's producers released.
__device__ __forceinline__ bool wait_flag_geq(const int *flag, int target, volatile int *abort_flag,
                                              uint64_t limit_ns)
{
    auto ld_acquire = [](const int *f) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
        return v;
    };
    if (ld_acquire(flag) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        __nanosleep(64);
        if (ld_acquire(flag) >= target) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            *abort_flag = 1;
            return false;
        }
    }
}

// Which pairs of scores (index mod 8) take the software exp2; the rest use
// MUFU ex2.  Measured on B200 (motif-4K / 16K prefill, TFLOP/s): 4 of 8
// 790 / 931, 3 of 8 810 / 893, 2 of 8 860 / 909, 1 of 8 861 / 959, none
// 843 / 996: with the pipeline overlapped, issue slots matter more than
// MUFU time, so only one pair in eight goes to the FMA pipe.
constexpr uint32_t SOFT_EXP_MASK = 0x20u;  // pair 5 of every 8

// Softmax of one map for one 64-key step, for the query row this thread owns;
// keys lo..hi of the step are visible to it (a row may see none of a step's
// keys under a sliding window: its max stays -inf and its P row is 0).
// Reads S (fp32) from TMEM, updates the running max / sum, rescales the O row
// when the max moved (after the previous P.V product into it has finished),
// and writes P (fp16) over the first 32 columns of the S buffer.  Returns
// false if a bounded wait gave up.
template <bool WINDOW>
__device__ __forceinline__ bool softmax_step(uint32_t tS, uint32_t tO, bool first, int lo, int hi,
                                             float scale_log2, float &m_run, float &l_run,
                                             uint32_t bar_pv, uint32_t pv_parity,
                                             volatile int *abort_flag, uint64_t lim)
{
    uint32_t v[2][32];
    tmem_ld32(tS, v[0]);
    tmem_ld32(tS + 32, v[1]);
    tmem_wait_ld();

    if (hi < BN - 1) {  // diagonal (or ragged) step: hide keys past hi
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (32 * c + i > hi) v[c][i] = __float_as_uint(-INFINITY);
    }
    if (WINDOW && lo > 0) {  // sliding-window edge: hide keys before lo
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (32 * c + i < lo) v[c][i] = __float_as_uint(-INFINITY);
    }
    // Row max of the raw scores (scale > 0 commutes with max): four
    // independent chains of three-input maxima.
    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
            float &m = mx[(2 * c + (i >> 4)) & 3];
            m = fmax3(m, __uint_as_float(v[c][i]), __uint_as_float(v[c][i + 1]));
            m = fmax3(m, __uint_as_float(v[c][i + 2]), __uint_as_float(v[c][i + 3]));
            m = fmax3(m, __uint_as_float(v[c][i + 4]), __uint_as_float(v[c][i + 5]));
            m = fmax3(m, __uint_as_float(v[c][i + 6]), __uint_as_float(v[c][i + 7]));
        }
    const float tmax = fmax3(fmaxf(mx[0], mx[1]), mx[2], mx[3]) * scale_log2;

    const bool need = tmax > m_run + RESCALE_THRESHOLD;
    const float m_new = need ? tmax : m_run;
    // A row that has seen no key yet (m_run = -inf: every P of it so far was
    // 0, so its O row and l are 0) takes its first maximum without a rescale.
    // Under a sliding window that is most rows of a tile's first steps.
    const bool scale_o = need && m_run != -INFINITY;
    float alpha = 1.0f;
    if (__any_sync(0xffffffffu, scale_o)) {  // rare after a row's first visible step
      alpha = scale_o ? ex2_approx(m_run - m_new) : 1.0f;
      if (!first) {
        // O holds P.V products up to the previous step; the last one must be
        // finished before the row is rescaled.
        if (!mbar_wait_warp(bar_pv, pv_parity, abort_flag, lim)) return false;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + 32 * c, o);
        }
      }
    }
    l_run *= alpha;
    m_run = m_new;
    const float m_sub = (m_run == -INFINITY) ? 0.0f : m_run;

    // p = 2^(s * scale_log2 - m): one packed FMA per two scores, then MUFU or
    // software exp2; row sum in four packed accumulators.
    const float2 sc = make_float2(scale_log2, scale_log2), nm = make_float2(-m_sub, -m_sub);
    float2 acc[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
    uint32_t pk[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int c = i >> 4, e = (2 * i) & 31;
        const float2 x = ffma2(make_float2(__uint_as_float(v[c][e]), __uint_as_float(v[c][e + 1])), sc, nm);
        const float2 pp = ((SOFT_EXP_MASK >> (i & 7)) & 1u)
                              ? exp2_soft2(x)
                              : make_float2(ex2_approx(x.x), ex2_approx(x.y));
        acc[i & 3] = fadd2(acc[i & 3], pp);
        pk[i] = pack_half2(pp.x, pp.y);
    }
    tmem_st32(tS, pk);
    const float2 a = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
    l_run += a.x + a.y;
    tmem_wait_st();
    return true;
}

// WINDOW: the kernel of sliding-window calls (p.window > 0); GATED: of calls
// with an output gate (p.gate); SAVE: of calls that also save the state of
// the backward pass (p.save).  Without them their code is left out
// altogether: even untaken, the window's lower-edge mask cost the plain
// kernel 2-5 % and the gate's loads 2-5 % (measured).
template <bool WINDOW, bool GATED, bool SAVE>
__global__ void __launch_bounds__(NTHREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q1, const __grid_constant__ CUtensorMap tm_q2,
                   const __grid_constant__ CUtensorMap tm_k1, const __grid_constant__ CUtensorMap tm_k2,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_out,
                   const PrefillParams p)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_addr(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (sbase & 1023u) {  // the 128-byte-swizzled tiles need 1 KB alignment
        if (threadIdx.x == 0) report_error(p.dev_status, DIFFATTN_ERR_UNSUPPORTED);
        return;
    }
    const int total = p.B * p.units * p.num_qt * (p.mode == 1 ? p.pairs + 1 : 1);
    const int n_steps_all = (p.N + BN - 1) / BN;
    // Key steps of a work item: [kv_first, kv_first + steps_of).  Causal tiles
    // stop at the diagonal; under a sliding window of W keys they start at
    // the step holding key q0 - W + 1, the first one row q0 sees.
    auto kv_first = [&](const Work &w) {
        return WINDOW ? max(0, w.qt * BM - p.window + 1) / BN : 0;
    };
    auto steps_of = [&](const Work &w) {
        const int q0 = w.qt * BM;
        return (p.causal ? min(n_steps_all, (q0 + BM) / BN) : n_steps_all) - kv_first(w);
    };

    auto bar = [&](int i) { return sbase + OFF_BARS + 8 * i; };
    auto bar_full = [&](int s) { return bar(B_FULL + s); };
    auto bar_empty = [&](int s) { return bar(B_EMPTY + s); };
    auto bar_s = [&](int t, int b) { return bar(B_S + 2 * t + b); };
    auto bar_p = [&](int t, int b) { return bar(B_P + 2 * t + b); };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_ABORT);
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(smem + OFF_TMEM_PTR);
    float *sStat = reinterpret_cast<float *>(smem + OFF_STAT);

    if (threadIdx.x == 0) {
        mbar_init(bar(B_QFULL), 1);
        mbar_init(bar(B_QFREE), 2);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), 2);
        }
        for (int i = 0; i < 4; ++i) {
            mbar_init(bar(B_S + i), 1);
            mbar_init(bar(B_P + i), 4);   // one arrival per softmax warp
        }
        mbar_init(bar(B_PV), 1);
        mbar_init(bar(B_PV + 1), 1);
        mbar_init(bar(B_O), 2);
        mbar_init(bar(B_OFREE), 4);   // one arrival per epilogue warp
        mbar_init(bar(B_STAT), 8);    // one arrival per softmax warp
        mbar_init(bar(B_STAT + 1), 8);
        for (int i = 0; i < 4; ++i) mbar_init(bar(B_AN + i), 1);
        if (WINDOW)
            for (int s = 0; s < STAGES; ++s) mbar_init(bar(B_VCVT + s), 1);
        for (int i = 0; i < ITEM_SLOTS; ++i) {
            mbar_init(bar(B_ITEM + i), 1);
            mbar_init(bar(B_ITEMFREE + i), ITEM_READERS + (WINDOW ? 1 : 0));
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(sbase + OFF_TMEM_PTR, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_ptr;
    // The prologue above overlaps the end of the staging kernel (or, for the
    // second grouped launch, of the first): everything below reads what they
    // wrote -- the fp16 V and rotated Q/K copies, the work counters, the
    // exported noise outputs.
    grid_dependency_wait();
    const uint64_t lim = p.timeout_ns;

    // Work items are handed out dynamically (an atomic counter in global
    // memory, zeroed by the V staging kernel that runs first): the producer
    // takes the next one, decodes it (tile, heads, key steps) and publishes
    // it in a ring of ITEM_SLOTS; the other roles read item k from slot
    // k % ITEM_SLOTS and release the slot.  The producer reuses a slot only
    // after all fourteen reader warps released it (with short tiles it can
    // run several tiles ahead).  b < 0 ends the loop.
    struct Item {
        Work w;
        Heads hd;
        int nkv, kv0;
    };
    auto read_item = [&](int k, Item &it) -> bool {
        const int slot = k % ITEM_SLOTS;
        if (!mbar_wait_warp(bar(B_ITEM + slot), (k / ITEM_SLOTS) & 1, abort_flag, p.timeout_ns)) return false;
        const uint32_t a = sbase + OFF_ITEM + ITEM_BYTES * slot;
        const uint4 x = ld_shared_v4(a), y = ld_shared_v4(a + 16), z = ld_shared_v4(a + 32);
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_ITEMFREE + slot));
        it.w = Work{int(x.x), int(x.y), int(x.z)};
        it.nkv = int(x.w);
        it.kv0 = int(y.x);
        it.hd = Heads{int(y.y), int(y.z), int(y.w), int(z.x), (z.y & 1u) != 0, (z.y & 2u) != 0};
        return it.w.b >= 0;
    };

    // Register split: 4 x REGS_LAUNCH = REGS_IO + 2 x REGS_SOFTMAX + REGS_EPI per thread slot
    // (the host launches only when the kernel was built with REGS_LAUNCH).
    // Each budget change opens its role's branch so that the compiler
    // allocates each branch within its own budget.
    if (warp < 4) {
      regs_decrease<REGS_IO>();
      if (warp == 0) {
        // ------------------------------------------------------------ producer
        // The whole warp runs the loop; an elected lane issues the copies.
        const uint64_t keep = policy_evict_last(), stream = policy_evict_first();
        if (elect_one()) {
            prefetch_tensormap(&tm_q1);
            prefetch_tensormap(&tm_q2);
            prefetch_tensormap(&tm_k1);
            prefetch_tensormap(&tm_k2);
            prefetch_tensormap(&tm_v);
        }
        __syncwarp();
        int g = 0, tiles = 0, q_loads = 0;
        bool ok = true;
        for (;; ++tiles) {
            const int slot = tiles % ITEM_SLOTS;
            if (tiles >= ITEM_SLOTS &&
                !(ok = mbar_wait_warp(bar(B_ITEMFREE + slot), ((tiles / ITEM_SLOTS) - 1) & 1, abort_flag, lim)))
                break;
            int item = -1;
            if (lane == 0) item = *abort_flag ? total : atomicAdd(p.tile_counter, 1);
            item = __shfl_sync(0xffffffffu, item, 0);
            const Work w = item < total ? work_of(item, p) : Work{-1, 0, 0};
            const Heads hd = heads_of(item < total ? w.u : 0, p);
            const int nkv = item < total ? steps_of(w) : 0, kv0 = item < total ? kv_first(w) : 0;
            if (lane == 0) {  // the decoded item, for the other roles
                const uint32_t a = sbase + OFF_ITEM + ITEM_BYTES * slot;
                st_shared_v4(a, uint32_t(w.b), uint32_t(w.u), uint32_t(w.qt), uint32_t(nkv));
                st_shared_v4(a + 16, uint32_t(kv0), uint32_t(hd.a), uint32_t(hd.b), uint32_t(hd.vh));
                st_shared_v4(a + 32, uint32_t(hd.n), (hd.b_noise ? 1u : 0u) | (hd.own ? 2u : 0u), 0u, 0u);
                mbar_arrive(bar(B_ITEM + slot));
            }
            if (item >= total) break;
            const CUtensorMap *mq2 = hd.b_noise ? &tm_q2 : &tm_q1;
            const CUtensorMap *mk2 = hd.b_noise ? &tm_k2 : &tm_k1;
            // Q waits until the previous tile's last score MMAs are done with
            // it.  The first two key steps' stages were last used by the
            // previous tile, so their loads go out first (often while that
            // tile still runs); a stage that this tile's own steps free is
            // only waited for once Q is on its way.
            auto load_q = [&]() -> bool {
                if (tiles > 0 && !mbar_wait_warp(bar(B_QFREE), (tiles - 1) & 1, abort_flag, lim)) return false;
                if (elect_one()) {
                    mbar_arrive_expect_tx(bar(B_QFULL), 2 * Q_BYTES);
                    tma_load_4d(sbase + OFF_Q1, &tm_q1, bar(B_QFULL), 0, w.qt * BM, hd.a, w.b, stream);
                    tma_load_4d(sbase + OFF_Q2, mq2, bar(B_QFULL), 0, w.qt * BM, hd.b, w.b, stream);
                }
                __syncwarp();
                ++q_loads;
                return true;
            };
            const int q_at = nkv < 2 ? nkv : 2;
            static_assert(STAGES > 2, "the steps loaded before Q must not depend on this tile");
            for (int j = 0; j < nkv; ++j, ++g) {
                if (j == q_at && !(ok = load_q())) break;
                const int s = g % STAGES;
                if (g >= STAGES &&
                    !(ok = mbar_wait_warp(bar_empty(s), ((g / STAGES) - 1) & 1, abort_flag, lim)))
                    break;
                const uint32_t st = sbase + OFF_STAGE0 + s * STAGE_BYTES;
                const int k0 = (kv0 + j) * BN;
                if (p.withhold_load && g == 0) continue;  // test hook: this stage never fills
                if (elect_one()) {
                    // Warm L2 with the K/V tiles of a later step of this tile
                    // (the stage ring alone cannot hide an HBM miss).
                    if (j + L2_PREFETCH_STEPS < nkv) {
                        const int kp = k0 + L2_PREFETCH_STEPS * BN;
                        tma_prefetch_l2_4d(&tm_k1, 0, kp, hd.a, w.b);
                        tma_prefetch_l2_4d(mk2, 0, kp, hd.b, w.b);
                        tma_prefetch_l2_4d(&tm_v, 0, kp, hd.vh, w.b);
                        tma_prefetch_l2_4d(&tm_v, 64, kp, hd.vh, w.b);
                    }
                    mbar_arrive_expect_tx(bar_full(s), STAGE_BYTES);
                    tma_load_4d(st, &tm_k1, bar_full(s), 0, k0, hd.a, w.b, keep);
                    tma_load_4d(st + K_BYTES, mk2, bar_full(s), 0, k0, hd.b, w.b, keep);
                    tma_load_4d(st + 2 * K_BYTES, &tm_v, bar_full(s), 0, k0, hd.vh, w.b, keep);
                    tma_load_4d(st + 2 * K_BYTES + VHALF_BYTES, &tm_v, bar_full(s), 64, k0, hd.vh, w.b, keep);
                }
                __syncwarp();
            }
            if (ok && q_at == nkv) ok = load_q();
            if (!ok) {
                ++tiles;
                break;
            }
        }
        // No load of ours may land after the CTA has gone: wait for all of them.
        bool drained = true;
        if (q_loads > 0) drained = mbar_wait_drain(bar(B_QFULL), (q_loads - 1) & 1, lim);
        for (int k = (g > STAGES ? g - STAGES : 0); k < g; ++k)
            if (!(p.withhold_load && k == 0))  // the withheld load was never issued
                drained &= mbar_wait_drain(bar_full(k % STAGES), (k / STAGES) & 1, lim);
        if (!__all_sync(0xffffffffu, drained) && lane == 0) *abort_flag = 1;
      } else if (warp == 1 || warp == 2) {
        // ------------------------------------------------------------ MMA issuers
        // Warp 1 issues map 1's MMAs, warp 2 map 2's.  The maps use disjoint
        // TMEM, so each warp only needs its own MMAs in order, and neither map
        // waits for the other's softmax.  The whole warp runs the loop
        // (descriptors stay warp-uniform); an elected lane issues.
        const int t = warp - 1;
        // Scores: bf16 x bf16, or f16 x f16 on rotated fp16 copies; both K-major.
        const uint32_t ID_S = p.qk_f16 ? idesc_f16(0, 0, 0, BM, BN) : idesc_f16(1, 1, 0, BM, BN);
        constexpr uint32_t ID_PV = idesc_f16(0, 0, 1, BM, HDV);  // f16 x f16, B (V) MN-major
        const uint32_t qa = sbase + (t ? OFF_Q2 : OFF_Q1);
        const uint32_t tS = tbase + (t ? TM_S2 : TM_S1), tO = tbase + (t ? TM_O2 : TM_O1);
        const uint32_t bar_pv = bar(B_PV + t);
        auto issue_s = [&](int s, int buf) {
            const uint32_t ka = sbase + OFF_STAGE0 + s * STAGE_BYTES + (t ? K_BYTES : 0);
#pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk) {
                if (elect_one())
                    mma_ss(tS + BN * buf, smem_desc_sw128(qa + 32 * kk, 16, 1024),
                           smem_desc_sw128(ka + 32 * kk, 16, 1024), ID_S, kk > 0);
                __syncwarp();
            }
        };
        auto issue_pv = [&](int s, int buf, bool acc) {
            const uint32_t va = sbase + OFF_STAGE0 + s * STAGE_BYTES + 2 * K_BYTES;
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) {
                if (elect_one())
                    mma_ts(tO, tS + BN * buf + 8 * kk, smem_desc_sw128(va + 2048 * kk, VHALF_BYTES, 1024),
                           ID_PV, (acc || kk > 0) ? 1u : 0u);
                __syncwarp();
            }
        };
        auto commit = [&](uint32_t b) {
            if (elect_one()) mma_commit(b);
            __syncwarp();
        };
        int g = 0;
        bool ok = true;
        // The next item is read during the current tile's last step (while
        // this warp waits for its P), so that the first score MMAs of the
        // next tile follow the tile's last P.V at once.
        Item nxt;
        bool have = read_item(0, nxt);
        for (int tiles = 0; have; ++tiles) {
            const int nkv = nxt.nkv;
            if (!(ok = mbar_wait_warp(bar(B_QFULL), tiles & 1, abort_flag, lim))) break;
            for (int jj = 0; jj < 2 && jj < nkv; ++jj) {
                const int gg = g + jj;
                if (!(ok = mbar_wait_warp(bar_full(gg % STAGES), (gg / STAGES) & 1, abort_flag, lim))) break;
                tc_fence_after();
                issue_s(gg % STAGES, gg & 1);
                commit(bar_s(t, gg & 1));
                if (jj == nkv - 1) commit(bar(B_QFREE));
            }
            for (int j = 0; ok && j < nkv; ++j) {
                const int gg = g + j, s = gg % STAGES, buf = gg & 1;
                if (j == nkv - 1) have = read_item(tiles + 1, nxt);
                if (!(ok = mbar_wait_warp(bar_p(t, buf), (gg >> 1) & 1, abort_flag, lim))) break;
                // The first P.V of a tile overwrites O: the previous tile's
                // epilogue must have read it.
                if (j == 0 && tiles > 0 &&
                    !(ok = mbar_wait_warp(bar(B_OFREE), (tiles - 1) & 1, abort_flag, lim)))
                    break;
                // Under a window V arrives in bf16 and warp 3 converts it.
                if (WINDOW && !(ok = mbar_wait_warp(bar(B_VCVT + s), (gg / STAGES) & 1, abort_flag, lim)))
                    break;
                tc_fence_after();
                issue_pv(s, buf, j > 0);
                commit(bar_pv);
                commit(bar_empty(s));  // the stage is free once both maps' P.V have read it
                if (j + 2 < nkv) {
                    const int g2 = gg + 2;
                    if (!(ok = mbar_wait_warp(bar_full(g2 % STAGES), (g2 / STAGES) & 1, abort_flag, lim)))
                        break;
                    tc_fence_after();
                    issue_s(g2 % STAGES, buf);
                    commit(bar_s(t, buf));
                    if (j + 2 == nkv - 1) commit(bar(B_QFREE));
                }
            }
            if (!ok) break;
            commit(bar(B_O));  // completes once both maps' MMAs of the tile are done
            g += nkv;
        }
        // Nothing of ours may still run on the tensor cores at teardown.
        commit(bar(B_PV + t));
        const bool drained = mbar_wait_drain(bar(B_PV + t), g & 1, lim);
        if (!__all_sync(0xffffffffu, drained) && lane == 0) *abort_flag = 1;
      } else if (WINDOW) {
        // ------------------------------------------------------------ V converter (window kernels)
        // A window tile has only a few key steps, so each V step is used by
        // about two tiles: converting it here, once per use, costs less than
        // a separate pass over all of V.  Each landed stage's V (bf16, in
        // the 128-byte swizzle) is rewritten in place as fp16 -- the swizzle
        // moves 16-byte chunks, so the layout is unchanged -- and released
        // to the P.V MMAs.
        int g = 0;
        bool ok = true, overflow = false;
        for (int tiles = 0;; ++tiles) {
            Item it;
            if (!read_item(tiles, it)) break;
            for (int j = 0; j < it.nkv; ++j, ++g) {
                const int s = g % STAGES;
                if (!(ok = mbar_wait_warp(bar_full(s), (g / STAGES) & 1, abort_flag, lim))) break;
                const uint32_t va = sbase + OFF_STAGE0 + s * STAGE_BYTES + 2 * K_BYTES;
                float big = 0.0f;
#pragma unroll 4
                for (int k = 0; k < int(V_BYTES / 16 / 32); ++k) {
                    const uint32_t a = va + 16u * (32u * k + lane);
                    const uint4 x = ld_shared_v4(a);
                    const uint32_t in[4] = {x.x, x.y, x.z, x.w};
                    uint32_t o[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float lo = __uint_as_float(in[e] << 16), hi = __uint_as_float(in[e] & 0xffff0000u);
                        big = fmaxf(big, fmaxf(fabsf(lo), fabsf(hi)));
                        o[e] = pack_half2(lo, hi);
                    }
                    st_shared_v4(a, o[0], o[1], o[2], o[3]);
                }
                overflow |= big > 65504.0f;
                // the generic-proxy writes, visible to the tensor cores' reads
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(B_VCVT + s));
            }
            if (!ok) break;
        }
        if (__any_sync(0xffffffffu, overflow) && lane == 0) report_error(p.dev_status, DIFFATTN_ERR_UNSUPPORTED);
      }
    } else if (warp < 12) {
        regs_increase<REGS_SOFTMAX>();
        // ------------------------------------------------------------ softmax
        const int t = (warp >= 8) ? 1 : 0;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
        const uint32_t tS0 = tbase + lane_off + (t ? TM_S2 : TM_S1);
        const uint32_t tO = tbase + lane_off + (t ? TM_O2 : TM_O1);
        const uint32_t bar_pv = bar(B_PV + t);
        int g = 0;
        bool ok = true;
        for (int tiles = 0;; ++tiles) {
            Item it;
            if (!read_item(tiles, it)) break;
            const Work w = it.w;
            const int nkv = it.nkv, kv0 = it.kv0;
            const int qrow = w.qt * BM + r;
            float m_run = -INFINITY, l_run = 0.0f;
            for (int j = 0; j < nkv; ++j) {
                const int gg = g + j, buf = gg & 1;
                if (!(ok = mbar_wait_warp(bar_s(t, buf), (gg >> 1) & 1, abort_flag, lim))) break;
                tc_fence_after();
                const int k0 = (kv0 + j) * BN;
                const int hi = p.causal ? qrow - k0 : p.N - 1 - k0;
                const int lo = WINDOW ? qrow - p.window + 1 - k0 : INT_MIN;
                if (!(ok = softmax_step<WINDOW>(tS0 + BN * buf, tO, j == 0, lo, hi, p.scale_log2, m_run, l_run,
                                        bar_pv, (gg - 1) & 1, abort_flag, lim)))
                    break;
                // Every lane's P store has completed (tcgen05.wait::st in the
                // step); after the warp sync one arrival stands for the warp.
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_p(t, buf));
            }
            if (!ok) break;
            g += nkv;
            if constexpr (SAVE) {
                // Saved for the backward pass: this map's lse = m + log2(l)
                // (the running max and sum are in units of scale * log2(e) *
                // score), at float 2 * 128 * 128 + 128 t + r of the tile's state.
                const int head = it.hd.a;
                p.save[((size_t)(w.b * p.H + head) * p.num_qt + w.qt) * kSaveTileFloats + 2 * BM * HDV + t * BM + r] =
                    m_run + log2f(l_run);
            }
            // The row's running sum goes to the epilogue warps, in the slot of
            // the tile's parity.  The epilogue reads the slot before it
            // releases O; this warp writes the slot again two tiles later,
            // after the MMA warps have waited for that release.
            sStat[(tiles & 1) * (2 * BM) + t * BM + r] = l_run;
            __syncwarp();  // every lane's sum is written: one arrival for the warp
            if (lane == 0) mbar_arrive(bar(B_STAT + (tiles & 1)));
        }
    } else {
        regs_increase<REGS_EPI>();
        // ------------------------------------------------------------ epilogue
        // Warp 12 + e finishes tile rows 32 e .. 32 e + 31 (its TMEM lanes)
        // over all 128 output columns, while the softmax warps run the next
        // tile.  Per item it waits for the softmax warps' row sums and for
        // the tile's last P.V, reads O1 and O2, and writes the output rows.
        const int ew = warp & 3;
        const int r = 32 * ew + lane;
        const uint32_t lane_off = uint32_t(32 * ew) << 16;
        const uint32_t tO1 = tbase + lane_off + TM_O1, tO2 = tbase + lane_off + TM_O2;
        // This warp's 16 KB of shared memory: the staged output boxes (two 32
        // x 64 bf16 boxes per output head, 128-byte swizzle) and, in a
        // one-head item, first D itself in fp32.
        const uint32_t wbuf = sbase + OFF_OUT + ew * EPI_WARP_BYTES;
        // 16-byte chunk ch of row `lane` of an output box (the TMA swizzle).
        auto box_at = [&](uint32_t box, int ch) { return box + 128 * lane + ((ch ^ (lane & 7)) << 4); };
        const uint32_t abar = bar(B_AN + ew);  // this warp's A_N copies landed
        int an_loads = 0;
        bool ok = true;
        for (int tiles = 0;; ++tiles) {
            Item it;
            if (!read_item(tiles, it)) break;
            const Work w = it.w;
            const Heads hd = it.hd;
            const bool own = hd.own;
            const int qrow = w.qt * BM + r;
            const int64_t qrow_c = min(qrow, p.N - 1);
            const int r0 = w.qt * BM + 32 * ew;  // first row of this warp's boxes
            // The per-item inputs of the epilogue -- lambda (per head, or the
            // token-dependent logit of this row), the gain rows, the gate
            // logits' rows -- are loaded or prefetched now: the wait below
            // hides their latency.
            auto lam_load = [&](int head) {
                return ld_early_f32(p.lam_logits ? p.lam_logits + w.b * p.ll_sb + qrow_c * p.ll_sn + head * p.ll_sh
                                                 : p.lambda + head);
            };
            const float lam_a = lam_load(hd.a);
            const float lam_b = own ? lam_load(hd.b) : 0.0f;
            const float *gain_a = p.gain ? p.gain + (size_t)hd.a * HDV : nullptr;
            const float *gain_b = p.gain ? p.gain + (size_t)hd.b * HDV : nullptr;
            if (gain_a && lane < 4) prefetch_l1(gain_a + 32 * lane);
            if (own && gain_b && lane < 4) prefetch_l1(gain_b + 32 * lane);
            const uint4 *gate_a = nullptr, *gate_b = nullptr;  // this row's 128 logits: 16 chunks of 8
            if constexpr (GATED) {
                const __nv_bfloat16 *g0 =
                    static_cast<const __nv_bfloat16 *>(p.gate) + w.b * p.gate_sb + qrow_c * p.gate_sn;
                gate_a = reinterpret_cast<const uint4 *>(g0 + hd.a * p.gate_sh);
                prefetch_l2(gate_a);
                prefetch_l2(gate_a + 8);
                if (own) {
                    gate_b = reinterpret_cast<const uint4 *>(g0 + hd.b * p.gate_sh);
                    prefetch_l2(gate_b);
                    prefetch_l2(gate_b + 8);
                }
            }
            const size_t noise_tile = ((size_t)w.b * p.H_N + hd.n) * p.num_qt + w.qt;
            // Gain times output gate for 16 columns (16 c ..) of one head; gq:
            // the gate logits of those columns, loaded one step ahead.
            auto scale16 = [&](const float *gain, const uint4 (&gq)[2], int c, float (&gv)[16]) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float4 g4 = gain ? __ldg(reinterpret_cast<const float4 *>(gain) + 4 * c + k)
                                           : make_float4(1.f, 1.f, 1.f, 1.f);
                    gv[4 * k] = g4.x;
                    gv[4 * k + 1] = g4.y;
                    gv[4 * k + 2] = g4.z;
                    gv[4 * k + 3] = g4.w;
                }
                if constexpr (GATED) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t qw[4] = {gq[h].x, gq[h].y, gq[h].z, gq[h].w};
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            gv[8 * h + 2 * k] *= logistic_tanh(__uint_as_float(qw[k] << 16));
                            gv[8 * h + 2 * k + 1] *= logistic_tanh(__uint_as_float(qw[k] & 0xffff0000u));
                        }
                    }
                }
            };
            // Row sums of the tile, from the softmax warps.
            if (!(ok = mbar_wait_warp(bar(B_STAT + (tiles & 1)), (tiles >> 1) & 1, abort_flag, lim))) break;
            const float l1 = sStat[(tiles & 1) * (2 * BM) + r], l2 = sStat[(tiles & 1) * (2 * BM) + BM + r];
            // The previous item's output stores must have read the buffer.
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
            if (!own) {
                // -------------------------------------------- one output head
                // D = (O1 - r2 O2) / l1 with r2 = lambda l1 / l2 (identical
                // maps with lambda = 1 cancel exactly), then the RMS norm over
                // the row's 128 columns, gain, gate, bf16.
                if (!(ok = mbar_wait_warp(bar(B_O), tiles & 1, abort_flag, lim))) break;
                tc_fence_after();
                const float lam = p.lam_logits ? logistic_fast(lam_a) : lam_a;
                const float inv1 = 1.0f / l1, inv2 = 1.0f / l2, r2 = lam * l1 / l2;
                const uint32_t drow = wbuf + 64 * lane;
                const int rot = (lane >> 1) & 3;
                float4 *sa = SAVE ? reinterpret_cast<float4 *>(p.save + ((size_t)(w.b * p.H + hd.a) * p.num_qt + w.qt) *
                                                                            kSaveTileFloats) + r
                                  : nullptr;
                float4 *an = p.mode == 1
                                 ? reinterpret_cast<float4 *>(p.noise_out) + noise_tile * (HDV / 4) * BM + r
                                 : nullptr;
                float ss = 0.0f;
#pragma unroll 2
                for (int c = 0; c < 8; ++c) {
                    uint32_t oa[16], ob[16];
                    tmem_ld16(tO1 + 16 * c, oa);
                    tmem_ld16(tO2 + 16 * c, ob);
                    tmem_wait_ld();
                    if (c == 7) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(B_OFREE));
                    }
                    float d[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        d[i] = fmaf(-r2, __uint_as_float(ob[i]), __uint_as_float(oa[i]));
                        ss = fmaf(d[i], d[i], ss);
                    }
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        st_shared_v4(drow + 2048 * c + ((k ^ rot) << 4), __float_as_uint(d[4 * k]),
                                     __float_as_uint(d[4 * k + 1]), __float_as_uint(d[4 * k + 2]),
                                     __float_as_uint(d[4 * k + 3]));
                    if constexpr (SAVE) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            sa[(4 * c + k) * BM] = make_float4(
                                __uint_as_float(oa[4 * k]) * inv1, __uint_as_float(oa[4 * k + 1]) * inv1,
                                __uint_as_float(oa[4 * k + 2]) * inv1, __uint_as_float(oa[4 * k + 3]) * inv1);
                            sa[(32 + 4 * c + k) * BM] = make_float4(
                                __uint_as_float(ob[4 * k]) * inv2, __uint_as_float(ob[4 * k + 1]) * inv2,
                                __uint_as_float(ob[4 * k + 2]) * inv2, __uint_as_float(ob[4 * k + 3]) * inv2);
                        }
                    }
                    if (an) {
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            an[(4 * c + k) * BM] = make_float4(
                                __uint_as_float(ob[4 * k]) * inv2, __uint_as_float(ob[4 * k + 1]) * inv2,
                                __uint_as_float(ob[4 * k + 2]) * inv2, __uint_as_float(ob[4 * k + 3]) * inv2);
                    }
                }
                ss *= inv1 * inv1;
                const float rn = (p.apply_norm ? rsqrtf(ss * (1.0f / HDV) + p.eps) : 1.0f) * inv1;
                // Pass 2, 32 columns at a time: D' back from shared memory,
                // normalised, scaled and rounded to bf16 into the output boxes,
                // which overlay the first 8 KB of the buffer: box half h holds
                // columns 64 h .. 64 h + 63 over D chunks 2 h and 2 h + 1.
                // Columns 32 q .. 32 q + 31 go to box half q / 2, whose D chunks
                // every lane has read by then (this pass or the one before),
                // hence the warp sync between the reads and the writes.
                uint4 gcur[2][2], gnext[2][2];  // gate logits of columns 32 q .. 32 q + 31, then of the next q
                if constexpr (GATED) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        gcur[h][0] = __ldg(gate_a + 2 * h);
                        gcur[h][1] = __ldg(gate_a + 2 * h + 1);
                    }
                }
#pragma unroll 1
                for (int q = 0; q < 4; ++q) {
                    if (GATED && q < 3) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            gnext[h][0] = __ldg(gate_a + 4 * (q + 1) + 2 * h);
                            gnext[h][1] = __ldg(gate_a + 4 * (q + 1) + 2 * h + 1);
                        }
                    }
                    float d[2][16];
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint4 v = ld_shared_v4(drow + 2048 * (2 * q + h) + ((k ^ rot) << 4));
                            d[h][4 * k] = __uint_as_float(v.x);
                            d[h][4 * k + 1] = __uint_as_float(v.y);
                            d[h][4 * k + 2] = __uint_as_float(v.z);
                            d[h][4 * k + 3] = __uint_as_float(v.w);
                        }
                    __syncwarp();
                    const uint32_t box = wbuf + (q >> 1) * OUT_HALF_BYTES;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float gv[16];
                        scale16(gain_a, gcur[h], 2 * q + h, gv);
                        uint32_t y[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            y[i] = pack_bf162(d[h][2 * i] * rn * gv[2 * i], d[h][2 * i + 1] * rn * gv[2 * i + 1]);
                        const int ch = 4 * (q & 1) + 2 * h;  // 16-byte chunk of the box row
                        st_shared_v4(box_at(box, ch), y[0], y[1], y[2], y[3]);
                        st_shared_v4(box_at(box, ch + 1), y[4], y[5], y[6], y[7]);
                    }
                    if constexpr (GATED) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            gcur[h][0] = gnext[h][0];
                            gcur[h][1] = gnext[h][1];
                        }
                    }
                }
            } else {
                // -------------------------------------------- pair item
                // Two output heads, one per map: D_h = O_h / l_h - lambda_h A_N
                // with A_N the group's normalised noise output (written by the
                // tile's export item), then each head's RMS norm.  This warp's
                // 32 rows of A_N (16 KB) come into its buffer by bulk copies,
                // 512 contiguous bytes per float4 chunk (chunk j of row `lane`
                // at 512 j + 16 lane).  O is read twice (sums of squares, then
                // the output) and released after the second read; the output
                // rows go straight from registers to global memory.
                bool ready = true;
                if (lane == 0) ready = wait_flag_geq(p.noise_ready + noise_tile, 4, abort_flag, lim);
                if (!(ok = __shfl_sync(0xffffffffu, ready, 0))) break;
                // The buffer's last generic-proxy reads and writes (the previous
                // item's) come before the copies into it; the acquired A_N
                // comes before the copies' reads of it.
                fence_proxy_async_smem();
                __syncwarp();
                if (elect_one()) {
                    fence_proxy_async_global();
                    const float4 *src = reinterpret_cast<const float4 *>(p.noise_out) + noise_tile * (HDV / 4) * BM +
                                        32 * ew;
                    mbar_arrive_expect_tx(abar, 32 * 512);
                    for (int j = 0; j < 32; ++j) bulk_load_g2s(wbuf + 512 * j, src + j * BM, 512, abar);
                }
                __syncwarp();
                ++an_loads;
                if (!(ok = mbar_wait_warp(bar(B_O), tiles & 1, abort_flag, lim))) break;
                tc_fence_after();
                if (!(ok = mbar_wait_warp(abar, (an_loads - 1) & 1, abort_flag, lim))) break;
                const float la = p.lam_logits ? logistic_fast(lam_a) : lam_a;
                const float lb = p.lam_logits ? logistic_fast(lam_b) : lam_b;
                const float inv1 = 1.0f / l1, inv2 = 1.0f / l2;
                // D_h' = O_h - (lambda_h l_h) A_N = l_h D_h: one fused
                // multiply-add per element; 1 / l_h goes into the output scale.
                const float2 ka = make_float2(-la * l1, -la * l1), kb = make_float2(-lb * l2, -lb * l2);
                auto an16 = [&](int c, float (&av)[16]) {  // A_N of columns 16 c .. 16 c + 15
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint4 v = ld_shared_v4(wbuf + 512 * (4 * c + k) + 16 * lane);
                        av[4 * k] = __uint_as_float(v.x);
                        av[4 * k + 1] = __uint_as_float(v.y);
                        av[4 * k + 2] = __uint_as_float(v.z);
                        av[4 * k + 3] = __uint_as_float(v.w);
                    }
                };
                float2 ssa2 = make_float2(0.0f, 0.0f), ssb2 = make_float2(0.0f, 0.0f);
#pragma unroll 1
                for (int c2 = 0; c2 < 4; ++c2) {  // pass 1, 32 columns at a time
                    uint32_t oa[32], ob[32];
                    tmem_ld32(tO1 + 32 * c2, oa);
                    tmem_ld32(tO2 + 32 * c2, ob);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float av[16];
                        an16(2 * c2 + h, av);
                        if (h == 0) tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float2 a2 = make_float2(av[2 * i], av[2 * i + 1]);
                            const float2 da = ffma2(a2, ka, make_float2(__uint_as_float(oa[16 * h + 2 * i]),
                                                                        __uint_as_float(oa[16 * h + 2 * i + 1])));
                            const float2 db = ffma2(a2, kb, make_float2(__uint_as_float(ob[16 * h + 2 * i]),
                                                                        __uint_as_float(ob[16 * h + 2 * i + 1])));
                            ssa2 = ffma2(da, da, ssa2);
                            ssb2 = ffma2(db, db, ssb2);
                        }
                    }
                }
                const float rna = (p.apply_norm ? rsqrtf((ssa2.x + ssa2.y) * inv1 * inv1 * (1.0f / HDV) + p.eps) : 1.0f) * inv1;
                const float rnb = (p.apply_norm ? rsqrtf((ssb2.x + ssb2.y) * inv2 * inv2 * (1.0f / HDV) + p.eps) : 1.0f) * inv2;
                const bool row_ok = qrow < p.N;
                __nv_bfloat16 *out_row = static_cast<__nv_bfloat16 *>(p.out) + w.b * p.out_sb + qrow_c * p.out_sn;
                uint4 gcur[2][2], gnext[2][2];  // [head][half]: gate logits of the current / next chunk
                if constexpr (GATED) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        gcur[0][h] = __ldg(gate_a + h);
                        gcur[1][h] = __ldg(gate_b + h);
                    }
                }
#pragma unroll 1
                for (int c = 0; c < 8; ++c) {
                    uint32_t oa[16], ob[16];
                    tmem_ld16(tO1 + 16 * c, oa);
                    tmem_ld16(tO2 + 16 * c, ob);
                    if (GATED && c < 7) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            gnext[0][h] = __ldg(gate_a + 2 * (c + 1) + h);
                            gnext[1][h] = __ldg(gate_b + 2 * (c + 1) + h);
                        }
                    }
                    float av[16];
                    an16(c, av);
                    tmem_wait_ld();
                    if (c == 7) {  // every lane has read all of O: release it, once per warp
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(B_OFREE));
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t *o = h ? ob : oa;
                        const float2 kl = h ? kb : ka;
                        const float rn = h ? rnb : rna;
                        float gv[16];
                        scale16(h ? gain_b : gain_a, gcur[h], c, gv);
                        uint32_t y[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float2 dd = ffma2(make_float2(av[2 * i], av[2 * i + 1]), kl,
                                                    make_float2(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1])));
                            y[i] = pack_bf162(dd.x * rn * gv[2 * i], dd.y * rn * gv[2 * i + 1]);
                        }
                        if (row_ok) {
                            uint4 *dst = reinterpret_cast<uint4 *>(out_row + (h ? hd.b : hd.a) * p.out_sh + 16 * c);
                            dst[0] = make_uint4(y[0], y[1], y[2], y[3]);
                            dst[1] = make_uint4(y[4], y[5], y[6], y[7]);
                        }
                    }
                    if constexpr (GATED) {
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            gcur[h][0] = gnext[h][0];
                            gcur[h][1] = gnext[h][1];
                        }
                    }
                }
            }
            if (!own) {
                // The staged boxes go out by TMA (rows past N are clipped; a
                // box wholly past N is not issued).
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && r0 < p.N) {
                    tma_store_4d(&tm_out, wbuf, 0, r0, hd.a, w.b);
                    tma_store_4d(&tm_out, wbuf + OUT_HALF_BYTES, 64, r0, hd.a, w.b);
                    bulk_commit_group();
                }
            }
            if (p.mode == 1 && !own) {
                // Publish this warp's rows of the noise output (stored in pass
                // 1, so the stores have had pass 2 to drain): every lane's
                // stores, then one release per warp; the pair items wait for
                // all four epilogue warps of the tile.
                __syncwarp();
                if (lane == 0) {
                    __threadfence();
                    atomicAdd(p.noise_ready + noise_tile, 1);
                }
            }
        }
        // No copy of ours may land after the CTA has gone.
        if (an_loads > 0 && !__all_sync(0xffffffffu, mbar_wait_drain(abar, (an_loads - 1) & 1, lim)) && lane == 0)
            *abort_flag = 1;
    }

    if (warp >= 12 && lane == 0) bulk_wait_all();  // output stores done before the CTA exits
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) report_error(p.dev_status, DIFFATTN_ERR_TIMEOUT);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, TMEM_COLS);
    }
}

__global__ void v_to_f16_kernel(const __nv_bfloat16 *__restrict__ v, int64_t sb, int64_t sn,
                                int64_t sh, __half *__restrict__ dst, int B, int N, int H_V,
                                int32_t *dev_status, int *tile_counter, int *zero, int64_t n_zero,
                                const RopeStage rope, int stage_v)
{
    // The prefill launch that follows may become resident and run its
    // prologue now; it waits for this kernel to finish before reading.
    grid_launch_dependents();
    // The prefill launches that follow on the stream hand out their work
    // items from these two counters (one per launch), and the grouped pairs
    // count their exports in `zero`.
    if (blockIdx.x == 0 && threadIdx.x < 2) tile_counter[threadIdx.x] = 0;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n_zero;
         i += (int64_t)gridDim.x * blockDim.x)
        zero[i] = 0;
    // One thread per 8 consecutive V elements (16 bytes in, 16 bytes out).
    // A dense V ([B, N, H_V, 128] with no gaps, the common case) is one flat
    // array, so its chunk i needs no index arithmetic, and each thread keeps
    // four loads in flight; otherwise chunk i is decomposed into (b, n, head,
    // column) -- 64-bit divisions that made the pass compute-bound.
    const int64_t total = stage_v ? (int64_t)B * N * H_V * (HDV / 8) : 0;
    const bool dense = sh == HDV && sn == (int64_t)H_V * HDV && sb == (int64_t)N * H_V * HDV;
    bool overflow = false;
    auto to_f16 = [&](const uint4 src) {
        const uint32_t in[4] = {src.x, src.y, src.z, src.w};
        uint32_t out[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162 *>(&in[k]);
            const float2 f = __bfloat1622float2(x);
            overflow |= fabsf(f.x) > 65504.0f || fabsf(f.y) > 65504.0f;
            out[k] = pack_half2(f.x, f.y);
        }
        return make_uint4(out[0], out[1], out[2], out[3]);
    };
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (dense) {
        const uint4 *src = reinterpret_cast<const uint4 *>(v);
        uint4 *out = reinterpret_cast<uint4 *>(dst);
        for (; i + 3 * stride < total; i += 4 * stride) {
            uint4 x[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) x[u] = __ldcs(src + i + u * stride);  // read once: streaming
#pragma unroll
            for (int u = 0; u < 4; ++u) out[i + u * stride] = to_f16(x[u]);
        }
        for (; i < total; i += stride) out[i] = to_f16(__ldcs(src + i));
    } else {
        for (; i < total; i += stride) {
            const int c8 = int(i % (HDV / 8));
            const int64_t row = i / (HDV / 8);
            const int hv = int(row % H_V);
            const int64_t bn = row / H_V;
            const int n = int(bn % N), b = int(bn / N);
            const int64_t off = b * sb + n * sn + hv * sh + 8 * c8;
            reinterpret_cast<uint4 *>(dst)[i] = to_f16(__ldg(reinterpret_cast<const uint4 *>(v + off)));
        }
    }
    if (overflow) report_error(dev_status, DIFFATTN_ERR_UNSUPPORTED);
    if (!rope.enabled) return;
    // Rotary embedding of Q1, K1, Q2, K2 (Motif 2.6B explainer, "The block"):
    // one thread per 8 consecutive elements = 4 interleaved pairs of a 64-wide
    // row, written as fp16 (2^-11 rounding: bf16 copies added enough logit
    // error to break the mean tolerance).  The angle n g[c] 2 pi is reduced to a fraction of a turn in double
    // precision (n up to 2^24), so the float sincos sees an angle in [-pi, pi).
    for (int t = 0; t < 4; ++t) {
        const int heads = rope.heads[t];
        const int64_t tot = (int64_t)B * N * heads * 8;
        const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(rope.src[t]);
        uint4 *out = static_cast<uint4 *>(rope.dst[t]);
        const bool qk_dense = rope.sh[t] == 64 && rope.sn[t] == (int64_t)heads * 64 &&
                              rope.sb[t] == (int64_t)N * heads * 64;
        for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < tot;
             i += (int64_t)gridDim.x * blockDim.x) {
            const int c8 = int(i & 7);
            const int64_t row = i >> 3;
            // the token position n is needed for the angle in any case; the
            // source offset needs the full decomposition only when not dense
            const int64_t bn = row / heads;
            const int n = int(bn % N);
            int64_t off = 8 * i;
            if (!qk_dense) {
                const int h = int(row - bn * heads), b = int(bn / N);
                off = b * rope.sb[t] + n * rope.sn[t] + h * rope.sh[t] + 8 * c8;
            }
            const uint4 x = __ldg(reinterpret_cast<const uint4 *>(src + off));
            const uint32_t in[4] = {x.x, x.y, x.z, x.w};
            uint32_t o[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const double turns = (double)n * rope.g[4 * c8 + k];
                const float frac = (float)(turns - rint(turns));  // in [-1/2, 1/2]
                float sn_, cs;  // |angle| <= pi: the fast intrinsic errs by ~2^-21, below fp16 rounding
                __sincosf(6.283185307179586f * frac, &sn_, &cs);
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&in[k]));
                const float r0 = f.x * cs - f.y * sn_, r1 = f.x * sn_ + f.y * cs;
                overflow |= fabsf(r0) > 65504.0f || fabsf(r1) > 65504.0f;
                o[k] = pack_half2(r0, r1);
            }
            out[i] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
    if (overflow) report_error(dev_status, DIFFATTN_ERR_UNSUPPORTED);
}

}  // namespace

cudaError_t launch_prefill(const CUtensorMap &q1, const CUtensorMap &q2, const CUtensorMap &k1,
                           const CUtensorMap &k2, const CUtensorMap &v16, const CUtensorMap &out,
                           const PrefillParams &p,
                           cudaStream_t stream, int *launches)
{
    // Per device, once (first calls from several host threads serialise on
    // the mutex): the kernel attributes.
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
      std::lock_guard<std::mutex> lock(attr_mutex);
      if (!attr_set[dev].load(std::memory_order_relaxed)) {
        // The register split inside the kernel is only valid for a build that
        // launches with exactly REGS_LAUNCH registers per thread: with fewer,
        // the softmax warpgroups' increase could never be granted.  Refuse to
        // launch such a build.
        for (const void *k : {(const void *)prefill_kernel<false, false, false>,
                              (const void *)prefill_kernel<true, false, false>,
                              (const void *)prefill_kernel<false, true, false>,
                              (const void *)prefill_kernel<true, true, false>,
                              (const void *)prefill_kernel<false, false, true>,
                              (const void *)prefill_kernel<true, false, true>,
                              (const void *)prefill_kernel<false, true, true>,
                              (const void *)prefill_kernel<true, true, true>}) {
            cudaFuncAttributes fa;
            e = cudaFuncGetAttributes(&fa, k);
            if (e != cudaSuccess) return e;
            if (fa.numRegs != REGS_LAUNCH || fa.maxThreadsPerBlock < NTHREADS) {
                set_internal_error("prefill_kernel built with an unexpected register count");
                return cudaErrorInvalidConfiguration;
            }
            e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
            if (e != cudaSuccess) return e;
        }
        attr_set[dev].store(true, std::memory_order_release);
      }
    }
    const int sms = device_sm_count();
    const int total = p.B * p.units * p.num_qt * (p.mode == 1 ? p.pairs + 1 : 1);
    if (total == 0) return cudaSuccess;
    const int grid = total < sms ? total : sms;  // persistent: one CTA per SM
    using Kernel = decltype(&prefill_kernel<false, false, false>);
    static const Kernel kernels[2][2][2] = {  // [save][gate][window]
        {{prefill_kernel<false, false, false>, prefill_kernel<true, false, false>},
         {prefill_kernel<false, true, false>, prefill_kernel<true, true, false>}},
        {{prefill_kernel<false, false, true>, prefill_kernel<true, false, true>},
         {prefill_kernel<false, true, true>, prefill_kernel<true, true, true>}}};
    const Kernel kernel = kernels[p.save != nullptr][p.gate != nullptr][p.window > 0];
    // Programmatic dependent launch: the prologue (barriers, TMEM) overlaps
    // the tail of the kernel before it; the kernel waits (griddepcontrol)
    // before touching that kernel's results.
    cudaLaunchAttribute attr{};
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = stream;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    cudaError_t le = cudaLaunchKernelEx(&cfg, kernel, q1, q2, k1, k2, v16, out, p);
    if (le != cudaSuccess) return le;
    ++*launches;
    return cudaGetLastError();
}

cudaError_t launch_v_to_f16(const void *v, int64_t sb, int64_t sn, int64_t sh, void *dst, int B,
                            int N, int H_V, int32_t *dev_status, int *tile_counter,
                            int *zero, int64_t n_zero, const RopeStage &rope, int sm_count,
                            cudaStream_t stream, int *launches, bool stage_v)
{
    const int64_t total = (int64_t)B * N * H_V * (HDV / 8);
    if (total == 0) return cudaSuccess;  // nothing to stage; the prefill is skipped too
    const int threads = 256;
    // Without the V copy (and without RoPE) only the counters are cleared.
    const int64_t work = stage_v || rope.enabled ? total : (n_zero > 0 ? n_zero : 1);
    int blocks = (int)((work + threads - 1) / threads);
    if (blocks > sm_count * 8) blocks = sm_count * 8;  // resident at once (2048 threads per SM); grid-stride beyond
    v_to_f16_kernel<<<blocks, threads, 0, stream>>>(static_cast<const __nv_bfloat16 *>(v), sb, sn,
                                                    sh, static_cast<__half *>(dst), B, N, H_V,
                                                    dev_status, tile_counter, zero, n_zero, rope,
                                                    stage_v ? 1 : 0);
    ++*launches;
    return cudaGetLastError();
}

}  // namespace da
