// decode.cu -- single-query differential-attention decode on sm_100a.
//
// The query of sequence b sits at position kv_len[b]-1 and attends to every
// cached key 0..kv_len[b]-1 of both maps; the two softmax-weighted V sums are
// subtracted and normalised as in the prefill (Motif 2.6B explainer, section
// "Differential attention" and figure 1).  One token reads the whole cache
// once (K1, K2: 128 B per key; V: 256 B per key), so the path is bound by HBM
// bandwidth, not arithmetic.
//
// split kernel   grid = B*H*splits, 256 threads.  Each CTA streams one chunk
//                of keys of one (b, h) with 128-bit non-allocating loads:
//                  phase 1  logits of both maps (8 lanes per key, shuffles)
//                           into shared memory;
//                  phase 2  chunk max and exp2 weights, chunk sums;
//                  phase 3  weighted V sums (16 lanes per key row, 8 columns
//                           per lane), reduced across the CTA;
//                and writes the partial state (m1, l1, m2, l2, acc1, acc2) of
//                the chunk.  Logits are kept in the log2 domain.
// combine kernel grid = B*H, 128 threads (one per V column): merges the
//                chunks (m = max m_s, l = sum l_s 2^(m_s - m), same for acc),
//                then D = acc1/l1 - lambda acc2/l2, RMS norm, gain, the optional
//                output gate sigma(G) (lambda optionally sigma of a per-token
//                logit; Motif 3 summary, section 2.2), bf16.
#include <cuda_bf16.h>

#include <mutex>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace da {

// Partial-state storage for diffattn_decode_noalloc, for callers that cannot
// hand the library a workspace.  It lives in the module's static device
// memory, so every GPU that loads this library holds it until the process
// exits, and every no-allocation call on a device shares it.
static __device__ __align__(256) float g_decode_scratch[kNoAllocScratchBytes / sizeof(float)];

namespace {

constexpr int DHDV = 128;
constexpr int SPLIT_THREADS = 256;
constexpr int PF = kDecodePartialFloats;

__device__ __forceinline__ uint4 ld_stream(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void bf16x8_to_float(const uint4 &u, float (&f)[8])
{
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[k]));
        f[2 * k] = t.x;
        f[2 * k + 1] = t.y;
    }
}

__device__ __forceinline__ float warp_max(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Reduce two values across the CTA (max or sum); every thread gets results.
template <bool IS_MAX>
__device__ __forceinline__ float2 block_reduce2(float a, float b, float *scratch)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    a = IS_MAX ? warp_max(a) : warp_sum(a);
    b = IS_MAX ? warp_max(b) : warp_sum(b);
    __syncthreads();
    if (lane == 0) {
        scratch[warp] = a;
        scratch[32 + warp] = b;
    }
    __syncthreads();
    a = scratch[0];
    b = scratch[32];
    for (int i = 1; i < nw; ++i) {
        a = IS_MAX ? fmaxf(a, scratch[i]) : a + scratch[i];
        b = IS_MAX ? fmaxf(b, scratch[32 + i]) : b + scratch[32 + i];
    }
    return make_float2(a, b);
}

// WINDOW: the kernel of sliding-window calls.  The unwindowed kernel keeps
// the window offset out: with it, the kernel needed 88 registers, fit two CTAs
// per SM instead of three and lost 12 % of its bandwidth (measured).
template <bool WINDOW>
__global__ void __launch_bounds__(SPLIT_THREADS)
    decode_split_kernel(const DecodeParams p)
{
    extern __shared__ float dsm[];
    float *z1 = dsm;                 // [chunk] logits, then weights, of map 1
    float *z2 = dsm + p.chunk;       // [chunk] of map 2
    float *red = dsm + 2 * p.chunk;  // [16][2][128] partial V sums
    __shared__ float scratch[64];

    const int split = blockIdx.x % p.splits;
    const int bh = blockIdx.x / p.splits;
    const int b = bh / p.H, h = bh % p.H;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    int kv = p.L;
    if (p.kv_len) {
        kv = p.kv_len[b];
        if (kv < 1 || kv > p.L) {
            if (tid == 0 && split == 0) report_error(p.dev_status, DIFFATTN_ERR_INVALID_ARG);
            kv = kv < 0 ? 0 : (kv > p.L ? p.L : kv);
        }
    }
    // Under a window the keys start at kv - window.
    const int kv_lo = (WINDOW && kv > p.window) ? kv - p.window : 0;
    const int k_begin = kv_lo + split * p.chunk;
    const int n = max(0, min(p.chunk, kv - k_begin));
    float *out = p.partials + ((size_t)bh * p.splits + split) * PF;

    if (n == 0) {
        for (int i = tid; i < PF; i += SPLIT_THREADS) out[i] = (i == 0 || i == 2) ? -INFINITY : 0.0f;
        return;
    }

    // ---- phase 1: logits.  Lane group g = lane / 8 owns one key, part = lane % 8
    // owns dims [8 part, 8 part + 8).
    const int part = lane & 7, g = lane >> 3;
    float q1f[8], q2f[8];
    {
        const __nv_bfloat16 *q1 = static_cast<const __nv_bfloat16 *>(p.q1) + b * p.q1_sb + h * p.q1_sh;
        const __nv_bfloat16 *q2 = static_cast<const __nv_bfloat16 *>(p.q2) + b * p.q2_sb + h * p.q2_sh;
        bf16x8_to_float(*reinterpret_cast<const uint4 *>(q1 + 8 * part), q1f);
        bf16x8_to_float(*reinterpret_cast<const uint4 *>(q2 + 8 * part), q2f);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            q1f[e] *= p.scale_log2;
            q2f[e] *= p.scale_log2;
        }
    }
    const __nv_bfloat16 *k1 = static_cast<const __nv_bfloat16 *>(p.k1) + b * p.k1_sb + h * p.k1_sh +
                              (int64_t)k_begin * p.k1_sl + 8 * part;
    const __nv_bfloat16 *k2 = static_cast<const __nv_bfloat16 *>(p.k2) + b * p.k2_sb + h * p.k2_sh +
                              (int64_t)k_begin * p.k2_sl + 8 * part;
    constexpr int KEYS_PER_PASS = SPLIT_THREADS / 8;  // 32 keys per CTA pass
    constexpr int U1 = 4;
    for (int base = 0; base < n; base += KEYS_PER_PASS * U1) {
        uint4 a[U1], c[U1];
#pragma unroll
        for (int u = 0; u < U1; ++u) {
            const int key = base + u * KEYS_PER_PASS + warp * 4 + g;
            if (key < n) {
                a[u] = ld_stream(k1 + (int64_t)key * p.k1_sl);
                c[u] = ld_stream(k2 + (int64_t)key * p.k2_sl);
            }
        }
#pragma unroll
        for (int u = 0; u < U1; ++u) {
            const int key = base + u * KEYS_PER_PASS + warp * 4 + g;
            float s1 = 0.0f, s2 = 0.0f;
            if (key < n) {
                float f[8];
                bf16x8_to_float(a[u], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) s1 = fmaf(q1f[e], f[e], s1);
                bf16x8_to_float(c[u], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) s2 = fmaf(q2f[e], f[e], s2);
            }
            s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
            s2 += __shfl_xor_sync(0xffffffffu, s2, 1);
            s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
            s2 += __shfl_xor_sync(0xffffffffu, s2, 2);
            s1 += __shfl_xor_sync(0xffffffffu, s1, 4);
            s2 += __shfl_xor_sync(0xffffffffu, s2, 4);
            if (part == 0 && key < n) {
                z1[key] = s1;
                z2[key] = s2;
            }
        }
    }
    __syncthreads();

    // ---- phase 2: chunk max, weights, chunk sums.
    float m1 = -INFINITY, m2 = -INFINITY;
    for (int i = tid; i < n; i += SPLIT_THREADS) {
        m1 = fmaxf(m1, z1[i]);
        m2 = fmaxf(m2, z2[i]);
    }
    const float2 mm = block_reduce2<true>(m1, m2, scratch);
    m1 = mm.x;
    m2 = mm.y;
    float l1 = 0.0f, l2 = 0.0f;
    for (int i = tid; i < n; i += SPLIT_THREADS) {
        const float w1 = ex2_approx(z1[i] - m1), w2 = ex2_approx(z2[i] - m2);
        z1[i] = w1;
        z2[i] = w2;
        l1 += w1;
        l2 += w2;
    }
    const float2 ll = block_reduce2<false>(l1, l2, scratch);  // also orders the z writes
    // ---- phase 3: weighted V sums.  cg = tid % 16 owns columns [8 cg, 8 cg + 8);
    // ko = tid / 16 walks keys ko, ko + 16, ...
    const int cg = tid & 15, ko = tid >> 4;
    const __nv_bfloat16 *vb = static_cast<const __nv_bfloat16 *>(p.v) + b * p.v_sb + h * p.v_sh +
                              (int64_t)k_begin * p.v_sl + 8 * cg;
    float acc1[8], acc2[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc1[e] = acc2[e] = 0.0f;
    constexpr int U3 = 8;
    for (int base = ko; base < n; base += 16 * U3) {
        uint4 vv[U3];
#pragma unroll
        for (int u = 0; u < U3; ++u) {
            const int key = base + 16 * u;
            if (key < n) vv[u] = ld_stream(vb + (int64_t)key * p.v_sl);
        }
#pragma unroll
        for (int u = 0; u < U3; ++u) {
            const int key = base + 16 * u;
            if (key < n) {
                const float w1 = z1[key], w2 = z2[key];
                float f[8];
                bf16x8_to_float(vv[u], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    acc1[e] = fmaf(w1, f[e], acc1[e]);
                    acc2[e] = fmaf(w2, f[e], acc2[e]);
                }
            }
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        red[(ko * 2 + 0) * DHDV + 8 * cg + e] = acc1[e];
        red[(ko * 2 + 1) * DHDV + 8 * cg + e] = acc2[e];
    }
    __syncthreads();
    {
        const int map = tid >> 7, c = tid & 127;
        float s = 0.0f;
#pragma unroll
        for (int k = 0; k < 16; ++k) s += red[(k * 2 + map) * DHDV + c];
        out[4 + map * DHDV + c] = s;
    }
    if (tid == 0) {
        out[0] = m1;
        out[1] = ll.x;
        out[2] = m2;
        out[3] = ll.y;
    }
}

__global__ void __launch_bounds__(DHDV) decode_combine_kernel(const DecodeParams p)
{
    __shared__ float scratch[64];
    const int bh = blockIdx.x, h = bh % p.H, b = bh / p.H;
    const int c = threadIdx.x;
    const float *part = p.partials + (size_t)bh * p.splits * PF;
    float M1 = -INFINITY, M2 = -INFINITY;
    for (int s = 0; s < p.splits; ++s) {
        M1 = fmaxf(M1, part[s * PF + 0]);
        M2 = fmaxf(M2, part[s * PF + 2]);
    }
    float L1 = 0.0f, L2 = 0.0f, A1 = 0.0f, A2 = 0.0f;
    for (int s = 0; s < p.splits; ++s) {
        const float *ps = part + s * PF;
        const float e1 = (ps[0] == -INFINITY) ? 0.0f : ex2_approx(ps[0] - M1);
        const float e2 = (ps[2] == -INFINITY) ? 0.0f : ex2_approx(ps[2] - M2);
        L1 = fmaf(ps[1], e1, L1);
        L2 = fmaf(ps[3], e2, L2);
        A1 = fmaf(ps[4 + c], e1, A1);
        A2 = fmaf(ps[4 + DHDV + c], e2, A2);
    }
    float d = 0.0f;
    // lambda of this (b, h): per head, or sigma of its token-dependent logit
    // (Motif 3 summary, section 2.2).
    const float lam = p.lam_logits ? logistic_fast(p.lam_logits[b * p.ll_sb + h * p.ll_sh]) : p.lambda[h];
    // D = (A1 - r A2) / L1 with r = lambda L1 / L2 (one rounding in the difference).
    if (L1 > 0.0f && L2 > 0.0f) d = fmaf(-(lam * L1 / L2), A2, A1) / L1;
    float y = d;
    if (p.apply_norm) {
        const float ss = warp_sum(d * d);
        if ((c & 31) == 0) scratch[c >> 5] = ss;
        __syncthreads();
        const float tot = scratch[0] + scratch[1] + scratch[2] + scratch[3];
        y = d * rsqrtf(tot * (1.0f / DHDV) + p.eps);
        if (p.gain) y *= p.gain[h * DHDV + c];
    }
    if (p.gate) {  // output gate sigma(G) (same section, "Output Gating"), the last step
        const __nv_bfloat16 *g = static_cast<const __nv_bfloat16 *>(p.gate) + b * p.gate_sb + h * p.gate_sh;
        y *= logistic_tanh(__bfloat162float(g[c]));
    }
    __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.out) + b * p.out_sb + h * p.out_sh;
    o[c] = __float2bfloat16_rn(y);
}

}  // namespace

cudaError_t decode_noalloc_scratch(float **ptr)
{
    // Host code cannot use g_decode_scratch's name as a device address; ask
    // the runtime for the address on the current device, once per device.
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static float *addr[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = static_cast<float *>(p);
    }
    *ptr = addr[dev];
    return cudaSuccess;
}

cudaError_t launch_decode(const DecodeParams &p, cudaStream_t stream, int *launches,
                          const ProfileEvents &ev)
{
    const int BH = p.B * p.H;
    if (BH == 0) return cudaSuccess;
    const size_t smem = (size_t)(2 * p.chunk + 16 * 2 * DHDV) * sizeof(float);
    if (smem > 48 * 1024) {
        // The opt-in shared-memory size is a per-device attribute of the
        // kernel: remember the largest size set on each device (under a
        // mutex, for first calls from several host threads).
        constexpr int kMaxDevices = 64;
        static size_t smem_set[kMaxDevices] = {};
        static std::mutex smem_mutex;
        std::lock_guard<std::mutex> lock(smem_mutex);
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kMaxDevices || smem > smem_set[dev]) {
            for (const void *k : {(const void *)decode_split_kernel<false>,
                                  (const void *)decode_split_kernel<true>}) {
                e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
                if (e != cudaSuccess) return e;
            }
            if (dev >= 0 && dev < kMaxDevices) smem_set[dev] = smem;
        }
    }
    if (ev.start) cudaEventRecord(ev.start, stream);
    if (p.window > 0)
        decode_split_kernel<true><<<BH * p.splits, SPLIT_THREADS, smem, stream>>>(p);
    else
        decode_split_kernel<false><<<BH * p.splits, SPLIT_THREADS, smem, stream>>>(p);
    ++*launches;
    if (ev.stop) cudaEventRecord(ev.stop, stream);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_combine_kernel<<<BH, DHDV, 0, stream>>>(p);
    ++*launches;
    return cudaGetLastError();
}

}  // namespace da
