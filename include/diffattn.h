/*
 * diffattn.h -- C ABI of libdiffattn, the B200 (sm_100a) differential-attention
 * forward pass.
 *
 * The operation (Motif 2.6B explainer, section "Differential attention" and
 * figure 1): per batch b, signal head h and query row i,
 *
 *   A_t = softmax(scale * Q_t[i] K_t^T) V          for the two maps t = 1, 2
 *   D   = A_1 - lambda[h] * A_2                      (the subtraction)
 *   Y   = D / sqrt(mean_c D[c]^2 + eps) * gain[h]    (the norm after it)
 *
 * with causal masking (key j is visible to query i when j <= i).  The pages
 * call the norm "GroupNorm"; this library reads it as an RMS norm over each
 * head's dv channels of each token, with a learned per-channel gain.
 * The grouped variant (Motif 3 summary, section 2.2, eq. "grouped differential
 * output" D_t = H_S,t - lambda_t (.) Repeat_g(H_N,t)) takes map 2 of signal
 * head h from noise head h / (H / H_N) and V from V head h / (H / H_V).
 * The same section makes lambda token-dependent, lambda_t = sigma(x_t W^lambda),
 * and gates the output, vec(sigma(G_t) (.) D_t) W^O ("Output Gating"): both
 * are optional inputs of every entry point (the logits x_t W^lambda and G_t,
 * produced by projections outside this library; sigma(z) = 1 / (1 + e^-z)).
 * The gate multiplies the result element-wise as the last step: Y above when
 * the norm is applied, D when it is not.
 *
 * Conventions for every entry point:
 *  - Element type of Q/K/V/out is bf16.  Only d = 64 (Q/K head dim) and
 *    dv = 128 (V head dim) are built; anything else is DIFFATTN_ERR_UNSUPPORTED.
 *  - Tensor pointers are DEVICE pointers owned by the caller.  Every base
 *    pointer must be 16-byte aligned and every stride a multiple of 8 elements
 *    (16 bytes); the last dimension is contiguous.  Strides are in elements.
 *  - The library allocates no device memory.  Scratch is the caller's
 *    `workspace` (device memory, 256-byte aligned) of at least the size the
 *    matching *_workspace_size function returns.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 *    is the legacy default stream).  Nothing is synchronised.
 *  - Argument errors are reported by the return value before anything is
 *    launched.  Errors that only the device can see (a bounded wait that ran
 *    out, a V value outside the fp16 range, a kv_len out of range) are written
 *    to `dev_status` (device int32, nullable): the first error code wins, 0
 *    means none.  The caller reads it after synchronising.  A kernel that sees
 *    such an error finishes without writing the rows it could not compute.
 *  - Every device-side wait is bounded by `timeout_ms` (0 selects 2000 ms).
 */
#ifndef DIFFATTN_H
#define DIFFATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum diffattn_status {
    DIFFATTN_OK = 0,
    DIFFATTN_ERR_INVALID_ARG = 1,  /* null pointer, bad size, inconsistent heads */
    DIFFATTN_ERR_UNSUPPORTED = 2,  /* head dims other than 64 / 128, V beyond fp16 range */
    DIFFATTN_ERR_ALIGNMENT = 3,    /* pointer not 16-byte aligned or stride not 8-element */
    DIFFATTN_ERR_WORKSPACE = 4,    /* workspace missing or too small */
    DIFFATTN_ERR_CUDA = 5,         /* a CUDA runtime / driver call failed */
    DIFFATTN_ERR_TIMEOUT = 6       /* (device) a bounded wait ran out */
} diffattn_status;

#define DIFFATTN_FLAG_CAUSAL 1u      /* key j visible to query i iff j <= i */
#define DIFFATTN_FLAG_APPLY_NORM 2u  /* apply the RMS norm + gain; else write D */
/* Sliding window (Motif 3 summary, section 2.1: sliding-window attention
 * layers; "Practical Implications": 128-token windows): with `window` = W > 0
 * the query at position i sees only keys i-W < j <= i, the W most recent
 * including itself (prefill: needs DIFFATTN_FLAG_CAUSAL; decode: the W most
 * recent cached keys).  0 means no window.                                   */
/* Test hook for the failure path: the prefill kernel withholds the K/V load
 * of the first key step of the first tile each CTA takes, so its bounded
 * waits run out (after timeout_ms) and the call reports
 * DIFFATTN_ERR_TIMEOUT in dev_status without writing the output.  Nothing
 * faults or hangs; the device stays usable.  Not for production use.       */
#define DIFFATTN_FLAG_TEST_WITHHOLD_LOAD 0x80000000u

/* Prefill arguments.  Layout of each tensor: element (b, n, head, c) sits at
 * ptr + b*stride[0] + n*stride[1] + head*stride[2] + c.
 *   q1, k1: [B, N, H,   64]     q2, k2: [B, N, H_N, 64]
 *   v:      [B, N, H_V, 128]    out:    [B, N, H,   128]
 *   lambda: [H] fp32 device     gain:   [H, 128] fp32 device (16-byte aligned,
 *                                       contiguous), or NULL for 1.
 *   lambda_logits: [B, N, H] fp32 device, element (b, n, h) at
 *       ptr + b*s[0] + n*s[1] + h*s[2] (4-byte aligned, any strides), or NULL.
 *       When set, signal head h of token n uses lambda = sigma(logit) and
 *       `lambda` may be NULL.
 *   gate: [B, N, H, 128] bf16 device gate logits, laid out like `out` (16-byte
 *       aligned base, strides multiples of 8 elements), or NULL for no gate. */
typedef struct diffattn_fwd_args {
    int64_t B, N, H, H_N, H_V;
    int64_t d, dv;
    float scale, eps;
    uint32_t flags;
    uint32_t timeout_ms;
    const void *q1; int64_t q1_stride[3];
    const void *q2; int64_t q2_stride[3];
    const void *k1; int64_t k1_stride[3];
    const void *k2; int64_t k2_stride[3];
    const void *v;  int64_t v_stride[3];
    void *out;      int64_t out_stride[3];
    const float *lambda;
    const float *gain;
    int32_t *dev_status;
    const float *lambda_logits; int64_t lambda_logits_stride[3];
    const void *gate;           int64_t gate_stride[3];
    int32_t window;             /* sliding window in keys, 0 = none (causal only) */
    /* Rotary position embedding (Motif 2.6B explainer, "The block": RoPE with
     * theta = 500,000): with rope_theta > 0 every 64-wide row of Q1, K1, Q2
     * and K2 at token position n is rotated before the scores, in interleaved
     * pairs: (x[2c], x[2c+1]) turned by the angle n * rope_theta^(-2c/64).
     * The rotated copies live in the workspace as fp16 (see
     * diffattn_fwd_workspace_size); the caller's tensors are not modified.
     * Rotated values beyond the fp16 range report DIFFATTN_ERR_UNSUPPORTED
     * in dev_status.
     * 0 = no rotation.  Decode has no rotation: it reads its cache as
     * stored.                                                               */
    float rope_theta;
    /* State saved for diffattn_bwd: NULL, or device memory (16-byte aligned)
     * of diffattn_fwd_save_size(args) bytes that the forward fills, besides
     * `out`, with what the backward pass needs: per row and map the
     * normalised map output A_t = softmax(scale Q_t K_t^T) V (fp32) and the
     * base-2 log of the row's softmax denominator.  Its layout is private to
     * the library; it stays valid until the caller reuses the memory.
     * Every option of the forward call can save.  A grouped call that saves
     * computes each noise map once per signal head (the state is per signal
     * head), not once per group.                                            */
    void *save;
} diffattn_fwd_args;

/* Causal (or full) prefill, one noise map per signal head: H_N and H_V must be
 * 0 or equal to H.  N_q == N_k == N.  Differential attention as defined in the
 * Motif 2.6B explainer, section "Differential attention".                    */
diffattn_status diffattn_fwd(const diffattn_fwd_args *args, void *workspace, size_t ws_bytes,
                             void *stream);

/* Grouped prefill: H % H_N == 0 and H % H_V == 0; signal head h uses Q2/K2 of
 * noise head h / (H / H_N) and V head h / (H / H_V) (Motif 3 summary,
 * section 2.2).  With H_N == H_V == H it is diffattn_fwd.                    */
diffattn_status diffattn_grouped_fwd(const diffattn_fwd_args *args, void *workspace,
                                     size_t ws_bytes, void *stream);

/* Bytes of workspace diffattn_fwd / diffattn_grouped_fwd need for `args`
 * (an fp16 copy of V for the tensor-core P.V product -- not under a sliding
 * window, whose kernel converts each V step itself --, the work counters,
 * and depending on the arguments the grouped heads' noise outputs and the
 * rotated copies of Q1, K1, Q2, K2).                                        */
size_t diffattn_fwd_workspace_size(const diffattn_fwd_args *args);

/* Bytes of the `save` buffer a diffattn_fwd call with `args` fills (0 for
 * an empty problem).                                                        */
size_t diffattn_fwd_save_size(const diffattn_fwd_args *args);

/* Backward pass of diffattn_fwd / diffattn_grouped_fwd: the gradients of
 * sum(dout * out) with respect to q1, q2, k1, k2, v, lambda (or the lambda
 * logits), gain and the gate logits.  The pages define the forward pass only
 * (Motif 2.6B explainer, section "Differential attention"; the model is
 * trained with it, same page, "A schedule for the data"), so this is its
 * exact gradient.  With lambda_i the row's lambda, Yn the output before the
 * gate and r = (mean_c D^2 + eps)^-1/2:
 *
 *   dYn = dY sigma(G), dG = dY Yn sigma(G) (1 - sigma(G))   (no gate: dYn = dY)
 *   dgain = sum_i dYn D r,  dD = r (dYn gain) - (r^3 / dv) D sum_c(dYn gain D)
 *   dA_1 = dD, dA_2 = -lambda_i dD, dlambda_i = -sum_c dD A_2
 *   per map: dP = dA_t V^T, dS = P (dP - rowsum(dA_t A_t)),
 *            dQ_t = scale dS K_t, dK_t = scale dS^T Q_t, dV += P^T dA_t
 *
 * (without DIFFATTN_FLAG_APPLY_NORM, dD = dYn and dgain = 0; with lambda
 * logits, dlogit_i = dlambda_i sigma'(logit_i) and grad_lambda = 0; with a
 * window, the masked pairs take no part; with rope_theta, the products use
 * the rotated Q/K and dQ, dK are rotated back).  Grouped heads (H_N, H_V as
 * in the forward) sum the gradients of a shared noise or V head over its
 * signal heads.  Inputs are those of the forward call that filled `save`,
 * with the same sizes, scale, eps, flags, lambda / logits, gate, window and
 * rope_theta.  Layouts as in the forward:
 *   q1, k1, grad_q1, grad_k1: [B, N, H, 64] bf16
 *   q2, k2, grad_q2, grad_k2: [B, N, H_N, 64] bf16
 *   v, grad_v: [B, N, H_V, 128] bf16;  dout: [B, N, H, 128] bf16
 *   lambda: [H] fp32 device (or NULL with lambda_logits); gain: [H, 128]
 *   fp32 device or NULL for 1.
 *   grad_lambda: [H] fp32 device or NULL; grad_gain: [H, 128] fp32 device,
 *   contiguous, or NULL.
 *   lambda_logits / grad_lambda_logits: [B, N, H] fp32 (any strides), or
 *   NULL; gate / grad_gate: [B, N, H, 128] bf16 laid out like dout, or NULL.
 * Every gradient is overwritten, not accumulated into.  Intermediate
 * quantities beyond the fp16 range (the normalised-output gradient dD is
 * staged in fp16 for the tensor cores, and with rope_theta so are the score
 * gradients) report DIFFATTN_ERR_UNSUPPORTED in dev_status; the kernels
 * still run to the end, and every gradient of such a call is undefined (it
 * may hold inf or NaN).  Check dev_status before using the gradients.       */
typedef struct diffattn_bwd_args {
    int64_t B, N, H;
    int64_t d, dv;
    float scale, eps;
    uint32_t flags;         /* CAUSAL, APPLY_NORM: as in the forward call */
    uint32_t timeout_ms;
    const void *q1; int64_t q1_stride[3];
    const void *q2; int64_t q2_stride[3];
    const void *k1; int64_t k1_stride[3];
    const void *k2; int64_t k2_stride[3];
    const void *v;  int64_t v_stride[3];
    const void *dout; int64_t dout_stride[3];
    const void *save;       /* filled by the forward call */
    const float *lambda;
    const float *gain;
    void *grad_q1; int64_t grad_q1_stride[3];
    void *grad_q2; int64_t grad_q2_stride[3];
    void *grad_k1; int64_t grad_k1_stride[3];
    void *grad_k2; int64_t grad_k2_stride[3];
    void *grad_v;  int64_t grad_v_stride[3];
    float *grad_lambda;
    float *grad_gain;
    int32_t *dev_status;
    int64_t H_N, H_V;       /* noise / V heads; 0 means H */
    const float *lambda_logits; int64_t lambda_logits_stride[3];
    const void *gate;           int64_t gate_stride[3];
    int32_t window;             /* as in the forward call; 0 = none */
    float rope_theta;           /* as in the forward call; 0 = none */
    float *grad_lambda_logits;  int64_t grad_lambda_logits_stride[3];
    void *grad_gate;            int64_t grad_gate_stride[3];
} diffattn_bwd_args;

diffattn_status diffattn_bwd(const diffattn_bwd_args *args, void *workspace, size_t ws_bytes,
                             void *stream);

/* Workspace bytes of diffattn_bwd (fp16 copies of V and of dD, per-row
 * statistics, the two tile kernels' work counters, and depending on the
 * arguments the rotated copies of Q1, K1, Q2, K2 and fp32 sums of the
 * gradients of shared noise and V heads).                                   */
size_t diffattn_bwd_workspace_size(const diffattn_bwd_args *args);

/* Host-only argument check of a prefill call: the status diffattn_fwd (or,
 * with grouped != 0, diffattn_grouped_fwd) would return before launching,
 * with the workspace check skipped.  Touches no device.                      */
diffattn_status diffattn_fwd_validate(const diffattn_fwd_args *args, int grouped);

/* Single-query decode arguments.  The query of sequence b sits at position
 * kv_len[b]-1 and attends to cached keys 0..kv_len[b]-1 (no mask needed).
 *   q1, q2: [B, H, 64]            element (b, h, c) at ptr + b*s[0] + h*s[1] + c
 *   k1, k2: [B, H, L, 64]         element (b, h, j, c) at ptr + b*s[0] + h*s[1] + j*s[2] + c
 *   v:      [B, H, L, 128]
 *   out:    [B, H, 128]
 *   kv_len: [B] int32 device, 1 <= kv_len[b] <= L, or NULL for L.
 *   num_splits: KV splits per (b, h); 0 picks one.
 *   lambda_logits: [B, H] fp32 device (element (b, h) at ptr + b*s[0] + h*s[1])
 *       or NULL; when set, lambda = sigma(logit) and `lambda` may be NULL.
 *   gate: [B, H, 128] bf16 device gate logits laid out like `out`, or NULL. */
typedef struct diffattn_decode_args {
    int64_t B, H, L;
    int64_t d, dv;
    float scale, eps;
    uint32_t flags;         /* DIFFATTN_FLAG_APPLY_NORM; CAUSAL is ignored */
    int32_t num_splits;
    const void *q1; int64_t q1_stride[2];
    const void *q2; int64_t q2_stride[2];
    const void *k1; int64_t k1_stride[3];
    const void *k2; int64_t k2_stride[3];
    const void *v;  int64_t v_stride[3];
    void *out;      int64_t out_stride[2];
    const int32_t *kv_len;
    const float *lambda;
    const float *gain;
    int32_t *dev_status;
    const float *lambda_logits; int64_t lambda_logits_stride[2];
    const void *gate;           int64_t gate_stride[2];
    int32_t window;             /* the query sees the `window` most recent keys; 0 = all */
} diffattn_decode_args;

/* Split-KV decode: a split kernel writes per-split partial softmax states
 * (running max, sum and unnormalised V sum for both maps) into the workspace;
 * a combine kernel merges them and applies the subtraction and the norm.    */
diffattn_status diffattn_decode(const diffattn_decode_args *args, void *workspace,
                                size_t ws_bytes, void *stream);

/* Decode without a workspace.  The pages have no counterpart to this entry
 * point: it exists for callers that cannot allocate device memory or pass
 * a workspace -- for instance code inside a serving engine whose allocator
 * already owns all of the GPU's memory (a KV-cache pool), code on a
 * latency-critical path that must not call cudaMalloc (which can
 * synchronise the device), or a plugin that has no allocator handle to take
 * a workspace from.  It computes exactly what diffattn_decode computes, with
 * the per-split partial states kept in a fixed static device array of
 * DIFFATTN_DECODE_NOALLOC_SCRATCH_BYTES that the library carries (every GPU
 * that loads the library holds it until the process exits).
 *  - Sizes whose partials (diffattn_decode_workspace_size) exceed that array
 *    return DIFFATTN_ERR_WORKSPACE; diffattn_last_error() says by how much.
 *  - The first call on a device looks up the array's device address and
 *    keeps it for the rest of the process; make that first call before any
 *    stream capture.  The kept address dies with the device's context: after
 *    cudaDeviceReset (or anything else that destroys and recreates the
 *    primary context) do not call this entry point on that device again.
 *  - Every call on a device shares the one array and leaves its partials
 *    there; nothing in it has to start at zero.  Calls that overlap on the
 *    GPU (other streams, other host threads) race on it: serialise them.
 *  - Nothing is allocated or freed, by the library or on its behalf.        */
#define DIFFATTN_DECODE_NOALLOC_SCRATCH_BYTES (8u << 20)
diffattn_status diffattn_decode_noalloc(const diffattn_decode_args *args, void *stream);

/* Workspace bytes diffattn_decode needs for these sizes (num_splits 0 = the
 * count diffattn_decode picks).                                              */
size_t diffattn_decode_workspace_size(int64_t B, int64_t H, int64_t L, int32_t num_splits);

/* The split count diffattn_decode uses for these sizes (chosen for about
 * four CTAs per SM of the current device).                                   */
int32_t diffattn_decode_num_splits(int64_t B, int64_t H, int64_t L, int32_t num_splits);

/* Host-only argument check of a decode call (workspace check skipped).      */
diffattn_status diffattn_decode_validate(const diffattn_decode_args *args);

/* Static, human-readable name of a status code.                              */
const char *diffattn_status_str(diffattn_status status);

/* Number of kernels the last successful call on this thread launched (for
 * launch accounting in benchmarks).                                          */
int32_t diffattn_last_launch_count(void);

/* Text of the CUDA error (or internal check) behind the last
 * DIFFATTN_ERR_CUDA returned on this thread; "" when there was none.  The
 * string is owned by the library and valid until the next call.             */
const char *diffattn_last_error(void);

/* Timing hook for benchmarks: while set (non-NULL), every later call on this
 * thread records `start` (a cudaEvent_t passed as void*) on its stream just
 * before its main kernel (the prefill kernel, or the decode split kernel) and
 * `stop` just after it, so the caller can time that kernel alone.  Pass NULL,
 * NULL to switch it off.  The events are the caller's.                       */
void diffattn_set_profile_events(void *start, void *stop);

#ifdef __cplusplus
}
#endif

#endif /* DIFFATTN_H */
