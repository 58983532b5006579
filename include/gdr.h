/*
 * gdr.h - C ABI of libgdr, a B200 (sm_100a) library for the gated delta rule.
 *
 * The operation (NextTransformer, "Source notes", section "Linear attention",
 * rows gdn and kda; Frontier-model atlas, items 01, 03 and 08):
 *
 *   for each batch row b and value head h (key head hk = h / (Hv / Hk)):
 *     S_t = (I - beta_t k_t k_t^T) diag(exp(g_t)) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * S is the Dk x Dv ("K x V") state, stored row-major as [Dk][Dv] in fp32.
 * g_t <= 0 is the log of the decay alpha_t: one scalar per head (Gated
 * DeltaNet, GDR_GATE_SCALAR) or one value per key channel (Kimi Delta
 * Attention, GDR_GATE_CHANNEL); in both cases the decay acts before the delta
 * update. beta_t in (0,1) is the write strength. The readout uses the state
 * after the update and no scale (scale = 1, "Backend and numerical limits" on
 * the same page). q and k are used as given: the library does not normalise them.
 * DeltaNet is the special case g = 0.
 *
 * Layouts (all row-major and contiguous; "bf16 or fp32" follows `dtype`):
 *   q, k      [B, T, Hk, Dk]   bf16 or fp32
 *   v         [B, T, Hv, Dv]   bf16 or fp32
 *   o         [B, T, Hv, Dv]   bf16 or fp32 (fp32 for GDR_BF16_OUT_F32)
 *   g         [B, T, Hv]       fp32 (GDR_GATE_SCALAR)
 *             [B, T, Hv, Dk]   fp32 (GDR_GATE_CHANNEL)
 *   beta      [B, T, Hv]       fp32
 *   h0, hT    [B, Hv, Dk, Dv]  fp32
 * Decode uses the same layouts with T = 1 ([B, H, D]) and an fp32 state.
 *
 * Grouped value heads: Hv must be a multiple of Hk; value head h reads key
 * head h / (Hv / Hk) (contiguous groups, as repeat-interleaving q and k).
 *
 * Ownership and execution: every pointer is device memory owned by the
 * caller. The library never allocates, frees or synchronises; all work is
 * enqueued on `stream` (a cudaStream_t passed as void*, NULL = legacy default
 * stream) and GDR_OK means "enqueued". gdr_fwd_chunked needs every pointer
 * 16-byte aligned; gdr_decode_step needs the state 16-byte aligned and the
 * other pointers aligned to their element size.
 * h0 and hT may be the same buffer (in-place state update); o must not alias
 * any input. No C++ exception crosses this boundary.
 *
 * Errors: arguments are checked on the host before anything is launched.
 * A non-zero status means nothing was enqueued (except GDR_ERR_CUDA, which
 * reports a launch failure) and gdr_last_error() returns a message for the
 * calling thread.
 */
#ifndef GDR_H
#define GDR_H

#include <stddef.h>

#if defined(__GNUC__)
#define GDR_API __attribute__((visibility("default")))
#else
#define GDR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDR_OK = 0,
    GDR_ERR_INVALID_ARG = 1,   /* bad size, Hv % Hk != 0, NULL required pointer, bad enum */
    GDR_ERR_UNSUPPORTED = 2,   /* Dk or Dv not 64 or 128 */
    GDR_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned */
    GDR_ERR_WORKSPACE = 4,     /* workspace missing or smaller than gdr_fwd_workspace_size() (gdr_bwd_workspace_size() for gdr_bwd) */
    GDR_ERR_CUDA = 5           /* a CUDA launch or runtime call failed */
} gdr_status;

enum { GDR_GATE_SCALAR = 0, GDR_GATE_CHANNEL = 1 };
/* dtype of q, k, v and o: */
enum {
    GDR_BF16 = 0,          /* q, k, v, o bf16 */
    GDR_FP32 = 1,          /* q, k, v, o fp32 */
    GDR_BF16_OUT_F32 = 2   /* q, k, v bf16; o fp32 */
};

/* Library version, major * 10000 + minor * 100 + patch. */
GDR_API int gdr_version(void);

/* Message describing the last non-GDR_OK status returned on the calling thread. */
GDR_API const char *gdr_last_error(void);

/* Number of kernels this library has enqueued so far in this process (all
 * threads and devices); lets a caller count the launches inside a timed region. */
GDR_API unsigned long long gdr_kernel_launches(void);

/*
 * Backward of the recurrence (NextTransformer, "Source notes", "Linear attention":
 * the gdn and kda updates; their adjoint, step by step in reverse).
 *
 * Gradients of L = sum(dout * o) + sum(dhT * hT), where (o, hT) is what
 * gdr_fwd_chunked computes from the same q, k, v, g, beta, h0 (h0 == NULL: zero
 * state; dhT == NULL: zero):
 *   dq, dk  [B, T, Hk, Dk] fp32 (summed over the value heads sharing a key head)
 *   dv      [B, T, Hv, Dv] fp32
 *   dg      [B, T, Hv] or [B, T, Hv, Dk] fp32 (g's layout)
 *   dbeta   [B, T, Hv] fp32
 *   dh0     [B, Hv, Dk, Dv] fp32
 * Inputs as for gdr_fwd_chunked; dout [B, T, Hv, Dv] in the input dtype (GDR_BF16
 * or GDR_BF16_OUT_F32: bf16; GDR_FP32: fp32), dhT fp32. The arithmetic is fp32:
 * a forward pass stores the state before every 4th token in the workspace, then a
 * reverse pass recomputes each block of 4 tokens and reverses its steps.
 * Needs Dk of 64 or 128, Dv of 64 or 128 and B * Hv <= 65535 (else
 * GDR_ERR_UNSUPPORTED); the other
 * argument errors are those of gdr_fwd_chunked. All pointers 16-byte aligned;
 * the outputs must not alias the inputs or each other. T == 0 writes dh0 = dhT
 * (or zeros) and nothing else.
 *
 * workspace: device buffer of at least gdr_bwd_workspace_size(...) bytes
 * (B * Hv * ceil(T / 4) * Dk * Dv * 4), owned by the caller; two calls that
 * overlap in time must not share one. Asynchronous on `stream`.
 */
GDR_API size_t gdr_bwd_workspace_size(int B, int T, int Hk, int Hv, int Dk, int Dv, int gate_mode, int dtype);
GDR_API int gdr_bwd(const void *q, const void *k, const void *v, const float *g, const float *beta,
                    const float *h0, const void *dout, const float *dhT, float *dq, float *dk, float *dv,
                    float *dg, float *dbeta, float *dh0, int B, int T, int Hk, int Hv, int Dk, int Dv,
                    int gate_mode, int dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Chunked backward on tensor cores (NextTransformer, "Source notes", "Linear
 * attention": the gdn update's first-order backward). Same gradients, arguments,
 * layouts and outputs as gdr_bwd, for the scalar gate with bf16 inputs
 * (GDR_BF16 or GDR_BF16_OUT_F32: q, k, v and dout bf16) and Dk = Dv = 128; other
 * sizes or modes return GDR_ERR_UNSUPPORTED (gdr_bwd takes them).
 *
 * Three passes, chunks of 64 tokens: the tcgen05 forward stores each chunk's
 * entering state, its P, Qh and T = (I + A)^-1 (the chunk map of gdr_fwd_chunked)
 * in the workspace; a reverse scan over the chunks carries the state gradient
 * dS <- Gamma_C dS + P^T dS + Qh^T dout, the transposed chunk map, and stores it per
 * chunk; then every chunk forms its own gradients from its entering state, the
 * gradient of the state it leaves, dout and its inputs, all chunks at once. All
 * three passes run their products on the tcgen05 tensor cores with fp16 operands
 * and fp32 accumulation (the forward's precision), so results are of the
 * forward's accuracy class (about 1e-3 relative), not fp32: gdr_bwd is the fp32
 * path. q, k, v, dout and the states must stay inside the fp16 range. dv, dg,
 * dbeta and dh0 repeat bit for bit; so do dq and dk when Hv == Hk (one writer per
 * row). With grouped value heads dq and dk are sums over the value heads' work
 * (atomics), repeatable to rounding only.
 *
 * workspace: device buffer of at least gdr_bwd_chunked_workspace_size(...) bytes
 * (B * Hv * ceil(T / 64) * 120 KiB), owned by the caller; two calls that overlap
 * in time must not share one. Asynchronous on `stream`.
 */
GDR_API size_t gdr_bwd_chunked_workspace_size(int B, int T, int Hk, int Hv, int Dk, int Dv, int gate_mode,
                                              int dtype);
GDR_API int gdr_bwd_chunked(const void *q, const void *k, const void *v, const float *g, const float *beta,
                            const float *h0, const void *dout, const float *dhT, float *dq, float *dk, float *dv,
                            float *dg, float *dbeta, float *dh0, int B, int T, int Hk, int Hv, int Dk, int Dv,
                            int gate_mode, int dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Device-side failure counts of the tensor-core chunked kernels (bf16 inputs,
 * Dk = Dv = 128) on the current device, accumulated since the library was
 * loaded there. Either pointer may be NULL; returns the sum of the two.
 *   load_timeouts  waits inside the kernel (chunk input loads, or a hand-off
 *                  between its warp groups) that gave up after one second; the
 *                  (batch row, value head) unit stops, so that call's o and hT
 *                  are incomplete.
 *   range_errors   per-channel gate (warp-level kernel): chunks whose
 *                  per-key-channel gate factors left the fp16 range (a decay
 *                  stronger than about exp(-11) within 32 tokens); that
 *                  chunk's results are not valid. Scalar gate (tcgen05
 *                  kernel): (batch row, value head) units whose o or final
 *                  state came out inf or NaN. That happens when a value
 *                  rounded to an fp16 operand overflowed (the copy of the
 *                  state, A, M, the inverse, W, U, P, Qh), since a product
 *                  of an inf operand is never finite, or when an input was
 *                  inf or NaN; that unit's o and hT are not valid.
 * The chunked backward (gdr_bwd_chunked) adds its own: load_timeouts counts its
 * waits that gave up, range_errors its reverse-scan units whose dh0 and its
 * (unit, chunk) work items whose dq, dk, dv, dg or dbeta came out inf or NaN (an
 * fp16 operand that overflowed: an input, a stored chunk map, the state
 * gradient's copy or a tile formed from them); those gradients are not valid.
 * Reads device memory, so it waits for prior work on the default stream.
 */
GDR_API unsigned int gdr_fused_error_counts(unsigned int *load_timeouts, unsigned int *range_errors);

/*
 * Bytes of device workspace gdr_fwd_chunked needs for these sizes (0 when it
 * needs none). Returns 0 for invalid arguments as well; gdr_fwd_chunked then
 * reports the actual error. For the tcgen05 kernel with more (batch row, value
 * head) units than the current device has SMs, this is the workspace that lets
 * it spread the units' chunks evenly over the SMs (it depends on the device's
 * SM count); that kernel also runs with less, one CTA per unit.
 */
GDR_API size_t gdr_fwd_workspace_size(int B, int T, int Hk, int Hv, int Dk, int Dv,
                              int gate_mode, int dtype);

/*
 * Chunked forward over whole sequences (chunks of 64 tokens; the last chunk
 * of a sequence may be partial).
 *
 * Computes o_t for every t in [0, T) and, if hT != NULL, the state after the
 * last token. h0 == NULL means a zero initial state. The result equals the
 * token recurrence above (chunk by chunk, no approximation; SinkProbe (Attention-Sink)
 * README, description of its delta-rule layer): per 64-token chunk a UT/WY
 * transform A = tril(diag(beta)(K*Gamma)(K/Gamma)^T, -1), T = (I + A)^-1,
 * W = T diag(beta)(K*Gamma), U = T diag(beta) V, then the state scan
 * U' = U - W S, S <- diag(Gamma_C) S + (K*Gamma_C/Gamma)^T U', and the output
 * O = (Q*Gamma) S + tril((Q*Gamma)(K/Gamma)^T) U'.
 *
 * bf16 inputs with Dk = Dv = 128 run one tensor-core kernel: for the scalar
 * gate on tcgen05 (where the chunk's state map is used in the equivalent
 * affine form S <- Gamma_C S + P S + R, O = Qh S + Uh, with P = -(K*Gamma_C/
 * Gamma)^T W, R = (K*Gamma_C/Gamma)^T U, Qh = (Q*Gamma) - M W, Uh = M U and M
 * the masked (Q*Gamma)(K/Gamma)^T above), for the per-channel gate too, with
 * the decays carried by the Gram's operands (K exp(G - G_31), Q exp(G - G_31),
 * K exp(G_31 - G), G the in-chunk prefix per key channel and G_31 its value at
 * the chunk's row 31); with the layer options (gdr_fwd_chunked_norm) the
 * per-channel gate runs on the warp-level tensor cores. All use fp16 operands,
 * fp32 accumulation and an fp32 carried state; q, k, v and the state must stay inside the fp16 range,
 * |x| < 6.5e4 (both kernels count violations, see gdr_fused_error_counts;
 * the call still returns GDR_OK). Other shapes and fp32 inputs run fp32 CUDA-core kernels, which
 * take at most 65535 batch rows (else GDR_ERR_UNSUPPORTED).
 * B == 0 or T == 0 is a valid no-op that still writes hT = h0 (or zeros).
 *
 * workspace: device buffer of at least gdr_fwd_workspace_size(...) bytes,
 * 256-byte aligned, owned by the caller; may be NULL when that size is 0.
 * Its contents on entry are ignored. Two calls that overlap in time on the
 * GPU must not share one workspace. With the tcgen05 kernel and more units
 * than SMs it holds, per CTA boundary, a flag and the state of the unit cut
 * there: the first CTA runs the unit's first chunks and hands its state over,
 * the other runs the rest; each launch tags its flags, so stale contents are
 * harmless. A NULL or smaller workspace is not an error there: the kernel
 * then runs one CTA per unit (in more than one wave of SMs).
 */
GDR_API int gdr_fwd_chunked(const void *q, const void *k, const void *v, const float *g,
                    const float *beta, const float *h0, void *o, float *hT,
                    int B, int T, int Hk, int Hv, int Dk, int Dv,
                    int gate_mode, int dtype,
                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * Chunked forward over packed sequences of different lengths (no counterpart
 * on the source pages beyond their remark that the recurrent state is reset at
 * each packed row).
 *
 * N sequences are packed along one token axis of T_total tokens: sequence n
 * is tokens [cu_seqlens[n], cu_seqlens[n+1]) and starts from h0[n] (or zeros),
 * its final state goes to hT[n]. Layouts: q, k [T_total, Hk, Dk]; v, o
 * [T_total, Hv, Dv]; g [T_total, Hv] or [T_total, Hv, Dk]; beta [T_total, Hv];
 * h0, hT [N, Hv, Dk, Dv] fp32. cu_seqlens: device int32 [N + 1], non-decreasing,
 * cu_seqlens[0] = 0, cu_seqlens[N] = T_total (values are clamped into
 * [0, T_total], so a malformed array yields wrong results, never an
 * out-of-bounds access). Each sequence equals a gdr_fwd_chunked call on it
 * alone, bit for bit.
 *
 * Runs only on the tensor-core kernels: bf16 inputs (dtype GDR_BF16 or
 * GDR_BF16_OUT_F32) with Dk = Dv = 128; anything else returns
 * GDR_ERR_UNSUPPORTED. The scalar gate runs the same kernel as
 * gdr_fwd_chunked, so each packed sequence equals a separate call bit for bit. Needs no workspace. Pointers 16-byte aligned (cu_seqlens
 * 4-byte aligned); o must not alias q, k or v.
 */
GDR_API int gdr_fwd_chunked_varlen(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, const float *h0, void *o, float *hT,
                           const int *cu_seqlens, int N, int T_total, int Hk, int Hv, int Dk, int Dv,
                           int gate_mode, int dtype, void *stream);

/*
 * Chunked forward with the layer's normalisations fused into the kernel
 * (NextTransformer "Source notes", section "Linear attention": L2-normalized
 * Q/K in rows deltanet and kda; the GDN output RMSNorm x gain x SiLU gate in
 * row gdn; "Backend and numerical limits": a gated RMSNorm on the output).
 *
 * Arguments as gdr_fwd_chunked, plus:
 * - cu_seqlens: NULL, or packed sequences exactly as gdr_fwd_chunked_varlen (B
 *   is then N and T is T_total; q, k [T, Hk, Dk] and so on).
 * - qk_l2norm: non-zero to divide every q and k row (one head of one token) by
 *   sqrt(sum of squares + 1e-6) as it is loaded.
 * - z: NULL, or the output gate [B, T, Hv, Dv] bf16 (the layout of o). Then o
 *   receives o / sqrt(mean(o^2) + norm_eps) * norm_weight * SiLU(z) per row of
 *   Dv, where o is the recurrence's output; norm_weight [Dv] fp32 is required.
 *
 * Runs only on the tensor-core kernels: bf16 inputs (GDR_BF16 or
 * GDR_BF16_OUT_F32) with Dk = Dv = 128, else GDR_ERR_UNSUPPORTED. No workspace.
 * Without options it equals gdr_fwd_chunked bit for bit. A call with z keeps
 * each (b, h) in one CTA. Pointers 16-byte aligned (norm_weight 4-byte,
 * cu_seqlens 4-byte); o must not alias q, k, v or z.
 */
GDR_API int gdr_fwd_chunked_norm(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const float *h0, void *o, float *hT,
                                 const int *cu_seqlens, int B, int T, int Hk, int Hv, int Dk, int Dv,
                                 int gate_mode, int dtype, int qk_l2norm, const void *z,
                                 const float *norm_weight, float norm_eps, void *stream);

/*
 * One decode step for B independent sequences (the recurrence with T = 1):
 *   S' = diag(exp(g)) S;  u = beta (v - S'^T k);  S <- S' + k u^T;  o = S^T q.
 * state [B, Hv, Dk, Dv] fp32 is read and overwritten in place; q, k [B, Hk, Dk],
 * v, o [B, Hv, Dv] in `dtype`; g [B, Hv] or [B, Hv, Dk] fp32; beta [B, Hv] fp32.
 * Needs no workspace. Frontier-model atlas, item 03: decay, memory
 * prediction, delta correction and recurrent read, in that order.
 */
GDR_API int gdr_decode_step(const void *q, const void *k, const void *v, const float *g,
                    const float *beta, float *state, void *o,
                    int B, int Hk, int Hv, int Dk, int Dv,
                    int gate_mode, int dtype, void *stream);

/*
 * Chunked forward for callers that cannot allocate device memory. The source
 * pages have no counterpart to this entry point; it exists for users of the
 * library, not for the method.
 *
 * Who needs it: code that may not call cudaMalloc - an engine that owns all
 * device memory through its own pool and forbids side allocations, or a
 * latency-bound serving loop where allocating (and the device
 * synchronisation cudaMalloc/cudaFree can trigger) is not allowed after
 * start-up. Such a caller cannot provide gdr_fwd_chunked's workspace.
 *
 * Same arguments and results as gdr_fwd_chunked without the workspace. The
 * scratch is a fixed array of GDR_NOALLOC_SCRATCH_BYTES in the library's own
 * device memory; sizes whose gdr_fwd_workspace_size() exceeds it are
 * rejected with GDR_ERR_WORKSPACE before anything runs. The array is reserved
 * on every GPU where the library's no-allocation code is loaded and stays
 * reserved until the process exits. The first call on a device looks up the
 * array's address on that device: make that first call before any stream
 * capture. That address belongs to the device's context at the time; after a
 * device reset (cudaDeviceReset) the first call in the new context looks it up
 * again, so make that call before any capture too. Every call shares the one array and it keeps the previous call's
 * contents (each call writes every part it reads before reading it), so
 * calls that overlap in time on one GPU race and must be serialised by the
 * caller. Nothing here calls cudaMalloc, cudaFree or any allocating routine.
 */
#define GDR_NOALLOC_SCRATCH_BYTES (64u << 20)
GDR_API int gdr_fwd_chunked_noalloc(const void *q, const void *k, const void *v, const float *g,
                                    const float *beta, const float *h0, void *o, float *hT,
                                    int B, int T, int Hk, int Hv, int Dk, int Dv,
                                    int gate_mode, int dtype, void *stream);

/*
 * The layer's short causal convolution with SiLU, applied to the q/k/v
 * projections before the recurrence (NextTransformer "Source notes", section
 * "Linear attention", rows deltanet and kda: causal conv + SiLU; "Backend and
 * numerical limits": a causal convolution with SiLU activation; Atlas entry 03,
 * a four-token causal convolution). Depthwise over channels:
 *   y[t, c] = SiLU(bias[c] + sum_{j=0..3} w[c, j] x[t - 3 + j, c]),
 *   SiLU(a) = a / (1 + e^-a),
 * with the inputs before a sequence's first token taken from state_in (else 0).
 *
 * x, y: [B, T, Ch] (or, with cu_seqlens, [T, Ch]: B sequences packed along T
 * tokens, sequence n is tokens [cu_seqlens[n], cu_seqlens[n+1]), cu_seqlens a
 * device int32 [B + 1], non-decreasing, from 0 to T). w: [Ch, 4] fp32 (tap 3 on
 * the current token), bias: [Ch] fp32 or NULL. state_in, state_out: [B, Ch, 3]
 * in the dtype of x, the three inputs before each sequence / its last three
 * (oldest first), each may be NULL (state_out of an empty sequence is state_in,
 * or zeros). dtype: GDR_BF16 or GDR_FP32 for x, y and the states; arithmetic in
 * fp32. width must be 4 and Ch a multiple of 8 (else GDR_ERR_UNSUPPORTED).
 * x, w, y 16-byte aligned; y must not alias x. The caller owns every buffer.
 */
GDR_API int gdr_causal_conv_silu(const void *x, const float *w, const float *bias, const void *state_in,
                                 void *state_out, void *y, const int *cu_seqlens, int B, int T, int Ch,
                                 int width, int dtype, void *stream);

/*
 * The gated RMSNorm on the recurrence's output (NextTransformer "Source notes",
 * row gdn: output RMSNorm x gain x SiLU gate; "Backend and numerical limits"):
 *   y = o / sqrt(mean(o^2) + eps) * weight * SiLU(z)
 * per row of D elements (one head of one token). o, z, y: [rows, D] in `dtype`
 * (GDR_BF16 or GDR_FP32; arithmetic in fp32); weight: [D] fp32. D must be 64
 * or 128 (else GDR_ERR_UNSUPPORTED). y may alias o (in place). o, z and y
 * 16-byte aligned, weight 4-byte aligned.
 */
GDR_API int gdr_rmsnorm_gated(const void *o, const void *z, const float *weight, void *y, long rows, int D,
                              float eps, int dtype, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H */
