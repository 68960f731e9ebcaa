/*
 * gswa.h -- C ABI of the ZGCM-1 attention core on B200 (sm_100a).
 *
 * The operation (ZGCM-1, §2.1 Model overview and Figure 3 caption; §2.3
 * KV-cache analysis; §3.2 Mid-training): for projected queries q, keys k,
 * values v and gate logits g of one attention layer,
 *
 *   q~ = RoPE(RMSNorm(q) * w_q),  k~ = RoPE(RMSNorm(k) * w_k)
 *        RMSNorm per (token, head) over the head dim, eps inside the root;
 *        RoPE rotates the first R dims as pairs (p, p + R/2) by the angle
 *        pos * rope_base^(-2p/R), pos = 0-based token index;
 *   s_ij = scale * <q~_i, k~_j>, query head h reads KV head h / (Hq/Hkv);
 *   gated sliding-window layers: key j visible to query i iff i-W < j <= i,
 *        y_i = softmax_j(s_ij) V  ⊙  sigmoid(g_i)        (GatedSWA core)
 *   global layers: key j visible iff j <= i, y_i = softmax_j(s_ij) V.
 * The q/k/v/g projections before and o_proj after are not part of it.
 *
 * Conventions shared by every entry point:
 *   - Layouts are dense row-major: q, g, y, dq, dg, dy: [B, T, Hq, D];
 *     k, v, dk, dv: [B, T, Hkv, D]; w_q, w_k: [D]; lse: [B, Hq, T].
 *     Tensors are bf16 unless stated; lse and dw are float32.
 *   - Pointers marked "device" must point to device memory of the current
 *     CUDA device; tensor pointers must be 16-byte aligned.
 *   - Ownership: the caller owns every buffer.  The library allocates no
 *     device memory, keeps no pointer past the call and frees nothing.
 *     Workspace, when an operation needs one, is caller-provided and sized
 *     by gswa_workspace_bytes().
 *   - Execution: asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  Argument errors are reported synchronously by the
 *     return value; a device-side wait that gave up (a bounded wait that
 *     timed out) is reported by gswa_check_status().
 *   - Supported shapes: D = 128, Hq = 4 * Hkv, R in {0, 42, 64, 128},
 *     1 <= window <= 128 for the sliding-window entry points.
 *   - No C++ exception crosses this interface.
 */
#ifndef GSWA_H
#define GSWA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define GSWA_OK 0
#define GSWA_ERR_INVALID_ARG (-1)       /* null pointer, negative size, bad enum */
#define GSWA_ERR_UNSUPPORTED_SHAPE (-2) /* D != 128, Hq != 4*Hkv, window out of range ... */
#define GSWA_ERR_MISALIGNED (-3)        /* a tensor pointer is not 16-byte aligned */
#define GSWA_ERR_WORKSPACE_TOO_SMALL (-4)
#define GSWA_ERR_LAUNCH (-5)            /* a CUDA runtime call failed */
#define GSWA_ERR_TIMEOUT (-6)           /* a bounded device wait gave up */
#define GSWA_ERR_UNIMPLEMENTED (-7)
#define GSWA_ERR_NO_DEVICE (-8)         /* no sm_100 device current */
#define GSWA_ERR_SCRATCH_LIMIT (-9)     /* full_decode_noalloc: shape needs more than its fixed scratch */

/* Operation ids for gswa_workspace_bytes(). */
#define GSWA_OP_GSWA_FWD 0
#define GSWA_OP_FULL_FWD 1
#define GSWA_OP_GSWA_BWD 2
#define GSWA_OP_FULL_BWD 3
#define GSWA_OP_GSWA_DECODE 4
#define GSWA_OP_FULL_DECODE 5

/* Problem description (plain values, passed by pointer, read during the call only). */
typedef struct gswa_shape {
    int32_t B;         /* batch (sequences) */
    int32_t T;         /* tokens per sequence (prefill/backward); unused by decode */
    int32_t Hq;        /* query heads (32 in ZGCM-1) */
    int32_t Hkv;       /* key/value heads (8 in ZGCM-1); Hq = 4 * Hkv */
    int32_t D;         /* head dim; must be 128 */
    int32_t window;    /* W of the sliding window (128 in ZGCM-1); ring-cache slots in decode */
    int32_t rope_dims; /* R rotated dims (42 = 0.33 of 128, rounded to even) */
    int32_t cache_len; /* decode with a linear cache: capacity Tmax of the cache */
    double rope_base;  /* 1e4, or 1e7 for the 256K stage (§3.2) */
    float eps;         /* RMSNorm epsilon (1e-6) */
    float scale;       /* softmax scale (1/sqrt(D)) */
} gswa_shape_t;

/*
 * Gated sliding-window attention forward (§2.1 Figure 3: A_SWA(q,k,v) ⊙ σ(g)).
 *   q, g [B,T,Hq,D], k, v [B,T,Hkv,D], w_q, w_k [D]: device, bf16, read.
 *   y [B,T,Hq,D] bf16: device, written (gated output).
 *   lse [B,Hq,T] f32: device, written (natural-log softmax normaliser of each
 *     row, for the backward); may be NULL.
 *   workspace: gswa_workspace_bytes(GSWA_OP_GSWA_FWD) bytes (device, 16-byte
 *     aligned), overwritten; it receives the prepared keys k~ [B,T,Hkv,D]
 *     (each key block is read by five consecutive query blocks, so it is
 *     normed and rotated once).  GSWA_ERR_WORKSPACE_TOO_SMALL if smaller.
 */
int gswa_fwd(const gswa_shape_t *shape, const void *q, const void *k, const void *v,
             const void *g, const void *w_q, const void *w_k, void *y, float *lse,
             void *workspace, size_t workspace_bytes, void *stream);

/*
 * Full causal attention forward of the 5 global layers (§2.1: global
 * layers attend over the whole context and drop the gate).  Same layouts
 * as gswa_fwd without g; shape->window is ignored.  Needs a workspace of
 * gswa_workspace_bytes(GSWA_OP_FULL_FWD) bytes (device, 16-byte aligned):
 * it receives the prepared keys and queries (each key tile is reused by
 * every later query block, so it is normed and rotated once).
 */
int full_attn_fwd(const gswa_shape_t *shape, const void *q, const void *k, const void *v,
                  const void *w_q, const void *w_k, void *y, float *lse, void *workspace,
                  size_t workspace_bytes, void *stream);

/*
 * Backward of gswa_fwd: the gradients a training step of the gated-SWA layers
 * needs (ZGCM-1 §2.2 hybrid-attention experiments, whose models are trained
 * at sequence length 4,096; §3.1 pre-training hyperparameters).  With
 * σ = sigmoid(g), A = y / σ and the forward's P:
 *   dA = dy ⊙ σ, dg = dy ⊙ y ⊙ (1 - σ), D_i = Σ_d dy_i y_i,
 *   dV = Σ_heads P^T dA, dS = P ⊙ (dA V^T - D), dq~ = scale dS K~,
 *   dk~ = scale Σ_heads dS^T Q~, then back through RoPE (the transposed
 *   rotation) and RMSNorm to dq, dk, dw_q, dw_k.
 *   Reads q, k, v, g, w_q, w_k, the forward's y and lse (as gswa_fwd wrote
 *   them; the softmax is recomputed from lse, not stored), and the upstream
 *   gradient dy [B,T,Hq,D].  Writes dq, dg [B,T,Hq,D], dk, dv [B,T,Hkv,D]
 *   (bf16) and dw_q, dw_k [D] (f32, summed over every token and head).  All
 *   device.  workspace: gswa_workspace_bytes(GSWA_OP_GSWA_BWD) bytes (device,
 *   16-byte aligned), overwritten.  Results are bitwise reproducible.
 *   B * T = 0 writes zero weight gradients and nothing else.
 */
int gswa_bwd(const gswa_shape_t *shape, const void *q, const void *k, const void *v,
             const void *g, const void *w_q, const void *w_k, const void *y, const float *lse,
             const void *dy, void *dq, void *dk, void *dv, void *dg, float *dw_q, float *dw_k,
             void *workspace, size_t workspace_bytes, void *stream);

/*
 * Backward of full_attn_fwd, the global layers' share of a training step
 * (ZGCM-1 §2.1: global layers attend over the whole causal context, no gate;
 * §2.2 and §3.1 as for gswa_bwd).  The formulas of gswa_bwd with σ = 1
 * (dA = dy) over every key j <= i; no g, no dg.  Layouts, workspace
 * (gswa_workspace_bytes(GSWA_OP_FULL_BWD)) and ownership as for gswa_bwd.
 * dk, dv and dw_k are bitwise reproducible; dq~ is summed in f32 by
 * atomic adds whose order across key tiles is not fixed, so dq and dw_q may
 * differ between runs in their last bits.
 */
int full_attn_bwd(const gswa_shape_t *shape, const void *q, const void *k, const void *v,
                  const void *w_q, const void *w_k, const void *y, const float *lse,
                  const void *dy, void *dq, void *dk, void *dv, float *dw_q, float *dw_k,
                  void *workspace, size_t workspace_bytes, void *stream);

/*
 * One decode step of a gated sliding-window layer over a ring KV cache
 * (§2.3: the SWA layers keep a fixed window of W tokens in the cache).
 *   q, g [B,Hq,D], k, v [B,Hkv,D]: the new token's projections (device, bf16).
 *   k_ring, v_ring [B,Hkv,W,D] bf16 (device, read and written): the token at
 *     position t lives in slot t mod W; k_ring holds normed+rotated keys,
 *     v_ring raw values.  The new token is written to slot pos mod W and is
 *     part of its own window; slots holding positions < 0 are ignored.
 *   pos [B] int64 (device): position of the new token of each sequence.
 *   y [B,Hq,D] bf16 (device, written).  shape->window = W = ring slots
 *   (1..128).  No workspace.  A negative pos skips that sequence and is
 *   reported by gswa_check_status().
 */
int gswa_decode(const gswa_shape_t *shape, const void *q, const void *k, const void *v,
                const void *g, const void *w_q, const void *w_k, void *k_ring, void *v_ring,
                const int64_t *pos, void *y, void *workspace, size_t workspace_bytes,
                void *stream);

/*
 * One decode step of a global layer over a linear cache [B,Hkv,Tmax,D]
 * (Tmax = shape->cache_len): writes the prepared key and the value of the
 * new token at row pos and attends over rows 0..pos (positions must lie in
 * [0, Tmax); others skip the sequence and are reported by
 * gswa_check_status()).  q, k, v, pos, y as in gswa_decode (no gate).
 * Split over the cache length in 4096-key chunks whose partial softmax states
 * are merged by log-sum-exp weight; needs gswa_workspace_bytes(
 * GSWA_OP_FULL_DECODE) bytes of workspace (device, 16-byte aligned).
 */
int full_decode(const gswa_shape_t *shape, const void *q, const void *k, const void *v,
                const void *w_q, const void *w_k, void *k_cache, void *v_cache,
                const int64_t *pos, void *y, void *workspace, size_t workspace_bytes,
                void *stream);

/*
 * full_decode without a caller-supplied workspace, for callers that may not
 * allocate device memory at all: an inference loop that runs under a fixed
 * memory budget or must never stall on an allocator, or plain C code with no
 * allocator of its own to draw a workspace from.  The ZGCM-1 report has no
 * counterpart of this entry point; it is a convenience of this library.
 *
 * Arguments, layouts, results and the position rules are those of
 * full_decode.  The scratch it needs (the same gswa_workspace_bytes(
 * GSWA_OP_FULL_DECODE) bytes) comes from one array of
 * GSWA_NOALLOC_SCRATCH_BYTES (36 MiB) that the library holds in device
 * memory, one per device, set aside when the library's kernels are loaded on
 * that device.  Nothing in that scratch needs to start at zero: every byte a
 * call reads was written earlier in the same call.
 *
 * - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library.
 * - The first call on a device does a one-time set-up (it looks up the
 *   scratch's device address with that device current); make that first call
 *   before any stream capture begins.
 * - Shapes that need more than GSWA_NOALLOC_SCRATCH_BYTES are rejected with
 *   GSWA_ERR_SCRATCH_LIMIT before anything runs.  36 MiB covers, for
 *   example, 32 sequences of 8 KV heads over a 262,144-token cache
 *   (33.5 MiB).
 * - All calls on one device share the one scratch: two calls whose work can
 *   overlap in time (on different streams, or from different host threads
 *   without ordering between them) race on it and give wrong results.  Issue
 *   them on one stream, or order them with events.
 */
#define GSWA_NOALLOC_SCRATCH_BYTES ((size_t)36 << 20)
int full_decode_noalloc(const gswa_shape_t *shape, const void *q, const void *k, const void *v,
                        const void *w_q, const void *w_k, void *k_cache, void *v_cache,
                        const int64_t *pos, void *y, void *stream);

/*
 * QK-RMSNorm + partial RoPE of a head tensor on its own (§2.1 Figure 3: the
 * prologue of the attention core): out[b,t,h,:] = RoPE_{pos0+t}(RMSNorm(
 * x[b,t,h,:]) * w).  x, out [B,T,H,D] bf16 (device; may not alias), w [D]
 * bf16 (device).  Uses shape->B, T, D, rope_dims, rope_base, eps.  Fills
 * decode caches, which hold prepared keys.
 */
int gswa_qk_prep(const gswa_shape_t *shape, int H, const void *x, const void *w, void *out,
                 int64_t pos0, void *stream);

/* Workspace bytes an operation needs for `shape` (0 when none). */
size_t gswa_workspace_bytes(int op, const gswa_shape_t *shape);

/*
 * KV-cache bytes of a layer stack at context length T (§2.3): every cached
 * token costs 2 * Hkv * D * bytes_per_elem bytes per layer; a global layer
 * caches all T tokens, a sliding-window layer min(T, window).  Host only.
 * Returns -1 on a negative argument.
 */
int64_t gswa_kv_cache_bytes(int n_global_layers, int n_window_layers, int window, int Hkv,
                            int D, int bytes_per_elem, int64_t T);

/*
 * Synchronises `stream`, then reads and clears the device status word of the
 * current device: GSWA_OK, GSWA_ERR_TIMEOUT if a bounded wait inside a
 * kernel gave up since the last check, GSWA_ERR_INVALID_ARG if a decode step
 * found a position outside its cache (that sequence was skipped), or
 * GSWA_ERR_LAUNCH on a CUDA error.
 */
int gswa_check_status(void *stream);

/*
 * Failure-detection hook: every bounded wait inside the kernels of this
 * library gives up after `ns` nanoseconds of wall time on the current device
 * instead of the default 4 s (ns = 0 restores the default).  A kernel whose
 * wait gives up stops all of its roles, lets its in-flight copies land,
 * frees its tensor memory and returns; gswa_check_status() then reports
 * GSWA_ERR_TIMEOUT and the outputs of that call are undefined.  Meant for
 * tests that exercise that path; synchronous (it waits for the device).
 * Returns GSWA_OK or GSWA_ERR_LAUNCH.
 */
int gswa_set_wait_limit_ns(uint64_t ns);

/* Human-readable name of a return code (static string). */
const char *gswa_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* GSWA_H */
