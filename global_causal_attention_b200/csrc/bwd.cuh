// bwd.cuh -- backward of the gated sliding-window attention core, and the
// pieces the full causal backward (bwd_full.cuh) shares with it, for sm_100a.
//
// The forward (ZGCM-1 §2.1, Figure 3 caption) is, per query row i of head h
// (kv head h / 4), with q~ = RoPE(RMSNorm(q) w_q), k~ = RoPE(RMSNorm(k) w_k):
//   S_ij = scale <q~_i, k~_j>,  P_ij = exp(S_ij - lse_i) over the visible j,
//   A_i = sum_j P_ij v_j,  y_i = A_i ⊙ σ(g_i) (gated) or A_i (global layers).
// Its gradients, given dy:
//   dA = dy ⊙ σ(g),  dg = dy ⊙ y ⊙ (1 - σ(g))            (ungated: dA = dy)
//   D_i = sum_d dA_i A_i = sum_d dy_i y_i
//   dV_j = sum_i P_ij dA_i,  dP_ij = <dA_i, v_j>,  dS_ij = P_ij (dP_ij - D_i)
//   dq~_i = scale sum_j dS_ij k~_j,  dk~_j = scale sum_i dS_ij q~_i
//   dq = RMSNorm'(RoPE^T(dq~)), dk likewise, dw_q = sum dq^ ⊙ n_q, dw_k likewise.
//
// Kernels:
//   bwd_prep     per row: D and lse log2 e into a row-ordered record, dA and
//                dg (gated only); shared with the full causal backward
//   bwd_dq_swa   query-stationary (M = 128 rows = 4 heads x 32 tokens): S =
//                Q~K~^T and dP = dA V^T into TMEM over the unit's 160-key
//                span from K~/V rings kept across consecutive units; P from
//                the forward's lse; dS (bf16); dQ~ += dS K~ in TMEM;
//                epilogue: RoPE^T and the RMSNorm backward against the raw q,
//                per-warp dw_q partials
//   bwd_dkdv     key-stationary (M = 128 keys of one kv head): per 64-row
//                query chunk (16 tokens x 4 heads) S^T = K~Q~^T and
//                dP^T = V dA^T; P^T and dS^T (bf16, shared memory);
//                dV += P^T dA and dK~ += dS^T Q~ in TMEM; epilogue: dv, and
//                RoPE^T + RMSNorm backward against the raw k, dw_k partials
//   dw_reduce    fixed-order sum of the weight-gradient partials
// q~ and k~ come from qk_prep (workspace).  No atomics on global memory: the
// results do not depend on scheduling.
#pragma once

#include <cuda.h>

#include "ptx.cuh"
#include "swa_fwd.cuh"

namespace gswa {
namespace bwd {

constexpr int kD = 128;
constexpr int kThreads = 384;
constexpr int kMaxGrid = 256;                 // bound on CTAs of the main kernels (partials sizing)
constexpr uint32_t kHalfRowBytes = 128;       // one swizzled 64-dim half row

// ------------------------------------------------------------------ pre-pass
// Row record of the attention backward: {lse_i log2 e, D_i}, rows ordered
// [B, Hkv, Tp, 4] (Tp = T rounded up to 32) so that the rows of one tile are
// contiguous; rows t >= T hold {+inf, 0}, which makes their P exactly 0.
struct PrepParams {
    const __nv_bfloat16 *y, *dy, *g;   // g null: ungated
    const float *lse;                  // [B, Hq, T]
    __nv_bfloat16 *dA, *dg;            // [B, T, Hq, D]; null when ungated
    float2 *ld;                        // [B, Hkv, Tp, 4]
    long long rows;                    // B * Tp * Hq
    int T, Tp, Hq;
};

constexpr int kPrepUnroll = 4;   // heads (rows) in flight per half-warp

// A half-warp takes one token (b, t) at a time and walks its Hq rows four
// heads at a time (one kv group, so the four records are contiguous); lane =
// 8 dims, 16-byte accesses.  Tokens t >= T (the padding up to Tp) get
// records only.
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __grid_constant__ PrepParams p)
{
    const int lane = threadIdx.x & 31, l16 = lane & 15;
    // the two half-warps of a warp may take different branches: shuffle within one
    const unsigned half_mask = 0xFFFFu << (lane & 16);
    const unsigned nhw = gridDim.x * 16u;   // half-warps in the grid
    const unsigned ntok = (unsigned)(p.rows / p.Hq);   // B * Tp
    const int Hkv = p.Hq / 4;
    for (unsigned bt = blockIdx.x * 16u + (threadIdx.x >> 4); bt < ntok; bt += nhw) {
        const unsigned b = bt / (unsigned)p.Tp;
        const int t = (int)(bt - b * (unsigned)p.Tp);
        float2 *rec = p.ld + ((long long)b * Hkv * p.Tp + t) * 4;   // + (kvh Tp) 4 + h % 4
        if (t >= p.T) {
            // padded token: P = 0 for every key
            if (l16 < Hkv * 4)
                for (int h = l16; h < p.Hq; h += 16)
                    rec[(long long)(h >> 2) * p.Tp * 4 + (h & 3)] = make_float2(INFINITY, 0.f);
            continue;
        }
        const long long row0 = ((long long)b * p.T + t) * p.Hq;
        for (int h0 = 0; h0 < p.Hq; h0 += kPrepUnroll) {
            uint4 yv[kPrepUnroll], dv[kPrepUnroll], gv[kPrepUnroll];
#pragma unroll
            for (int u = 0; u < kPrepUnroll; ++u) {
                const long long off = (row0 + h0 + u) * kD + 8 * l16;
                yv[u] = *reinterpret_cast<const uint4 *>(p.y + off);
                dv[u] = *reinterpret_cast<const uint4 *>(p.dy + off);
                if (p.g != nullptr) gv[u] = *reinterpret_cast<const uint4 *>(p.g + off);
            }
            float dsum[kPrepUnroll];
#pragma unroll
            for (int u = 0; u < kPrepUnroll; ++u) {
                const uint32_t ya[4] = {yv[u].x, yv[u].y, yv[u].z, yv[u].w};
                const uint32_t da[4] = {dv[u].x, dv[u].y, dv[u].z, dv[u].w};
                float s = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 yy = unpack_bf16(ya[e]), dd = unpack_bf16(da[e]);
                    s = fmaf(dd.x, yy.x, fmaf(dd.y, yy.y, s));
                }
                dsum[u] = s;
                if (p.g != nullptr) {
                    const uint32_t ga[4] = {gv[u].x, gv[u].y, gv[u].z, gv[u].w};
                    uint32_t oa[4], og[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 gg = unpack_bf16(ga[e]), yy = unpack_bf16(ya[e]), dd = unpack_bf16(da[e]);
                        const float s0 = 1.f / (1.f + __expf(-gg.x)), s1 = 1.f / (1.f + __expf(-gg.y));
                        oa[e] = pack_bf16(dd.x * s0, dd.y * s1);
                        og[e] = pack_bf16(dd.x * yy.x * (1.f - s0), dd.y * yy.y * (1.f - s1));
                    }
                    const long long off = (row0 + h0 + u) * kD + 8 * l16;
                    *reinterpret_cast<uint4 *>(p.dA + off) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
                    *reinterpret_cast<uint4 *>(p.dg + off) = make_uint4(og[0], og[1], og[2], og[3]);
                }
            }
#pragma unroll
            for (int o = 8; o > 0; o >>= 1)
#pragma unroll
                for (int u = 0; u < kPrepUnroll; ++u) dsum[u] += __shfl_xor_sync(half_mask, dsum[u], o);
            if (l16 < kPrepUnroll) {
                // lane u of the half-warp writes the record of head h0 + u
                float dv_u = dsum[0];
#pragma unroll
                for (int u = 1; u < kPrepUnroll; ++u) dv_u = (l16 == u) ? dsum[u] : dv_u;
                const int h = h0 + l16;
                rec[(long long)(h >> 2) * p.Tp * 4 + (h & 3)] =
                    make_float2(p.lse[((long long)b * p.Hq + h) * p.T + t] * 1.4426950408889634f, dv_u);
            }
        }
    }
}

// dw[d] = sum over the partials, in a fixed order (deterministic): thread
// (slice s, dim d) sums partials s, s + 8, ... in order, then the 8 slice
// sums are added in slice order.
constexpr int kReduceSlices = 8;
__global__ void __launch_bounds__(kD * kReduceSlices) dw_reduce_kernel(const float *part, int nparts, float *dw)
{
    __shared__ float acc[kReduceSlices][kD];
    const int d = threadIdx.x & (kD - 1), sl = threadIdx.x / kD;
    float s0 = 0.f, s1 = 0.f;
    int i = sl;
    for (; i + kReduceSlices < nparts; i += 2 * kReduceSlices) {
        s0 += part[(long long)i * kD + d];
        s1 += part[(long long)(i + kReduceSlices) * kD + d];
    }
    if (i < nparts) s0 += part[(long long)i * kD + d];
    acc[sl][d] = s0 + s1;
    __syncthreads();
    if (sl == 0) {
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < kReduceSlices; ++k) s += acc[k][d];
        dw[d] = s;
    }
}

// --------------------------------------------------------- shared machinery
struct Params {
    int B, T, Tp, Hq, Hkv, window;   // window: sliding-window width (ignored by the full kernels)
    int nq;                          // query blocks of 32 tokens
    int nkt;                         // key tiles (dq: of kN keys; dkdv: of 128 keys)
    long long units;
    float eps, sl2, scale;           // sl2 = scale log2 e
    const float2 *ld;                // row records (see PrepParams)
    const __nv_bfloat16 *x;          // raw q (dq kernel) or raw k (dkdv kernel)
    const __nv_bfloat16 *w;          // w_q or w_k
    __nv_bfloat16 *dx;               // dq or dk
    __nv_bfloat16 *dv;               // dkdv kernel: dv
    float *dw_part;                  // [gridDim.x * 4][128] per-warp partial weight gradients
    double theta[64];
};

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity)
{
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer() - t0 > 200000000ull) break;
}

// k-th unit of this CTA in a longest-first "snake" order over `units`
// (unit u of the order goes to CTA u mod 2G or 2G - 1 - u mod 2G).
__device__ __forceinline__ long long snake_unit(int k)
{
    const long long G = gridDim.x, c = blockIdx.x;
    return (k & 1) ? ((long long)(k + 1) * G - 1 - c) : ((long long)k * G + c);
}

__device__ __forceinline__ int snake_count(long long units)
{
    const long long G = gridDim.x, c = blockIdx.x;
    const long long full = units / (2 * G), rem = units - full * 2 * G;
    return (int)(2 * full + (c < rem ? 1 : 0) + (2 * G - 1 - c < rem ? 1 : 0));
}

// Warp reduce-scatter: on return, lane l holds the warp-wide sum of a[l].
__device__ __forceinline__ float warp_reduce_scatter32(float (&a)[32])
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 16; k >= 1; k >>= 1) {
        const bool upper = (lane & k) != 0;
#pragma unroll
        for (int i = 0; i < k; ++i) {
            const float send = upper ? a[i] : a[i + k];
            const float keep = upper ? a[i + k] : a[i];
            a[i] = keep + __shfl_xor_sync(0xffffffffu, send, k);
        }
    }
    return a[0];
}

// Rotate one TMEM row of 128 f32 gradients back through RoPE_pos^T, in place:
//   (g_p, g_{p+R/2}) <- (g_p c + g_{p+R/2} s, g_{p+R/2} c - g_p s).
template <int R>
__device__ __forceinline__ void rope_back_tmem(uint32_t trow, int pos, const double *theta)
{
    constexpr int H = R / 2;
    if constexpr (R > 0) {
        constexpr int kRounds = (R == 128) ? 2 : 1;
        static_assert(R <= 64 || R == 128, "rotary width");
#pragma unroll
        for (int rd = 0; rd < kRounds; ++rd) {
            // R <= 64: dims 0..63 (chunks 0, 1); R = 128: chunk rd pairs with chunk rd + 2
            const uint32_t ca = trow + 32 * rd, cb = trow + ((R == 128) ? 32 * (rd + 2) : 32);
            uint32_t a[32], b[32];
            tmem_ld32(ca, a);
            tmem_ld32(cb, b);
            tmem_wait_ld();
            if constexpr (R == 128) {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    float c, s;
                    swa::rope_cs(theta[32 * rd + e], pos, c, s);
                    const float g1 = __uint_as_float(a[e]), g2 = __uint_as_float(b[e]);
                    a[e] = __float_as_uint(g1 * c + g2 * s);
                    b[e] = __float_as_uint(g2 * c - g1 * s);
                }
            } else {
                float u[64];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    u[e] = __uint_as_float(a[e]);
                    u[32 + e] = __uint_as_float(b[e]);
                }
#pragma unroll
                for (int pp = 0; pp < H; ++pp) {
                    float c, s;
                    swa::rope_cs(theta[pp], pos, c, s);
                    const float g1 = u[pp], g2 = u[pp + H];
                    u[pp] = g1 * c + g2 * s;
                    u[pp + H] = g2 * c - g1 * s;
                }
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    a[e] = __float_as_uint(u[e]);
                    b[e] = __float_as_uint(u[32 + e]);
                }
            }
            uint32_t lo[16], hi[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                lo[e] = a[e];
                hi[e] = a[16 + e];
            }
            tmem_st16(ca, lo);
            tmem_st16(ca + 16, hi);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                lo[e] = b[e];
                hi[e] = b[16 + e];
            }
            tmem_st16(cb, lo);
            tmem_st16(cb + 16, hi);
        }
        tmem_wait_st();
    }
}

// RoPE^T and RMSNorm backward of one row.  The gradient w.r.t. the prepared
// row is `gscale` times the f32 row at TMEM address `trow` (this thread's
// lane); x is the raw row (bf16, global), pos its position:
//   du = RoPE_pos^T(g);  r = (mean x^2 + eps)^-1/2;  n = x r;
//   dx = r (w ⊙ du - n mean(w ⊙ du ⊙ n));  dw += du ⊙ n.
// Every lane of the warp must call it (TMEM loads are warp-wide); a lane
// with valid == false contributes nothing and writes nothing.  dwacc[c] of
// lane l accumulates dim 32 c + l of the warp's dw sum.
template <int R>
__device__ __forceinline__ void norm_rope_backward(uint32_t trow, float gscale, const __nv_bfloat16 *xrow,
                                                   bool valid, const float *w, float eps, int pos,
                                                   const double *theta, __nv_bfloat16 *dxrow, float (&dwacc)[4])
{
    rope_back_tmem<R>(trow, pos, theta);
    const float gs = valid ? gscale : 0.f;
    const uint4 *xr = reinterpret_cast<const uint4 *>(xrow);
    // pass 1: sum x^2 and sum w g x
    float ss = 0.f, wgx = 0.f;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld32(trow + 32 * c, v);
        uint4 xv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) xv[q] = xr[4 * c + q];
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t x4[4] = {xv[q].x, xv[q].y, xv[q].z, xv[q].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int d = 32 * c + 8 * q + 2 * e;
                const float2 f = unpack_bf16(x4[e]);
                ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
                wgx = fmaf(w[d] * __uint_as_float(v[8 * q + 2 * e]), f.x,
                           fmaf(w[d + 1] * __uint_as_float(v[8 * q + 2 * e + 1]), f.y, wgx));
            }
        }
    }
    const float r = rsqrtf(ss * (1.0f / kD) + eps);
    const float m = gs * r * wgx * (1.0f / kD);   // mean(w du n)
    // pass 2: dx and dw
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld32(trow + 32 * c, v);
        uint4 xv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) xv[q] = xr[4 * c + q];
        tmem_wait_ld();
        float pw[32];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t x4[4] = {xv[q].x, xv[q].y, xv[q].z, xv[q].w};
            uint32_t o4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int d = 32 * c + 8 * q + 2 * e;
                const float2 f = unpack_bf16(x4[e]);
                const float du0 = gs * __uint_as_float(v[8 * q + 2 * e]);
                const float du1 = gs * __uint_as_float(v[8 * q + 2 * e + 1]);
                const float n0 = f.x * r, n1 = f.y * r;
                o4[e] = pack_bf16(r * fmaf(w[d], du0, -n0 * m), r * fmaf(w[d + 1], du1, -n1 * m));
                pw[8 * q + 2 * e] = du0 * n0;
                pw[8 * q + 2 * e + 1] = du1 * n1;
            }
            if (valid) reinterpret_cast<uint4 *>(dxrow)[4 * c + q] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
        dwacc[c] += warp_reduce_scatter32(pw);
    }
}

// ====================================================== dq kernel, sliding window
// Query-stationary: unit = 32 query tokens x 4 heads (M = 128 rows) of one
// (sequence, KV head); its keys are the 160 keys [32 s - 128, 32 s + 32), five
// 32-key blocks.  Persistent CTAs walk a contiguous range of units, strip by
// strip, and keep the K~ and V blocks in six-slot rings (each block is loaded
// once per CTA and serves the five units whose window covers it); Q~ and dA
// tiles have two slots each.  S = Q~K~^T and dP = dA V^T (N = 160, split where
// the window wraps the ring) go to one TMEM buffer; dS = P (dP - D) is written
// as bf16 over S; dQ~ += dS K~ is a TMEM-A MMA over the K~ ring.
struct DqSwaCfg {
    static constexpr int kTok = 32, kSpanBlocks = 5, kRing = 6, kSpan = kSpanBlocks * kTok;
    static constexpr uint32_t kBlockHalf = kTok * kHalfRowBytes;    // 4 KiB: 32 keys x 64 dims
    static constexpr uint32_t kRingHalf = kRing * kBlockHalf;       // 24 KiB
    static constexpr uint32_t kTileHalf = 128 * kHalfRowBytes;      // 16 KiB: 128 rows x 64 dims
    static constexpr uint32_t kTile = 2 * kTileHalf;                // 32 KiB
    static constexpr uint32_t kOffK = 0;
    static constexpr uint32_t kOffV = kOffK + 2 * kRingHalf;        // rings: 48 KiB each
    static constexpr uint32_t kOffQ = kOffV + 2 * kRingHalf;        // Q~: 2 slots
    static constexpr uint32_t kOffA = kOffQ + 2 * kTile;            // dA: 2 slots
    static constexpr uint32_t kOffW = kOffA + 2 * kTile;            // f32[128]
    static constexpr uint32_t kOffBar = kOffW + 512;
    static constexpr int kNumBars = 34;
    static constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
    static constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
    static constexpr uint32_t kSmemBytes = kOffAbort + 4 + 1024;
    static_assert(kSmemBytes <= 232448, "shared memory budget of one sm_100 CTA");
    // TMEM columns: S (dS as bf16 over its first 80), dP, dQ~
    static constexpr uint32_t kColS = 0, kColDP = kSpan, kColDQ = 2 * kSpan;
    static_assert(kColDQ + 128 <= 512, "TMEM budget");
    static constexpr int BQ_FULL = 0, BQ_EMPTY = 2, BK_FULL = 4, BK_EMPTY = BK_FULL + kRing,
                         BV_FULL = BK_EMPTY + kRing, BV_EMPTY = BV_FULL + kRing, BS_FULL = BV_EMPTY + kRing,
                         BS_FREE = BS_FULL + 1, BDS_READY = BS_FREE + 1, BACC_FULL = BDS_READY + 1,
                         BACC_FREE = BACC_FULL + 1, B_DRAIN = BACC_FREE + 1;
    static_assert(B_DRAIN < kNumBars, "barrier count");
};

// Walks units [u0, u1) of a CTA in order: (sequence b, kv head, query block s).
struct SwaWalk {
    int b, kvh, s;
    __device__ __forceinline__ void init(const Params &p, long long u0)
    {
        const long long strip = u0 / p.nq;
        s = (int)(u0 - strip * p.nq);
        b = (int)(strip / p.Hkv);
        kvh = (int)(strip - (long long)b * p.Hkv);
    }
    __device__ __forceinline__ void next(const Params &p)
    {
        if (++s == p.nq) {
            s = 0;
            if (++kvh == p.Hkv) {
                kvh = 0;
                ++b;
            }
        }
    }
    // first unit of the CTA or of a strip: its window's older blocks are not in the ring yet
    __device__ __forceinline__ bool first(int idx) const { return idx == 0 || s == 0; }
    // last unit of the CTA or of a strip: no later unit reads its window's blocks
    __device__ __forceinline__ bool last(const Params &p, int idx, int n) const
    {
        return idx == n - 1 || s == p.nq - 1;
    }
};

__device__ __forceinline__ int dq_ring_slot(int kb)
{
    return ((kb % DqSwaCfg::kRing) + DqSwaCfg::kRing) % DqSwaCfg::kRing;
}

template <int R>
__global__ void __launch_bounds__(kThreads, 1)
bwd_dq_swa_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_a,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ Params p)
{
    using C = DqSwaCfg;
    constexpr int kRing = C::kRing, kSpanBlocks = C::kSpanBlocks, kTok = C::kTok;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffTmemSlot);
    Abort ab{reinterpret_cast<volatile int *>(smem + C::kOffAbort)};
    auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8u * (uint32_t)i; };
    const long long u0 = (long long)blockIdx.x * p.units / gridDim.x;
    const long long u1 = (long long)(blockIdx.x + 1) * p.units / gridDim.x;
    const int n = (int)(u1 - u0);

    if (tid == 0) {
        *ab.flag = 0;
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(C::BQ_FULL + i), 1);
            mbar_init(bar(C::BQ_EMPTY + i), 1);
        }
        for (int i = 0; i < kRing; ++i) {
            mbar_init(bar(C::BK_FULL + i), 1);
            mbar_init(bar(C::BK_EMPTY + i), 1);
            mbar_init(bar(C::BV_FULL + i), 1);
            mbar_init(bar(C::BV_EMPTY + i), 1);
        }
        mbar_init(bar(C::BS_FULL), 1);
        mbar_init(bar(C::BS_FREE), 1);
        mbar_init(bar(C::BDS_READY), 4);
        mbar_init(bar(C::BACC_FULL), 1);
        mbar_init(bar(C::BACC_FREE), 4);
        mbar_init(bar(C::B_DRAIN), 1);
        fence_barrier_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (tid < 128) reinterpret_cast<float *>(smem + C::kOffW)[tid] = __bfloat162float(p.w[tid]);
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 || warp == 2) {
        // ================================================= ring producers: K~ (warp 0), V (warp 2)
        if (lane == 0) {
            const bool is_k = warp == 0;
            const CUtensorMap *tm = is_k ? &tm_k : &tm_v;
            const uint32_t ring = sbase + (is_k ? C::kOffK : C::kOffV);
            const int b_full = is_k ? C::BK_FULL : C::BV_FULL, b_empty = is_k ? C::BK_EMPTY : C::BV_EMPTY;
            uint32_t fills = 0, armed = 0;   // fill parity per slot; slots loaded at least once
            SwaWalk w;
            w.init(p, u0);
            auto load = [&](int kb) -> bool {
                const int slot = dq_ring_slot(kb);
                if (!mbar_wait(bar(b_empty + slot), ((fills >> slot) & 1u) ^ 1u, ab)) return false;
                fills ^= 1u << slot;
                armed |= 1u << slot;
                mbar_arrive_expect_tx(bar(b_full + slot), 2 * C::kBlockHalf);
                for (int h = 0; h < 2; ++h)
                    tma_load_4d(ring + h * C::kRingHalf + slot * C::kBlockHalf, tm, bar(b_full + slot), h * 64,
                                w.kvh, kb * kTok, w.b);
                return true;
            };
            bool ok = true;
            for (int idx = 0; idx < n && ok; ++idx, w.next(p)) {
                if (w.first(idx))
                    for (int kb = w.s - 4; kb < w.s && ok; ++kb) ok = load(kb);
                if (ok) ok = load(w.s);
            }
            for (int slot = 0; slot < kRing; ++slot)
                if (armed & (1u << slot)) drain_wait(bar(b_full + slot), ((fills >> slot) & 1u) ^ 1u);
        }
    } else if (warp == 3) {
        // ================================================= Q~ and dA tiles (two slots)
        if (lane == 0) {
            SwaWalk w;
            w.init(p, u0);
            int idx = 0;
            bool ok = true;
            for (; idx < n && ok; ++idx, w.next(p)) {
                const int j = idx & 1;
                ok = mbar_wait(bar(C::BQ_EMPTY + j), ((idx >> 1) & 1) ^ 1u, ab);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(C::BQ_FULL + j), 2 * C::kTile);
                for (int h = 0; h < 2; ++h) {
                    tma_load_4d(sbase + C::kOffQ + j * C::kTile + h * C::kTileHalf, &tm_q, bar(C::BQ_FULL + j),
                                h * 64, w.kvh * 4, w.s * kTok, w.b);
                    tma_load_4d(sbase + C::kOffA + j * C::kTile + h * C::kTileHalf, &tm_a, bar(C::BQ_FULL + j),
                                h * 64, w.kvh * 4, w.s * kTok, w.b);
                }
            }
            for (int i = (idx > 2 ? idx - 2 : 0); i < idx; ++i) drain_wait(bar(C::BQ_FULL + (i & 1)), (i >> 1) & 1);
        }
    } else if (warp == 1) {
        // ================================================= MMA issuer
        if (lane == 0) {
            const uint32_t idesc_dq = idesc_bf16_f32(128, 128, 0, 1);
            // shared-memory descriptors built once: Q~/dA tiles and the K~/V rings
            // K-major, the K~ ring MN-major as the B operand of dQ~ += dS K~
            const SmemDesc dQt = make_desc(sbase + C::kOffQ, 16, 1024), dAt = make_desc(sbase + C::kOffA, 16, 1024);
            const SmemDesc dKr = make_desc(sbase + C::kOffK, 16, 1024), dVr = make_desc(sbase + C::kOffV, 16, 1024);
            const SmemDesc dKmn = make_desc(sbase + C::kOffK, C::kRingHalf, 1024);
            SwaWalk ws, wd;
            ws.init(p, u0);
            wd.init(p, u0);
            int ns = 0, nd = 0;
            // K~ and V loads are confirmed in their producers' order: block kkb
            // (vkb) is the next one of unit ns's window not yet seen landed
            uint32_t k_fills = 0, v_fills = 0;
            int kkb = ws.s - 4, vkb = ws.s - 4;
            PollWatch watch;
            while (nd < n) {
                bool progressed = false;
                // S(ns) = Q~ K~^T and dP(ns) = dA V^T, once dQ(ns - 1) has read dS(ns - 1)
                if (ns < n && ns == nd) {
                    while (kkb <= ws.s) {
                        const int ks = dq_ring_slot(kkb);
                        if (!mbar_test(bar(C::BK_FULL + ks), (k_fills >> ks) & 1u)) break;
                        k_fills ^= 1u << ks;
                        ++kkb;
                        progressed = true;
                    }
                    while (vkb <= ws.s) {
                        const int vs = dq_ring_slot(vkb);
                        if (!mbar_test(bar(C::BV_FULL + vs), (v_fills >> vs) & 1u)) break;
                        v_fills ^= 1u << vs;
                        ++vkb;
                        progressed = true;
                    }
                    const int j = ns & 1;
                    if (kkb > ws.s && vkb > ws.s && mbar_test(bar(C::BQ_FULL + j), (ns >> 1) & 1) &&
                        mbar_test(bar(C::BS_FREE), (ns & 1) ^ 1u)) {
                        tc_fence_after();
                        const int a = dq_ring_slot(ws.s - 4);
                        const int n1 = (kRing - a) < kSpanBlocks ? (kRing - a) : kSpanBlocks;
                        const int n2 = kSpanBlocks - n1;
                        const uint32_t id1 = idesc_bf16_f32(128, n1 * kTok, 0, 0);
                        const uint32_t id2 = idesc_bf16_f32(128, n2 > 0 ? n2 * kTok : 32, 0, 0);
                        const uint32_t to = (uint32_t)j * C::kTile, ro = (uint32_t)a * C::kBlockHalf;
#pragma unroll
                        for (int op = 0; op < 2; ++op) {
                            // op 0: S from Q~ and the K~ ring; op 1: dP from dA and the V ring
                            const uint32_t dst = tmem + (op == 0 ? C::kColS : C::kColDP);
                            const SmemDesc &dt = op == 0 ? dQt : dAt;
                            const SmemDesc &dr = op == 0 ? dKr : dVr;
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk) {
                                const uint32_t h = kk >> 2, ko = (kk & 3) * 32;
                                const uint64_t ad = dt.at(to + h * C::kTileHalf + ko);
                                mma_ss(dst, ad, dr.at(h * C::kRingHalf + ko + ro), id1, kk > 0);
                                if (n2 > 0) mma_ss(dst + n1 * kTok, ad, dr.at(h * C::kRingHalf + ko), id2, kk > 0);
                            }
                        }
                        mma_commit(bar(C::BS_FULL));
                        mma_commit(bar(C::BQ_EMPTY + j));
                        // V slots that no later unit of this CTA reads (dP was their last use)
                        if (ws.last(p, ns, n)) {
                            for (int i = 0; i < kSpanBlocks; ++i) mma_commit(bar(C::BV_EMPTY + (a + i) % kRing));
                        } else {
                            mma_commit(bar(C::BV_EMPTY + a));
                        }
                        ws.next(p);
                        ++ns;
                        kkb = vkb = ws.first(ns) ? ws.s - 4 : ws.s;
                        progressed = true;
                    }
                }
                // dQ~(nd) = dS K~ over the same window, once the epilogue has read dQ~(nd - 1)
                if (nd < ns && mbar_test(bar(C::BDS_READY), nd & 1) &&
                    mbar_test(bar(C::BACC_FREE), (nd & 1) ^ 1u)) {
                    tc_fence_after();
                    const int a = dq_ring_slot(wd.s - 4);
#pragma unroll
                    for (int kk = 0; kk < C::kSpan / 16; ++kk) {
                        const int sl = a + (kk >> 1);
                        const int slot = sl >= kRing ? sl - kRing : sl;   // a + i < 2 kRing
                        mma_ts(tmem + C::kColDQ, tmem + C::kColS + kk * 8,
                               dKmn.at((uint32_t)slot * C::kBlockHalf + (kk & 1) * 16 * kHalfRowBytes), idesc_dq, kk > 0);
                    }
                    mma_commit(bar(C::BS_FREE));
                    mma_commit(bar(C::BACC_FULL));
                    // K~ slots that no later unit of this CTA reads
                    if (wd.last(p, nd, n)) {
                        for (int i = 0; i < kSpanBlocks; ++i) mma_commit(bar(C::BK_EMPTY + (a + i) % kRing));
                    } else {
                        mma_commit(bar(C::BK_EMPTY + a));
                    }
                    wd.next(p);
                    ++nd;
                    progressed = true;
                }
                if (!watch.tick(progressed, ab)) break;
            }
            mma_commit(bar(C::B_DRAIN));
            drain_wait(bar(C::B_DRAIN), 0);
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 8) {
        // ================================================= dS = P (dP - D), bf16 over S
        const int r = tid - 128;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const int W = p.window;
        const uint64_t sl2_2 = f2_pack(p.sl2, p.sl2);
        SwaWalk w;
        w.init(p, u0);
        bool ok = true;
        for (int idx = 0; idx < n && ok; ++idx, w.next(p)) {
            const float2 rec = p.ld[(((long long)w.b * p.Hkv + w.kvh) * p.Tp + w.s * kTok) * 4 + r];
            const uint64_t nlse2 = f2_pack(-rec.x, -rec.x), nD2 = f2_pack(-rec.y, -rec.y);
            const int i = w.s * kTok + (r >> 2);
            const int key0 = w.s * kTok - 128;
            const int hi = i - key0;                     // visible columns: lo <= c <= hi
            const int lo = max(-key0, hi - W + 1);
            ok = warp_wait(bar(C::BS_FULL), idx & 1, ab);
            if (!ok) break;
            tc_fence_after();
            const uint32_t ts = tmem + lane_base + C::kColS, td = tmem + lane_base + C::kColDP;
#pragma unroll 1
            for (int c = 0; c < kSpanBlocks; ++c) {
                uint32_t sv[32], dv[32], pk[16];
                tmem_ld32(ts + 32 * c, sv);
                tmem_ld32(td + 32 * c, dv);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    // two columns per f32x2 instruction (same per-lane rounding as the scalar form)
                    const int col = 32 * c + e;
                    const float2 x = f2_unpack(
                        f2_fma(f2_pack(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sl2_2, nlse2));
                    float p0 = ex2(x.x);
                    float p1 = ex2(x.y);
                    p0 = (col >= lo && col <= hi) ? p0 : 0.f;
                    p1 = (col + 1 >= lo && col + 1 <= hi) ? p1 : 0.f;
                    const uint64_t dd = f2_add(f2_pack(__uint_as_float(dv[e]), __uint_as_float(dv[e + 1])), nD2);
                    const float2 ds = f2_unpack(f2_mul(f2_pack(p0, p1), dd));
                    pk[e >> 1] = pack_bf16(ds.x, ds.y);
                }
                // dS of chunk c lands on S columns 16 c .. 16 c + 15 (chunk c / 2, already read)
                tmem_st16(ts + 16 * c, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::BDS_READY));
        }
    } else if (warp >= 8) {
        // ================================================= epilogue: dq, dw_q
        const int r = tid - 256;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const float *w = reinterpret_cast<const float *>(smem + C::kOffW);
        float dwacc[4] = {0.f, 0.f, 0.f, 0.f};
        SwaWalk wk;
        wk.init(p, u0);
        bool ok = true;
        for (int idx = 0; idx < n && ok; ++idx, wk.next(p)) {
            const int i = wk.s * kTok + (r >> 2);
            const bool valid = i < p.T;
            const long long off = valid ? (((long long)wk.b * p.T + i) * p.Hq + wk.kvh * 4 + (r & 3)) * kD : 0;
            // the raw q row (two 128-byte lines) is read twice below: start it toward L2 while dQ~ is computed
            if (valid) {
                prefetch_l2(p.x + off);
                prefetch_l2(p.x + off + 64);
            }
            ok = warp_wait(bar(C::BACC_FULL), idx & 1, ab);
            if (!ok) break;
            tc_fence_after();
            norm_rope_backward<R>(tmem + lane_base + C::kColDQ, p.scale, p.x + off, valid, w, p.eps, i, p.theta,
                                  p.dx + off, dwacc);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::BACC_FREE));
        }
        float *dst = p.dw_part + ((long long)blockIdx.x * 4 + (warp & 3)) * kD;
#pragma unroll
        for (int c = 0; c < 4; ++c) dst[32 * c + lane] = dwacc[c];
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Store 32 consecutive bf16 (16 packed words) as chunks c0 .. c0 + 3 of row
// `row` of a single-half swizzled K-major tile (128-byte rows).
__device__ __forceinline__ void sts_row_chunks(uint32_t tile, int row, int c0, const uint32_t (&w)[16])
{
#pragma unroll
    for (int q = 0; q < 4; ++q)
        sts128(tile + (uint32_t)row * kHalfRowBytes + ((uint32_t)((c0 + q) ^ (row & 7)) << 4),
               make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]));
}

// ============================================================ dk/dv kernel
// Key-stationary (M = 128 keys of one KV head).  Per 64-row query chunk (16
// tokens x 4 heads): S^T = K~ Q~^T and dP^T = V dA^T into one of two TMEM
// buffers; eight warps (two per TMEM lane quarter, each taking 32 of the 64
// columns) load them, release the buffer at once, and write P^T and dS^T as
// bf16 into shared memory, from where dV += P^T dA and dK~ += dS^T Q~ read
// them.  So the next chunk's scores are computed while this chunk's
// probabilities are formed, and every contraction runs at N >= 64 from
// shared memory.  Two threads issue the MMAs (warp 1 the scores, warp 2 dV
// and dK~), each committing only its own products.  The same eight warps run
// the epilogue: dv (warps 4-7), dk through RoPE^T and the RMSNorm backward
// (warps 8-11).  The sliding-window backward only: the full causal one is the
// fused kernel of bwd_full.cuh.
struct KvCfg {
    static constexpr int kM = 64;                    // query rows per chunk (16 tokens x 4 heads)
    static constexpr int kChTok = 16;
    static constexpr int kStages = 3;
    static constexpr uint32_t kKHalf = 128 * kHalfRowBytes;   // 16 KiB
    static constexpr uint32_t kKTile = 2 * kKHalf;
    static constexpr uint32_t kCHalf = kM * kHalfRowBytes;    // 8 KiB
    static constexpr uint32_t kCTile = 2 * kCHalf;
    static constexpr uint32_t kRecBytes = kM * 8;             // {lse log2 e, D} per row
    static constexpr uint32_t kStageBytes = 2 * kCTile + 1024;   // Q~ chunk, dA chunk, records
    static constexpr uint32_t kPTile = 128 * kHalfRowBytes;   // P^T or dS^T: 128 keys x 64 rows bf16
    static constexpr uint32_t kOffK = 0;
    static constexpr uint32_t kOffV = kOffK + kKTile;
    static constexpr uint32_t kOffCh = kOffV + kKTile;
    static constexpr uint32_t kOffP = kOffCh + kStages * kStageBytes;
    static constexpr uint32_t kOffDS = kOffP + kPTile;
    static constexpr uint32_t kOffW = kOffDS + kPTile;
    static constexpr uint32_t kOffBar = kOffW + 512;
    static constexpr int kNumBars = 24;
    static constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
    static constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
    static constexpr uint32_t kSmemBytes = kOffAbort + 4 + 1024;
    // TMEM columns: two {S^T, dP^T} buffers, dV, dK~
    static constexpr uint32_t kColBuf = 0, kBufStride = 128, kColDV = 256, kColDK = 384;
    static_assert(kSmemBytes <= 232448, "shared memory budget of one sm_100 CTA");
    static constexpr int BKV_FULL = 0, BKV_EMPTY = 1, BCH_FULL = 2, BCH_EMPTY = BCH_FULL + kStages,
                         BS_FULL = BCH_EMPTY + kStages, BS_FREE = BS_FULL + 2, BPS_READY = BS_FREE + 2,
                         BPS_FREE = BPS_READY + 1, BACC_FULL = BPS_FREE + 1, BACC_FREE = BACC_FULL + 1,
                         B_DRAIN = BACC_FREE + 1 /* 2: one per issuer */;
    static_assert(B_DRAIN + 1 < kNumBars, "barrier count");
};

struct KUnit {
    int b, kvh, kt, n;   // n: query chunks of the unit
};

__device__ __forceinline__ bool kv_unit_at(const Params &p, int k, KUnit &x)
{
    const long long u = snake_unit(k);
    if (u >= p.units) return false;
    const long long per = (long long)p.B * p.Hkv;
    x.kt = (int)(u / per);
    const long long strip = u % per;
    x.b = (int)(strip / p.Hkv);
    x.kvh = (int)(strip % p.Hkv);
    const int k0 = 128 * x.kt;
    // queries that see keys [k0, k0 + 128): i in [k0, k0 + 127 + W - 1]
    const int span = min(127 + p.window, p.T - k0);
    x.n = (span + KvCfg::kChTok - 1) / KvCfg::kChTok;
    return true;
}

struct KvWalk {
    int k = 0, j = 0;
    KUnit x;
    bool valid = false;
    __device__ __forceinline__ void init(const Params &p) { k = 0; j = 0; valid = kv_unit_at(p, 0, x); }
    __device__ __forceinline__ bool last() const { return j == x.n - 1; }
    __device__ __forceinline__ void next(const Params &p)
    {
        if (++j == x.n) {
            j = 0;
            ++k;
            valid = kv_unit_at(p, k, x);
        }
    }
};

template <int R>
__global__ void __launch_bounds__(kThreads, 1)
bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_a,
                const __grid_constant__ Params p)
{
    using C = KvCfg;
    constexpr int kM = C::kM, kStages = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffTmemSlot);
    Abort ab{reinterpret_cast<volatile int *>(smem + C::kOffAbort)};
    auto bar = [&](int i) -> uint32_t { return sbase + C::kOffBar + 8u * (uint32_t)i; };
    auto stage = [&](int st) -> uint32_t { return sbase + C::kOffCh + (uint32_t)st * C::kStageBytes; };
    const int nunits = snake_count(p.units);

    if (tid == 0) {
        *ab.flag = 0;
        mbar_init(bar(C::BKV_FULL), 1);
        mbar_init(bar(C::BKV_EMPTY), 1);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(bar(C::BCH_FULL + i), 1);
            mbar_init(bar(C::BCH_EMPTY + i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(C::BS_FULL + i), 1);
            mbar_init(bar(C::BS_FREE + i), 8);
        }
        mbar_init(bar(C::BPS_READY), 8);
        mbar_init(bar(C::BPS_FREE), 1);
        mbar_init(bar(C::BACC_FULL), 1);
        mbar_init(bar(C::BACC_FREE), 8);
        mbar_init(bar(C::B_DRAIN), 1);
        mbar_init(bar(C::B_DRAIN + 1), 1);
        fence_barrier_init();
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_a);
    }
    if (tid < 128) reinterpret_cast<float *>(smem + C::kOffW)[tid] = __bfloat162float(p.w[tid]);
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ================================================= TMA producer
        if (lane == 0) {
            int g = 0, k = 0;
            KUnit x;
            bool ok = true;
            for (; k < nunits && ok; ++k) {
                kv_unit_at(p, k, x);
                ok = mbar_wait(bar(C::BKV_EMPTY), (k & 1) ^ 1u, ab);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(C::BKV_FULL), 2 * C::kKTile);
                for (int h = 0; h < 2; ++h) {
                    tma_load_4d(sbase + C::kOffK + h * C::kKHalf, &tm_k, bar(C::BKV_FULL), h * 64, x.kvh,
                                128 * x.kt, x.b);
                    tma_load_4d(sbase + C::kOffV + h * C::kKHalf, &tm_v, bar(C::BKV_FULL), h * 64, x.kvh,
                                128 * x.kt, x.b);
                }
                for (int j = 0; j < x.n && ok; ++j, ++g) {
                    const int st = g % kStages;
                    ok = mbar_wait(bar(C::BCH_EMPTY + st), ((g / kStages) & 1) ^ 1u, ab);
                    if (!ok) break;
                    const int t0 = 128 * x.kt + C::kChTok * j;
                    mbar_arrive_expect_tx(bar(C::BCH_FULL + st), 2 * C::kCTile + C::kRecBytes);
                    for (int h = 0; h < 2; ++h) {
                        tma_load_4d(stage(st) + h * C::kCHalf, &tm_q, bar(C::BCH_FULL + st), h * 64, x.kvh * 4, t0,
                                    x.b);
                        tma_load_4d(stage(st) + C::kCTile + h * C::kCHalf, &tm_a, bar(C::BCH_FULL + st), h * 64,
                                    x.kvh * 4, t0, x.b);
                    }
                    bulk_load(stage(st) + 2 * C::kCTile, p.ld + (((long long)x.b * p.Hkv + x.kvh) * p.Tp + t0) * 4,
                              C::kRecBytes, bar(C::BCH_FULL + st));
                }
            }
            for (int i = (g > kStages ? g - kStages : 0); i < g; ++i)
                drain_wait(bar(C::BCH_FULL + i % kStages), (i / kStages) & 1);
            if (k > 0) drain_wait(bar(C::BKV_FULL), (k - 1) & 1);
        }
    } else if (warp == 1 || warp == 2) {
        // ================================================= MMA issuers: warp 1 the scores (S^T, dP^T),
        // warp 2 the accumulations (dV, dK~); each thread's commits cover its own products
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16_f32(128, kM, 0, 0);
            const uint32_t idesc_acc = idesc_bf16_f32(128, 128, 0, 1);
            // shared-memory descriptors built once (stage 0; the stages differ by a
            // constant byte offset): K~, V, P^T, dS^T and the chunk tiles K-major, the
            // chunk tiles MN-major as the B operands of dV and dK~
            const SmemDesc dC = make_desc(stage(0), 16, 1024), dCmn = make_desc(stage(0), C::kCHalf, 1024);
            KvWalk w;
            w.init(p);
            bool ok = true;
            int g = 0;
            if (warp == 1) {
                const SmemDesc dK = make_desc(sbase + C::kOffK, 16, 1024), dV = make_desc(sbase + C::kOffV, 16, 1024);
                for (; w.valid && ok; w.next(p), ++g) {
                    if (w.j == 0 && !(ok = mbar_wait(bar(C::BKV_FULL), w.k & 1, ab))) break;
                    if (!(ok = mbar_wait(bar(C::BCH_FULL + g % kStages), (g / kStages) & 1, ab))) break;
                    // the buffer's previous scores (chunk g - 2) are in the softmax warps' registers
                    if (!(ok = mbar_wait(bar(C::BS_FREE + (g & 1)), ((g >> 1) & 1) ^ 1u, ab))) break;
                    tc_fence_after();
                    const uint32_t dS = tmem + C::kColBuf + (g & 1) * C::kBufStride;
                    const uint32_t qo = (uint32_t)(g % kStages) * C::kStageBytes, ao = qo + C::kCTile;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t ok_ = (kk >> 2) * C::kKHalf + (kk & 3) * 32;
                        const uint32_t oc = (kk >> 2) * C::kCHalf + (kk & 3) * 32;
                        mma_ss(dS, dK.at(ok_), dC.at(qo + oc), idesc_s, kk > 0);
                    }
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t ok_ = (kk >> 2) * C::kKHalf + (kk & 3) * 32;
                        const uint32_t oc = (kk >> 2) * C::kCHalf + (kk & 3) * 32;
                        mma_ss(dS + kM, dV.at(ok_), dC.at(ao + oc), idesc_s, kk > 0);
                    }
                    mma_commit(bar(C::BS_FULL + (g & 1)));
                    if (w.last()) mma_commit(bar(C::BKV_EMPTY));   // K~ and V are read by the scores alone
                }
            } else {
                const SmemDesc dP = make_desc(sbase + C::kOffP, 16, 1024), dDS = make_desc(sbase + C::kOffDS, 16, 1024);
                for (; w.valid && ok; w.next(p), ++g) {
                    // P^T and dS^T of the chunk are in shared memory (the softmax warps saw
                    // its scores complete, so the scores' reads of the stage are done)
                    if (!(ok = mbar_wait(bar(C::BPS_READY), g & 1, ab))) break;
                    if (w.j == 0 && !(ok = mbar_wait(bar(C::BACC_FREE), (w.k & 1) ^ 1u, ab))) break;
                    tc_fence_after();
                    const uint32_t qo = (uint32_t)(g % kStages) * C::kStageBytes, ao = qo + C::kCTile;
                    const uint32_t acc0 = w.j > 0;
#pragma unroll
                    for (int kk = 0; kk < kM / 16; ++kk)
                        mma_ss(tmem + C::kColDV, dP.at(kk * 32), dCmn.at(ao + kk * 16 * 128), idesc_acc, acc0 | (kk > 0));
#pragma unroll
                    for (int kk = 0; kk < kM / 16; ++kk)
                        mma_ss(tmem + C::kColDK, dDS.at(kk * 32), dCmn.at(qo + kk * 16 * 128), idesc_acc, acc0 | (kk > 0));
                    mma_commit(bar(C::BCH_EMPTY + g % kStages));
                    mma_commit(bar(C::BPS_FREE));
                    if (w.last()) mma_commit(bar(C::BACC_FULL));
                }
            }
            mma_commit(bar(C::B_DRAIN + (warp - 1)));
            drain_wait(bar(C::B_DRAIN + (warp - 1)), 0);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ================================================= P^T, dS^T (8 warps) and the epilogue
        const int grp = (warp - 4) >> 2;           // column half of each chunk: rows 32 grp .. 32 grp + 31
        const int r = 32 * (warp & 3) + lane;      // key of the tile (TMEM lane)
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const float *w = reinterpret_cast<const float *>(smem + C::kOffW);
        const int W = p.window;
        float dwacc[4] = {0.f, 0.f, 0.f, 0.f};
        bool ok = true;
        int g = 0;
        KUnit x;
        for (int k = 0; k < nunits && ok; ++k) {
            kv_unit_at(p, k, x);
            const int jkey = 128 * x.kt + r;
            for (int j = 0; j < x.n && ok; ++j, ++g) {
                const int bb = g & 1, st = g % kStages;
                ok = warp_wait(bar(C::BS_FULL + bb), (g >> 1) & 1, ab);
                // the stage's records: its load completed before the MMA read the stage
                if (ok) ok = warp_wait(bar(C::BCH_FULL + st), (g / kStages) & 1, ab);
                if (!ok) break;
                tc_fence_after();
                uint32_t s[32], d[32];
                const uint32_t ts = tmem + lane_base + C::kColBuf + bb * C::kBufStride + 32 * grp;
                tmem_ld32(ts, s);
                tmem_ld32(ts + kM, d);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::BS_FREE + bb));   // the scores are in registers
                const int t0 = 128 * x.kt + C::kChTok * j;
                const int lo = jkey - t0, hi = jkey - t0 + W - 1;   // visible chunk tokens
                const uint32_t rec = stage(st) + 2 * C::kCTile + 32 * grp * 8;
                uint32_t pk[16], dk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    // records of rows 32 grp + e .. + 3 (one token, four heads)
                    const uint4 ra = lds128(rec + e * 8);
                    const uint4 rb = lds128(rec + (e + 2) * 8);
                    const float l2[4] = {__uint_as_float(ra.x), __uint_as_float(ra.z), __uint_as_float(rb.x),
                                         __uint_as_float(rb.z)};
                    const float dv[4] = {__uint_as_float(ra.y), __uint_as_float(ra.w), __uint_as_float(rb.y),
                                         __uint_as_float(rb.w)};
                    const int tok = (32 * grp + e) >> 2;
                    const bool vis = tok >= lo && tok <= hi;
                    float pp[4], ds[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        pp[q] = vis ? ex2(fmaf(__uint_as_float(s[e + q]), p.sl2, -l2[q])) : 0.f;
                        ds[q] = pp[q] * (__uint_as_float(d[e + q]) - dv[q]);
                    }
                    pk[e >> 1] = pack_bf16(pp[0], pp[1]);
                    pk[(e >> 1) + 1] = pack_bf16(pp[2], pp[3]);
                    dk[e >> 1] = pack_bf16(ds[0], ds[1]);
                    dk[(e >> 1) + 1] = pack_bf16(ds[2], ds[3]);
                }
                // the previous chunk's dV/dK have read the P^T / dS^T tiles
                ok = warp_wait(bar(C::BPS_FREE), (g & 1) ^ 1u, ab);
                if (!ok) break;
                sts_row_chunks(sbase + C::kOffP, r, 4 * grp, pk);
                sts_row_chunks(sbase + C::kOffDS, r, 4 * grp, dk);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::BPS_READY));
            }
            if (!ok) break;
            // ---- epilogue of the unit: dv (warps 4-7), dk and dw_k (warps 8-11)
            ok = warp_wait(bar(C::BACC_FULL), k & 1, ab);
            if (!ok) break;
            tc_fence_after();
            const bool valid = jkey < p.T;
            const long long off = valid ? (((long long)x.b * p.T + jkey) * p.Hkv + x.kvh) * kD : 0;
            if (grp == 0) {
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t v[32];
                    tmem_ld32(tmem + lane_base + C::kColDV + 32 * c, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 o = make_uint4(
                            pack_bf16(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1])),
                            pack_bf16(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                            pack_bf16(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                            pack_bf16(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
                        if (valid) reinterpret_cast<uint4 *>(p.dv + off)[4 * c + q] = o;
                    }
                }
            } else {
                norm_rope_backward<R>(tmem + lane_base + C::kColDK, p.scale, p.x + off, valid, w, p.eps, jkey,
                                      p.theta, p.dx + off, dwacc);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::BACC_FREE));
        }
        if (grp == 1) {
            float *dst = p.dw_part + ((long long)blockIdx.x * 4 + (warp & 3)) * kD;
#pragma unroll
            for (int c = 0; c < 4; ++c) dst[32 * c + lane] = dwacc[c];
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace bwd
}  // namespace gswa
