// swa_fwd.cuh -- gated sliding-window attention forward for sm_100a.
//
// Computes, for one ZGCM-1 gated-SWA layer (ZGCM-1 §2.1 Model overview and
// Figure 3 caption: 128-token sliding window, GQA 32 q / 8 kv heads of dim
// 128, QK RMSNorm, partial RoPE; GatedSWA(h) = o_proj(A_SWA(q,k,v) ⊙ σ(g)))
//   y_i = softmax_{i-W < j <= i}(scale <q~_i, k~_j>) V  ⊙  σ(g_i)
// with q~, k~ the RMS-normed, partially rotated queries and keys, and the
// natural-log normaliser lse_i of each row.  The keys arrive prepared (k~,
// written once by qk_prep: each key block serves five query blocks, and one
// key warp per CTA preparing them in-line overloaded its scheduler); the
// queries are prepared here, in shared memory, as their tiles land.
//
// Work unit: a 32-token query block of one (sequence, KV head) pair, i.e. the
// 4 query heads of a GQA group packed as M = 128 tensor-core rows
// (row r = 4 * token + head-in-group).  Its keys are the 160 keys
// [i0 - 128, i0 + 32): five 32-key blocks, so one QK^T MMA of N = 160 covers
// every key any of its rows can see and the softmax needs a single pass (no
// running rescale).  Persistent CTAs walk consecutive blocks of a strip, so
// each K/V block is fetched from HBM once and kept in a six-slot shared-memory
// ring while the window slides over it.
//
// Warp roles (16 warps):
//   warp 0      TMA producer of k~ blocks (ring)
//   warp 1      TMEM owner and tcgen05.mma issuer; it polls S-, PV- and
//               Q-slot readiness independently (so none waits behind another)
//               and also issues the TMA loads of the Q tiles (2 stages)
//   warp 2      idle
//   warp 3      TMA producer of V blocks (ring)
// K and V slots have their own barriers: a K slot is handed back as soon as
// the last QK^T that reads it completes, a V slot after the last PV, so the
// next K block's load never waits behind a softmax.
//   warps 4-7   query prologue: RMSNorm + RoPE of the 128 Q rows, in place
//   warps 8-11  softmax: S (TMEM) -> P (bf16, TMEM), 1/l (TMEM), lse
//   warps 12-15 epilogue: σ(g) (f32, stored as f16) into the gate tile ahead of time, then
//               O (TMEM) * 1/l * σ -> y in the gate tile, TMA store; its thread 0
//               also loads the gate tiles (2 stages), reusing each slot as soon
//               as the y store has read it
//
// TMEM (512 columns) holds two buffers of 256 columns: S at +0 (160 f32
// columns), P at +0 (80 columns of bf16 pairs, written over S once read),
// 1/l at +80, and O at +128 (128 f32 columns, written only after P is done).
#pragma once

#include <cuda.h>

#include <type_traits>

#include "ptx.cuh"

namespace gswa {
namespace swa {

constexpr int kD = 128;
constexpr int kTok = 32;                  // query tokens per unit
constexpr int kRows = 128;                // MMA M
constexpr int kSpanBlocks = 5;            // 160-key window span in 32-key blocks
constexpr int kRing = 6;                  // K/V ring slots
constexpr int kSpan = kSpanBlocks * kTok; // 160
constexpr int kThreads = 512;
constexpr int kColInvL = 80;              // TMEM column of 1/l inside a buffer

// Shared-memory map (offsets from a 1024-byte-aligned base).
constexpr uint32_t kHalfRowBytes = 128;                       // 64 bf16 per swizzled row
constexpr uint32_t kBlockHalfBytes = kTok * kHalfRowBytes;    // 4096: 32 rows x 64 dims
constexpr uint32_t kRingHalfBytes = kRing * kBlockHalfBytes;  // 24576
constexpr uint32_t kTileHalfBytes = kRows * kHalfRowBytes;    // 16384: 128 rows x 64 dims
constexpr uint32_t kTileBytes = 2 * kTileHalfBytes;           // 32768
constexpr uint32_t kOffK = 0;
constexpr uint32_t kOffV = kOffK + 2 * kRingHalfBytes;        // 49152
constexpr uint32_t kOffQ = kOffV + 2 * kRingHalfBytes;        // 98304
constexpr uint32_t kOffG = kOffQ + 2 * kTileBytes;            // 163840
constexpr uint32_t kOffWq = kOffG + 2 * kTileBytes;           // 229376 (f32[128])
constexpr uint32_t kOffBar = kOffWq + 512;
constexpr int kNumBars = 45;
constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
constexpr uint32_t kSmemUsed = kOffAbort + 4;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;             // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget of one sm_100 CTA");

// Barrier indices.
enum : int {
    BQ_FULL = 0, BQ_PREP = 2, BQ_EMPTY = 4, BG_FULL = 6, BG_EMPTY = 8,
    BK_FULL = 10, BK_EMPTY = 16, BS_FULL = 22, BP_READY = 24, BO_FULL = 26,
    BT_EMPTY = 28, BY_READY = 30, B_DRAIN = 32, BV_FULL = 33, BV_EMPTY = 39
};

struct Params {
    int B, T, Hq, Hkv, window;
    int nsteps;        // ceil(T / 32)
    long long units;   // B * Hkv * nsteps
    float eps;
    float sl2;         // softmax scale * log2(e)
    const __nv_bfloat16 *wq, *wk;
    float *lse;        // [B, Hq, T] or null
    double theta[64];  // rope_base^(-2p/R), p < R/2
};

// Walks the units [u0, u1) of a CTA in order: (sequence b, kv head, step s).
struct Walker {
    int b, kvh, s;
    __device__ __forceinline__ void init(const Params &p, long long u0)
    {
        const long long strip = u0 / p.nsteps;
        s = (int)(u0 - strip * p.nsteps);
        b = (int)(strip / p.Hkv);
        kvh = (int)(strip - (long long)b * p.Hkv);
    }
    __device__ __forceinline__ void next(const Params &p)
    {
        if (++s == p.nsteps) {
            s = 0;
            if (++kvh == p.Hkv) {
                kvh = 0;
                ++b;
            }
        }
    }
    __device__ __forceinline__ bool first(int idx) const { return idx == 0 || s == 0; }
    __device__ __forceinline__ bool last(const Params &p, int idx, int n) const
    {
        return idx == n - 1 || s == p.nsteps - 1;
    }
};

__device__ __forceinline__ int ring_slot(int kb) { return ((kb % kRing) + kRing) % kRing; }

// Byte offset of 16-byte chunk c (0..15) of row r in a two-half swizzled tile
// whose halves are `half_stride` apart (TMA 128-byte swizzle pattern).
__device__ __forceinline__ uint32_t chunk_off(int r, int c, uint32_t half_stride)
{
    return (uint32_t)(c >> 3) * half_stride + (uint32_t)r * kHalfRowBytes +
           ((uint32_t)((c & 7) ^ (r & 7)) << 4);
}

// cos/sin of the rotary angle pos * theta, reduced modulo 2π in double
// precision first so that positions up to 2^18 keep full accuracy.
__device__ __forceinline__ void rope_cs(double theta, int pos, float &c, float &s)
{
    const double two_pi = 6.283185307179586;
    const double phi = (double)pos * theta;
    const double k = rint(phi * (1.0 / two_pi));
    const float r = (float)fma(-k, two_pi, phi);
    // |r| <= pi here, where the hardware sine/cosine are accurate to ~2^-21.
    __sincosf(r, &s, &c);
}

// cos/sin of the rotary angles of one thread's token, by angle addition:
// the angle (i0 + t) theta_p of token t of a 32-token block starting at i0 is
// split into a block part i0 theta_p, evaluated once per block (lane p of the
// warp evaluates pair p and the warp shares it by shuffle), and a row part
// t theta_p, evaluated once per kernel (t is fixed per thread).  Then
// cos = cA cB - sA sB and sin = sA cB + cA sB cost four FMAs per pair.
// kStride/kOffset select the pairs this thread owns (p = kOffset + k kStride).
template <int H, int kStride>
struct RopeTab {
    static constexpr int kN = (H + kStride - 1) / kStride;
    float cb[kN > 0 ? kN : 1], sb[kN > 0 ? kN : 1];  // row part of the owned pairs
    float ca, sa, ca2, sa2;                           // block part of pairs lane, lane + 32
    __device__ __forceinline__ void init_rows(int t, int offset, const double *theta)
    {
#pragma unroll
        for (int k = 0; k < kN; ++k) {
            const int pp = offset + k * kStride;
            cb[k] = 1.f;
            sb[k] = 0.f;
            if (pp < H) rope_cs(theta[pp], t, cb[k], sb[k]);
        }
    }
    __device__ __forceinline__ void set_block(int i0, const double *theta)
    {
        const int lane = threadIdx.x & 31;
        ca = ca2 = 1.f;
        sa = sa2 = 0.f;
        if (lane < H) rope_cs(theta[lane], i0, ca, sa);
        if (H > 32 && lane + 32 < H) rope_cs(theta[lane + 32], i0, ca2, sa2);
    }
    // cos/sin of owned pair k (pair index pp, a warp-uniform function of k
    // only when kStride == 1; otherwise each lane passes its own pp)
    __device__ __forceinline__ void get(int k, int pp, float &c, float &sn) const
    {
        const float a_c = __shfl_sync(0xffffffffu, (pp < 32) ? ca : ca2, pp & 31);
        const float a_s = __shfl_sync(0xffffffffu, (pp < 32) ? sa : sa2, pp & 31);
        c = a_c * cb[k] - a_s * sb[k];
        sn = a_s * cb[k] + a_c * sb[k];
    }
};

// Same interface as RopeTab for wide rotations (one lane per key row): each
// cos/sin is evaluated directly, keeping no per-pair registers.
template <int H>
struct RopeDirect {
    int pos0 = 0, t = 0;
    const double *theta = nullptr;
    __device__ __forceinline__ void init_rows(int row, int, const double *th)
    {
        t = row;
        theta = th;
    }
    __device__ __forceinline__ void set_block(int i0, const double *) { pos0 = i0; }
    __device__ __forceinline__ void get(int, int pp, float &c, float &sn) const
    {
        rope_cs(theta[pp], pos0 + t, c, sn);
    }
};

// RMSNorm then partial RoPE of one head row held in shared memory (bf16,
// swizzled), in place, one thread per row.
//   r = (mean_d x_d^2 + eps)^-1/2;  u_d = x_d r w_d;
//   (u_p, u_{p+R/2}) <- (u_p c - u_{p+R/2} s, u_{p+R/2} c + u_p s),  p < R/2
// computed in f32 and rounded to bf16 once.  The row streams through
// registers 16 bytes at a time; only the chunks taking part in the rotation
// are held together.  `tile` is the shared-memory address of the tile, `hs`
// the byte distance between its two 64-dim halves, `w` the f32 weights
// (16-byte aligned).  kQuad: the 4 lanes of a quad hold 4 heads of one token;
// lane q evaluates the cos/sin of pairs p = q mod 4 and the quad swaps them.
template <int R, bool kQuad, class Tab>
__device__ __forceinline__ void prep_row(uint32_t tile, uint32_t hs, int row, const float *w, float eps,
                                         const Tab &tab)
{
    constexpr int H = R / 2;
    constexpr bool kAligned = (H % 8) == 0;
    constexpr int kRot = (R + 7) / 8;      // leading chunks holding a rotated dim
    constexpr int kPair = kAligned ? H / 8 : 0;  // aligned: chunk c pairs with chunk c + kPair
    const float4 *w4 = reinterpret_cast<const float4 *>(w);
    const int lane = threadIdx.x & 31;
    // pass 1: mean square of the raw row (eight independent accumulators,
    // updated in pairs by f32x2 FMAs)
    uint64_t ss2[4] = {0, 0, 0, 0};
#pragma unroll 4
    for (int c = 0; c < 16; ++c) {
        const uint4 v = lds128(tile + chunk_off(row, c, hs));
        const uint32_t u4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = unpack_bf16(u4[e]);
            const uint64_t x2 = f2_pack(f.x, f.y);
            ss2[e] = f2_fma(x2, x2, ss2[e]);
        }
    }
    float ss[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 t = f2_unpack(ss2[e]);
        ss[2 * e] = t.x;
        ss[2 * e + 1] = t.y;
    }
    const float r = rsqrtf(((ss[0] + ss[1]) + (ss[2] + ss[3]) + ((ss[4] + ss[5]) + (ss[6] + ss[7]))) *
                               (1.0f / kD) + eps);
    const uint64_t r2 = f2_pack(r, r);
    // scaled values x (r w) of one chunk, two dims per instruction
    auto scale8 = [&](const uint4 v, int c, float (&u)[8]) {
        const float4 wa = w4[2 * c], wb = w4[2 * c + 1];
        const uint64_t w2[4] = {f2_pack(wa.x, wa.y), f2_pack(wa.z, wa.w), f2_pack(wb.x, wb.y), f2_pack(wb.z, wb.w)};
        const uint32_t u4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = unpack_bf16(u4[e]);
            const float2 y = f2_unpack(f2_mul(f2_pack(f.x, f.y), f2_mul(r2, w2[e])));
            u[2 * e] = y.x;
            u[2 * e + 1] = y.y;
        }
    };
    auto pack8 = [](const float *u) {
        return make_uint4(pack_bf16(u[0], u[1]), pack_bf16(u[2], u[3]), pack_bf16(u[4], u[5]),
                          pack_bf16(u[6], u[7]));
    };
    // cos/sin of pair p0 + j: from the table (this lane owns p0 + j) or, in quad
    // mode, from the lane of the quad that owns it
    auto cs_round = [&](int p0, float &cm, float &sm) {  // quad mode: own pair p0 + (lane & 3)
        cm = 1.f;
        sm = 0.f;
        const int pp = p0 + (lane & 3);
        tab.get(p0 >> 2, pp < H ? pp : 0, cm, sm);
    };
    auto cs_get = [&](int p0, int j, float cm, float sm, float &cc, float &sn) {
        if constexpr (kQuad) {
            cc = __shfl_sync(0xffffffffu, cm, (lane & ~3) | j);
            sn = __shfl_sync(0xffffffffu, sm, (lane & ~3) | j);
        } else {
            tab.get(p0 + j, p0 + j, cc, sn);
        }
    };
    // pass 2: chunks without a rotated dim, the next chunk's load ahead of this store
    constexpr int kPlain0 = kRot;
    if constexpr (kPlain0 < 16) {
        uint4 cur = lds128(tile + chunk_off(row, kPlain0, hs));
#pragma unroll 2
        for (int c = kPlain0; c < 16; ++c) {
            uint4 nxt = cur;
            if (c + 1 < 16) nxt = lds128(tile + chunk_off(row, c + 1, hs));
            float u[8];
            scale8(cur, c, u);
            sts128(tile + chunk_off(row, c, hs), pack8(u));
            cur = nxt;
        }
    }
    if constexpr (R > 0 && kAligned) {
        // pairs (p, p + H), H a multiple of 8: chunk c pairs with chunk c + H/8
#pragma unroll
        for (int c = 0; c < kPair; ++c) {
            const uint32_t a1 = tile + chunk_off(row, c, hs);
            const uint32_t a2 = tile + chunk_off(row, c + kPair, hs);
            float u1[8], u2[8];
            scale8(lds128(a1), c, u1);
            scale8(lds128(a2), c + kPair, u2);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int p0 = 8 * c + 4 * half;
                float cm = 1.f, sm = 0.f;
                if constexpr (kQuad) cs_round(p0, cm, sm);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float cc, sn;
                    cs_get(p0, j, cm, sm, cc, sn);
                    const int e = 4 * half + j;
                    const float x1 = u1[e], x2 = u2[e];
                    u1[e] = x1 * cc - x2 * sn;
                    u2[e] = x2 * cc + x1 * sn;
                }
            }
            sts128(a1, pack8(u1));
            sts128(a2, pack8(u2));
        }
    } else if constexpr (R > 0) {
        // general H: hold the kRot leading chunks (<= 48 dims) as floats
        static_assert(R <= 48, "unaligned rotary widths are held in registers");
        float u[8 * kRot];
#pragma unroll
        for (int c = 0; c < kRot; ++c) {
            float t8[8];
            scale8(lds128(tile + chunk_off(row, c, hs)), c, t8);
#pragma unroll
            for (int e = 0; e < 8; ++e) u[8 * c + e] = t8[e];
        }
#pragma unroll
        for (int p0 = 0; p0 < H; p0 += 4) {
            float cm = 1.f, sm = 0.f;
            if constexpr (kQuad) cs_round(p0, cm, sm);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (p0 + j < H) {
                    float cc, sn;
                    cs_get(p0, j, cm, sm, cc, sn);
                    const float x1 = u[p0 + j], x2 = u[p0 + j + H];
                    u[p0 + j] = x1 * cc - x2 * sn;
                    u[p0 + j + H] = x2 * cc + x1 * sn;
                }
            }
        }
#pragma unroll
        for (int c = 0; c < kRot; ++c) sts128(tile + chunk_off(row, c, hs), pack8(&u[8 * c]));
    }
}

// Row max over the visible columns [lo, hi] of one 32-column chunk m of S
// (four independent accumulators).
__device__ __forceinline__ void chunk_max(const uint32_t (&v)[32], int m, int lo, int hi, float (&mx)[4])
{
    const int kl = lo - 32 * m, kh = hi - 32 * m;  // visible e: kl <= e <= kh
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const float x = (e >= kl && e <= kh) ? __uint_as_float(v[e]) : -INFINITY;
        mx[e & 3] = fmaxf(mx[e & 3], x);
    }
}

// P = 2^(S sl2 - mxs) over one 32-column chunk m (0 outside [lo, hi]), packed
// as bf16 pairs; accumulates the row sum in f32.  (One masked form for every
// chunk: a second, unmasked copy for the interior chunks saves arithmetic but
// costs more in instruction fetch than it saves.)
__device__ __forceinline__ void chunk_exp(const uint32_t (&v)[32], int m, int lo, int hi, float sl2, float mxs,
                                          uint64_t (&sum2)[4], uint32_t (&pk)[16])
{
    const int kl = lo - 32 * m, kh = hi - 32 * m;
    const uint64_t sl2_2 = f2_pack(sl2, sl2), nm2 = f2_pack(-mxs, -mxs);
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        const float2 x = f2_unpack(f2_fma(f2_pack(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), sl2_2, nm2));
        float p0 = ex2(x.x);
        float p1 = ex2(x.y);
        p0 = (e >= kl && e <= kh) ? p0 : 0.f;
        p1 = (e + 1 >= kl && e + 1 <= kh) ? p1 : 0.f;
        sum2[(e >> 1) & 3] = f2_add(sum2[(e >> 1) & 3], f2_pack(p0, p1));
        pk[e >> 1] = pack_bf16(p0, p1);
    }
}

// Bounded wait used only while tearing down: ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity)
{
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer() - t0 > 200000000ull) break;
}

template <int R>
__global__ void __launch_bounds__(kThreads, 1)
swa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
               const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffTmemSlot);
    Abort ab{reinterpret_cast<volatile int *>(smem + kOffAbort)};
    auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * (uint32_t)i; };

    const long long u0 = (long long)blockIdx.x * p.units / gridDim.x;
    const long long u1 = (long long)(blockIdx.x + 1) * p.units / gridDim.x;
    const int n = (int)(u1 - u0);

    // ---- set-up
    if (tid == 0) {
        *ab.flag = 0;
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(BQ_FULL + i), 1);
            mbar_init(bar(BQ_PREP + i), 4);   // query-prologue warps
            mbar_init(bar(BQ_EMPTY + i), 1);
            mbar_init(bar(BG_FULL + i), 1);
            mbar_init(bar(BG_EMPTY + i), 1);
            mbar_init(bar(BS_FULL + i), 1);
            mbar_init(bar(BP_READY + i), 4);  // softmax warps
            mbar_init(bar(BO_FULL + i), 1);
            mbar_init(bar(BT_EMPTY + i), 4);  // epilogue warps
            mbar_init(bar(BY_READY + i), 4);  // epilogue warps
        }
        for (int i = 0; i < kRing; ++i) {
            mbar_init(bar(BK_FULL + i), 1);
            mbar_init(bar(BK_EMPTY + i), 1);
            mbar_init(bar(BV_FULL + i), 1);
            mbar_init(bar(BV_EMPTY + i), 1);
        }
        mbar_init(bar(B_DRAIN), 1);
        fence_barrier_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_g);
        tma_prefetch_desc(&tm_y);
    }
    if (tid < 128) {
        reinterpret_cast<float *>(smem + kOffWq)[tid] = __bfloat162float(p.wq[tid]);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 || warp == 3) {
        // ================================================= TMA producers: K ring (warp 0), V ring (warp 3)
        if (lane == 0) {
            const bool is_k = warp == 0;
            const CUtensorMap *tm = is_k ? &tm_k : &tm_v;
            const uint32_t ring = sbase + (is_k ? kOffK : kOffV);
            const int b_full = is_k ? BK_FULL : BV_FULL, b_empty = is_k ? BK_EMPTY : BV_EMPTY;
            uint32_t fills = 0;     // parity of fills per ring slot
            uint32_t armed = 0;     // ring slots loaded at least once
            Walker w;
            w.init(p, u0);
            auto load = [&](int kb) -> bool {
                const int slot = ring_slot(kb);
                if (!mbar_wait(bar(b_empty + slot), ((fills >> slot) & 1u) ^ 1u, ab)) return false;
                fills ^= 1u << slot;
                armed |= 1u << slot;
                mbar_arrive_expect_tx(bar(b_full + slot), 2 * kBlockHalfBytes);
                for (int h = 0; h < 2; ++h)
                    tma_load_4d(ring + h * kRingHalfBytes + slot * kBlockHalfBytes, tm, bar(b_full + slot), h * 64,
                                w.kvh, kb * kTok, w.b);
                return true;
            };
            bool ok = true;
            for (int idx = 0; idx < n && ok; ++idx, w.next(p)) {
                if (w.first(idx))
                    for (int kb = w.s - 4; kb < w.s && ok; ++kb) ok = load(kb);
                if (ok) ok = load(w.s);
            }
            // Teardown: every load this thread issued must have landed before
            // the CTA's shared memory is released.
            for (int slot = 0; slot < kRing; ++slot)
                if (armed & (1u << slot)) drain_wait(bar(b_full + slot), ((fills >> slot) & 1u) ^ 1u);
        }
    } else if (warp == 1) {
        // ================================================= MMA issuer
        if (lane == 0) {
            const uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
            // shared-memory descriptors built once: Q tiles and the K ring K-major, the V
            // ring MN-major (32-key blocks, halves kRingHalfBytes apart)
            const SmemDesc dQt = make_desc(sbase + kOffQ, 16, 1024), dKr = make_desc(sbase + kOffK, 16, 1024);
            const SmemDesc dVr = make_desc(sbase + kOffV, kRingHalfBytes, 1024);
            Walker ws, wp, wq;
            ws.init(p, u0);
            wp.init(p, u0);
            wq.init(p, u0);
            int ns = 0, npv = 0, nq = 0;
            // K and V loads are confirmed in their producers' order: block kkb
            // (vkb) is the next one of unit ns's (npv's) window not yet seen
            // landed; a ring slot's fill parity flips with every load into it
            uint32_t k_fills = 0, v_fills = 0;
            int kkb = ws.s - 4, vkb = wp.s - 4;
            PollWatch watch;
            while (npv < n) {
                bool progressed = false;
                // Q tile of unit nq into slot nq & 1 once S(nq - 2) has consumed it
                if (nq < n && mbar_test(bar(BQ_EMPTY + (nq & 1)), ((nq >> 1) & 1) ^ 1u)) {
                    const int j = nq & 1;
                    mbar_arrive_expect_tx(bar(BQ_FULL + j), kTileBytes);
                    for (int h = 0; h < 2; ++h)
                        tma_load_4d(sbase + kOffQ + j * kTileBytes + h * kTileHalfBytes, &tm_q, bar(BQ_FULL + j),
                                    h * 64, wq.kvh * 4, wq.s * kTok, wq.b);
                    wq.next(p);
                    ++nq;
                    progressed = true;
                }
                // S(ns) = Q~ K~^T over the 160-key window, at most one unit ahead of PV
                if (ns < n && ns <= npv + 1) {
                    const int bb = ns & 1;
                    const uint32_t ph = (ns >> 1) & 1;
                    while (kkb <= ws.s) {
                        const int ks = ring_slot(kkb);
                        if (!mbar_test(bar(BK_FULL + ks), (k_fills >> ks) & 1u)) break;
                        k_fills ^= 1u << ks;
                        ++kkb;
                        progressed = true;
                    }
                    if (kkb > ws.s && mbar_test(bar(BT_EMPTY + bb), ph ^ 1u) && mbar_test(bar(BQ_PREP + bb), ph)) {
                        tc_fence_after();
                        const int a = ring_slot(ws.s - 4);
                        const int n1 = (kRing - a) < kSpanBlocks ? (kRing - a) : kSpanBlocks;
                        const int n2 = kSpanBlocks - n1;
                        const uint32_t id1 = idesc_bf16_f32(128, n1 * kTok, 0, 0);
                        const uint32_t id2 = idesc_bf16_f32(128, n2 > 0 ? n2 * kTok : 32, 0, 0);
                        const uint32_t dS = tmem + bb * 256;
                        const uint32_t qo = (uint32_t)bb * kTileBytes, ao = (uint32_t)a * kBlockHalfBytes;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t h = kk >> 2, ko = (kk & 3) * 32;
                            const uint64_t ad = dQt.at(qo + h * kTileHalfBytes + ko);
                            mma_ss(dS, ad, dKr.at(h * kRingHalfBytes + ko + ao), id1, kk > 0);
                            if (n2 > 0) mma_ss(dS + n1 * kTok, ad, dKr.at(h * kRingHalfBytes + ko), id2, kk > 0);
                        }
                        mma_commit(bar(BS_FULL + bb));
                        mma_commit(bar(BQ_EMPTY + bb));
                        // K slots that no later unit of this CTA reads
                        if (ws.last(p, ns, n)) {
                            for (int i = 0; i < kSpanBlocks; ++i) mma_commit(bar(BK_EMPTY + (a + i) % kRing));
                        } else {
                            mma_commit(bar(BK_EMPTY + a));
                        }
                        ws.next(p);
                        ++ns;
                        kkb = ws.first(ns) ? ws.s - 4 : ws.s;
                        progressed = true;
                    }
                }
                // O(npv) = P V over the same window
                if (npv < ns) {
                    const int bb = npv & 1;
                    const uint32_t ph = (npv >> 1) & 1;
                    while (vkb <= wp.s) {
                        const int vs = ring_slot(vkb);
                        if (!mbar_test(bar(BV_FULL + vs), (v_fills >> vs) & 1u)) break;
                        v_fills ^= 1u << vs;
                        ++vkb;
                        progressed = true;
                    }
                    if (vkb > wp.s && mbar_test(bar(BP_READY + bb), ph)) {
                        tc_fence_after();
                        const int a = ring_slot(wp.s - 4);
                        const uint32_t dO = tmem + bb * 256 + 128;
#pragma unroll
                        for (int kk = 0; kk < kSpan / 16; ++kk) {
                            const int sl = a + (kk >> 1);
                            const int slot = sl >= kRing ? sl - kRing : sl;   // a + i < 2 kRing
                            mma_ts(dO, tmem + bb * 256 + kk * 8,
                                   dVr.at((uint32_t)slot * kBlockHalfBytes + (kk & 1) * 16 * kHalfRowBytes), idesc_pv,
                                   kk > 0);
                        }
                        mma_commit(bar(BO_FULL + bb));
                        // V slots that no later unit of this CTA reads
                        if (wp.last(p, npv, n)) {
                            for (int i = 0; i < kSpanBlocks; ++i) mma_commit(bar(BV_EMPTY + (a + i) % kRing));
                        } else {
                            mma_commit(bar(BV_EMPTY + a));
                        }
                        wp.next(p);
                        ++npv;
                        vkb = wp.first(npv) ? wp.s - 4 : wp.s;
                        progressed = true;
                    }
                }
                if (!watch.tick(progressed, ab)) break;
            }
            // all MMAs issued by this thread complete before TMEM is freed, and
            // every Q load it issued has landed before shared memory is released
            mma_commit(bar(B_DRAIN));
            drain_wait(bar(B_DRAIN), 0);
            for (int i = (nq > 2 ? nq - 2 : 0); i < nq; ++i) drain_wait(bar(BQ_FULL + (i & 1)), (i >> 1) & 1);
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 8) {
        // ================================================= query prologue
        const int r = tid - 128;
        const float *wq = reinterpret_cast<const float *>(smem + kOffWq);
        RopeTab<R / 2, 4> tab;   // this lane's pairs p = lane & 3 (mod 4) of token r / 4
        tab.init_rows(r >> 2, lane & 3, p.theta);
        Walker w;
        w.init(p, u0);
        bool ok = true;
        for (int idx = 0; idx < n && ok; ++idx, w.next(p)) {
            const int j = idx & 1;
            tab.set_block(w.s * kTok, p.theta);
            ok = warp_wait(bar(BQ_FULL + j), (idx >> 1) & 1, ab);
            if (ok)
                prep_row<R, true>(sbase + kOffQ + j * kTileBytes, kTileHalfBytes, r, wq, p.eps, tab);
            fence_proxy_async_smem();
            __syncwarp();
            if (ok && lane == 0) mbar_arrive(bar(BQ_PREP + j));
        }
    } else if (warp >= 8 && warp < 12) {
        // ================================================= softmax
        const int r = tid - 256;
        const int t = r >> 2;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const float ln2 = 0.6931471805599453f;
        // Softmax reference: the QK norm bounds every raw score by
        // D max|w_q| max|w_k|, and softmax is shift-invariant, so while that
        // bound (times scale log2 e, 2 % headroom) is at most 60 it serves as
        // the reference and the max pass is skipped (no P of a visible key
        // falls below 2^-120); otherwise the exact row max is used.
        float wmax_q = 0.f, wmax_k = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            wmax_q = fmaxf(wmax_q, fabsf(__bfloat162float(p.wq[4 * lane + e])));
            wmax_k = fmaxf(wmax_k, fabsf(__bfloat162float(p.wk[4 * lane + e])));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            wmax_q = fmaxf(wmax_q, __shfl_xor_sync(0xffffffffu, wmax_q, o));
            wmax_k = fmaxf(wmax_k, __shfl_xor_sync(0xffffffffu, wmax_k, o));
        }
        const float ref_fixed = 1.02f * 128.0f * wmax_q * wmax_k * fabsf(p.sl2);
        const bool fixed = ref_fixed <= 60.0f;
        Walker w;
        w.init(p, u0);
        bool ok = true;
        for (int idx = 0; idx < n && ok; ++idx, w.next(p)) {
            const int bb = idx & 1;
            ok = warp_wait(bar(BS_FULL + bb), (idx >> 1) & 1, ab);
            if (!ok) break;
            tc_fence_after();
            // visible window columns c (key j = 32 s - 128 + c): i - W < j <= i, j >= 0
            const int lo = max(t + 129 - p.window, 128 - kTok * w.s);
            const int hi = t + 128;
            const uint32_t ts = tmem + lane_base + bb * 256;
            float mxs = ref_fixed;   // reference in log2 units
            if (!fixed) {
                // pass 1: row max over the visible columns (the next chunk's TMEM
                // load is in flight while the current one is reduced)
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                {
                    uint32_t va[32], vb[32];
                    tmem_ld32(ts, va);
#pragma unroll 1
                    for (int m = 0; m < kSpanBlocks - 1; m += 2) {
                        tmem_wait_ld();
                        tmem_ld32(ts + (m + 1) * 32, vb);
                        chunk_max(va, m, lo, hi, mx4);
                        tmem_wait_ld();
                        tmem_ld32(ts + (m + 2) * 32, va);
                        chunk_max(vb, m + 1, lo, hi, mx4);
                    }
                    tmem_wait_ld();
                    chunk_max(va, kSpanBlocks - 1, lo, hi, mx4);
                }
                mxs = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * p.sl2;
            }
            // pass 2: P = 2^(S sl2 - max sl2) in bf16 over S's first 80 columns
            // (P of chunk m lands on S columns of chunk m/2, already consumed)
            uint64_t sum2[4] = {0, 0, 0, 0};   // eight partial sums, in pairs
            {
                uint32_t va[32], pk[16];
#pragma unroll 1
                for (int m = 0; m < kSpanBlocks; ++m) {
                    tmem_ld32(ts + m * 32, va);
                    tmem_wait_ld();
                    chunk_exp(va, m, lo, hi, p.sl2, mxs, sum2, pk);
                    tmem_st16(ts + m * 16, pk);
                }
            }
            const float2 s01 = f2_unpack(f2_add(sum2[0], sum2[1])), s23 = f2_unpack(f2_add(sum2[2], sum2[3]));
            const float sum = (s01.x + s01.y) + (s23.x + s23.y);
            tmem_st1(ts + kColInvL, __float_as_uint(1.0f / sum));
            tmem_wait_st();
            const int i = w.s * kTok + t;
            if (p.lse != nullptr && i < p.T)
                p.lse[((long long)w.b * p.Hq + w.kvh * 4 + (r & 3)) * p.T + i] = (mxs + __log2f(sum)) * ln2;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BP_READY + bb));
        }
    } else if (warp >= 12) {
        // ================================================= epilogue
        // Phase A (off the critical path): as soon as a gate tile lands, σ(g)
        // replaces g in place, as f16.  Phase B (once O is ready): y = O (1/l) σ
        // replaces σ in place as bf16; TMEM is released as soon as the last O
        // chunk is in registers; thread 0 stores y by TMA and reloads the slot.
        const int r = tid - 384;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        Walker w;
        w.init(p, u0);
        Walker wg;   // unit of the next gate tile to load (thread 0)
        wg.init(p, u0);
        int g_issued = 0;
        auto load_gate = [&]() {
            const int j = g_issued & 1;
            mbar_arrive_expect_tx(bar(BG_FULL + j), kTileBytes);
            for (int h = 0; h < 2; ++h)
                tma_load_4d(sbase + kOffG + j * kTileBytes + h * kTileHalfBytes, &tm_g, bar(BG_FULL + j),
                            h * 64, wg.kvh * 4, wg.s * kTok, wg.b);
            wg.next(p);
            ++g_issued;
        };
        if (r == 0)
            while (g_issued < n && g_issued < 2) load_gate();
        // σ(g) = (1 + tanh(g/2)) / 2 (f32, kept as f16) over this thread's row of gate tile `idx`
        auto sigma_row = [&](int idx) -> bool {
            if (!warp_wait(bar(BG_FULL + (idx & 1)), (idx >> 1) & 1, ab)) return false;
            const uint32_t ga = sbase + kOffG + (idx & 1) * kTileBytes;
            uint4 cur = lds128(ga + chunk_off(r, 0, kTileHalfBytes));
#pragma unroll 2
            for (int c = 0; c < 16; ++c) {
                uint4 nxt = cur;
                if (c + 1 < 16) nxt = lds128(ga + chunk_off(r, c + 1, kTileHalfBytes));
                sts128(ga + chunk_off(r, c, kTileHalfBytes),
                       make_uint4(sigmoid_bf16x2_f16x2(cur.x), sigmoid_bf16x2_f16x2(cur.y),
                                  sigmoid_bf16x2_f16x2(cur.z), sigmoid_bf16x2_f16x2(cur.w)));
                cur = nxt;
            }
            return true;
        };
        bool ok = n > 0 ? sigma_row(0) : true;
        for (int idx = 0; idx < n && ok; ++idx, w.next(p)) {
            const int bb = idx & 1;
            const uint32_t ph = (idx >> 1) & 1;
            // p_ready also orders the softmax's 1/l store before this warp's TMEM read
            ok = warp_wait(bar(BP_READY + bb), ph, ab) && warp_wait(bar(BO_FULL + bb), ph, ab);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tb = tmem + lane_base + bb * 256;
            const uint32_t gaddr = sbase + kOffG + bb * kTileBytes;
            const float inv = __uint_as_float(tmem_ld1(tb + kColInvL));
            const uint64_t inv2 = f2_pack(inv, inv);
            auto load_s = [&](int m, uint4 (&sv)[4]) {
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) sv[c4] = lds128(gaddr + chunk_off(r, m * 4 + c4, kTileHalfBytes));
            };
            // y = O * (1/l) * σ over one 32-column chunk m
            auto out_chunk = [&](const uint32_t (&o)[32], const uint4 (&sv)[4], int m) {
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const uint32_t su[4] = {sv[c4].x, sv[c4].y, sv[c4].z, sv[c4].w};
                    uint32_t yu[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 sg = unpack_f16(su[e]);
                        const uint64_t o2 = f2_pack(__uint_as_float(o[c4 * 8 + 2 * e]), __uint_as_float(o[c4 * 8 + 2 * e + 1]));
                        const float2 y = f2_unpack(f2_mul(f2_mul(o2, inv2), f2_pack(sg.x, sg.y)));
                        yu[e] = pack_bf16(y.x, y.y);
                    }
                    sts128(gaddr + chunk_off(r, m * 4 + c4, kTileHalfBytes), make_uint4(yu[0], yu[1], yu[2], yu[3]));
                }
            };
            {
                uint32_t oa[32], ob[32];
                uint4 sa[4], sb[4];
                tmem_ld32(tb + 128, oa);
                load_s(0, sa);
#pragma unroll 1
                for (int m = 0; m < 4; m += 2) {
                    tmem_wait_ld();
                    tmem_ld32(tb + 128 + (m + 1) * 32, ob);
                    load_s(m + 1, sb);
                    out_chunk(oa, sa, m);
                    tmem_wait_ld();
                    if (m + 2 < 4) {
                        tmem_ld32(tb + 128 + (m + 2) * 32, oa);
                        load_s(m + 2, sa);
                    } else {
                        // every O column of this buffer is in registers: hand it back
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar(BT_EMPTY + bb));
                    }
                    out_chunk(ob, sb, m + 1);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BY_READY + bb));
            if (r == 0 && mbar_wait(bar(BY_READY + bb), ph, ab)) {
                for (int h = 0; h < 2; ++h)
                    tma_store_4d(&tm_y, sbase + kOffG + bb * kTileBytes + h * kTileHalfBytes, h * 64,
                                 w.kvh * 4, w.s * kTok, w.b);
                bulk_commit_group();
                bulk_wait_group_read<0>();
                if (g_issued < n) load_gate();  // the slot just read is free again
            }
            if (idx + 1 < n) ok = sigma_row(idx + 1);
        }
        if (r == 0) {
            bulk_wait_group<0>();
            // loads of gate tiles that no step consumed (only after an abort)
            for (int i = (g_issued > 2 ? g_issued - 2 : 0); i < g_issued; ++i)
                drain_wait(bar(BG_FULL + (i & 1)), (i >> 1) & 1);
        }
    }

    // ---- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace swa
}  // namespace gswa
