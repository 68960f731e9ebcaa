// swa_fwd.cuh -- gated sliding-window attention forward for sm_100a.
//
// Computes, for one ZGCM-1 gated-SWA layer (ZGCM-1 §2.1 Model overview and
// Figure 3 caption: 128-token sliding window, GQA 32 q / 8 kv heads of dim
// 128, QK RMSNorm, partial RoPE; GatedSWA(h) = o_proj(A_SWA(q,k,v) ⊙ σ(g)))
//   y_i = softmax_{i-W < j <= i}(scale <q~_i, k~_j>) V  ⊙  σ(g_i)
// with q~, k~ the RMS-normed, partially rotated queries and keys, and the
// natural-log normaliser lse_i of each row.
//
// Work unit: a 32-token query block of one (sequence, KV head) pair, i.e. the
// 4 query heads of a GQA group packed as M = 128 tensor-core rows
// (row r = 4 * token + head-in-group).  Its keys are the 160 keys
// [i0 - 128, i0 + 32): five 32-key blocks.  Persistent CTAs walk consecutive
// blocks of a strip, so each K/V block is fetched from HBM once and kept in
// a six-slot shared-memory ring while the window slides over it.
//
// Warp roles (16 warps):
//   warp 0      TMA producer: Q, g tiles (2 stages) and K/V blocks (ring)
//   warp 1      TMEM owner and tcgen05.mma issuer
//   warp 2      key prologue: RMSNorm + RoPE of each new K block, in place
//   warp 3      idle
//   warps 4-7   query prologue: RMSNorm + RoPE of the 128 Q rows, in place
//   warps 8-11  softmax: S (TMEM) -> P (bf16, TMEM), row max/sum, lse
//   warps 12-15 epilogue: O (TMEM) / l ⊙ σ(g) -> y, TMA store
//
// TMEM (512 columns) holds two buffers of 256 columns: S at +0 (160 f32
// columns), P at +0 (80 columns of bf16 pairs, written over S once read)
// and O at +128 (128 f32 columns, written only after P is complete).
#pragma once

#include <cuda.h>

#include "ptx.cuh"

namespace gswa {
namespace swa {

constexpr int kD = 128;
constexpr int kTok = 32;                 // query tokens per unit
constexpr int kRows = 128;               // MMA M
constexpr int kSpanBlocks = 5;           // 160-key window span in 32-key blocks
constexpr int kRing = 6;                 // K/V ring slots
constexpr int kSpan = kSpanBlocks * kTok; // 160
constexpr int kThreads = 512;

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
constexpr uint32_t kOffWq = kOffG + 2 * kTileBytes;           // 229376 (bf16[128])
constexpr uint32_t kOffWk = kOffWq + 256;
constexpr uint32_t kOffInvL = kOffWk + 256;                   // f32[2][128]
constexpr uint32_t kOffBar = kOffInvL + 2 * kRows * 4;
constexpr int kNumBars = 33;
constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
constexpr uint32_t kSmemUsed = kOffAbort + 4;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;             // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget of one sm_100 CTA");

// Barrier indices.
enum : int {
    BQ_FULL = 0, BQ_PREP = 2, BQ_EMPTY = 4, BG_FULL = 6, BG_EMPTY = 8,
    BKV_FULL = 10, BKV_EMPTY = 16, BS_FULL = 22, BP_READY = 24, BO_FULL = 26,
    BT_EMPTY = 28, BY_READY = 30, B_DRAIN = 32
};

struct Params {
    int B, T, Hq, Hkv, window, R;
    int nsteps;        // ceil(T / 32)
    long long units;   // B * Hkv * nsteps
    float eps;
    float sl2;         // softmax scale * log2(e)
    const __nv_bfloat16 *wq, *wk;
    float *lse;        // [B, Hq, T] or null
    double theta[64];  // rope_base^(-2p/R), p < R/2
};

struct Unit {
    int b, kvh, s;
    bool first, last;
};

__device__ __forceinline__ Unit unit_of(const Params &p, long long u, long long u0, long long u1)
{
    Unit x;
    long long strip = u / p.nsteps;
    x.s = (int)(u - strip * p.nsteps);
    x.b = (int)(strip / p.Hkv);
    x.kvh = (int)(strip - (long long)x.b * p.Hkv);
    x.first = (u == u0) || (x.s == 0);
    x.last = (u == u1 - 1) || (x.s == p.nsteps - 1);
    return x;
}

__device__ __forceinline__ int ring_slot(int kb) { return ((kb % kRing) + kRing) % kRing; }

// Byte offset of 16-byte chunk c (0..15) of row r in a two-half swizzled tile
// whose halves are `half_stride` apart (TMA 128-byte swizzle pattern).
__device__ __forceinline__ uint32_t chunk_off(int r, int c, uint32_t half_stride)
{
    return (uint32_t)(c >> 3) * half_stride + (uint32_t)r * kHalfRowBytes +
           ((uint32_t)((c & 7) ^ (r & 7)) << 4);
}

// Byte offset of element d of row r (same layout).
__device__ __forceinline__ uint32_t elem_off(int r, int d, uint32_t half_stride)
{
    return chunk_off(r, d >> 3, half_stride) + (uint32_t)(d & 7) * 2;
}

// cos/sin of the rotary angle pos * theta, reduced in double precision first
// so that positions up to 2^18 keep full single-precision accuracy.
__device__ __forceinline__ void rope_cs(double theta, int pos, float &c, float &s)
{
    const double two_pi = 6.283185307179586;
    double phi = (double)pos * theta;
    double k = rint(phi * (1.0 / two_pi));
    float r = (float)fma(-k, two_pi, phi);
    sincosf(r, &s, &c);
}

// RMSNorm then partial RoPE of one head row held in shared memory (bf16,
// swizzled), in place, one thread per row.  Dims >= R are scaled only; the
// rotated pairs (p, p + R/2) are normalised and rotated in f32 and rounded
// once.  `cs_from_group` lets 4 neighbouring lanes that share a token split
// the cos/sin evaluations (each computes every 4th pair, then they swap).
template <bool kShareInQuad>
__device__ __forceinline__ void prep_row_smem(uint8_t *tile, uint32_t half_stride, int row,
                                              const __nv_bfloat16 *w, int R, float eps, int pos,
                                              const double *theta)
{
    // pass 1: mean square of the raw row
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        uint4 v = *reinterpret_cast<const uint4 *>(tile + chunk_off(row, c, half_stride));
        uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float2 f = unpack_bf16(u[e]);
            ss = fmaf(f.x, f.x, ss);
            ss = fmaf(f.y, f.y, ss);
        }
    }
    const float r = rsqrtf(ss * (1.0f / kD) + eps);
    // pass 2: plain scaling of the dims past the rotated slice
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        const int d0 = c * 8;
        if (d0 + 8 <= R) continue;
        uint4 *ptr = reinterpret_cast<uint4 *>(tile + chunk_off(row, c, half_stride));
        uint4 v = *ptr;
        uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float2 f = unpack_bf16(u[e]);
            const int d = d0 + 2 * e;
            float a = (d >= R) ? f.x * r * __bfloat162float(w[d]) : f.x;
            float b = (d + 1 >= R) ? f.y * r * __bfloat162float(w[d + 1]) : f.y;
            // dims below R keep their raw bits for pass 3
            u[e] = (d >= R) ? pack_bf16(a, b)
                            : ((d + 1 >= R) ? ((u[e] & 0xFFFFu) | (pack_bf16(a, b) & 0xFFFF0000u))
                                            : u[e]);
        }
        *ptr = make_uint4(u[0], u[1], u[2], u[3]);
    }
    // pass 3: rotate the pairs (p, p + R/2)
    const int half = R >> 1;
    if (kShareInQuad) {
        const int lane = threadIdx.x & 31;
        const int q = lane & 3;
        for (int p0 = 0; p0 < half; p0 += 4) {
            float cm = 1.f, sm = 0.f;
            if (p0 + q < half) rope_cs(theta[p0 + q], pos, cm, sm);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float c = __shfl_sync(0xffffffffu, cm, (lane & ~3) | j);
                const float s = __shfl_sync(0xffffffffu, sm, (lane & ~3) | j);
                const int pp = p0 + j;
                if (pp < half) {
                    __nv_bfloat16 *x1 = reinterpret_cast<__nv_bfloat16 *>(tile + elem_off(row, pp, half_stride));
                    __nv_bfloat16 *x2 = reinterpret_cast<__nv_bfloat16 *>(tile + elem_off(row, pp + half, half_stride));
                    const float n1 = __bfloat162float(*x1) * r * __bfloat162float(w[pp]);
                    const float n2 = __bfloat162float(*x2) * r * __bfloat162float(w[pp + half]);
                    *x1 = __float2bfloat16_rn(n1 * c - n2 * s);
                    *x2 = __float2bfloat16_rn(n2 * c + n1 * s);
                }
            }
        }
    } else {
        for (int pp = 0; pp < half; ++pp) {
            float c, s;
            rope_cs(theta[pp], pos, c, s);
            __nv_bfloat16 *x1 = reinterpret_cast<__nv_bfloat16 *>(tile + elem_off(row, pp, half_stride));
            __nv_bfloat16 *x2 = reinterpret_cast<__nv_bfloat16 *>(tile + elem_off(row, pp + half, half_stride));
            const float n1 = __bfloat162float(*x1) * r * __bfloat162float(w[pp]);
            const float n2 = __bfloat162float(*x2) * r * __bfloat162float(w[pp + half]);
            *x1 = __float2bfloat16_rn(n1 * c - n2 * s);
            *x2 = __float2bfloat16_rn(n2 * c + n1 * s);
        }
    }
}

// Bounded wait used only while tearing down: ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity)
{
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer() - t0 > 200000000ull) break;
}

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
    const int nunits = (int)(u1 - u0);

    // ---- set-up
    if (tid == 0) {
        *ab.flag = 0;
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(BQ_FULL + i), 1);
            mbar_init(bar(BQ_PREP + i), 5);   // 4 query-prologue warps + key warp
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
            mbar_init(bar(BKV_FULL + i), 1);
            mbar_init(bar(BKV_EMPTY + i), 1);
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
        reinterpret_cast<__nv_bfloat16 *>(smem + kOffWq)[tid] = p.wq[tid];
        reinterpret_cast<__nv_bfloat16 *>(smem + kOffWk)[tid] = p.wk[tid];
    }
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
            uint32_t kv_fills = 0;     // parity of fills per ring slot
            uint32_t armed = 0;        // ring slots with a load in flight at least once
            auto load_kv = [&](const Unit &x, int kb) -> bool {
                const int slot = ring_slot(kb);
                const uint32_t f = (kv_fills >> slot) & 1u;
                if (!mbar_wait(bar(BKV_EMPTY + slot), f ^ 1u, ab)) return false;
                kv_fills ^= 1u << slot;
                armed |= 1u << slot;
                mbar_arrive_expect_tx(bar(BKV_FULL + slot), 4 * kBlockHalfBytes);
                for (int h = 0; h < 2; ++h) {
                    tma_load_4d(sbase + kOffK + h * kRingHalfBytes + slot * kBlockHalfBytes, &tm_k,
                                bar(BKV_FULL + slot), h * 64, x.kvh, kb * kTok, x.b);
                    tma_load_4d(sbase + kOffV + h * kRingHalfBytes + slot * kBlockHalfBytes, &tm_v,
                                bar(BKV_FULL + slot), h * 64, x.kvh, kb * kTok, x.b);
                }
                return true;
            };
            bool ok = true;
            for (int idx = 0; idx < nunits && ok; ++idx) {
                const Unit x = unit_of(p, u0 + idx, u0, u1);
                if (x.first)
                    for (int kb = x.s - 4; kb < x.s && ok; ++kb) ok = load_kv(x, kb);
                if (ok) ok = load_kv(x, x.s);
                const int j = idx & 1;
                const uint32_t ph = (idx >> 1) & 1;
                if (ok) ok = mbar_wait(bar(BQ_EMPTY + j), ph ^ 1u, ab);
                if (ok) {
                    mbar_arrive_expect_tx(bar(BQ_FULL + j), kTileBytes);
                    for (int h = 0; h < 2; ++h)
                        tma_load_4d(sbase + kOffQ + j * kTileBytes + h * kTileHalfBytes, &tm_q,
                                    bar(BQ_FULL + j), h * 64, x.kvh * 4, x.s * kTok, x.b);
                }
                if (ok) ok = mbar_wait(bar(BG_EMPTY + j), ph ^ 1u, ab);
                if (ok) {
                    mbar_arrive_expect_tx(bar(BG_FULL + j), kTileBytes);
                    for (int h = 0; h < 2; ++h)
                        tma_load_4d(sbase + kOffG + j * kTileBytes + h * kTileHalfBytes, &tm_g,
                                    bar(BG_FULL + j), h * 64, x.kvh * 4, x.s * kTok, x.b);
                }
            }
            // Teardown: every load this thread issued must have landed before
            // the CTA's shared memory is released.
            for (int slot = 0; slot < kRing; ++slot)
                if (armed & (1u << slot)) drain_wait(bar(BKV_FULL + slot), ((kv_fills >> slot) & 1u) ^ 1u);
            for (int idx = (nunits > 2 ? nunits - 2 : 0); idx < nunits; ++idx) {
                drain_wait(bar(BQ_FULL + (idx & 1)), (idx >> 1) & 1);
                drain_wait(bar(BG_FULL + (idx & 1)), (idx >> 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ================================================= MMA issuer
        if (lane == 0) {
            const uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
            bool ok = true;
            auto issue_S = [&](int idx) -> bool {
                const Unit x = unit_of(p, u0 + idx, u0, u1);
                const int bb = idx & 1;
                const uint32_t ph = (idx >> 1) & 1;
                if (!mbar_wait(bar(BT_EMPTY + bb), ph ^ 1u, ab)) return false;
                if (!mbar_wait(bar(BQ_PREP + bb), ph, ab)) return false;
                tc_fence_after();
                const int a = ring_slot(x.s - 4);
                const int n1 = (kRing - a) < kSpanBlocks ? (kRing - a) : kSpanBlocks;
                const int n2 = kSpanBlocks - n1;
                const uint32_t id1 = idesc_bf16_f32(128, n1 * kTok, 0, 0);
                const uint32_t id2 = idesc_bf16_f32(128, n2 > 0 ? n2 * kTok : 32, 0, 0);
                const uint32_t dS = tmem + bb * 256;
                const uint32_t qs = sbase + kOffQ + bb * kTileBytes;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t h = kk >> 2, ko = (kk & 3) * 32;
                    const uint64_t ad = smem_desc_sw128(qs + h * kTileHalfBytes + ko, 16, 1024);
                    const uint32_t kbase = sbase + kOffK + h * kRingHalfBytes + ko;
                    mma_ss(dS, ad, smem_desc_sw128(kbase + a * kBlockHalfBytes, 16, 1024), id1, kk > 0);
                    if (n2 > 0)
                        mma_ss(dS + n1 * kTok, ad, smem_desc_sw128(kbase, 16, 1024), id2, kk > 0);
                }
                mma_commit(bar(BS_FULL + bb));
                mma_commit(bar(BQ_EMPTY + bb));
                return true;
            };
            auto issue_PV = [&](int idx) -> bool {
                const Unit x = unit_of(p, u0 + idx, u0, u1);
                const int bb = idx & 1;
                const uint32_t ph = (idx >> 1) & 1;
                if (!mbar_wait(bar(BP_READY + bb), ph, ab)) return false;
                tc_fence_after();
                const int a = ring_slot(x.s - 4);
                const uint32_t dO = tmem + bb * 256 + 128;
#pragma unroll
                for (int kk = 0; kk < kSpan / 16; ++kk) {
                    const int slot = (a + (kk >> 1)) % kRing;
                    const uint32_t vaddr = sbase + kOffV + slot * kBlockHalfBytes + (kk & 1) * 16 * kHalfRowBytes;
                    mma_ts(dO, tmem + bb * 256 + kk * 8, smem_desc_sw128(vaddr, kRingHalfBytes, 1024),
                           idesc_pv, kk > 0);
                }
                mma_commit(bar(BO_FULL + bb));
                // Release ring slots no later step of this CTA reads.
                if (x.last) {
                    for (int i = 0; i < kSpanBlocks; ++i) mma_commit(bar(BKV_EMPTY + (a + i) % kRing));
                } else {
                    mma_commit(bar(BKV_EMPTY + a));
                }
                return true;
            };
            if (nunits > 0) ok = issue_S(0);
            for (int idx = 0; idx < nunits && ok; ++idx) {
                const Unit x = unit_of(p, u0 + idx, u0, u1);
                const bool has_next = idx + 1 < nunits;
                if (has_next && !x.last) ok = issue_S(idx + 1);
                if (ok) ok = issue_PV(idx);
                if (ok && has_next && x.last) ok = issue_S(idx + 1);
            }
            // all MMAs issued by this thread complete before TMEM is freed
            mma_commit(bar(B_DRAIN));
            drain_wait(bar(B_DRAIN), 0);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ================================================= key prologue
        uint32_t kv_fills = 0;
        const __nv_bfloat16 *wk = reinterpret_cast<const __nv_bfloat16 *>(smem + kOffWk);
        bool ok = true;
        for (int idx = 0; idx < nunits && ok; ++idx) {
            const Unit x = unit_of(p, u0 + idx, u0, u1);
            for (int kb = x.first ? x.s - 4 : x.s; kb <= x.s && ok; ++kb) {
                const int slot = ring_slot(kb);
                ok = warp_wait(bar(BKV_FULL + slot), (kv_fills >> slot) & 1u, ab);
                kv_fills ^= 1u << slot;
                if (ok)
                    prep_row_smem<false>(smem + kOffK + slot * kBlockHalfBytes, kRingHalfBytes, lane, wk,
                                         p.R, p.eps, kb * kTok + lane, p.theta);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (ok && lane == 0) mbar_arrive(bar(BQ_PREP + (idx & 1)));
        }
    } else if (warp >= 4 && warp < 8) {
        // ================================================= query prologue
        const int r = tid - 128;
        const __nv_bfloat16 *wq = reinterpret_cast<const __nv_bfloat16 *>(smem + kOffWq);
        bool ok = true;
        for (int idx = 0; idx < nunits && ok; ++idx) {
            const Unit x = unit_of(p, u0 + idx, u0, u1);
            const int j = idx & 1;
            ok = warp_wait(bar(BQ_FULL + j), (idx >> 1) & 1, ab);
            if (ok)
                prep_row_smem<true>(smem + kOffQ + j * kTileBytes, kTileHalfBytes, r, wq, p.R, p.eps,
                                    x.s * kTok + (r >> 2), p.theta);
            fence_proxy_async_smem();
            __syncwarp();
            if (ok && lane == 0) mbar_arrive(bar(BQ_PREP + j));
        }
    } else if (warp >= 8 && warp < 12) {
        // ================================================= softmax
        const int r = tid - 256;
        const int t = r >> 2;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        float *inv_l = reinterpret_cast<float *>(smem + kOffInvL);
        const float ln2 = 0.6931471805599453f;
        bool ok = true;
        for (int idx = 0; idx < nunits && ok; ++idx) {
            const Unit x = unit_of(p, u0 + idx, u0, u1);
            const int bb = idx & 1;
            ok = warp_wait(bar(BS_FULL + bb), (idx >> 1) & 1, ab);
            if (!ok) break;
            tc_fence_after();
            // visible window columns c: key j = 32 s - 128 + c, i - W < j <= i, j >= 0
            const int lo = max(t + 129 - p.window, 128 - kTok * x.s);
            const int hi = t + 128;
            const uint32_t ts = tmem + lane_base + bb * 256;
            float mx = -INFINITY;
#pragma unroll
            for (int m = 0; m < kSpanBlocks; ++m) {
                uint32_t v[32];
                tmem_ld32(ts + m * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int c = m * 32 + e;
                    if (c >= lo && c <= hi) mx = fmaxf(mx, __uint_as_float(v[e]));
                }
            }
            const float mxs = mx * p.sl2;
            float sum = 0.f;
#pragma unroll
            for (int m = 0; m < kSpanBlocks; ++m) {
                uint32_t v[32];
                tmem_ld32(ts + m * 32, v);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int c = m * 32 + e;
                    float p0 = (c >= lo && c <= hi) ? ex2(fmaf(__uint_as_float(v[e]), p.sl2, -mxs)) : 0.f;
                    float p1 = (c + 1 >= lo && c + 1 <= hi) ? ex2(fmaf(__uint_as_float(v[e + 1]), p.sl2, -mxs)) : 0.f;
                    sum += p0 + p1;
                    pk[e >> 1] = pack_bf16(p0, p1);
                }
                tmem_st16(ts + m * 16, pk);
            }
            tmem_wait_st();
            inv_l[bb * kRows + r] = 1.0f / sum;
            const int i = x.s * kTok + t;
            if (p.lse != nullptr && i < p.T)
                p.lse[((long long)x.b * p.Hq + x.kvh * 4 + (r & 3)) * p.T + i] = (mxs + __log2f(sum)) * ln2;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BP_READY + bb));
        }
    } else if (warp >= 12) {
        // ================================================= epilogue
        const int r = tid - 384;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const float *inv_l = reinterpret_cast<const float *>(smem + kOffInvL);
        const float log2e = 1.4426950408889634f;
        bool ok = true;
        int done = 0;
        for (int idx = 0; idx < nunits && ok; ++idx) {
            const Unit x = unit_of(p, u0 + idx, u0, u1);
            const int bb = idx & 1;
            const uint32_t ph = (idx >> 1) & 1;
            ok = warp_wait(bar(BP_READY + bb), ph, ab) && warp_wait(bar(BO_FULL + bb), ph, ab) &&
                 warp_wait(bar(BG_FULL + bb), ph, ab);
            if (!ok) break;
            tc_fence_after();
            const float inv = inv_l[bb * kRows + r];
            uint8_t *gt = smem + kOffG + bb * kTileBytes;
            const uint32_t to = tmem + lane_base + bb * 256 + 128;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                uint32_t o[32];
                tmem_ld32(to + m * 32, o);
                tmem_wait_ld();
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint4 *ptr = reinterpret_cast<uint4 *>(gt + chunk_off(r, m * 4 + c4, kTileHalfBytes));
                    uint4 gv = *ptr;
                    uint32_t gu[4] = {gv.x, gv.y, gv.z, gv.w};
                    uint32_t yu[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 gf = unpack_bf16(gu[e]);
                        const float s0 = __frcp_rn(1.0f + ex2(-gf.x * log2e));
                        const float s1 = __frcp_rn(1.0f + ex2(-gf.y * log2e));
                        const float y0 = __uint_as_float(o[c4 * 8 + 2 * e]) * inv * s0;
                        const float y1 = __uint_as_float(o[c4 * 8 + 2 * e + 1]) * inv * s1;
                        yu[e] = pack_bf16(y0, y1);
                    }
                    *ptr = make_uint4(yu[0], yu[1], yu[2], yu[3]);
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(BT_EMPTY + bb));
                mbar_arrive(bar(BY_READY + bb));
            }
            if (r == 0 && mbar_wait(bar(BY_READY + bb), ph, ab)) {
                for (int h = 0; h < 2; ++h)
                    tma_store_4d(&tm_y, sbase + kOffG + bb * kTileBytes + h * kTileHalfBytes, h * 64,
                                 x.kvh * 4, x.s * kTok, x.b);
                bulk_commit_group();
                bulk_wait_group_read<1>();
                if (idx >= 1) mbar_arrive(bar(BG_EMPTY + ((idx - 1) & 1)));
            }
            done = idx + 1;
        }
        if (r == 0) {
            bulk_wait_group<0>();
            if (done >= 1) mbar_arrive(bar(BG_EMPTY + ((done - 1) & 1)));
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
