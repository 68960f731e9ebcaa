// full_fwd.cuh -- full causal attention forward (the 5 global layers) for sm_100a.
//
// ZGCM-1 §2.1 and Figure 3 caption: global layers attend over the whole
// context (causal) and drop the gate; they use the same QK RMSNorm and
// partial RoPE.  y_i = softmax_{j <= i}(scale <q~_i, k~_j>) V, lse_i.
//
// Queries and keys arrive prepared (q~, k~ from qk_prep, in the workspace): a
// key tile is reused by every later query block, and preparing the queries
// up front frees the warps that would otherwise do it for the softmax.
//
// Unit: 32 query tokens of one (sequence, KV head) -- the 4 heads of the GQA
// group as M = 128 tensor-core rows (row = 4 * token + head) -- against the
// 128-key tiles 0 .. (32 qb + 31) / 128.  Persistent CTAs take units in a
// longest-first "snake" order (unit u of the order goes to CTA u mod 2G or
// 2G - 1 - u mod 2G), which balances the causal triangle.
//
// Pipeline per tile j: S = Q~ K~^T (TMEM, two buffers) -> softmax -> P (bf16,
// its own two TMEM buffers) -> O += P V (TMEM-A MMA).  K and V tiles have
// separate shared-memory stages and producers: a K stage is released as soon
// as its QK^T is done, a V stage after its PV, so the next K load starts
// early.  Eight softmax warps -- two per TMEM lane quarter, 64 of the 128
// columns each -- hold their scores in registers (the S buffer is released
// at once), exchange row maxima through shared memory, and run the epilogue.
//
// Softmax reference.  The queries and keys are RMS-normed, so every raw score
// is bounded: |<q~, k~>| <= |q~| |k~| <= D max|w_q| max|w_k| (a normed row has
// norm sqrt(D) before the weights).  Softmax is shift-invariant, so that bound
// (times scale log2 e, with 2 % headroom for bf16 rounding) serves as a fixed
// reference: P = 2^(S scale log2 e - M) never overflows, and while M <= 60 no
// P of a visible key falls below 2^-120, inside the float range.  Then no
// row max, no exchange between the two halves of a row and no rescaling of O
// are needed.  With larger norm weights the kernel falls back to a lazy
// running max: the reference is raised only when a tile's max exceeds it by
// more than 2^8, so the O accumulator in TMEM is rescaled rarely.
//
// Warp roles (12 warps): 0 K~ producer, 1 TMEM owner and MMA issuer, 2 V
// producer, 3 Q~ producer, 4-11 softmax, O correction and epilogue.
// TMEM: S buffers at columns 0 and 128, O at 256, P buffers at 384 and 448.
#pragma once

#include <cuda.h>

#include "ptx.cuh"
#include "swa_fwd.cuh"

namespace gswa {
namespace full {

constexpr int kTok = 32;
constexpr int kRows = 128;
constexpr int kKeys = 128;                 // keys per tile
constexpr int kThreads = 384;
constexpr float kRescaleLog2 = 8.0f;       // raise the reference max past 2^8

constexpr uint32_t kHalf = kRows * 128;                 // 16 KiB: 128 rows x 64 dims
constexpr uint32_t kTile = 2 * kHalf;                    // 32 KiB
constexpr uint32_t kOffK = 0;                            // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTile;            // 2 stages
constexpr uint32_t kOffQ = kOffV + 2 * kTile;            // 2 slots
constexpr uint32_t kOffMax = kOffQ + 2 * kTile;          // f32 [2 tile parity][2 halves][128 rows]
constexpr uint32_t kOffL = kOffMax + 2 * 2 * 128 * 4;    // f32 [2 halves][128 rows]
constexpr uint32_t kOffBar = kOffL + 2 * 128 * 4;
constexpr int kNumBars = 27;
constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
constexpr uint32_t kSmemBytes = kOffAbort + 4 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget of one sm_100 CTA");

constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;   // TMEM columns

enum : int {
    BK_FULL = 0, BK_EMPTY = 2, BV_FULL = 4, BV_EMPTY = 6, BQ_FULL = 8, BQ_EMPTY = 10, BS_FULL = 12,
    BS_FREE = 14, BP_READY = 16, BP_FREE = 18, BO_FULL = 20, BO_FREE = 21, B_DRAIN = 22,
    BX = 23   // 4 barriers: exchange between the two softmax warps of a TMEM lane quarter
};

struct Params {
    int B, T, Hq, Hkv;
    int nq;            // query blocks: ceil(T / 32)
    int nkt;           // key tiles: ceil(T / 128)
    long long units;   // B * Hkv * nq
    float sl2;         // softmax scale * log2(e)
    const __nv_bfloat16 *wq, *wk;   // norm weights, for the score bound
    __nv_bfloat16 *y;  // [B, T, Hq, D]
    float *lse;        // [B, Hq, T] or null
};

struct Unit {
    int b, kvh, qb, nt;
};

// k-th unit of this CTA in the longest-first snake order; false past the end.
__device__ __forceinline__ bool unit_at(const Params &p, int k, Unit &x)
{
    const long long G = gridDim.x, c = blockIdx.x;
    const long long u = (k & 1) ? ((long long)(k + 1) * G - 1 - c) : ((long long)k * G + c);
    if (u >= p.units) return false;
    const long long per = (long long)p.B * p.Hkv;
    x.qb = p.nq - 1 - (int)(u / per);
    const long long strip = u % per;
    x.b = (int)(strip / p.Hkv);
    x.kvh = (int)(strip % p.Hkv);
    x.nt = min(p.nkt, (kTok * x.qb + kTok - 1) / kKeys + 1);
    return true;
}

// Number of units of this CTA: pairs k = 2q, 2q + 1 take units 2qG + c and
// 2qG + 2G - 1 - c, so every full pair fits and the last pair fits partly.
__device__ __forceinline__ int num_units(const Params &p)
{
    const long long G = gridDim.x, c = blockIdx.x;
    const long long full = p.units / (2 * G), rem = p.units - full * 2 * G;
    return (int)(2 * full + (c < rem ? 1 : 0) + (2 * G - 1 - c < rem ? 1 : 0));
}

// Walks (unit, tile) pairs of this CTA in order.
struct TileWalk {
    int k = 0, j = 0;
    Unit x;
    bool valid = false;
    __device__ __forceinline__ void init(const Params &p) { k = 0; j = 0; valid = unit_at(p, 0, x); }
    __device__ __forceinline__ bool last_tile() const { return j == x.nt - 1; }
    __device__ __forceinline__ void next(const Params &p)
    {
        if (++j == x.nt) {
            j = 0;
            ++k;
            valid = unit_at(p, k, x);
        }
    }
};

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity)
{
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer() - t0 > 200000000ull) break;
}

// Producer of one operand stream (K~ or V): a tile per (unit, key tile) into
// two shared-memory stages.
__device__ __forceinline__ void tile_producer(const Params &p, const CUtensorMap *tm, uint32_t dst,
                                              uint32_t full, uint32_t empty, const Abort &ab)
{
    TileWalk w;
    w.init(p);
    int g = 0;
    bool ok = true;
    for (; w.valid && ok; w.next(p), ++g) {
        const int st = g & 1;
        ok = mbar_wait(empty + 8 * st, ((g >> 1) & 1) ^ 1u, ab);
        if (!ok) break;
        mbar_arrive_expect_tx(full + 8 * st, kTile);
        for (int h = 0; h < 2; ++h)
            tma_load_4d(dst + st * kTile + h * kHalf, tm, full + 8 * st, h * 64, w.x.kvh, w.j * kKeys, w.x.b);
    }
    for (int i = (g > 2 ? g - 2 : 0); i < g; ++i) drain_wait(full + 8 * (i & 1), (i >> 1) & 1);
}

__global__ void __launch_bounds__(kThreads, 1)
full_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffTmemSlot);
    Abort ab{reinterpret_cast<volatile int *>(smem + kOffAbort)};
    auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * (uint32_t)i; };
    const int n = num_units(p);

    if (tid == 0) {
        *ab.flag = 0;
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(BK_FULL + i), 1);
            mbar_init(bar(BK_EMPTY + i), 1);
            mbar_init(bar(BV_FULL + i), 1);
            mbar_init(bar(BV_EMPTY + i), 1);
            mbar_init(bar(BQ_FULL + i), 1);
            mbar_init(bar(BQ_EMPTY + i), 1);
            mbar_init(bar(BS_FULL + i), 1);
            mbar_init(bar(BS_FREE + i), 8);
            mbar_init(bar(BP_READY + i), 8);
            mbar_init(bar(BP_FREE + i), 1);
        }
        mbar_init(bar(BO_FULL), 1);
        mbar_init(bar(BO_FREE), 8);
        mbar_init(bar(B_DRAIN), 1);
        for (int i = 0; i < 4; ++i) mbar_init(bar(BX + i), 2);
        fence_barrier_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
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
        // ================================================= K~ producer
        if (lane == 0) tile_producer(p, &tm_k, sbase + kOffK, bar(BK_FULL), bar(BK_EMPTY), ab);
    } else if (warp == 2) {
        // ================================================= V producer
        if (lane == 0) tile_producer(p, &tm_v, sbase + kOffV, bar(BV_FULL), bar(BV_EMPTY), ab);
    } else if (warp == 3) {
        // ================================================= Q~ producer (one tile per unit, two slots)
        if (lane == 0) {
            Unit x;
            int k = 0;
            bool ok = true;
            for (; k < n && ok; ++k) {
                unit_at(p, k, x);
                ok = mbar_wait(bar(BQ_EMPTY + (k & 1)), ((k >> 1) & 1) ^ 1u, ab);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(BQ_FULL + (k & 1)), kTile);
                for (int h = 0; h < 2; ++h)
                    tma_load_4d(sbase + kOffQ + (k & 1) * kTile + h * kHalf, &tm_q, bar(BQ_FULL + (k & 1)), h * 64,
                                x.kvh * 4, x.qb * kTok, x.b);
            }
            for (int i = (k > 2 ? k - 2 : 0); i < k; ++i) drain_wait(bar(BQ_FULL + (i & 1)), (i >> 1) & 1);
        }
    } else if (warp == 1) {
        // ================================================= MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16_f32(128, kKeys, 0, 0);
            const uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
            TileWalk ws, wp;
            ws.init(p);
            wp.init(p);
            int ns = 0, npv = 0;
            PollWatch watch;
            while (wp.valid) {
                bool progressed = false;
                if (ws.valid && ns < npv + 2 && mbar_test(bar(BQ_FULL + (ws.k & 1)), (ws.k >> 1) & 1) &&
                    mbar_test(bar(BK_FULL + (ns & 1)), (ns >> 1) & 1) &&
                    mbar_test(bar(BS_FREE + (ns & 1)), ((ns >> 1) & 1) ^ 1u)) {
                    tc_fence_after();
                    const uint32_t dS = tmem + kColS + (ns & 1) * 128;
                    const uint32_t qs = sbase + kOffQ + (ws.k & 1) * kTile;
                    const uint32_t ks = sbase + kOffK + (ns & 1) * kTile;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
                        mma_ss(dS, smem_desc_sw128(qs + off, 16, 1024), smem_desc_sw128(ks + off, 16, 1024),
                               idesc_s, kk > 0);
                    }
                    mma_commit(bar(BS_FULL + (ns & 1)));
                    mma_commit(bar(BK_EMPTY + (ns & 1)));
                    if (ws.last_tile()) mma_commit(bar(BQ_EMPTY + (ws.k & 1)));
                    ws.next(p);
                    ++ns;
                    progressed = true;
                }
                if (npv < ns && mbar_test(bar(BP_READY + (npv & 1)), (npv >> 1) & 1) &&
                    mbar_test(bar(BV_FULL + (npv & 1)), (npv >> 1) & 1) &&
                    (wp.j != 0 || mbar_test(bar(BO_FREE), (wp.k & 1) ^ 1u))) {
                    tc_fence_after();
                    const uint32_t vs = sbase + kOffV + (npv & 1) * kTile;
                    const uint32_t pa = tmem + kColP + (npv & 1) * 64;
#pragma unroll
                    for (int kk = 0; kk < kKeys / 16; ++kk)
                        mma_ts(tmem + kColO, pa + kk * 8, smem_desc_sw128(vs + kk * 16 * 128, kHalf, 1024), idesc_pv,
                               (wp.j > 0 || kk > 0));
                    mma_commit(bar(BV_EMPTY + (npv & 1)));
                    mma_commit(bar(BP_FREE + (npv & 1)));
                    if (wp.last_tile()) mma_commit(bar(BO_FULL));
                    wp.next(p);
                    ++npv;
                    progressed = true;
                }
                if (!watch.tick(progressed, ab)) break;
            }
            mma_commit(bar(B_DRAIN));
            drain_wait(bar(B_DRAIN), 0);
        }
        __syncwarp();
    } else {
        // ================================================= softmax, correction, epilogue (8 warps)
        const int grp = (warp - 4) >> 2;           // column half: keys 64 grp .. 64 grp + 63 of each tile
        const int q = warp & 3;                    // TMEM lane quarter
        const int r = 32 * q + lane;               // row of the unit
        const int t = r >> 2;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        float *xmax = reinterpret_cast<float *>(smem + kOffMax);   // [parity][grp][row]
        float *xl = reinterpret_cast<float *>(smem + kOffL);       // [grp][row]
        const float ln2 = 0.6931471805599453f;
        // fixed softmax reference from the score bound (see the header)
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
        const float ref_fixed = 1.02f * 128.0f * wmax_q * wmax_k * fabsf(p.sl2);   // bound of |S scale log2 e|
        const bool fixed = ref_fixed <= 60.0f;
        // exchange with the partner warp (same rows, other half): every lane has
        // written its value before lane 0 arrives; both warps take the same
        // sequence of exchanges, so one counter gives the phase
        uint32_t xphase = 0;
        auto exchange = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BX + q));
            const bool done = warp_wait(bar(BX + q), xphase & 1u, ab);
            ++xphase;
            return done;
        };
        bool ok = true;
        int g = 0;   // global tile counter of this CTA
        Unit x;
        for (int k = 0; k < n && ok; ++k) {
            unit_at(p, k, x);
            const int i = x.qb * kTok + t;   // this row's query position
            float m_ref = -INFINITY;         // reference max (raw score units)
            float l = 0.f;                   // this half's share of the row sum
            for (int j = 0; j < x.nt && ok; ++j, ++g) {
                const int bb = g & 1;
                ok = warp_wait(bar(BS_FULL + bb), (g >> 1) & 1, ab);
                if (!ok) break;
                tc_fence_after();
                uint32_t s0[32], s1[32];
                const uint32_t ts = tmem + lane_base + kColS + bb * 128 + 64 * grp;
                tmem_ld32(ts, s0);
                tmem_ld32(ts + 32, s1);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(BS_FREE + bb));   // the scores are in registers
                const int hi = i - j * kKeys - 64 * grp;         // visible local columns e <= hi
                float mxs = ref_fixed;   // reference of this tile, in log2 units
                if (!fixed) {
                    float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        mx4[e & 3] = fmaxf(mx4[e & 3], (e <= hi) ? __uint_as_float(s0[e]) : -INFINITY);
                        mx4[e & 3] = fmaxf(mx4[e & 3], (e + 32 <= hi) ? __uint_as_float(s1[e]) : -INFINITY);
                    }
                    float mt = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
                    // row max over both halves (slot by tile parity: the partner read the
                    // previous use of this slot before it arrived at the next exchange)
                    xmax[(bb * 2 + grp) * 128 + r] = mt;
                    ok = exchange();
                    if (!ok) break;
                    mt = fmaxf(mt, xmax[(bb * 2 + (grp ^ 1)) * 128 + r]);
                    // lazy running max: raise the reference only past 2^8 (same decision in both halves)
                    float alpha = 1.f;
                    const bool raise = (m_ref == -INFINITY) || ((mt - m_ref) * p.sl2 > kRescaleLog2);
                    if (raise) {
                        if (m_ref != -INFINITY) alpha = ex2((m_ref - mt) * p.sl2);
                        m_ref = mt;
                        l *= alpha;
                    }
                    if (j > 0 && __any_sync(0xffffffffu, raise && alpha != 1.f)) {
                        // O holds the tiles before this one: wait for their PV, rescale this half in TMEM
                        ok = warp_wait(bar(BP_FREE + ((g - 1) & 1)), ((g - 1) >> 1) & 1, ab);
                        if (!ok) break;
                        tc_fence_after();
#pragma unroll 1
                        for (int c = 0; c < 2; ++c) {
                            const uint32_t oa = tmem + lane_base + kColO + 64 * grp + 32 * c;
                            uint32_t o[32];
                            tmem_ld32(oa, o);
                            tmem_wait_ld();
                            uint32_t lo16[16], hi16[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                lo16[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                                hi16[e] = __float_as_uint(__uint_as_float(o[16 + e]) * alpha);
                            }
                            tmem_st16(oa, lo16);
                            tmem_st16(oa + 16, hi16);
                        }
                        tmem_wait_st();
                    }
                    mxs = m_ref * p.sl2;
                }
                uint32_t pa16[16], pb16[16];
                float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    float p0 = ex2(fmaf(__uint_as_float(s0[e]), p.sl2, -mxs));
                    float p1 = ex2(fmaf(__uint_as_float(s0[e + 1]), p.sl2, -mxs));
                    p0 = (e <= hi) ? p0 : 0.f;
                    p1 = (e + 1 <= hi) ? p1 : 0.f;
                    sum4[(e >> 1) & 3] += p0 + p1;
                    pa16[e >> 1] = pack_bf16(p0, p1);
                    float p2 = ex2(fmaf(__uint_as_float(s1[e]), p.sl2, -mxs));
                    float p3 = ex2(fmaf(__uint_as_float(s1[e + 1]), p.sl2, -mxs));
                    p2 = (e + 32 <= hi) ? p2 : 0.f;
                    p3 = (e + 33 <= hi) ? p3 : 0.f;
                    sum4[(e >> 1) & 3] += p2 + p3;
                    pb16[e >> 1] = pack_bf16(p2, p3);
                }
                l += (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
                // the PV two tiles back has read this P buffer
                ok = warp_wait(bar(BP_FREE + bb), ((g >> 1) & 1) ^ 1u, ab);
                if (!ok) break;
                const uint32_t pa = tmem + lane_base + kColP + bb * 64 + 32 * grp;
                tmem_st16(pa, pa16);
                tmem_st16(pa + 16, pb16);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(BP_READY + bb));
            }
            if (!ok) break;
            // ---- epilogue of the unit: y = O / l (this half's 64 dims), lse.  The partner
            // reads this slot before its next exchange, which precedes the next write here.
            xl[grp * 128 + r] = l;
            ok = exchange();
            if (!ok) break;
            const float lt = xl[r] + xl[128 + r];
            ok = warp_wait(bar(BO_FULL), k & 1, ab);
            if (!ok) break;
            tc_fence_after();
            const float inv = 1.0f / lt;
            uint32_t o0[32], o1[32];
            tmem_ld32(tmem + lane_base + kColO + 64 * grp, o0);
            tmem_ld32(tmem + lane_base + kColO + 64 * grp + 32, o1);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BO_FREE));
            if (i < p.T) {
                uint4 *yrow = reinterpret_cast<uint4 *>(
                    p.y + (((long long)x.b * p.T + i) * p.Hq + x.kvh * 4 + (r & 3)) * 128 + 64 * grp);
                auto ychunk = [&](const uint32_t(&o)[32], int c) {
                    return make_uint4(pack_bf16(__uint_as_float(o[8 * c + 0]) * inv, __uint_as_float(o[8 * c + 1]) * inv),
                                      pack_bf16(__uint_as_float(o[8 * c + 2]) * inv, __uint_as_float(o[8 * c + 3]) * inv),
                                      pack_bf16(__uint_as_float(o[8 * c + 4]) * inv, __uint_as_float(o[8 * c + 5]) * inv),
                                      pack_bf16(__uint_as_float(o[8 * c + 6]) * inv, __uint_as_float(o[8 * c + 7]) * inv));
                };
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    yrow[c] = ychunk(o0, c);
                    yrow[4 + c] = ychunk(o1, c);
                }
                if (grp == 0 && p.lse != nullptr)
                    p.lse[((long long)x.b * p.Hq + x.kvh * 4 + (r & 3)) * p.T + i] =
                        ((fixed ? ref_fixed : m_ref * p.sl2) + __log2f(lt)) * ln2;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace full
}  // namespace gswa
