// full_fwd.cuh -- full causal attention forward (the 5 global layers) for sm_100a.
//
// ZGCM-1 §2.1 and Figure 3 caption: global layers attend over the whole
// context (causal) and drop the gate; they use the same QK RMSNorm and
// partial RoPE.  y_i = softmax_{j <= i}(scale <q~_i, k~_j>) V, lse_i.
//
// The keys arrive prepared (k~ from qk_prep): a key tile is reused by every
// later query block, so it is normed and rotated once, not per use.  Queries
// are prepared in the prologue, as in the sliding-window kernel.
//
// Unit: 32 query tokens of one (sequence, KV head) -- the 4 heads of the GQA
// group as M = 128 tensor-core rows (row = 4 * token + head) -- against the
// 128-key tiles 0 .. (32 qb + 31) / 128.  Persistent CTAs take units in a
// longest-first "snake" order (unit u of the order goes to CTA u mod 2G or
// 2G - 1 - u mod 2G), which balances the causal triangle.
//
// Online softmax with a lazy running max: the reference max m used for
// P = 2^((S - m) scale log2 e) is raised only when a tile's max exceeds it by
// more than 2^8, so the O accumulator in TMEM is rescaled rarely; 1/l and m
// stay in the softmax thread's registers for the whole unit.
//
// Warp roles (12 warps): 0 K~/V TMA producer (2 stages); 1 TMEM owner, MMA
// issuer and Q TMA loads; 2-3 idle; 4-7 query prologue; 8-11 softmax,
// O correction and epilogue (y by TMA store, lse).
// TMEM: S/P buffers at columns 0 and 128 (P as bf16 pairs over S's first 64
// columns), O at 256.
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
constexpr uint32_t kOffY = kOffQ + 2 * kTile;            // 1 staging tile
constexpr uint32_t kOffWq = kOffY + kTile;               // f32[128]
constexpr uint32_t kOffBar = kOffWq + 512;
constexpr int kNumBars = 20;
constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
constexpr uint32_t kSmemBytes = kOffAbort + 4 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget of one sm_100 CTA");

enum : int {
    BKV_FULL = 0, BKV_EMPTY = 2, BQ_FULL = 4, BQ_PREP = 6, BQ_EMPTY = 8, BS_FULL = 10,
    BP_READY = 12, BS_FREE = 14, BO_FULL = 16, BO_FREE = 17, BY_READY = 18, B_DRAIN = 19
};

struct Params {
    int B, T, Hq, Hkv;
    int nq;            // query blocks: ceil(T / 32)
    int nkt;           // key tiles: ceil(T / 128)
    long long units;   // B * Hkv * nq
    float eps, sl2;
    const __nv_bfloat16 *wq;
    float *lse;
    double theta[64];
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

// Max of the visible scores of one 32-column chunk (columns c with c <= hi).
__device__ __forceinline__ void tile_chunk_max(const uint32_t (&v)[32], int c0, int hi, float (&mx)[4])
{
    const int kh = hi - c0;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const float x = (e <= kh) ? __uint_as_float(v[e]) : -INFINITY;
        mx[e & 3] = fmaxf(mx[e & 3], x);
    }
}

__device__ __forceinline__ void tile_chunk_exp(const uint32_t (&v)[32], int c0, int hi, float sl2, float mxs,
                                               float (&sum)[4], uint32_t (&pk)[16])
{
    const int kh = hi - c0;
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
        float p0 = ex2(fmaf(__uint_as_float(v[e]), sl2, -mxs));
        float p1 = ex2(fmaf(__uint_as_float(v[e + 1]), sl2, -mxs));
        p0 = (e <= kh) ? p0 : 0.f;
        p1 = (e + 1 <= kh) ? p1 : 0.f;
        sum[(e >> 1) & 3] += p0 + p1;
        pk[e >> 1] = pack_bf16(p0, p1);
    }
}

template <int R>
__global__ void __launch_bounds__(kThreads, 1)
full_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_y,
                const __grid_constant__ Params p)
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
            mbar_init(bar(BKV_FULL + i), 1);
            mbar_init(bar(BKV_EMPTY + i), 1);
            mbar_init(bar(BQ_FULL + i), 1);
            mbar_init(bar(BQ_PREP + i), 4);
            mbar_init(bar(BQ_EMPTY + i), 1);
            mbar_init(bar(BS_FULL + i), 1);
            mbar_init(bar(BP_READY + i), 4);
            mbar_init(bar(BS_FREE + i), 1);
        }
        mbar_init(bar(BO_FULL), 1);
        mbar_init(bar(BO_FREE), 4);
        mbar_init(bar(BY_READY), 4);
        mbar_init(bar(B_DRAIN), 1);
        fence_barrier_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_y);
    }
    if (tid < 128) reinterpret_cast<float *>(smem + kOffWq)[tid] = __bfloat162float(p.wq[tid]);
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ================================================= K~/V producer
        if (lane == 0) {
            TileWalk w;
            w.init(p);
            int g = 0;
            bool ok = true;
            for (; w.valid && ok; w.next(p), ++g) {
                const int st = g & 1;
                ok = mbar_wait(bar(BKV_EMPTY + st), ((g >> 1) & 1) ^ 1u, ab);
                if (!ok) break;
                mbar_arrive_expect_tx(bar(BKV_FULL + st), 2 * kTile);
                for (int h = 0; h < 2; ++h) {
                    tma_load_4d(sbase + kOffK + st * kTile + h * kHalf, &tm_k, bar(BKV_FULL + st), h * 64,
                                w.x.kvh, w.j * kKeys, w.x.b);
                    tma_load_4d(sbase + kOffV + st * kTile + h * kHalf, &tm_v, bar(BKV_FULL + st), h * 64,
                                w.x.kvh, w.j * kKeys, w.x.b);
                }
            }
            for (int i = (g > 2 ? g - 2 : 0); i < g; ++i) drain_wait(bar(BKV_FULL + (i & 1)), (i >> 1) & 1);
        }
    } else if (warp == 1) {
        // ================================================= MMA issuer + Q loads
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16_f32(128, kKeys, 0, 0);
            const uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
            TileWalk ws, wp;
            ws.init(p);
            wp.init(p);
            int kq = 0, ns = 0, npv = 0;
            Unit xq;
            bool q_more = unit_at(p, 0, xq);
            PollWatch watch;
            while (wp.valid) {
                bool progressed = false;
                if (q_more && mbar_test(bar(BQ_EMPTY + (kq & 1)), ((kq >> 1) & 1) ^ 1u)) {
                    const int j = kq & 1;
                    mbar_arrive_expect_tx(bar(BQ_FULL + j), kTile);
                    for (int h = 0; h < 2; ++h)
                        tma_load_4d(sbase + kOffQ + j * kTile + h * kHalf, &tm_q, bar(BQ_FULL + j), h * 64,
                                    xq.kvh * 4, xq.qb * kTok, xq.b);
                    ++kq;
                    q_more = unit_at(p, kq, xq);
                    progressed = true;
                }
                if (ws.valid && ns <= npv + 1 && mbar_test(bar(BQ_PREP + (ws.k & 1)), (ws.k >> 1) & 1) &&
                    mbar_test(bar(BKV_FULL + (ns & 1)), (ns >> 1) & 1) &&
                    mbar_test(bar(BS_FREE + (ns & 1)), ((ns >> 1) & 1) ^ 1u)) {
                    tc_fence_after();
                    const uint32_t dS = tmem + (ns & 1) * 128;
                    const uint32_t qs = sbase + kOffQ + (ws.k & 1) * kTile;
                    const uint32_t ks = sbase + kOffK + (ns & 1) * kTile;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
                        mma_ss(dS, smem_desc_sw128(qs + off, 16, 1024), smem_desc_sw128(ks + off, 16, 1024),
                               idesc_s, kk > 0);
                    }
                    mma_commit(bar(BS_FULL + (ns & 1)));
                    if (ws.last_tile()) mma_commit(bar(BQ_EMPTY + (ws.k & 1)));
                    ws.next(p);
                    ++ns;
                    progressed = true;
                }
                if (npv < ns && mbar_test(bar(BP_READY + (npv & 1)), (npv >> 1) & 1) &&
                    (wp.j != 0 || mbar_test(bar(BO_FREE), (wp.k & 1) ^ 1u))) {
                    tc_fence_after();
                    const uint32_t vs = sbase + kOffV + (npv & 1) * kTile;
#pragma unroll
                    for (int kk = 0; kk < kKeys / 16; ++kk)
                        mma_ts(tmem + 256, tmem + (npv & 1) * 128 + kk * 8,
                               smem_desc_sw128(vs + kk * 16 * 128, kHalf, 1024), idesc_pv, (wp.j > 0 || kk > 0));
                    mma_commit(bar(BKV_EMPTY + (npv & 1)));
                    mma_commit(bar(BS_FREE + (npv & 1)));
                    if (wp.last_tile()) mma_commit(bar(BO_FULL));
                    wp.next(p);
                    ++npv;
                    progressed = true;
                }
                if (!watch.tick(progressed, ab)) break;
            }
            mma_commit(bar(B_DRAIN));
            drain_wait(bar(B_DRAIN), 0);
            for (int i = (kq > 2 ? kq - 2 : 0); i < kq; ++i) drain_wait(bar(BQ_FULL + (i & 1)), (i >> 1) & 1);
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 8) {
        // ================================================= query prologue
        const int r = tid - 128;
        const float *wq = reinterpret_cast<const float *>(smem + kOffWq);
        swa::RopeTab<R / 2, 4> tab;
        tab.init_rows(r >> 2, lane & 3, p.theta);
        bool ok = true;
        Unit x;
        for (int k = 0; k < n && ok; ++k) {
            unit_at(p, k, x);
            tab.set_block(x.qb * kTok, p.theta);
            ok = warp_wait(bar(BQ_FULL + (k & 1)), (k >> 1) & 1, ab);
            if (ok) swa::prep_row<R, true>(sbase + kOffQ + (k & 1) * kTile, kHalf, r, wq, p.eps, tab);
            fence_proxy_async_smem();
            __syncwarp();
            if (ok && lane == 0) mbar_arrive(bar(BQ_PREP + (k & 1)));
        }
    } else if (warp >= 8) {
        // ================================================= softmax, correction, epilogue
        const int r = tid - 256;
        const int t = r >> 2;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const float ln2 = 0.6931471805599453f;
        bool ok = true;
        int g = 0;   // global tile counter of this CTA
        Unit x;
        for (int k = 0; k < n && ok; ++k) {
            unit_at(p, k, x);
            const int i = x.qb * kTok + t;   // this row's query position
            float m_ref = -INFINITY;         // reference max (raw score units)
            float l = 0.f;
            for (int j = 0; j < x.nt && ok; ++j, ++g) {
                const int bb = g & 1;
                ok = warp_wait(bar(BS_FULL + bb), (g >> 1) & 1, ab);
                if (!ok) break;
                tc_fence_after();
                const uint32_t ts = tmem + lane_base + bb * 128;
                const int hi = i - j * kKeys;   // visible columns c <= hi (hi >= 0 always)
                // pass 1: max of this tile's visible scores
                float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                {
                    uint32_t va[32], vb[32];
                    tmem_ld32(ts, va);
#pragma unroll 1
                    for (int c = 0; c < 4; c += 2) {
                        tmem_wait_ld();
                        tmem_ld32(ts + (c + 1) * 32, vb);
                        tile_chunk_max(va, c * 32, hi, mx4);
                        tmem_wait_ld();
                        if (c + 2 < 4) tmem_ld32(ts + (c + 2) * 32, va);
                        tile_chunk_max(vb, (c + 1) * 32, hi, mx4);
                    }
                }
                const float mt = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
                // lazy running max: raise the reference only past 2^8
                float alpha = 1.f;
                const bool raise = (m_ref == -INFINITY) || ((mt - m_ref) * p.sl2 > kRescaleLog2);
                if (raise) {
                    if (m_ref != -INFINITY) alpha = ex2((m_ref - mt) * p.sl2);
                    m_ref = mt;
                    l *= alpha;
                }
                if (j > 0 && __any_sync(0xffffffffu, raise && alpha != 1.f)) {
                    // O holds the tiles before this one: wait for their PV, rescale in TMEM
                    ok = warp_wait(bar(BS_FREE + ((g - 1) & 1)), ((g - 1) >> 1) & 1, ab);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t o[32];
                        tmem_ld32(tmem + lane_base + 256 + c * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        uint32_t lo16[16], hi16[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            lo16[e] = o[e];
                            hi16[e] = o[16 + e];
                        }
                        tmem_st16(tmem + lane_base + 256 + c * 32, lo16);
                        tmem_st16(tmem + lane_base + 256 + c * 32 + 16, hi16);
                    }
                    tmem_wait_st();
                }
                const float mxs = m_ref * p.sl2;
                // pass 2: P over S's first 64 columns (P of chunk c lands on S chunk c/2)
                float sum4[4] = {0.f, 0.f, 0.f, 0.f};
                {
                    uint32_t va[32], vb[32], pk[16];
                    tmem_ld32(ts, va);
#pragma unroll 1
                    for (int c = 0; c < 4; c += 2) {
                        tmem_wait_ld();
                        tmem_ld32(ts + (c + 1) * 32, vb);
                        tile_chunk_exp(va, c * 32, hi, p.sl2, mxs, sum4, pk);
                        tmem_st16(ts + c * 16, pk);
                        tmem_wait_ld();
                        if (c + 2 < 4) tmem_ld32(ts + (c + 2) * 32, va);
                        tile_chunk_exp(vb, (c + 1) * 32, hi, p.sl2, mxs, sum4, pk);
                        tmem_st16(ts + (c + 1) * 16, pk);
                    }
                }
                l += (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(BP_READY + bb));
            }
            if (!ok) break;
            // ---- epilogue of the unit: y = O / l, lse
            ok = warp_wait(bar(BO_FULL), k & 1, ab);
            if (!ok) break;
            tc_fence_after();
            const float inv = 1.0f / l;
            const uint32_t ya = sbase + kOffY;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_base + 256 + c * 32, o);
                tmem_wait_ld();
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint32_t yu[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        yu[e] = pack_bf16(__uint_as_float(o[c4 * 8 + 2 * e]) * inv,
                                          __uint_as_float(o[c4 * 8 + 2 * e + 1]) * inv);
                    sts128(ya + swa::chunk_off(r, c * 4 + c4, kHalf), make_uint4(yu[0], yu[1], yu[2], yu[3]));
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(BO_FREE));
                mbar_arrive(bar(BY_READY));
            }
            if (p.lse != nullptr && i < p.T)
                p.lse[((long long)x.b * p.Hq + x.kvh * 4 + (r & 3)) * p.T + i] = (m_ref * p.sl2 + __log2f(l)) * ln2;
            if (r == 0 && mbar_wait(bar(BY_READY), k & 1, ab)) {
                for (int h = 0; h < 2; ++h)
                    tma_store_4d(&tm_y, ya + h * kHalf, h * 64, x.kvh * 4, x.qb * kTok, x.b);
                bulk_commit_group();
                bulk_wait_group_read<0>();
            }
        }
        if (r == 0) bulk_wait_group<0>();
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
