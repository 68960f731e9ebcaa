// bwd_full.cuh -- fused backward of full causal attention (the global layers),
// for sm_100a.
//
// ZGCM-1 §2.1: the global layers attend over the whole causal context with
// the same QK RMSNorm and partial RoPE as the sliding-window layers and no
// gate.  With q~, k~ the prepared queries and keys, P the forward's softmax
// (recomputed from its lse), dA = dy and D_i = sum_d dy_i y_i:
//   dV_j = sum_i P_ij dA_i,  dS_ij = P_ij (<dA_i, v_j> - D_i),
//   dk~_j = scale sum_i dS_ij q~_i,  dq~_i = scale sum_j dS_ij k~_j,
// then dq, dk through RoPE^T and the RMSNorm backward.
//
// One key-stationary kernel does all four contractions (plus the one
// recomputation of the scores): a unit is 128 keys of one (sequence, KV
// head), M = 128 TMEM lanes; its queries stream past in chunks of 64 rows (16
// tokens x the 4 heads of the GQA group, row = 4 token + head).  Per chunk:
//   S^T  = K~ Q~_c^T   (N = 64)      -> TMEM S buffer (two, alternating)
//   dP^T = V dA_c^T    (N = 64)      -> TMEM dP
//   softmax warps: P^T = 2^(S^T sl2 - lse log2 e) (bf16, over S^T in TMEM),
//                  dS^T = P^T (dP^T - D) (bf16, shared memory)
//   dV  += P^T dA_c    (TMEM A operand, N = 128 dims)
//   dK~ += dS^T Q~_c   (N = 128 dims)
//   dQ~_c^T = K~^T dS^T (M = 128 dims, N = 64 rows: both operands read
//                  transposed from the tiles already in shared memory)
// and dQ~_c^T leaves TMEM into registers and is added, one coalesced
// red.global.add per chunk row and warp, into an f32 accumulator [B, T, Hq, D]
// (bwd_dq_post then applies scale, RoPE^T and the RMSNorm backward).  TMEM: S buffers at 0 and
// 64, dP at 128, dQ at 192, dV at 256, dK at 384 -- all 512 columns, which
// lets the next chunk's S^T and dP^T run on the tensor pipe while the softmax
// warps work on this one.
//
// dk, dv and dw_k are bitwise reproducible (fixed-order sums); the f32
// accumulation of dq~ is not (the atomic adds of different key tiles land in
// any order), and with it dq and dw_q may differ in their last bits from run
// to run.
//
// Warp roles (16 warps): 0 TMA producer (K~/V once per unit; Q~, dA and the
// row records per chunk, four stages), 1 TMEM owner and issuer of the score
// products (S^T, dP^T), 2 issuer of the accumulating products (dV, dK~,
// dQ~^T), 3 idle, 4-11 softmax (two per TMEM lane quarter, 32 of the chunk's
// 64 rows each), 12-15 dQ~ adds and the unit epilogue (dv; dk through RoPE^T
// and the RMSNorm backward; dw_k partials).  Two issuing threads keep the
// tensor pipe fed while either one waits on a barrier or commits: each
// thread's commits track only the products that thread issued, and every
// hand-off between the two goes through a barrier (below).
#pragma once

#include <cuda.h>

#include "bwd.cuh"
#include "ptx.cuh"
#include "swa_fwd.cuh"

namespace gswa {
namespace bwdf {

using bwd::kD;
using bwd::kHalfRowBytes;

constexpr int kThreads = 512;
constexpr int kKeys = 128;                  // keys per unit (MMA M)
constexpr int kChTok = 16;                  // tokens per query chunk
constexpr int kChRows = 4 * kChTok;         // 64 query rows per chunk (MMA N of the score products)
constexpr int kStages = 4;
constexpr int kMaxGrid = 256;               // CTAs (dw_k partials sizing)

constexpr uint32_t kKHalf = kKeys * kHalfRowBytes;        // 16 KiB: 128 keys x 64 dims
constexpr uint32_t kKTile = 2 * kKHalf;                   // 32 KiB
constexpr uint32_t kCHalf = kChRows * kHalfRowBytes;      // 8 KiB: 64 rows x 64 dims
constexpr uint32_t kCTile = 2 * kCHalf;                   // 16 KiB
constexpr uint32_t kStageBytes = 2 * kCTile;              // Q~ and dA of one chunk
constexpr uint32_t kRecBytes = kChRows * 8;               // {lse log2 e, D} per row
constexpr uint32_t kDSTile = kKeys * kHalfRowBytes;       // dS^T: 128 keys x 64 rows bf16
constexpr uint32_t kOffK = 0;
constexpr uint32_t kOffV = kOffK + kKTile;
constexpr uint32_t kOffSt = kOffV + kKTile;
constexpr uint32_t kOffDS = kOffSt + kStages * kStageBytes;
constexpr uint32_t kOffRec = kOffDS + kDSTile;            // records of each stage
constexpr uint32_t kOffW = kOffRec + kStages * kRecBytes; // f32[128] w_k
constexpr uint32_t kOffBar = kOffW + 512;
constexpr int kNumBars = 26;
constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
// No alignment slack: the kernel checks that the dynamic shared memory starts
// on a 1 KiB boundary (it does, as the only allocation of a one-CTA-per-SM
// kernel) and reports GSWA_ERR_LAUNCH through the status word otherwise.
constexpr uint32_t kSmemBytes = kOffAbort + 4;
static_assert(kSmemBytes <= 232448, "shared memory budget of one sm_100 CTA");
static_assert((kOffSt % 1024) == 0 && (kStageBytes % 1024) == 0 && (kOffDS % 1024) == 0,
              "swizzled tiles are 1 KiB aligned");

// TMEM columns
constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 192, kColDV = 256, kColDK = 384;

// Every barrier below completes at most one phase ahead of each of its
// waiters, which is what the parity waits need: a barrier's next phase always
// depends, through the chain of hand-offs, on each waiter having passed its
// wait for the current one.  The accumulation issuer waits on two barriers
// per chunk: P_READY, and DS_READY, which counts the softmax warps' dS^T
// writes and the readout warps' release of the previous chunk's dQ~^T
// columns (the readout warps arrive once up front for chunk 0).  It commits
// once per chunk, DQ_FULL after dK~ and dQ~^T, which covers everything that
// thread issued for the chunk: the readout warps learn that dQ~^T is in TMEM,
// the softmax warps that dS^T may be overwritten, the first readout warp
// passes the chunk's stage back to the producer, and the score issuer learns
// that dV has read P^T out of the S buffer that chunk g + 2's scores
// overwrite (the one hand-off between the two issuers).  P_READY and DQ_FULL
// come in pairs, one per chunk parity (= S buffer): the score issuer waits
// for chunk g - 2's DQ_FULL before chunk g's scores, and while it waits the
// accumulation issuer may already finish chunk g - 1 -- on the other barrier
// of the pair; the next phase of chunk g - 2's barrier is chunk g itself,
// which needs those scores first.  Likewise the softmax warps can finish
// chunk g + 1 before the accumulation issuer has looked at chunk g's
// P_READY.  The stage and K~/V releases follow the accumulation issuer's
// products alone, which start only after the softmax has seen that chunk's
// S^T and dP^T complete.
enum : int {
    BKV_FULL = 0, BKV_EMPTY = 1, BST_FULL = 2, BST_EMPTY = BST_FULL + kStages, BS_FULL = BST_EMPTY + kStages,
    BDP_FREE = BS_FULL + 1, BP_READY = BDP_FREE + 1 /* 2 */, BDS_READY = BP_READY + 2,
    BDQ_FULL = BDS_READY + 1 /* 2 */, BACC_FULL = BDQ_FULL + 2,
    BACC_FREE = BACC_FULL + 1, B_DRAIN = BACC_FREE + 1 /* 2: one per issuer */
};
static_assert(B_DRAIN + 1 < kNumBars, "barrier count");

struct Params {
    int B, T, Tp, Hq, Hkv;
    int nkt;                         // key tiles of 128
    long long units;                 // B * Hkv * nkt
    float eps, sl2, scale;           // sl2 = scale log2 e
    const float2 *ld;                // row records [B, Hkv, Tp, 4]
    const __nv_bfloat16 *k;          // raw k (RMSNorm backward)
    const __nv_bfloat16 *wk;
    __nv_bfloat16 *dk, *dv;
    float *dq_acc;                   // [B, T, Hq, D] f32 dq~ sums (zeroed by the caller)
    float *dw_part;                  // [gridDim.x * 4][128] dw_k partials
    double theta[64];
};

struct Unit {
    int b, kvh, kt, n;   // n: query chunks of 16 tokens from token 128 kt to T
};

// k-th unit of this CTA, longest first (key tile 0 has the most queries), in
// a snake order over the CTAs that balances the causal triangle.
__device__ __forceinline__ bool unit_at(const Params &p, int k, Unit &x)
{
    const long long u = bwd::snake_unit(k);
    if (u >= p.units) return false;
    const long long per = (long long)p.B * p.Hkv;
    x.kt = (int)(u / per);
    const long long strip = u % per;
    x.b = (int)(strip / p.Hkv);
    x.kvh = (int)(strip % p.Hkv);
    x.n = (p.T - kKeys * x.kt + kChTok - 1) / kChTok;
    return true;
}

// Walks the (unit, chunk) pairs of this CTA in order; g counts chunks over units.
struct Walk {
    int k = 0, j = 0, g = 0;
    Unit x;
    bool valid = false;
    __device__ __forceinline__ void init(const Params &p) { k = j = g = 0; valid = unit_at(p, 0, x); }
    __device__ __forceinline__ bool last() const { return j == x.n - 1; }
    __device__ __forceinline__ void next(const Params &p)
    {
        ++g;
        if (++j == x.n) {
            j = 0;
            ++k;
            valid = unit_at(p, k, x);
        }
    }
    __device__ __forceinline__ int t0() const { return kKeys * x.kt + kChTok * j; }
};

template <int R>
__global__ void __launch_bounds__(kThreads, 1)
bwd_full_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_a,
                const __grid_constant__ Params p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw;
    const uint32_t sbase = smem_u32(smem);
    if ((sbase & 1023u) != 0) {   // the swizzled tiles need 1 KiB alignment (uniform over the CTA)
        if (threadIdx.x == 0) atomicExch(&g_status, kStatusSetup);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffTmemSlot);
    Abort ab{reinterpret_cast<volatile int *>(smem + kOffAbort)};
    auto bar = [&](int i) -> uint32_t { return sbase + kOffBar + 8u * (uint32_t)i; };
    auto stage = [&](int st) -> uint32_t { return sbase + kOffSt + (uint32_t)st * kStageBytes; };
    auto recs = [&](int st) -> uint32_t { return sbase + kOffRec + (uint32_t)st * kRecBytes; };

    if (tid == 0) {
        *ab.flag = 0;
        mbar_init(bar(BKV_FULL), 1);
        mbar_init(bar(BKV_EMPTY), 1);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(bar(BST_FULL + i), 1);
            mbar_init(bar(BST_EMPTY + i), 1);
        }
        mbar_init(bar(BS_FULL), 1);
        mbar_init(bar(BDP_FREE), 8);
        mbar_init(bar(BP_READY), 8);
        mbar_init(bar(BP_READY + 1), 8);
        mbar_init(bar(BDS_READY), 8 + 4);
        mbar_init(bar(BDQ_FULL), 1);
        mbar_init(bar(BDQ_FULL + 1), 1);
        mbar_init(bar(BACC_FULL), 1);
        mbar_init(bar(BACC_FREE), 4);
        mbar_init(bar(B_DRAIN), 1);
        mbar_init(bar(B_DRAIN + 1), 1);
        fence_barrier_init();
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_a);
    }
    if (tid < 128) reinterpret_cast<float *>(smem + kOffW)[tid] = __bfloat162float(p.wk[tid]);
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
            Walk w;
            w.init(p);
            bool ok = true;
            int nkv = 0;
            for (; w.valid && ok; w.next(p)) {
                if (w.j == 0) {
                    ok = mbar_wait(bar(BKV_EMPTY), (w.k & 1) ^ 1u, ab);
                    if (!ok) break;
                    mbar_arrive_expect_tx(bar(BKV_FULL), 2 * kKTile);
                    for (int h = 0; h < 2; ++h) {
                        tma_load_4d(sbase + kOffK + h * kKHalf, &tm_k, bar(BKV_FULL), h * 64, w.x.kvh, kKeys * w.x.kt,
                                    w.x.b);
                        tma_load_4d(sbase + kOffV + h * kKHalf, &tm_v, bar(BKV_FULL), h * 64, w.x.kvh, kKeys * w.x.kt,
                                    w.x.b);
                    }
                    ++nkv;
                }
                const int st = w.g % kStages;
                ok = mbar_wait(bar(BST_EMPTY + st), ((w.g / kStages) & 1) ^ 1u, ab);
                if (!ok) break;
                const int t0 = w.t0();
                mbar_arrive_expect_tx(bar(BST_FULL + st), 2 * kCTile + kRecBytes);
                for (int h = 0; h < 2; ++h) {
                    tma_load_4d(stage(st) + h * kCHalf, &tm_q, bar(BST_FULL + st), h * 64, w.x.kvh * 4, t0, w.x.b);
                    tma_load_4d(stage(st) + kCTile + h * kCHalf, &tm_a, bar(BST_FULL + st), h * 64, w.x.kvh * 4, t0,
                                w.x.b);
                }
                bulk_load(recs(st), p.ld + (((long long)w.x.b * p.Hkv + w.x.kvh) * p.Tp + t0) * 4,
                          kRecBytes, bar(BST_FULL + st));
            }
            // every copy this thread issued lands before shared memory is released
            for (int i = (w.g > kStages ? w.g - kStages : 0); i < w.g; ++i)
                bwd::drain_wait(bar(BST_FULL + i % kStages), (i / kStages) & 1);
            if (nkv > 0) bwd::drain_wait(bar(BKV_FULL), (nkv - 1) & 1);
        }
    } else if (warp == 1 || warp == 2) {
        // ================================================= MMA issuers
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16_f32(128, kChRows, 0, 0);     // S^T, dP^T: both K-major
            const uint32_t id_acc = idesc_bf16_f32(128, 128, 0, 1);        // dV, dK: B (rows x dims) transposed
            const uint32_t id_dq = idesc_bf16_f32(128, kChRows, 1, 1);    // dQ^T: both operands transposed
            // shared-memory descriptors, built once: K-major (K~, V, dS^T, Q~ and dA of
            // stage 0 as A/B of the score products and dK) and MN-major (K~ as the A of
            // dQ^T; Q~, dA and dS^T as transposed B operands); the stages differ by a
            // constant byte offset
            const SmemDesc dC_k = make_desc(stage(0), 16, 1024), dC_mn = make_desc(stage(0), kCHalf, 1024);
            Walk w;
            w.init(p);
            bool ok = true;
            if (warp == 1) {
                // ---- S^T and dP^T of every chunk
                const SmemDesc dK_k = make_desc(sbase + kOffK, 16, 1024), dV_k = make_desc(sbase + kOffV, 16, 1024);
                for (; w.valid && ok; w.next(p)) {
                    const int g = w.g, st = g % kStages;
                    if (w.j == 0 && !(ok = mbar_wait(bar(BKV_FULL), w.k & 1, ab))) break;
                    if (!(ok = mbar_wait(bar(BST_FULL + st), (g / kStages) & 1, ab))) break;
                    // the S buffer's previous P^T (chunk g - 2) has been read by its dV: chunk
                    // g - 2's DQ_FULL commit follows that dV on the same issuing thread
                    if (g >= 2 && !(ok = mbar_wait(bar(BDQ_FULL + (g & 1)), ((g >> 1) - 1) & 1, ab))) break;
                    tc_fence_after();
                    const uint32_t qo = (uint32_t)st * kStageBytes, ao = qo + kCTile;   // stage offsets
                    const uint32_t ds = tmem + kColS + (g & 1) * 64;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(ds, dK_k.at((kk >> 2) * kKHalf + (kk & 3) * 32),
                               dC_k.at(qo + (kk >> 2) * kCHalf + (kk & 3) * 32), id_s, kk > 0);
                    // dP: the softmax warps have loaded the previous chunk's dP^T
                    if (!(ok = mbar_wait(bar(BDP_FREE), (g & 1) ^ 1u, ab))) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(tmem + kColDP, dV_k.at((kk >> 2) * kKHalf + (kk & 3) * 32),
                               dC_k.at(ao + (kk >> 2) * kCHalf + (kk & 3) * 32), id_s, kk > 0);
                    mma_commit(bar(BS_FULL));
                }
            } else {
                // ---- dV, dK~ and dQ~^T of every chunk
                const SmemDesc dK_mn = make_desc(sbase + kOffK, kKHalf, 1024);
                const SmemDesc dS_k = make_desc(sbase + kOffDS, 16, 1024),
                               dS_mn = make_desc(sbase + kOffDS, kDSTile, 1024);
                for (; w.valid && ok; w.next(p)) {
                    const int g = w.g;
                    const uint32_t qo = (uint32_t)(g % kStages) * kStageBytes, ao = qo + kCTile;
                    if (!(ok = mbar_wait(bar(BP_READY + (g & 1)), (g >> 1) & 1, ab))) break;
                    // the first chunk of a unit overwrites dV/dK: the previous unit's epilogue has read them
                    if (w.j == 0 && !(ok = mbar_wait(bar(BACC_FREE), (w.k & 1) ^ 1u, ab))) break;
                    tc_fence_after();
                    const uint32_t pt = tmem + kColS + (g & 1) * 64;
                    const uint32_t acc0 = w.j > 0;
#pragma unroll
                    for (int kk = 0; kk < kChRows / 16; ++kk)
                        mma_ts(tmem + kColDV, pt + (kk >> 1) * 32 + (kk & 1) * 8,
                               dC_mn.at(ao + kk * 16 * kHalfRowBytes), id_acc, acc0 | (kk > 0));
                    // dS^T written, and the previous chunk's dQ~^T read out of TMEM
                    if (!(ok = mbar_wait(bar(BDS_READY), g & 1, ab))) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kChRows / 16; ++kk)
                        mma_ss(tmem + kColDK, dS_k.at(kk * 32), dC_mn.at(qo + kk * 16 * kHalfRowBytes), id_acc,
                               acc0 | (kk > 0));
#pragma unroll
                    for (int kk = 0; kk < kKeys / 16; ++kk)
                        mma_ss(tmem + kColDQ, dK_mn.at(kk * 16 * kHalfRowBytes), dS_mn.at(kk * 16 * kHalfRowBytes),
                               id_dq, kk > 0);
                    mma_commit(bar(BDQ_FULL + (g & 1)));
                    if (w.last()) {
                        mma_commit(bar(BACC_FULL));
                        mma_commit(bar(BKV_EMPTY));
                    }
                }
            }
            // this thread's products have completed before TMEM and shared memory go away
            mma_commit(bar(B_DRAIN + (warp - 1)));
            bwd::drain_wait(bar(B_DRAIN + (warp - 1)), 0);
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 12) {
        // ================================================= P^T and dS^T (8 warps)
        const int grp = (warp - 4) >> 2;           // chunk rows 32 grp .. 32 grp + 31
        const int q4 = warp & 3;                   // TMEM lane quarter
        const int r = 32 * q4 + lane;              // key of the unit
        const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
        Walk w;
        w.init(p);
        bool ok = true;
        for (; w.valid && ok; w.next(p)) {
            const int g = w.g, st = g % kStages;
            const int jkey = kKeys * w.x.kt + r;
            ok = warp_wait(bar(BS_FULL), g & 1, ab);
            // the stage's records: its load completed before the MMA read the stage
            if (ok) ok = warp_wait(bar(BST_FULL + st), (g / kStages) & 1, ab);
            if (!ok) break;
            tc_fence_after();
            uint32_t s[32], d[32];
            const uint32_t ts = tmem + lane_base + kColS + (g & 1) * 64 + 32 * grp;
            tmem_ld32(ts, s);
            tmem_ld32(tmem + lane_base + kColDP + 32 * grp, d);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BDP_FREE));   // dP^T is in registers
            const int t0 = w.t0();
            const uint32_t rec = recs(st) + 32 * grp * 8;
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
                const bool vis = t0 + ((32 * grp + e) >> 2) >= jkey;
                float pp[4], ds[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    pp[u] = vis ? ex2(fmaf(__uint_as_float(s[e + u]), p.sl2, -l2[u])) : 0.f;
                    ds[u] = pp[u] * (__uint_as_float(d[e + u]) - dv[u]);
                }
                pk[e >> 1] = pack_bf16(pp[0], pp[1]);
                pk[(e >> 1) + 1] = pack_bf16(pp[2], pp[3]);
                dk[e >> 1] = pack_bf16(ds[0], ds[1]);
                dk[(e >> 1) + 1] = pack_bf16(ds[2], ds[3]);
            }
            // P^T over this warp's own S^T columns (the first 16 of its 32)
            tmem_st16(ts, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BP_READY + (g & 1)));
            // dS^T once the previous chunk's dK and dQ^T have read the tile
            if (g > 0) ok = warp_wait(bar(BDQ_FULL + ((g - 1) & 1)), ((g - 1) >> 1) & 1, ab);
            if (!ok) break;
            bwd::sts_row_chunks(sbase + kOffDS, r, 4 * grp, dk);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BDS_READY));
        }
    } else if (warp >= 12) {
        // ================================================= dQ~ adds, unit epilogue (4 warps)
        const int q4 = warp & 3;
        const int r = 32 * q4 + lane;              // dQ^T: dim r; dV/dK: key r
        const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
        const long long tstride = (long long)p.Hq * kD;   // accumulator floats per token
        const float *w = reinterpret_cast<const float *>(smem + kOffW);
        float dwacc[4] = {0.f, 0.f, 0.f, 0.f};
        Walk wk;
        wk.init(p);
        bool ok = true;
        if (lane == 0) mbar_arrive(bar(BDS_READY));   // chunk 0 has no previous dQ~^T to read out
        for (; wk.valid && ok; wk.next(p)) {
            const int g = wk.g;
            ok = warp_wait(bar(BDQ_FULL + (g & 1)), (g >> 1) & 1, ab);
            if (!ok) break;
            // the chunk's products have completed: its Q~/dA stage (and records) are free
            if (q4 == 0 && lane == 0) mbar_arrive(bar(BST_EMPTY + g % kStages));
            tc_fence_after();
            uint32_t a[32], b2[32];
            tmem_ld32(tmem + lane_base + kColDQ, a);        // rows 0..31 of the chunk, dim r
            tmem_ld32(tmem + lane_base + kColDQ + 32, b2);  // rows 32..63
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BDS_READY));   // dQ~^T columns free for the next chunk
            // dq~ += dQ~_c: chunk row c is token t0 + c / 4, head 4 kvh + c % 4; lane =
            // dim, so each warp-wide add covers 128 contiguous bytes of one row.  Rows of
            // tokens past T (the last chunk of a sequence) are skipped.
            {
                const int t0 = wk.t0();
                const int nt = min(kChTok, p.T - t0);
                float *dst = p.dq_acc + (((long long)wk.x.b * p.T + t0) * p.Hq + 4 * wk.x.kvh) * kD + r;
#pragma unroll
                for (int c = 0; c < kChRows; ++c)
                    if ((c >> 2) < nt)
                        red_add_f32(dst + (c >> 2) * tstride + (c & 3) * kD,
                                    __uint_as_float(c < 32 ? a[c] : b2[c - 32]));
            }
            if (!wk.last()) continue;
            // ---- epilogue of the unit: dv, and dk through RoPE^T and the RMSNorm backward
            ok = warp_wait(bar(BACC_FULL), wk.k & 1, ab);
            if (!ok) break;
            tc_fence_after();
            const int jkey = kKeys * wk.x.kt + r;
            const bool valid = jkey < p.T;
            const long long off = valid ? (((long long)wk.x.b * p.T + jkey) * p.Hkv + wk.x.kvh) * kD : 0;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_base + kColDV + 32 * c, v);
                tmem_wait_ld();
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const uint4 o = make_uint4(
                        pack_bf16(__uint_as_float(v[8 * qq + 0]), __uint_as_float(v[8 * qq + 1])),
                        pack_bf16(__uint_as_float(v[8 * qq + 2]), __uint_as_float(v[8 * qq + 3])),
                        pack_bf16(__uint_as_float(v[8 * qq + 4]), __uint_as_float(v[8 * qq + 5])),
                        pack_bf16(__uint_as_float(v[8 * qq + 6]), __uint_as_float(v[8 * qq + 7])));
                    if (valid) reinterpret_cast<uint4 *>(p.dv + off)[4 * c + qq] = o;
                }
            }
            bwd::norm_rope_backward<R>(tmem + lane_base + kColDK, p.scale, p.k + off, valid, w, p.eps, jkey, p.theta,
                                       p.dk + off, dwacc);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BACC_FREE));
        }
        float *dst = p.dw_part + ((long long)blockIdx.x * 4 + q4) * kD;
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

// ------------------------------------------------------------------ dq post
// dq = RMSNorm backward of RoPE^T(scale dq~), dq~ the f32 sums of the fused
// kernel, against the raw q.  A warp takes the 4 rows of one (token, KV
// head) at a time -- four independent row loads in flight, one set of rotary
// cos/sin for the four heads -- lane = dims 4 lane .. + 3; the warps walk the
// groups in a fixed order, so the dw_q partials (one per warp) are summed in a
// fixed order by dw_reduce.
struct PostParams {
    const float *acc;                // [B, T, Hq, D]
    const __nv_bfloat16 *q, *wq;
    __nv_bfloat16 *dq;
    float *dw_part;                  // [gridDim.x * 8][128]
    long long rows;                  // B * T * Hq
    int T, Hq;
    float eps, scale;
    double theta[64];
};

constexpr int kPostWarps = 8;
constexpr int kPostMaxGrid = 512;
constexpr int kPostRows = 4;         // rows per warp step: the 4 heads of a GQA group

template <int R>
__global__ void __launch_bounds__(kPostWarps * 32) bwd_dq_post_kernel(const __grid_constant__ PostParams p)
{
    constexpr int H = R / 2;
    __shared__ __align__(16) float ubuf[kPostWarps][kPostRows][kD];
    const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
    const long long gw = (long long)blockIdx.x * kPostWarps + wl, nw = (long long)gridDim.x * kPostWarps;
    const int d0 = 4 * lane;
    const uint2 wr = *reinterpret_cast<const uint2 *>(p.wq + d0);
    const float2 wa = unpack_bf16(wr.x), wb = unpack_bf16(wr.y);
    const float wv[4] = {wa.x, wa.y, wb.x, wb.y};
    float dwacc[4] = {0.f, 0.f, 0.f, 0.f};
    const long long groups = p.rows / kPostRows;
    for (long long grp = gw; grp < groups; grp += nw) {
        const long long row0 = grp * kPostRows;
        const int t = (int)((row0 / p.Hq) % p.T);
        float4 a4[kPostRows];
        uint2 xr[kPostRows];
#pragma unroll
        for (int u = 0; u < kPostRows; ++u) {
            a4[u] = *reinterpret_cast<const float4 *>(p.acc + (row0 + u) * kD + d0);
            xr[u] = *reinterpret_cast<const uint2 *>(p.q + (row0 + u) * kD + d0);
        }
        // rotary cos/sin of this lane's dims at position t (shared by the 4 heads)
        float cs[4] = {1.f, 1.f, 1.f, 1.f}, sn[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (R > 0) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int d = d0 + e;
                if (d < R) swa::rope_cs(p.theta[d < H ? d : d - H], t, cs[e], sn[e]);
            }
        }
        float du[kPostRows][4];
#pragma unroll
        for (int u = 0; u < kPostRows; ++u) {
            du[u][0] = a4[u].x * p.scale;
            du[u][1] = a4[u].y * p.scale;
            du[u][2] = a4[u].z * p.scale;
            du[u][3] = a4[u].w * p.scale;
        }
        if constexpr (R > 0) {
            // RoPE^T: (g_p, g_{p+H}) <- (g_p c + g_{p+H} s, g_{p+H} c - g_p s)
#pragma unroll
            for (int u = 0; u < kPostRows; ++u)
#pragma unroll
                for (int e = 0; e < 4; ++e) ubuf[wl][u][d0 + e] = du[u][e];
            __syncwarp();
#pragma unroll
            for (int u = 0; u < kPostRows; ++u)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int d = d0 + e;
                    if (d < R)
                        du[u][e] = d < H ? ubuf[wl][u][d] * cs[e] + ubuf[wl][u][d + H] * sn[e]
                                         : ubuf[wl][u][d] * cs[e] - ubuf[wl][u][d - H] * sn[e];
                }
            __syncwarp();
        }
        float x[kPostRows][4], ss[kPostRows], wgx[kPostRows];
#pragma unroll
        for (int u = 0; u < kPostRows; ++u) {
            const float2 xa = unpack_bf16(xr[u].x), xb = unpack_bf16(xr[u].y);
            x[u][0] = xa.x;
            x[u][1] = xa.y;
            x[u][2] = xb.x;
            x[u][3] = xb.y;
            ss[u] = 0.f;
            wgx[u] = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                ss[u] = fmaf(x[u][e], x[u][e], ss[u]);
                wgx[u] = fmaf(wv[e] * du[u][e], x[u][e], wgx[u]);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int u = 0; u < kPostRows; ++u) {
                ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], o);
                wgx[u] += __shfl_xor_sync(0xffffffffu, wgx[u], o);
            }
#pragma unroll
        for (int u = 0; u < kPostRows; ++u) {
            const float r = rsqrtf(ss[u] * (1.0f / kD) + p.eps);
            const float m = r * wgx[u] * (1.0f / kD);   // mean(w du n)
            float o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float n = x[u][e] * r;
                o[e] = r * fmaf(wv[e], du[u][e], -n * m);
                dwacc[e] = fmaf(du[u][e], n, dwacc[e]);
            }
            *reinterpret_cast<uint2 *>(p.dq + (row0 + u) * kD + d0) =
                make_uint2(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]));
        }
    }
    *reinterpret_cast<float4 *>(p.dw_part + gw * kD + d0) = make_float4(dwacc[0], dwacc[1], dwacc[2], dwacc[3]);
}

}  // namespace bwdf
}  // namespace gswa
