// decode.cuh -- one decode step of the ZGCM-1 attention core (§2.3: the SWA
// layers keep a fixed 128-token window in the KV cache, the global layers
// the whole sequence; autoregressive decoding is bound by memory bandwidth).
//
// Both paths prepare the new token's q and k (RMSNorm + partial RoPE at its
// position), write the prepared k and the raw v into the cache, then attend.
//
//   gswa_decode: ring cache [B, Hkv, W, D]; position t lives in slot t mod W.
//     One CTA per (sequence, KV head), one warp per query head of the group.
//   full_decode: linear cache [B, Hkv, Tmax, D], split over the cache length:
//     a prologue prepares q~ (f32, into the workspace) and appends k~, v; a
//     chunk kernel computes, per 4096-key chunk, the partial (max, sum, O) of
//     the 4 query heads from K/V rows streamed by TMA through a shared-memory
//     ring (lanes = keys for q.k with q~ broadcast from shared memory, lanes =
//     dims for P V); a combine kernel merges the chunks by their log-sum-exp
//     weights.
#pragma once

#include <cuda.h>

#include "ptx.cuh"
#include "swa_fwd.cuh"

namespace gswa {
namespace dec {

constexpr int kD = 128;
constexpr int kChunk = 4096;          // keys per chunk of the full-cache split
constexpr int kChunkWarps = 12;
constexpr int kPartial = 4 + kD;      // m, l, (2 pad), o[128] per (chunk, head): o 16-byte aligned

struct Params {
    int B, Hq, Hkv, R;
    int W;               // ring slots (sliding-window decode)
    long long Tmax;      // linear cache length (full decode)
    int nchunks;         // ceil(Tmax / kChunk)
    float eps, sl2;      // softmax scale * log2(e)
    const __nv_bfloat16 *q, *k, *v, *g, *wq, *wk;
    __nv_bfloat16 *kc, *vc;   // caches (written at the new position)
    const int64_t *pos;
    __nv_bfloat16 *y;
    float *qt;           // full decode: prepared queries [B, Hq, D] f32
    float *part;         // full decode: partials [B, Hkv, nchunks, 4, kPartial]
    double theta[64];
};

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ float warp_max(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

// RMSNorm then partial RoPE of one head row by one warp; lane l returns dims
// 4l .. 4l+3 (f32).  `ubuf` is 128 floats of shared memory for the rotation.
__device__ __forceinline__ float4 prep_head_warp(const __nv_bfloat16 *x, const __nv_bfloat16 *w, int R,
                                                 float eps, long long pos, const double *theta,
                                                 float *ubuf)
{
    const int lane = threadIdx.x & 31;
    const uint2 raw = *reinterpret_cast<const uint2 *>(x + 4 * lane);
    const uint2 wr = *reinterpret_cast<const uint2 *>(w + 4 * lane);
    const float2 a = unpack_bf16(raw.x), b = unpack_bf16(raw.y);
    const float2 wa = unpack_bf16(wr.x), wb = unpack_bf16(wr.y);
    const float ss = warp_sum(a.x * a.x + a.y * a.y + b.x * b.x + b.y * b.y);
    const float r = rsqrtf(ss * (1.0f / kD) + eps);
    float u[4] = {a.x * r * wa.x, a.y * r * wa.y, b.x * r * wb.x, b.y * r * wb.y};
    const int H = R / 2;
    if (R > 0) {
#pragma unroll
        for (int e = 0; e < 4; ++e) ubuf[4 * lane + e] = u[e];
        __syncwarp();
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int d = 4 * lane + e;
            if (d < R) {
                const int pp = d < H ? d : d - H;
                float c, s;
                swa::rope_cs(theta[pp], (int)pos, c, s);
                u[e] = d < H ? ubuf[d] * c - ubuf[d + H] * s : ubuf[d] * c + ubuf[d - H] * s;
            }
        }
        __syncwarp();
    }
    return make_float4(u[0], u[1], u[2], u[3]);
}

// ----------------------------------------------------------------- sliding window
// One CTA per (sequence, KV head), one warp per query head.  The whole ring
// (K and V, W rows each) is loaded by TMA into shared memory (128-byte
// swizzle: a lane per slot reads its K row without bank conflicts) while the
// new token's q, k and v are prepared; the new token's row is then written
// over its slot in shared memory (and in the ring), and the attention reads
// shared memory only.
constexpr uint32_t kRingHalfMax = 128 * 128;   // 128 slots x 64 dims bf16: 16 KiB

__device__ __forceinline__ uint32_t ring_half_bytes(int W)
{
    return (uint32_t)((W * 128 + 1023) / 1024 * 1024);   // halves stay 1024-byte aligned
}

constexpr uint32_t kSwaDecSmemBytes = 4 * kRingHalfMax + 16 + 1024;

__global__ void __launch_bounds__(128)
swa_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    __shared__ __align__(16) float qt[4][kD];
    __shared__ __align__(16) float ubuf[4][kD];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x / p.Hkv, kvh = blockIdx.x % p.Hkv;
    const int head = kvh * 4 + warp;
    const long long pos = p.pos[b];
    if (pos < 0) {
        if (threadIdx.x == 0) atomicExch(&g_status, kStatusBadArg);
        return;
    }
    const int W = p.W;
    const uint32_t hs = ring_half_bytes(W);
    const uint32_t ks = sbase, vs = sbase + 2 * hs;
    const uint32_t bar = sbase + 4 * hs;
    Abort ab{reinterpret_cast<volatile int *>(smem + 4 * hs + 8)};
    const int slot_new = (int)(pos % W);
    const long long cbase = ((long long)b * p.Hkv + kvh) * W;   // first row of this (b, kvh) ring
    if (threadIdx.x == 0) {
        *ab.flag = 0;
        mbar_init(bar, 1);
        fence_barrier_init();
        mbar_arrive_expect_tx(bar, 4u * (uint32_t)W * 128u);
        for (int h = 0; h < 2; ++h) {
            tma_load_2d(ks + h * hs, &tm_k, bar, h * 64, (int)cbase);
            tma_load_2d(vs + h * hs, &tm_v, bar, h * 64, (int)cbase);
        }
    }

    const float4 q4 = prep_head_warp(p.q + ((long long)b * p.Hq + head) * kD, p.wq, p.R, p.eps, pos,
                                     p.theta, ubuf[warp]);
    *reinterpret_cast<float4 *>(&qt[warp][4 * lane]) = q4;
    uint2 kbits = make_uint2(0, 0), vbits = make_uint2(0, 0);
    if (warp == 0) {
        // the new key, prepared and rounded as the cache stores it
        const float4 k4 = prep_head_warp(p.k + ((long long)b * p.Hkv + kvh) * kD, p.wk, p.R, p.eps, pos,
                                         p.theta, ubuf[0]);
        kbits = make_uint2(pack_bf16(k4.x, k4.y), pack_bf16(k4.z, k4.w));
        *reinterpret_cast<uint2 *>(p.kc + (cbase + slot_new) * kD + 4 * lane) = kbits;
    } else if (warp == 1) {
        vbits = *reinterpret_cast<const uint2 *>(p.v + ((long long)b * p.Hkv + kvh) * kD + 4 * lane);
        *reinterpret_cast<uint2 *>(p.vc + (cbase + slot_new) * kD + 4 * lane) = vbits;
    }
    __syncthreads();   // the barrier's initialisation is visible to every waiter
    const bool landed = warp_wait(bar, 0, ab);
    // the new token's row over its slot (the ring load may hold either version of it)
    if (landed && warp < 2) {
        const uint32_t tile = warp == 0 ? ks : vs;
        const uint32_t off = swa::chunk_off(slot_new, (4 * lane) / 8, hs) + ((4 * lane) % 8) * 2;
        const uint2 bits = warp == 0 ? kbits : vbits;
        asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(tile + off), "r"(bits.x), "r"(bits.y) : "memory");
    }
    __syncthreads();
    if (!landed) {
        // the wait gave up: the ring's copy must still land before the CTA exits
        if (threadIdx.x == 0) swa::drain_wait(bar, 0);
        return;
    }

    // scores: lane owns slots lane + 32 i; slot s holds position pos - ((slot_new - s) mod W)
    float sc[4];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int s = lane + 32 * i;
        sc[i] = -INFINITY;
        if (s < W) {
            const int age = (slot_new - s + W) % W;
            if (age <= pos) {
                float acc = 0.f;
#pragma unroll 4
                for (int c = 0; c < 16; ++c) {
                    const uint4 kv = lds128(ks + swa::chunk_off(s, c, hs));
                    const float4 qa = *reinterpret_cast<const float4 *>(&qt[warp][8 * c]);
                    const float4 qb = *reinterpret_cast<const float4 *>(&qt[warp][8 * c + 4]);
                    const float2 k0 = unpack_bf16(kv.x), k1 = unpack_bf16(kv.y), k2 = unpack_bf16(kv.z),
                                 k3 = unpack_bf16(kv.w);
                    acc = fmaf(qa.x, k0.x, fmaf(qa.y, k0.y, fmaf(qa.z, k1.x, fmaf(qa.w, k1.y, acc))));
                    acc = fmaf(qb.x, k2.x, fmaf(qb.y, k2.y, fmaf(qb.z, k3.x, fmaf(qb.w, k3.y, acc))));
                }
                sc[i] = acc * p.sl2;
            }
        }
        mx = fmaxf(mx, sc[i]);
    }
    mx = warp_max(mx);
    float pr[4], l = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        pr[i] = sc[i] == -INFINITY ? 0.f : ex2(sc[i] - mx);
        l += pr[i];
    }
    l = warp_sum(l);
    // P V: lane owns dims 4 lane .. 4 lane + 3 (half lane / 16, chunk (lane % 16) / 2, word lane % 2)
    const uint32_t v_half = (uint32_t)(lane >> 4) * hs, v_chunk = (uint32_t)((lane & 15) >> 1),
                   v_word = (uint32_t)(lane & 1) * 8;
    float o[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i = 0; i < 4; ++i) {
#pragma unroll 8
        for (int j = 0; j < 32; ++j) {
            const int s = 32 * i + j;
            const float ps = __shfl_sync(0xffffffffu, pr[i], j);
            if (s < W && ps != 0.f) {
                uint32_t v0, v1;
                const uint32_t va = vs + v_half + (uint32_t)s * 128 + ((v_chunk ^ (uint32_t)(s & 7)) << 4) + v_word;
                asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v0), "=r"(v1) : "r"(va));
                const float2 f0 = unpack_bf16(v0), f1 = unpack_bf16(v1);
                o[0] = fmaf(ps, f0.x, o[0]);
                o[1] = fmaf(ps, f0.y, o[1]);
                o[2] = fmaf(ps, f1.x, o[2]);
                o[3] = fmaf(ps, f1.y, o[3]);
            }
        }
    }
    const float inv = 1.0f / l;
    const uint2 gr = *reinterpret_cast<const uint2 *>(p.g + ((long long)b * p.Hq + head) * kD + 4 * lane);
    const float2 g0 = unpack_bf16(gr.x), g1 = unpack_bf16(gr.y);
    auto sig = [](float x) { return 1.0f / (1.0f + ex2(-1.4426950408889634f * x)); };
    *reinterpret_cast<uint2 *>(p.y + ((long long)b * p.Hq + head) * kD + 4 * lane) =
        make_uint2(pack_bf16(o[0] * inv * sig(g0.x), o[1] * inv * sig(g0.y)),
                   pack_bf16(o[2] * inv * sig(g1.x), o[3] * inv * sig(g1.y)));
}

// ----------------------------------------------------------------- full cache
// Prologue: q~ of the 4 heads (f32, workspace) and k~, v appended at `pos`.
__global__ void __launch_bounds__(128)
full_decode_prep_kernel(const __grid_constant__ Params p)
{
    __shared__ __align__(16) float ubuf[4][kD];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x / p.Hkv, kvh = blockIdx.x % p.Hkv;
    const int head = kvh * 4 + warp;
    const long long pos = p.pos[b];
    if (pos < 0 || pos >= p.Tmax) {
        if (threadIdx.x == 0) atomicExch(&g_status, kStatusBadArg);
        return;
    }
    const float4 q4 = prep_head_warp(p.q + ((long long)b * p.Hq + head) * kD, p.wq, p.R, p.eps, pos,
                                     p.theta, ubuf[warp]);
    *reinterpret_cast<float4 *>(p.qt + ((long long)b * p.Hq + head) * kD + 4 * lane) = q4;
    const long long row = ((long long)b * p.Hkv + kvh) * p.Tmax + pos;
    if (warp == 0) {
        const float4 k4 = prep_head_warp(p.k + ((long long)b * p.Hkv + kvh) * kD, p.wk, p.R, p.eps, pos,
                                         p.theta, ubuf[0]);
        *reinterpret_cast<uint2 *>(p.kc + row * kD + 4 * lane) =
            make_uint2(pack_bf16(k4.x, k4.y), pack_bf16(k4.z, k4.w));
    } else if (warp == 1) {
        *reinterpret_cast<uint2 *>(p.vc + row * kD + 4 * lane) =
            *reinterpret_cast<const uint2 *>(p.v + ((long long)b * p.Hkv + kvh) * kD + 4 * lane);
    }
}

__device__ __forceinline__ uint64_t f2_bits(float a, float b)
{
    return (uint64_t)__float_as_uint(a) | ((uint64_t)__float_as_uint(b) << 32);
}

// acc(2) += x(2) * s(broadcast)
__device__ __forceinline__ void ffma2(uint64_t &acc, uint64_t x, float s)
{
    const uint64_t ss = f2_bits(s, s);
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(x), "l"(ss));
}

// Chunk c of (b, kvh): partial softmax state of the 4 heads over keys
// [c * kChunk, (c + 1) * kChunk) intersected with [0, pos].
//
// The chunk's K and V rows stream through a ring of kDecStages shared-memory
// stages of kStageKeys keys, loaded by TMA (128-byte swizzle, so a lane per
// key reads its row without bank conflicts) by a producer warp; compute warp
// w takes stages w, w + kChunkWarps, ... and keeps its own running (max, sum,
// O) per head, merged at the end.  The loads of many stages are in flight at
// once, which is what keeps HBM busy.  There are as many stages as compute
// warps, so warp w always reads ring slot w and waits for the phases of that
// slot in order, each only after it has consumed the one before.  (With more
// warps than slots a warp's first wait could target a slot's second phase
// while its first load had not landed yet; the parity test would then take
// the slot's earlier phase for the one wanted.)
constexpr int kStageKeys = 32;
constexpr int kDecStages = kChunkWarps;   // one ring slot per compute warp
constexpr uint32_t kDecHalf = kStageKeys * 128;          // 32 keys x 64 dims bf16: 4 KiB
constexpr uint32_t kDecTile = 2 * kDecHalf;               // one operand of a stage: 8 KiB
constexpr uint32_t kDecStageBytes = 2 * kDecTile;          // K and V
constexpr uint32_t kDecOffBar = kDecStages * kDecStageBytes;
constexpr uint32_t kDecSmemBytes = kDecOffBar + 2 * kDecStages * 8 + 4 + 1024;
constexpr int kChunkThreads = (kChunkWarps + 1) * 32;     // compute warps + the producer warp

__global__ void __launch_bounds__(kChunkThreads, 1)
full_decode_chunk_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    __shared__ __align__(16) float qt[4][kD];
    __shared__ float wm[kChunkWarps][4], wl[kChunkWarps][4];
    __shared__ __align__(16) float wo[kChunkWarps][4][kD];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const int b = blockIdx.y / p.Hkv, kvh = blockIdx.y % p.Hkv;
    const long long pos = p.pos[b];
    if (pos < 0 || pos >= p.Tmax || (long long)c * kChunk > pos) return;   // nothing to attend here
    auto full = [&](int st) -> uint32_t { return sbase + kDecOffBar + 8u * st; };
    auto empty = [&](int st) -> uint32_t { return sbase + kDecOffBar + 8u * (kDecStages + st); };
    Abort ab{reinterpret_cast<volatile int *>(smem + kDecOffBar + 16 * kDecStages)};
    if (threadIdx.x == 0) {
        *ab.flag = 0;
        for (int i = 0; i < kDecStages; ++i) {
            mbar_init(full(i), 1);
            mbar_init(empty(i), 1);
        }
        fence_barrier_init();
    }
    for (int i = threadIdx.x; i < 4 * kD; i += blockDim.x)
        qt[i / kD][i % kD] = p.qt[((long long)b * p.Hq + kvh * 4) * kD + i];
    __syncthreads();
    const long long k0 = (long long)c * kChunk;
    const long long k1 = min(k0 + kChunk, pos + 1);   // exclusive end
    const int nst = (int)((k1 - k0 + kStageKeys - 1) / kStageKeys);
    const int row0 = (int)(((long long)b * p.Hkv + kvh) * p.Tmax + k0);   // first cache row of the chunk

    if (warp == kChunkWarps) {
        // ================================================= producer
        if (lane == 0) {
            bool ok = true;
            int s = 0;
            for (; s < nst && ok; ++s) {
                const int st = s % kDecStages;
                ok = mbar_wait(empty(st), ((s / kDecStages) & 1) ^ 1u, ab);
                if (!ok) break;
                mbar_arrive_expect_tx(full(st), kDecStageBytes);
                const uint32_t dst = sbase + st * kDecStageBytes;
                const int row = row0 + s * kStageKeys;
                for (int h = 0; h < 2; ++h) {
                    tma_load_2d(dst + h * kDecHalf, &tm_k, full(st), h * 64, row);
                    tma_load_2d(dst + kDecTile + h * kDecHalf, &tm_v, full(st), h * 64, row);
                }
            }
            // no copy may still be landing when the CTA exits
            const uint64_t t0 = globaltimer();
            for (int i = (s > kDecStages ? s - kDecStages : 0); i < s; ++i)
                while (!mbar_try_wait(full(i % kDecStages), (i / kDecStages) & 1))
                    if (globaltimer() - t0 > 200000000ull) break;
        }
    } else {
        // ================================================= compute warps
        float m[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // running max (log2 units)
        float l[4] = {0.f, 0.f, 0.f, 0.f};                          // this lane's keys' sums
        uint64_t o[4][2];                                           // dims 4 lane..+3, as 2 pairs
#pragma unroll
        for (int h = 0; h < 4; ++h) o[h][0] = o[h][1] = 0;
        // V row j, dims 4 lane .. 4 lane + 3: half lane / 16, 16-byte chunk (lane % 16) / 2, 8-byte word lane % 2
        const uint32_t v_half = (uint32_t)(lane >> 4) * kDecHalf, v_chunk = (uint32_t)((lane & 15) >> 1),
                       v_word = (uint32_t)(lane & 1) * 8;
        for (int s = warp; s < nst; s += kChunkWarps) {
            const int st = s % kDecStages;
            if (!warp_wait(full(st), (s / kDecStages) & 1, ab)) break;
            const uint32_t ks = sbase + st * kDecStageBytes, vs = ks + kDecTile;
            const long long t0 = k0 + (long long)s * kStageKeys;
            const int nk = (int)min((long long)kStageKeys, k1 - t0);
            float sc[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            if (lane < nk) {
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
                for (int ch = 0; ch < 16; ++ch) {
                    const uint4 kv = lds128(ks + swa::chunk_off(lane, ch, kDecHalf));
                    const float2 ka = unpack_bf16(kv.x), kb = unpack_bf16(kv.y), kc2 = unpack_bf16(kv.z),
                                 kd = unpack_bf16(kv.w);
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const float4 qa = *reinterpret_cast<const float4 *>(&qt[h][8 * ch]);
                        const float4 qb = *reinterpret_cast<const float4 *>(&qt[h][8 * ch + 4]);
                        float a = acc[h];
                        a = fmaf(qa.x, ka.x, fmaf(qa.y, ka.y, fmaf(qa.z, kb.x, fmaf(qa.w, kb.y, a))));
                        a = fmaf(qb.x, kc2.x, fmaf(qb.y, kc2.y, fmaf(qb.z, kd.x, fmaf(qb.w, kd.y, a))));
                        acc[h] = a;
                    }
                }
#pragma unroll
                for (int h = 0; h < 4; ++h) sc[h] = acc[h] * p.sl2;
            }
            float pr[4], alpha[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float tm = warp_max(sc[h]);
                const float mn = fmaxf(m[h], tm);
                alpha[h] = (m[h] == -INFINITY) ? 0.f : ex2(m[h] - mn);
                m[h] = mn;
                pr[h] = (sc[h] == -INFINITY) ? 0.f : ex2(sc[h] - mn);
                l[h] = l[h] * alpha[h] + pr[h];
                const uint64_t a2 = f2_bits(alpha[h], alpha[h]);
                asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(o[h][0]) : "l"(a2));
                asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(o[h][1]) : "l"(a2));
            }
            for (int j = 0; j < nk; ++j) {
                const uint32_t va = vs + v_half + (uint32_t)j * 128 + ((v_chunk ^ (uint32_t)(j & 7)) << 4) + v_word;
                uint32_t v0, v1;
                asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v0), "=r"(v1) : "r"(va));
                const float2 fa = unpack_bf16(v0), fb = unpack_bf16(v1);
                const uint64_t v01 = f2_bits(fa.x, fa.y), v23 = f2_bits(fb.x, fb.y);
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const float ps = __shfl_sync(0xffffffffu, pr[h], j);
                    ffma2(o[h][0], v01, ps);
                    ffma2(o[h][1], v23, ps);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty(st));
        }
        // this warp's state, for the merge
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const float lsum = warp_sum(l[h]);
            if (lane == 0) {
                wm[warp][h] = m[h];
                wl[warp][h] = lsum;
            }
            float2 a = *reinterpret_cast<float2 *>(&o[h][0]), bq = *reinterpret_cast<float2 *>(&o[h][1]);
            *reinterpret_cast<float4 *>(&wo[warp][h][4 * lane]) = make_float4(a.x, a.y, bq.x, bq.y);
        }
    }
    __syncthreads();
    // one warp per head merges the warps: lanes cover dims 4 lane .. + 3
    if (warp < 4) {
        const int h = warp;
        float M = -INFINITY;
        for (int w = 0; w < kChunkWarps; ++w) M = fmaxf(M, wm[w][h]);
        float L = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int w = 0; w < kChunkWarps; ++w) {
            if (wm[w][h] == -INFINITY) continue;
            const float f = ex2(wm[w][h] - M);
            L += wl[w][h] * f;
            const float4 ow = *reinterpret_cast<const float4 *>(&wo[w][h][4 * lane]);
            acc.x += ow.x * f;
            acc.y += ow.y * f;
            acc.z += ow.z * f;
            acc.w += ow.w * f;
        }
        float *dst = p.part + ((((long long)b * p.Hkv + kvh) * p.nchunks + c) * 4 + h) * kPartial;
        if (lane == 0) {
            dst[0] = M;
            dst[1] = L;
        }
        *reinterpret_cast<float4 *>(dst + 4 + 4 * lane) = acc;
    }
}

// Merge the chunks of (b, head): y = sum_c 2^(m_c - M) o_c / sum_c 2^(m_c - M) l_c.
__global__ void __launch_bounds__(kD)
full_decode_combine_kernel(const __grid_constant__ Params p)
{
    const int b = blockIdx.x / p.Hq, head = blockIdx.x % p.Hq;
    const int kvh = head / 4, h = head % 4;
    const int d = threadIdx.x;
    const long long pos = p.pos[b];
    if (pos < 0 || pos >= p.Tmax) return;
    const int nc = (int)(pos / kChunk) + 1;
    const float *base = p.part + (((long long)b * p.Hkv + kvh) * p.nchunks * 4 + h) * kPartial;
    float M = -INFINITY;
    for (int c = 0; c < nc; ++c) M = fmaxf(M, base[(long long)c * 4 * kPartial]);
    float L = 0.f, acc = 0.f;
    for (int c = 0; c < nc; ++c) {
        const float *pc = base + (long long)c * 4 * kPartial;
        if (pc[0] == -INFINITY) continue;
        const float f = ex2(pc[0] - M);
        L += pc[1] * f;
        acc += pc[4 + d] * f;
    }
    p.y[((long long)b * p.Hq + head) * kD + d] = __float2bfloat16_rn(acc / L);
}

}  // namespace dec
}  // namespace gswa
