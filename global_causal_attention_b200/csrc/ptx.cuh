// ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers with bounded
// waits, TMA tensor loads/stores, and the tcgen05 (5th-generation tensor
// core + tensor memory) instructions the attention kernels issue.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace gswa {

// Device status word of this library on the current device.  A bounded wait
// that gives up stores a nonzero code here; gswa_check_status() reads it.
__device__ int g_status;

constexpr int kStatusTimeout = 1;
constexpr int kStatusBadArg = 2;   // a device-side argument (a decode position) was out of range
constexpr int kStatusSetup = 3;    // a kernel found its launch set-up unusable (shared memory alignment)
// A wait gives up after this much wall time (the kernels' longest legitimate
// wait is a few microseconds; profilers that serialise passes stay far below).
constexpr uint64_t kWaitLimitNs = 4000000000ull;
// The limit the kernels apply: kWaitLimitNs unless gswa_set_wait_limit_ns()
// lowered it (a failure-detection test makes waits give up this way).  Read
// only once a wait has already spun, so it costs nothing on the fast path.
__device__ unsigned long long g_wait_limit_ns = kWaitLimitNs;

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking test of a phase (for threads that poll several barriers).
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// As mbar_try_wait, but the thread may be suspended (up to `hint_ns`) until
// the phase completes instead of spinning on the issue slots other warps need.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Shared abort flag of a CTA: once one role gives up, every other role stops
// waiting too, so that the whole CTA reaches its teardown.
struct Abort {
    volatile int *flag;
    __device__ __forceinline__ bool raised() const { return *flag != 0; }
    __device__ __forceinline__ void raise(int code) const
    {
        *flag = code;
        atomicExch(&g_status, code);
    }
};

// Wait for the phase of `bar` with the given parity to complete.  Returns
// false (and raises the CTA's abort flag) when the wait gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const Abort &ab)
{
    // fast path: a non-blocking test (a blocking try_wait could sit out a
    // lowered limit inside the hardware's own suspend window)
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    // a lowered limit (below 1 ms) is checked on every pass, with a suspend hint
    // no longer than the limit itself
    const unsigned long long lim = g_wait_limit_ns;
    const bool eager = lim < 1000000ull;
    const uint32_t hint = eager ? (uint32_t)lim : 1000000u;
    for (uint32_t spin = 0;; ++spin) {
        if (mbar_try_wait_sleep(bar, parity, hint)) return true;
        if (eager || (spin & 3u) == 3u) {
            if (ab.raised()) return false;
            if (globaltimer() - t0 > lim) {
                ab.raise(kStatusTimeout);
                return false;
            }
        }
    }
}

// Stall watchdog of a polling loop (a thread that tests several barriers in
// turn): call tick(progressed) once per pass.  The wall clock is a slow read,
// so it is consulted only every 512 idle passes (every 8 under a lowered
// limit).  Returns false (with the CTA's abort flag raised) once the loop has
// made no progress for g_wait_limit_ns, or when another role raised the flag.
struct PollWatch {
    uint32_t idle = 0;
    uint64_t t0 = 0;
    unsigned long long lim = g_wait_limit_ns;
    uint32_t mask = lim < 1000000ull ? 7u : 511u;
    __device__ __forceinline__ bool tick(bool progressed, const Abort &ab)
    {
        if (progressed) {
            idle = 0;
            return true;
        }
        if ((++idle & mask) != 0) return true;
        if (ab.raised()) return false;
        const uint64_t now = globaltimer();
        if (idle == mask + 1) {
            t0 = now;
            return true;
        }
        if (now - t0 > lim) {
            ab.raise(kStatusTimeout);
            return false;
        }
        return true;
    }
};

// Warp-uniform wait: every lane waits (and so acquires) itself, then the warp
// agrees, so a wait that gave up in one lane stops the whole warp.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const Abort &ab)
{
    const bool ok = mbar_wait(bar, parity, ab);
    return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------- fences
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const void *tmap)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const void *tmap, uint32_t bar, int c0,
                                            int c1, int c2, int c3)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// Prefetch the 128-byte line holding `p` into L2.
__device__ __forceinline__ void prefetch_l2(const void *p)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(p)));
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *tmap, uint32_t bar, int c0, int c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tma_store_4d(const void *tmap, uint32_t src, int c0, int c1, int c2,
                                             int c3)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(tmap)),
        "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// Relaxed atomic add of one float to global memory, result unused (a
// reduction at L2; a warp's 32 lanes on 32 consecutive floats make one
// 128-byte request).
__device__ __forceinline__ void red_add_f32(float *addr, float v)
{
    asm volatile("red.relaxed.gpu.global.add.f32 [%0], %1;" ::"l"(addr), "f"(v) : "memory");
}

// Untiled bulk copy global -> shared (16-byte aligned addresses, size a
// multiple of 16), completing on `bar` as transaction bytes.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void bulk_commit_group()
{
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait_group_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait_group()
{
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------- tcgen05
// TMEM address: bits [31:16] lane, bits [15:0] column.
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D(tmem) (+)= A(smem desc) * B(smem desc)^T
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D(tmem) (+)= A(tmem) * B(smem desc)^T
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05 op issued so far by this thread completes.
__device__ __forceinline__ void mma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

// One 32-bit column of this thread's TMEM lane.
__device__ __forceinline__ uint32_t tmem_ld1(uint32_t taddr)
{
    uint32_t r;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
    return r;
}

__device__ __forceinline__ void tmem_st1(uint32_t taddr, uint32_t v)
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(v) : "memory");
}

// 16 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

// ------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor (tcgen05 form): start address, leading and
// stride byte offsets (all >> 4), descriptor version 1 at bits 46-47, base
// offset 0 (tiles are 1024-byte aligned), layout type at bits 61-63
// (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// A shared-memory descriptor kept as its two 32-bit halves, built once per
// tile: the low half holds the start address (>> 4, 14 bits) and the leading
// byte offset, the high half the stride byte offset and the layout bits.
// Shared-memory addresses stay below 256 KiB, so advancing the start by a
// constant byte offset is one 32-bit add that never carries into the leading
// byte offset -- an MMA issue loop then spends one instruction per operand on
// its descriptor instead of rebuilding it.
struct SmemDesc {
    uint32_t lo, hi;
    __device__ __forceinline__ uint64_t at(uint32_t byte_off) const
    {
        uint64_t d;
        asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "r"(lo + (byte_off >> 4)), "r"(hi));
        return d;
    }
};

__device__ __forceinline__ SmemDesc make_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    const uint64_t d = smem_desc_sw128(saddr, lbo, sbo);
    return SmemDesc{(uint32_t)d, (uint32_t)(d >> 32)};
}

// Instruction descriptor of kind::f16 with bf16 A/B, f32 accumulator.
// a_mn/b_mn select MN-major operands (0 = K-major).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn)
{
    return (1u << 4)                       // D format: f32
           | (1u << 7)                     // A format: bf16
           | (1u << 10)                    // B format: bf16
           | ((uint32_t)a_mn << 15)        // A major
           | ((uint32_t)b_mn << 16)        // B major
           | ((uint32_t)(N >> 3) << 17)    // N / 8
           | ((uint32_t)(M >> 4) << 24);   // M / 16
}

// ------------------------------------------------------------- shared memory
__device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

// ------------------------------------------------------------- math helpers
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// σ(x) = (1 + tanh(x/2)) / 2 in f32 (one hardware tanh per element, relative
// error below 2^-10.9) of a packed bf16 pair, returned as a packed f16 pair
// (lo in the low half): the gate tile holds σ in place of g, two bytes per
// element, and f16 keeps 11 significant bits where bf16 would keep 8.  On
// one B200 this matched 1 / (1 + 2^(-x log2 e)) (hardware 2^x and reciprocal)
// in the output error, at the cost of the f16 tanh form, 13 % below it.
__device__ __forceinline__ uint32_t sigmoid_bf16x2_f16x2(uint32_t g)
{
    const float lo = __uint_as_float(g << 16), hi = __uint_as_float(g & 0xFFFF0000u);
    float tl, th;
    asm("tanh.approx.f32 %0, %1;" : "=f"(tl) : "f"(0.5f * lo));
    asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(0.5f * hi));
    uint32_t h;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(fmaf(0.5f, th, 0.5f)), "f"(fmaf(0.5f, tl, 0.5f)));
    return h;
}

// Packed f32 pairs: sm_100 executes add/mul/fma on .f32x2 operands as two
// IEEE f32 operations per instruction (same rounding as the scalar forms).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ float2 f2_unpack(uint64_t v)
{
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}

__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// 2^x of a pair of floats on the FMA pipe (the softmax runs part of its
// exponentials here so that the special-function unit, a quarter of the FMA
// pipe's width, stops being the bound).  Cody-Waite range reduction x = j + f
// with j = round(x) (adding 1.5 * 2^23 leaves round(x) in the low mantissa
// bits) and f in [-1/2, 1/2]; 2^f by a degree-3 polynomial whose
// coefficients minimise the maximum relative error on that interval (fitted
// by exp2_poly_fit.py: 7.5e-5, far below the bf16 rounding of P); 2^j by
// adding j to the exponent field (the low 9 bits of 1.5 * 2^23's pattern are
// zero, so shifting the sum's bits left by 23 leaves exactly j << 23).
// Valid for -125 <= x <= 127.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2)
{
    const uint64_t magic = f2_pack(12582912.0f, 12582912.0f);
    const uint64_t t = f2_add(x2, magic);
    const uint64_t f = f2_sub(x2, f2_sub(t, magic));
    uint64_t p = f2_fma(f, f2_pack(0.0551712066f, 0.0551712066f), f2_pack(0.242610276f, 0.242610276f));
    p = f2_fma(p, f, f2_pack(0.693260968f, 0.693260968f));
    p = f2_fma(p, f, f2_pack(0.999928117f, 0.999928117f));
    uint32_t tl, th, pl, ph;
    asm("mov.b64 {%0, %1}, %2;" : "=r"(tl), "=r"(th) : "l"(t));
    asm("mov.b64 {%0, %1}, %2;" : "=r"(pl), "=r"(ph) : "l"(p));
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(pl + (tl << 23)), "r"(ph + (th << 23)));
    return r;
}

// Two floats to a packed f16 pair (`lo` in the low half), round to nearest.
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi)
{
    uint32_t h;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(hi), "f"(lo));
    return h;
}

__device__ __forceinline__ float2 unpack_f16(uint32_t u)
{
    __half2 h = *reinterpret_cast<__half2 *>(&u);
    return __half22float2(h);
}

// Round two floats to bf16 (nearest-even) and pack them, `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// bf16 pair -> two floats.  A bf16 is the upper half of a float32, so the
// widening is a shift/mask on the integer pipe (exact), not a conversion.
__device__ __forceinline__ float2 unpack_bf16(uint32_t u)
{
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t h)
{
    return __uint_as_float((uint32_t)h << 16);
}

}  // namespace gswa
