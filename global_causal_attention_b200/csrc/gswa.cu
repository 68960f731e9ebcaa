// gswa.cu -- C ABI of the ZGCM-1 attention core (declared in include/gswa.h).
//
// Host-side argument validation, TMA tensor-map encoding and kernel launch.
// One translation unit: every kernel of the library is included here so that
// they share the device status word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "gswa.h"
#include "ptx.cuh"
#include "swa_fwd.cuh"
#include "qk_prep.cuh"
#include "full_fwd.cuh"
#include "decode.cuh"
#include "bwd.cuh"
#include "bwd_full.cuh"

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    int status = GSWA_OK;
    int num_sms = 0;
};

std::mutex g_mutex;
DeviceInfo g_dev[kMaxDevices];
EncodeTiledFn g_encode = nullptr;

template <typename K>
bool set_smem(K kernel, uint32_t bytes)
{
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) !=
           cudaSuccess;
}

template <int R>
bool set_bwd_smem()
{
    using namespace gswa::bwd;
    return set_smem(bwd_dq_swa_kernel<R>, DqSwaCfg::kSmemBytes) ||
           set_smem(bwd_dkdv_kernel<R>, KvCfg::kSmemBytes) ||
           set_smem(gswa::bwdf::bwd_full_kernel<R>, gswa::bwdf::kSmemBytes);
}

// Rotated dims the kernels are compiled for (the row is held in registers).
bool rope_dims_supported(int R) { return R == 0 || R == 42 || R == 64 || R == 128; }

// Per-device set-up (compute capability check, kernel attributes, SM count),
// done once per device under a lock.
int device_setup(int *num_sms)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GSWA_ERR_NO_DEVICE;
    if (dev < 0 || dev >= kMaxDevices) return GSWA_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo &d = g_dev[dev];
    if (!d.ready) {
        d.ready = true;
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            d.status = GSWA_ERR_NO_DEVICE;
        } else if (major != 10 || minor != 0) {
            d.status = GSWA_ERR_NO_DEVICE;  // built for sm_100a only
        } else if (set_smem(gswa::swa::swa_fwd_kernel<0>, gswa::swa::kSmemBytes) ||
                   set_smem(gswa::swa::swa_fwd_kernel<42>, gswa::swa::kSmemBytes) ||
                   set_smem(gswa::swa::swa_fwd_kernel<64>, gswa::swa::kSmemBytes) ||
                   set_smem(gswa::swa::swa_fwd_kernel<128>, gswa::swa::kSmemBytes) ||
                   set_smem(gswa::full::full_fwd_kernel, gswa::full::kSmemBytes) ||
                   set_smem(gswa::dec::full_decode_chunk_kernel, gswa::dec::kDecSmemBytes) ||
                   set_smem(gswa::dec::swa_decode_kernel, gswa::dec::kSwaDecSmemBytes) ||
                   set_bwd_smem<0>() || set_bwd_smem<42>() || set_bwd_smem<64>() || set_bwd_smem<128>()) {
            d.status = GSWA_ERR_LAUNCH;
        }
        if (d.status == GSWA_OK && g_encode == nullptr) {
            void *fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                    cudaSuccess ||
                q != cudaDriverEntryPointSuccess || fn == nullptr)
                d.status = GSWA_ERR_LAUNCH;
            else
                g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
    }
    *num_sms = d.num_sms;
    return d.status;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 4-D bf16 tensor map over [B, T, H, D] (innermost first: D, H, T, B) with a
// {64, box_h, box_t, 1} box and the 128-byte swizzle the MMA descriptors use.
int encode_bthd(CUtensorMap *m, const void *base, int B, int T, int H, int D, int box_h, int box_t)
{
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)box_h, (cuuint32_t)box_t, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                          strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GSWA_OK : GSWA_ERR_INVALID_ARG;
}

// 2-D bf16 tensor map over `rows` rows of 128 elements (a cache viewed as
// [B * Hkv * Tmax, 128]) with a {64, box_rows} box and the 128-byte swizzle.
int encode_rows(CUtensorMap *m, const void *base, long long rows, int box_rows)
{
    cuuint64_t dims[2] = {128, (cuuint64_t)rows};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GSWA_OK : GSWA_ERR_INVALID_ARG;
}

// Shape checks common to every entry point.
int check_common(const gswa_shape_t *s)
{
    if (s == nullptr) return GSWA_ERR_INVALID_ARG;
    if (s->B < 0 || s->T < 0 || s->Hq <= 0 || s->Hkv <= 0 || s->D <= 0) return GSWA_ERR_INVALID_ARG;
    if (!(s->eps >= 0.f) || !(s->rope_base > 0.0) || !std::isfinite(s->scale))
        return GSWA_ERR_INVALID_ARG;
    if (s->D != 128) return GSWA_ERR_UNSUPPORTED_SHAPE;
    if (s->Hq != 4 * s->Hkv) return GSWA_ERR_UNSUPPORTED_SHAPE;
    if (s->rope_dims < 0 || s->rope_dims > s->D || (s->rope_dims & 1)) return GSWA_ERR_UNSUPPORTED_SHAPE;
    return GSWA_OK;
}

void fill_theta(double *theta, int R, double base)
{
    for (int p = 0; p < 64; ++p)
        theta[p] = (p < R / 2) ? std::pow(base, -2.0 * (double)p / (double)R) : 0.0;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace of the full-cache decode: q~ [B, Hq, D] f32, then the chunk
// partials [B, Hkv, nchunks, 4, kPartial] f32.
size_t full_decode_ws(const gswa_shape_t *s)
{
    const size_t nch = ((size_t)s->cache_len + gswa::dec::kChunk - 1) / gswa::dec::kChunk;
    return align256((size_t)s->B * s->Hq * s->D * 4) +
           align256((size_t)s->B * s->Hkv * nch * 4 * gswa::dec::kPartial * 4);
}

void fill_dec(gswa::dec::Params &p, const gswa_shape_t *s)
{
    std::memset(&p, 0, sizeof p);
    p.B = s->B;
    p.Hq = s->Hq;
    p.Hkv = s->Hkv;
    p.R = s->rope_dims;
    p.W = s->window;
    p.Tmax = s->cache_len;
    p.nchunks = (int)((s->cache_len + gswa::dec::kChunk - 1) / gswa::dec::kChunk);
    p.eps = s->eps;
    p.sl2 = s->scale * 1.4426950408889634f;
    fill_theta(p.theta, s->rope_dims, s->rope_base);
}

// Workspace of the full causal forward: prepared keys k~ [B, T, Hkv, D] then
// prepared queries q~ [B, T, Hq, D], bf16.
size_t full_fwd_ws_keys(const gswa_shape_t *s)
{
    return align256((size_t)s->B * s->T * s->Hkv * s->D * 2);
}

// Workspace of the gated-SWA forward: prepared keys k~ [B, T, Hkv, D], bf16.
size_t swa_fwd_ws(const gswa_shape_t *s)
{
    return align256((size_t)s->B * s->T * s->Hkv * s->D * 2);
}

size_t full_fwd_ws(const gswa_shape_t *s)
{
    return full_fwd_ws_keys(s) + align256((size_t)s->B * s->T * s->Hq * s->D * 2);
}

// RMSNorm + partial RoPE of x [B, T, H, 128] into out, positions pos0 + t.
int launch_qk_prep(const gswa_shape_t *s, int H, const void *x, const void *w, void *out, long long pos0,
                   cudaStream_t st, int num_sms)
{
    gswa::prep::Params pp;
    std::memset(&pp, 0, sizeof pp);
    pp.x = static_cast<const __nv_bfloat16 *>(x);
    pp.out = static_cast<__nv_bfloat16 *>(out);
    pp.w = static_cast<const __nv_bfloat16 *>(w);
    pp.rows = (long long)s->B * s->T * H;
    pp.T = s->T;
    pp.H = H;
    pp.pos0 = pos0;
    pp.eps = s->eps;
    fill_theta(pp.theta, s->rope_dims, s->rope_base);
    const long long groups = (pp.rows + 31) / 32;
    long long grid = (groups + gswa::prep::kWarps - 1) / gswa::prep::kWarps;
    if (grid > 16LL * num_sms) grid = 16LL * num_sms;
    const dim3 gr((unsigned)grid), bl(gswa::prep::kWarps * 32);
    switch (s->rope_dims) {
    case 0: gswa::prep::qk_prep_kernel<0><<<gr, bl, 0, st>>>(pp); break;
    case 42: gswa::prep::qk_prep_kernel<42><<<gr, bl, 0, st>>>(pp); break;
    case 64: gswa::prep::qk_prep_kernel<64><<<gr, bl, 0, st>>>(pp); break;
    default: gswa::prep::qk_prep_kernel<128><<<gr, bl, 0, st>>>(pp); break;
    }
    return cudaGetLastError() == cudaSuccess ? GSWA_OK : GSWA_ERR_LAUNCH;
}

// ------------------------------------------------ allocation-free decode
// The fixed device scratch of full_decode_noalloc: one array per device,
// placed by the loader with the library's kernels; nothing is allocated at
// call time.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GSWA_NOALLOC_SCRATCH_BYTES];

struct NoAllocDevice {
    bool ready = false;       // set once the lookup succeeded
    void *scratch = nullptr;
};
NoAllocDevice g_noalloc[kMaxDevices];

// Device address of the scratch on the current device, looked up once per
// device (with that device current) under the library lock.
int noalloc_scratch(void **scratch)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GSWA_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lock(g_mutex);
    NoAllocDevice &d = g_noalloc[dev];
    if (!d.ready) {
        void *ptr = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || ptr == nullptr) {
            // not cached: clear the runtime's error state so that a later call
            // (say, one made outside a stream capture) can try again
            (void)cudaGetLastError();
            *scratch = nullptr;
            return GSWA_ERR_LAUNCH;
        }
        d.scratch = ptr;
        d.ready = true;
    }
    *scratch = d.scratch;
    return GSWA_OK;
}

// Backward workspace: prepared q~ [B,T,Hq,D] and k~ [B,T,Hkv,D] (bf16),
// dA [B,T,Hq,D] (gated only; ungated dA is dy), the row records
// [B,Hkv,Tp,4] float2, and the per-warp dw_q / dw_k partials.
struct BwdWs {
    size_t qt, kt, da, ld, pq, pk, total;
};

BwdWs bwd_ws_layout(const gswa_shape_t *s, bool gated)
{
    const size_t BT = (size_t)s->B * s->T;
    const size_t Tp = ((size_t)s->T + 31) / 32 * 32;
    const size_t part = align256((size_t)gswa::bwd::kMaxGrid * 4 * 128 * 4);
    BwdWs w;
    w.qt = 0;
    w.kt = w.qt + align256(BT * s->Hq * s->D * 2);
    w.da = w.kt + align256(BT * s->Hkv * s->D * 2);
    w.ld = w.da + (gated ? align256(BT * s->Hq * s->D * 2) : 0);
    w.pq = w.ld + align256((size_t)s->B * s->Hkv * Tp * 4 * 8);
    w.pk = w.pq + part;
    w.total = w.pk + part;
    return w;
}

// Full-causal backward workspace: prepared q~ [B,T,Hq,D] and k~ [B,T,Hkv,D]
// (bf16), the row records [B,Hkv,Tp,4] float2, the dq~ accumulator
// [B,T,Hq,D] f32, the dw_q partials of the post kernel and the dw_k partials
// of the fused kernel (f32 [n][128]).
struct FullBwdWs {
    size_t qt, kt, ld, acc, pq, pk, total;
};

FullBwdWs full_bwd_ws_layout(const gswa_shape_t *s)
{
    const size_t BT = (size_t)s->B * s->T;
    const size_t Tp = ((size_t)s->T + 31) / 32 * 32;
    FullBwdWs w;
    w.qt = 0;
    w.kt = w.qt + align256(BT * s->Hq * s->D * 2);
    w.ld = w.kt + align256(BT * s->Hkv * s->D * 2);
    w.acc = w.ld + align256((size_t)s->B * s->Hkv * Tp * 4 * 8);
    w.pq = w.acc + align256(BT * s->Hq * s->D * 4);
    w.pk = w.pq + align256((size_t)gswa::bwdf::kPostMaxGrid * gswa::bwdf::kPostWarps * 128 * 4);
    w.total = w.pk + align256((size_t)gswa::bwdf::kMaxGrid * 4 * 128 * 4);
    return w;
}

struct BwdMaps {
    CUtensorMap tq, ta, tk, tv;       // dq kernel
    CUtensorMap tk2, tv2, tq2, ta2;   // dk/dv kernel
};

// The gated sliding-window backward's two main kernels.
template <int R>
void launch_swa_bwd_main(const BwdMaps &m, const gswa::bwd::Params &pq, const gswa::bwd::Params &pk, unsigned gq,
                         unsigned gk, cudaStream_t st)
{
    using namespace gswa::bwd;
    bwd_dq_swa_kernel<R><<<gq, kThreads, DqSwaCfg::kSmemBytes, st>>>(m.tq, m.ta, m.tk, m.tv, pq);
    bwd_dkdv_kernel<R><<<gk, kThreads, KvCfg::kSmemBytes, st>>>(m.tk2, m.tv2, m.tq2, m.ta2, pk);
}

template <int R>
void launch_full_bwd(const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &tq, const CUtensorMap &ta,
                     const gswa::bwdf::Params &p, unsigned grid,
                     const gswa::bwdf::PostParams &pp, unsigned pgrid, cudaStream_t st)
{
    using namespace gswa::bwdf;
    bwd_full_kernel<R><<<grid, kThreads, kSmemBytes, st>>>(tk, tv, tq, ta, p);
    bwd_dq_post_kernel<R><<<pgrid, kPostWarps * 32, 0, st>>>(pp);
}

// full_attn_bwd after the argument checks: records, q~/k~, the fused
// key-stationary kernel (dk, dv, dw_k partials, dq~ sums), the dq post pass
// and the fixed-order weight-gradient sums.
int run_full_bwd(const gswa_shape_t *s, const void *q, const void *k, const void *v, const void *w_q,
                 const void *w_k, const void *y, const float *lse, const void *dy, void *dq, void *dk, void *dv,
                 float *dw_q, float *dw_k, void *workspace, int num_sms, cudaStream_t st)
{
    const FullBwdWs L = full_bwd_ws_layout(s);
    char *ws = static_cast<char *>(workspace);
    void *qt = ws + L.qt, *kt = ws + L.kt, *acc = ws + L.acc;
    float2 *ld = reinterpret_cast<float2 *>(ws + L.ld);
    float *part_q = reinterpret_cast<float *>(ws + L.pq), *part_k = reinterpret_cast<float *>(ws + L.pk);
    const int Tp = (s->T + 31) / 32 * 32;

    // 1. row records {lse log2 e, D = sum dy y}
    gswa::bwd::PrepParams pp;
    std::memset(&pp, 0, sizeof pp);
    pp.y = static_cast<const __nv_bfloat16 *>(y);
    pp.dy = static_cast<const __nv_bfloat16 *>(dy);
    pp.lse = lse;
    pp.ld = ld;
    pp.rows = (long long)s->B * Tp * s->Hq;
    pp.T = s->T;
    pp.Tp = Tp;
    pp.Hq = s->Hq;
    long long pgrid = ((long long)s->B * Tp + 15) / 16;
    if (pgrid > 16LL * num_sms) pgrid = 16LL * num_sms;
    gswa::bwd::bwd_prep_kernel<<<(unsigned)pgrid, 256, 0, st>>>(pp);
    // 2. prepared queries and keys; 3. the dq~ accumulator starts at zero
    int rc = launch_qk_prep(s, s->Hq, q, w_q, qt, 0, st, num_sms);
    if (rc == GSWA_OK) rc = launch_qk_prep(s, s->Hkv, k, w_k, kt, 0, st, num_sms);
    if (rc != GSWA_OK) return rc;
    if (cudaMemsetAsync(acc, 0, (size_t)s->B * s->T * s->Hq * s->D * 4, st) != cudaSuccess) return GSWA_ERR_LAUNCH;

    // 4. the fused kernel
    using namespace gswa::bwdf;
    CUtensorMap tk, tv, tq, ta;
    if (encode_bthd(&tk, kt, s->B, s->T, s->Hkv, s->D, 1, kKeys) ||
        encode_bthd(&tv, v, s->B, s->T, s->Hkv, s->D, 1, kKeys) ||
        encode_bthd(&tq, qt, s->B, s->T, s->Hq, s->D, 4, kChTok) ||
        encode_bthd(&ta, dy, s->B, s->T, s->Hq, s->D, 4, kChTok))
        return GSWA_ERR_INVALID_ARG;
    Params p;
    std::memset(&p, 0, sizeof p);
    p.B = s->B;
    p.T = s->T;
    p.Tp = Tp;
    p.Hq = s->Hq;
    p.Hkv = s->Hkv;
    p.nkt = (s->T + kKeys - 1) / kKeys;
    p.units = (long long)s->B * s->Hkv * p.nkt;
    p.eps = s->eps;
    p.scale = s->scale;
    p.sl2 = s->scale * 1.4426950408889634f;
    p.ld = ld;
    p.k = static_cast<const __nv_bfloat16 *>(k);
    p.wk = static_cast<const __nv_bfloat16 *>(w_k);
    p.dk = static_cast<__nv_bfloat16 *>(dk);
    p.dv = static_cast<__nv_bfloat16 *>(dv);
    p.dq_acc = static_cast<float *>(acc);
    p.dw_part = part_k;
    fill_theta(p.theta, s->rope_dims, s->rope_base);
    long long grid = p.units < num_sms ? p.units : num_sms;
    if (grid > kMaxGrid) grid = kMaxGrid;

    // 5. dq from the accumulated dq~
    PostParams q2;
    std::memset(&q2, 0, sizeof q2);
    q2.acc = static_cast<const float *>(acc);
    q2.q = static_cast<const __nv_bfloat16 *>(q);
    q2.wq = static_cast<const __nv_bfloat16 *>(w_q);
    q2.dq = static_cast<__nv_bfloat16 *>(dq);
    q2.dw_part = part_q;
    q2.rows = (long long)s->B * s->T * s->Hq;
    q2.T = s->T;
    q2.Hq = s->Hq;
    q2.eps = s->eps;
    q2.scale = s->scale;
    fill_theta(q2.theta, s->rope_dims, s->rope_base);
    long long qgrid = (q2.rows / kPostRows + kPostWarps - 1) / kPostWarps;
    if (qgrid > 3LL * num_sms) qgrid = 3LL * num_sms;
    if (qgrid > kPostMaxGrid) qgrid = kPostMaxGrid;

    switch (s->rope_dims) {
    case 0: launch_full_bwd<0>(tk, tv, tq, ta, p, (unsigned)grid, q2, (unsigned)qgrid, st); break;
    case 42: launch_full_bwd<42>(tk, tv, tq, ta, p, (unsigned)grid, q2, (unsigned)qgrid, st); break;
    case 64: launch_full_bwd<64>(tk, tv, tq, ta, p, (unsigned)grid, q2, (unsigned)qgrid, st); break;
    default: launch_full_bwd<128>(tk, tv, tq, ta, p, (unsigned)grid, q2, (unsigned)qgrid, st); break;
    }
    // 6. weight gradients, summed in a fixed order
    const unsigned rt = gswa::bwd::kD * gswa::bwd::kReduceSlices;
    gswa::bwd::dw_reduce_kernel<<<1, rt, 0, st>>>(part_q, (int)qgrid * kPostWarps, dw_q);
    gswa::bwd::dw_reduce_kernel<<<1, rt, 0, st>>>(part_k, (int)grid * 4, dw_k);
    return cudaGetLastError() == cudaSuccess ? GSWA_OK : GSWA_ERR_LAUNCH;
}

// Shared argument checks of gswa_bwd (swa: gated sliding window) and
// full_attn_bwd, then the gated path here or the full-causal one in run_full_bwd.
int run_bwd(bool swa, const gswa_shape_t *s, const void *q, const void *k, const void *v, const void *g,
            const void *w_q, const void *w_k, const void *y, const float *lse, const void *dy, void *dq,
            void *dk, void *dv, void *dg, float *dw_q, float *dw_k, void *workspace, size_t workspace_bytes,
            cudaStream_t st)
{
    int rc = check_common(s);
    if (rc != GSWA_OK) return rc;
    if (swa && (s->window < 1 || s->window > 128)) return GSWA_ERR_UNSUPPORTED_SHAPE;
    if (!rope_dims_supported(s->rope_dims)) return GSWA_ERR_UNSUPPORTED_SHAPE;
    if (!dw_q || !dw_k) return GSWA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(dw_q) & 3u) || (reinterpret_cast<uintptr_t>(dw_k) & 3u))
        return GSWA_ERR_MISALIGNED;
    int num_sms = 0;
    if ((long long)s->B * s->T == 0) {
        // nothing attends: the weight gradients are zero
        rc = device_setup(&num_sms);
        if (rc != GSWA_OK) return rc;
        if (cudaMemsetAsync(dw_q, 0, 128 * sizeof(float), st) != cudaSuccess ||
            cudaMemsetAsync(dw_k, 0, 128 * sizeof(float), st) != cudaSuccess)
            return GSWA_ERR_LAUNCH;
        return GSWA_OK;
    }
    if (!q || !k || !v || !w_q || !w_k || !y || !lse || !dy || !dq || !dk || !dv || (swa && (!g || !dg)))
        return GSWA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(y) || !aligned16(dy) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || (swa && (!aligned16(g) || !aligned16(dg))) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u))
        return GSWA_ERR_MISALIGNED;
    const size_t need = swa ? bwd_ws_layout(s, true).total : full_bwd_ws_layout(s).total;
    if (workspace == nullptr || workspace_bytes < need) return GSWA_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(workspace)) return GSWA_ERR_MISALIGNED;
    rc = device_setup(&num_sms);
    if (rc != GSWA_OK) return rc;
    if (!swa)
        return run_full_bwd(s, q, k, v, w_q, w_k, y, lse, dy, dq, dk, dv, dw_q, dw_k, workspace, num_sms, st);
    const BwdWs L = bwd_ws_layout(s, swa);

    char *ws = static_cast<char *>(workspace);
    void *qt = ws + L.qt, *kt = ws + L.kt;
    const void *da = swa ? static_cast<const void *>(ws + L.da) : dy;
    float2 *ld = reinterpret_cast<float2 *>(ws + L.ld);
    float *part_q = reinterpret_cast<float *>(ws + L.pq), *part_k = reinterpret_cast<float *>(ws + L.pk);
    const int Tp = (s->T + 31) / 32 * 32;

    // 1. D, lse records, dA, dg
    gswa::bwd::PrepParams pp;
    pp.y = static_cast<const __nv_bfloat16 *>(y);
    pp.dy = static_cast<const __nv_bfloat16 *>(dy);
    pp.g = static_cast<const __nv_bfloat16 *>(g);
    pp.lse = lse;
    pp.dA = swa ? reinterpret_cast<__nv_bfloat16 *>(ws + L.da) : nullptr;
    pp.dg = static_cast<__nv_bfloat16 *>(dg);
    pp.ld = ld;
    pp.rows = (long long)s->B * Tp * s->Hq;
    pp.T = s->T;
    pp.Tp = Tp;
    pp.Hq = s->Hq;
    long long pgrid = ((long long)s->B * Tp + 15) / 16;   // a half-warp per token
    if (pgrid > 16LL * num_sms) pgrid = 16LL * num_sms;
    gswa::bwd::bwd_prep_kernel<<<(unsigned)pgrid, 256, 0, st>>>(pp);
    // 2. prepared queries and keys
    rc = launch_qk_prep(s, s->Hq, q, w_q, qt, 0, st, num_sms);
    if (rc == GSWA_OK) rc = launch_qk_prep(s, s->Hkv, k, w_k, kt, 0, st, num_sms);
    if (rc != GSWA_OK) return rc;

    // 3. dq and dk/dv (the dq kernel's K~/V boxes are its 32-key ring blocks)
    const int kN = gswa::bwd::DqSwaCfg::kTok;
    BwdMaps m;
    if (encode_bthd(&m.tq, qt, s->B, s->T, s->Hq, s->D, 4, 32) ||
        encode_bthd(&m.ta, da, s->B, s->T, s->Hq, s->D, 4, 32) ||
        encode_bthd(&m.tk, kt, s->B, s->T, s->Hkv, s->D, 1, kN) ||
        encode_bthd(&m.tv, v, s->B, s->T, s->Hkv, s->D, 1, kN) ||
        encode_bthd(&m.tk2, kt, s->B, s->T, s->Hkv, s->D, 1, 128) ||
        encode_bthd(&m.tv2, v, s->B, s->T, s->Hkv, s->D, 1, 128) ||
        encode_bthd(&m.tq2, qt, s->B, s->T, s->Hq, s->D, 4, gswa::bwd::KvCfg::kChTok) ||
        encode_bthd(&m.ta2, da, s->B, s->T, s->Hq, s->D, 4, gswa::bwd::KvCfg::kChTok))
        return GSWA_ERR_INVALID_ARG;

    gswa::bwd::Params pq;
    std::memset(&pq, 0, sizeof pq);
    pq.B = s->B;
    pq.T = s->T;
    pq.Tp = Tp;
    pq.Hq = s->Hq;
    pq.Hkv = s->Hkv;
    pq.window = swa ? s->window : 0;
    pq.eps = s->eps;
    pq.scale = s->scale;
    pq.sl2 = s->scale * 1.4426950408889634f;
    pq.ld = ld;
    fill_theta(pq.theta, s->rope_dims, s->rope_base);
    gswa::bwd::Params pk = pq;

    pq.nq = Tp / 32;
    pq.nkt = (s->T + kN - 1) / kN;
    pq.units = (long long)s->B * s->Hkv * pq.nq;
    pq.x = static_cast<const __nv_bfloat16 *>(q);
    pq.w = static_cast<const __nv_bfloat16 *>(w_q);
    pq.dx = static_cast<__nv_bfloat16 *>(dq);
    pq.dw_part = part_q;

    pk.nq = pq.nq;
    pk.nkt = (s->T + 127) / 128;
    pk.units = (long long)s->B * s->Hkv * pk.nkt;
    pk.x = static_cast<const __nv_bfloat16 *>(k);
    pk.w = static_cast<const __nv_bfloat16 *>(w_k);
    pk.dx = static_cast<__nv_bfloat16 *>(dk);
    pk.dv = static_cast<__nv_bfloat16 *>(dv);
    pk.dw_part = part_k;

    auto grid_of = [&](long long units) {
        long long gsz = units < num_sms ? units : num_sms;
        return (unsigned)(gsz < gswa::bwd::kMaxGrid ? gsz : gswa::bwd::kMaxGrid);
    };
    const unsigned gq = grid_of(pq.units), gk = grid_of(pk.units);
    switch (s->rope_dims) {
    case 0: launch_swa_bwd_main<0>(m, pq, pk, gq, gk, st); break;
    case 42: launch_swa_bwd_main<42>(m, pq, pk, gq, gk, st); break;
    case 64: launch_swa_bwd_main<64>(m, pq, pk, gq, gk, st); break;
    default: launch_swa_bwd_main<128>(m, pq, pk, gq, gk, st); break;
    }
    // 4. weight gradients, summed in a fixed order
    const unsigned rt = gswa::bwd::kD * gswa::bwd::kReduceSlices;
    gswa::bwd::dw_reduce_kernel<<<1, rt, 0, st>>>(part_q, (int)gq * 4, dw_q);
    gswa::bwd::dw_reduce_kernel<<<1, rt, 0, st>>>(part_k, (int)gk * 4, dw_k);
    return cudaGetLastError() == cudaSuccess ? GSWA_OK : GSWA_ERR_LAUNCH;
}

// Argument checks of full_decode and full_decode_noalloc (everything but the
// scratch they run on).
int check_full_decode(const gswa_shape_t *s, const void *q, const void *k, const void *v, const void *w_q,
                      const void *w_k, const void *k_cache, const void *v_cache, const int64_t *pos,
                      const void *y)
{
    if (s == nullptr || s->B < 0 || s->Hq <= 0 || s->Hkv <= 0 || s->cache_len < 1) return GSWA_ERR_INVALID_ARG;
    if (!(s->eps >= 0.f) || !(s->rope_base > 0.0) || !std::isfinite(s->scale)) return GSWA_ERR_INVALID_ARG;
    if (s->D != 128 || s->Hq != 4 * s->Hkv || s->rope_dims < 0 || s->rope_dims > s->D || (s->rope_dims & 1))
        return GSWA_ERR_UNSUPPORTED_SHAPE;
    if (s->B == 0) return GSWA_OK;
    if (!q || !k || !v || !w_q || !w_k || !k_cache || !v_cache || !pos || !y) return GSWA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned16(y) || (reinterpret_cast<uintptr_t>(pos) & 7u))
        return GSWA_ERR_MISALIGNED;
    const long long cache_rows = (long long)s->B * s->Hkv * s->cache_len;
    if (cache_rows + gswa::dec::kStageKeys > 0x7fffffffLL) return GSWA_ERR_UNSUPPORTED_SHAPE;   // TMA row coordinates
    return GSWA_OK;
}

// The three launches of a full-cache decode step, on `scratch` laid out as
// full_decode_ws() describes: q~ [B, Hq, D] f32, then the chunk partials.
int launch_full_decode(const gswa_shape_t *s, const void *q, const void *k, const void *v, const void *w_q,
                       const void *w_k, void *k_cache, void *v_cache, const int64_t *pos, void *y, void *scratch,
                       cudaStream_t st)
{
    gswa::dec::Params p;
    fill_dec(p, s);
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.k = static_cast<const __nv_bfloat16 *>(k);
    p.v = static_cast<const __nv_bfloat16 *>(v);
    p.wq = static_cast<const __nv_bfloat16 *>(w_q);
    p.wk = static_cast<const __nv_bfloat16 *>(w_k);
    p.kc = static_cast<__nv_bfloat16 *>(k_cache);
    p.vc = static_cast<__nv_bfloat16 *>(v_cache);
    p.pos = pos;
    p.y = static_cast<__nv_bfloat16 *>(y);
    p.qt = static_cast<float *>(scratch);
    p.part = reinterpret_cast<float *>(static_cast<char *>(scratch) + align256((size_t)s->B * s->Hq * s->D * 4));
    CUtensorMap tkc, tvc;
    const long long cache_rows = (long long)s->B * s->Hkv * s->cache_len;
    if (encode_rows(&tkc, k_cache, cache_rows, gswa::dec::kStageKeys) ||
        encode_rows(&tvc, v_cache, cache_rows, gswa::dec::kStageKeys))
        return GSWA_ERR_INVALID_ARG;
    gswa::dec::full_decode_prep_kernel<<<s->B * s->Hkv, 128, 0, st>>>(p);
    gswa::dec::full_decode_chunk_kernel<<<dim3(p.nchunks, s->B * s->Hkv), gswa::dec::kChunkThreads,
                                          gswa::dec::kDecSmemBytes, st>>>(tkc, tvc, p);
    gswa::dec::full_decode_combine_kernel<<<s->B * s->Hq, gswa::dec::kD, 0, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? GSWA_OK : GSWA_ERR_LAUNCH;
}

}  // namespace

extern "C" {

int gswa_fwd(const gswa_shape_t *s, const void *q, const void *k, const void *v, const void *g,
             const void *w_q, const void *w_k, void *y, float *lse, void *workspace,
             size_t workspace_bytes, void *stream)
{
    int rc = check_common(s);
    if (rc != GSWA_OK) return rc;
    if (s->window < 1 || s->window > 128) return GSWA_ERR_UNSUPPORTED_SHAPE;
    if (!rope_dims_supported(s->rope_dims)) return GSWA_ERR_UNSUPPORTED_SHAPE;
    if ((long long)s->B * s->T == 0) return GSWA_OK;
    if (!q || !k || !v || !g || !w_q || !w_k || !y) return GSWA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(y) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return GSWA_ERR_MISALIGNED;
    if (workspace == nullptr || workspace_bytes < swa_fwd_ws(s)) return GSWA_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(workspace)) return GSWA_ERR_MISALIGNED;
    int num_sms = 0;
    rc = device_setup(&num_sms);
    if (rc != GSWA_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    // k~ = RoPE(RMSNorm(k) w_k) once into the workspace: each key block is
    // read by five consecutive query blocks.
    void *kt = workspace;
    rc = launch_qk_prep(s, s->Hkv, k, w_k, kt, 0, st, num_sms);
    if (rc != GSWA_OK) return rc;

    CUtensorMap tq, tk, tv, tg, ty;
    if (encode_bthd(&tq, q, s->B, s->T, s->Hq, s->D, 4, 32) ||
        encode_bthd(&tg, g, s->B, s->T, s->Hq, s->D, 4, 32) ||
        encode_bthd(&ty, y, s->B, s->T, s->Hq, s->D, 4, 32) ||
        encode_bthd(&tk, kt, s->B, s->T, s->Hkv, s->D, 1, 32) ||
        encode_bthd(&tv, v, s->B, s->T, s->Hkv, s->D, 1, 32))
        return GSWA_ERR_INVALID_ARG;

    gswa::swa::Params p;
    std::memset(&p, 0, sizeof p);
    p.B = s->B;
    p.T = s->T;
    p.Hq = s->Hq;
    p.Hkv = s->Hkv;
    p.window = s->window;
    p.nsteps = (s->T + gswa::swa::kTok - 1) / gswa::swa::kTok;
    p.units = (long long)s->B * s->Hkv * p.nsteps;
    p.eps = s->eps;
    p.sl2 = s->scale * 1.4426950408889634f;
    p.wq = static_cast<const __nv_bfloat16 *>(w_q);
    p.wk = static_cast<const __nv_bfloat16 *>(w_k);
    p.lse = lse;
    fill_theta(p.theta, s->rope_dims, s->rope_base);

    const long long grid = p.units < num_sms ? p.units : num_sms;
    const dim3 gr((unsigned)grid), bl(gswa::swa::kThreads);
    const uint32_t sm = gswa::swa::kSmemBytes;
    switch (s->rope_dims) {
    case 0: gswa::swa::swa_fwd_kernel<0><<<gr, bl, sm, st>>>(tq, tk, tv, tg, ty, p); break;
    case 42: gswa::swa::swa_fwd_kernel<42><<<gr, bl, sm, st>>>(tq, tk, tv, tg, ty, p); break;
    case 64: gswa::swa::swa_fwd_kernel<64><<<gr, bl, sm, st>>>(tq, tk, tv, tg, ty, p); break;
    default: gswa::swa::swa_fwd_kernel<128><<<gr, bl, sm, st>>>(tq, tk, tv, tg, ty, p); break;
    }
    return cudaGetLastError() == cudaSuccess ? GSWA_OK : GSWA_ERR_LAUNCH;
}

int full_attn_fwd(const gswa_shape_t *s, const void *q, const void *k, const void *v,
                  const void *w_q, const void *w_k, void *y, float *lse, void *workspace,
                  size_t workspace_bytes, void *stream)
{
    int rc = check_common(s);
    if (rc != GSWA_OK) return rc;
    if (!rope_dims_supported(s->rope_dims)) return GSWA_ERR_UNSUPPORTED_SHAPE;
    if ((long long)s->B * s->T == 0) return GSWA_OK;
    if (!q || !k || !v || !w_q || !w_k || !y) return GSWA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(y) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return GSWA_ERR_MISALIGNED;
    if (workspace == nullptr || workspace_bytes < full_fwd_ws(s)) return GSWA_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(workspace)) return GSWA_ERR_MISALIGNED;
    int num_sms = 0;
    rc = device_setup(&num_sms);
    if (rc != GSWA_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    // prepared keys and queries once, into the workspace
    void *kt = workspace;
    void *qt = static_cast<char *>(workspace) + full_fwd_ws_keys(s);
    rc = launch_qk_prep(s, s->Hkv, k, w_k, kt, 0, st, num_sms);
    if (rc == GSWA_OK) rc = launch_qk_prep(s, s->Hq, q, w_q, qt, 0, st, num_sms);
    if (rc != GSWA_OK) return rc;

    CUtensorMap tq, tk, tv;
    if (encode_bthd(&tq, qt, s->B, s->T, s->Hq, s->D, 4, 32) ||
        encode_bthd(&tk, kt, s->B, s->T, s->Hkv, s->D, 1, 128) ||
        encode_bthd(&tv, v, s->B, s->T, s->Hkv, s->D, 1, 128))
        return GSWA_ERR_INVALID_ARG;

    gswa::full::Params p;
    std::memset(&p, 0, sizeof p);
    p.B = s->B;
    p.T = s->T;
    p.Hq = s->Hq;
    p.Hkv = s->Hkv;
    p.nm = (s->T + gswa::full::kUnitTok - 1) / gswa::full::kUnitTok;
    p.nkt = (s->T + gswa::full::kKeys - 1) / gswa::full::kKeys;
    p.units = (long long)s->B * s->Hkv * p.nm;
    p.sl2 = s->scale * 1.4426950408889634f;
    p.wq = static_cast<const __nv_bfloat16 *>(w_q);
    p.wk = static_cast<const __nv_bfloat16 *>(w_k);
    p.y = static_cast<__nv_bfloat16 *>(y);
    p.lse = lse;

    const long long grid = p.units < num_sms ? p.units : num_sms;
    gswa::full::full_fwd_kernel<<<(unsigned)grid, gswa::full::kThreads, gswa::full::kSmemBytes, st>>>(tq, tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? GSWA_OK : GSWA_ERR_LAUNCH;
}

int gswa_qk_prep(const gswa_shape_t *s, int H, const void *x, const void *w, void *out, int64_t pos0,
                 void *stream)
{
    if (s == nullptr || H <= 0 || s->B < 0 || s->T < 0 || s->D != 128 || pos0 < 0)
        return s && s->D != 128 ? GSWA_ERR_UNSUPPORTED_SHAPE : GSWA_ERR_INVALID_ARG;
    if (!(s->eps >= 0.f) || !(s->rope_base > 0.0)) return GSWA_ERR_INVALID_ARG;
    if (!rope_dims_supported(s->rope_dims)) return GSWA_ERR_UNSUPPORTED_SHAPE;
    if ((long long)s->B * s->T == 0) return GSWA_OK;
    if (!x || !w || !out) return GSWA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(out)) return GSWA_ERR_MISALIGNED;
    int num_sms = 0;
    int rc = device_setup(&num_sms);
    if (rc != GSWA_OK) return rc;
    return launch_qk_prep(s, H, x, w, out, pos0, static_cast<cudaStream_t>(stream), num_sms);
}

int gswa_bwd(const gswa_shape_t *s, const void *q, const void *k, const void *v, const void *g,
             const void *w_q, const void *w_k, const void *y, const float *lse, const void *dy,
             void *dq, void *dk, void *dv, void *dg, float *dw_q, float *dw_k, void *workspace,
             size_t workspace_bytes, void *stream)
{
    return run_bwd(true, s, q, k, v, g, w_q, w_k, y, lse, dy, dq, dk, dv, dg, dw_q, dw_k, workspace,
                   workspace_bytes, static_cast<cudaStream_t>(stream));
}

int full_attn_bwd(const gswa_shape_t *s, const void *q, const void *k, const void *v,
                  const void *w_q, const void *w_k, const void *y, const float *lse,
                  const void *dy, void *dq, void *dk, void *dv, float *dw_q, float *dw_k,
                  void *workspace, size_t workspace_bytes, void *stream)
{
    return run_bwd(false, s, q, k, v, nullptr, w_q, w_k, y, lse, dy, dq, dk, dv, nullptr, dw_q, dw_k, workspace,
                   workspace_bytes, static_cast<cudaStream_t>(stream));
}

int gswa_decode(const gswa_shape_t *s, const void *q, const void *k, const void *v, const void *g,
                const void *w_q, const void *w_k, void *k_ring, void *v_ring, const int64_t *pos,
                void *y, void *workspace, size_t workspace_bytes, void *stream)
{
    (void)workspace;
    (void)workspace_bytes;
    if (s == nullptr || s->B < 0 || s->Hq <= 0 || s->Hkv <= 0) return GSWA_ERR_INVALID_ARG;
    if (!(s->eps >= 0.f) || !(s->rope_base > 0.0) || !std::isfinite(s->scale)) return GSWA_ERR_INVALID_ARG;
    if (s->D != 128 || s->Hq != 4 * s->Hkv || s->window < 1 || s->window > 128 ||
        s->rope_dims < 0 || s->rope_dims > s->D || (s->rope_dims & 1))
        return GSWA_ERR_UNSUPPORTED_SHAPE;
    if (s->B == 0) return GSWA_OK;
    if (!q || !k || !v || !g || !w_q || !w_k || !k_ring || !v_ring || !pos || !y) return GSWA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(k_ring) ||
        !aligned16(v_ring) || !aligned16(y) || (reinterpret_cast<uintptr_t>(pos) & 7u))
        return GSWA_ERR_MISALIGNED;
    int num_sms = 0;
    int rc = device_setup(&num_sms);
    if (rc != GSWA_OK) return rc;
    gswa::dec::Params p;
    fill_dec(p, s);
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.k = static_cast<const __nv_bfloat16 *>(k);
    p.v = static_cast<const __nv_bfloat16 *>(v);
    p.g = static_cast<const __nv_bfloat16 *>(g);
    p.wq = static_cast<const __nv_bfloat16 *>(w_q);
    p.wk = static_cast<const __nv_bfloat16 *>(w_k);
    p.kc = static_cast<__nv_bfloat16 *>(k_ring);
    p.vc = static_cast<__nv_bfloat16 *>(v_ring);
    p.pos = pos;
    p.y = static_cast<__nv_bfloat16 *>(y);
    // ring rows as TMA coordinates (32-bit)
    CUtensorMap tkr, tvr;
    const long long ring_rows = (long long)s->B * s->Hkv * s->window;
    if (ring_rows > 0x7fffffffLL) return GSWA_ERR_UNSUPPORTED_SHAPE;
    if (encode_rows(&tkr, k_ring, ring_rows, s->window) || encode_rows(&tvr, v_ring, ring_rows, s->window))
        return GSWA_ERR_INVALID_ARG;
    gswa::dec::swa_decode_kernel<<<s->B * s->Hkv, 128, gswa::dec::kSwaDecSmemBytes,
                                   static_cast<cudaStream_t>(stream)>>>(tkr, tvr, p);
    return cudaGetLastError() == cudaSuccess ? GSWA_OK : GSWA_ERR_LAUNCH;
}

int full_decode(const gswa_shape_t *s, const void *q, const void *k, const void *v,
                const void *w_q, const void *w_k, void *k_cache, void *v_cache,
                const int64_t *pos, void *y, void *workspace, size_t workspace_bytes,
                void *stream)
{
    int rc = check_full_decode(s, q, k, v, w_q, w_k, k_cache, v_cache, pos, y);
    if (rc != GSWA_OK || s->B == 0) return rc;
    if (workspace == nullptr || workspace_bytes < full_decode_ws(s)) return GSWA_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(workspace)) return GSWA_ERR_MISALIGNED;
    int num_sms = 0;
    rc = device_setup(&num_sms);
    if (rc != GSWA_OK) return rc;
    return launch_full_decode(s, q, k, v, w_q, w_k, k_cache, v_cache, pos, y, workspace,
                              static_cast<cudaStream_t>(stream));
}

int full_decode_noalloc(const gswa_shape_t *s, const void *q, const void *k, const void *v,
                        const void *w_q, const void *w_k, void *k_cache, void *v_cache,
                        const int64_t *pos, void *y, void *stream)
{
    int rc = check_full_decode(s, q, k, v, w_q, w_k, k_cache, v_cache, pos, y);
    if (rc != GSWA_OK || s->B == 0) return rc;
    // the same scratch layout full_decode takes from its workspace
    if (full_decode_ws(s) > GSWA_NOALLOC_SCRATCH_BYTES) return GSWA_ERR_SCRATCH_LIMIT;
    int num_sms = 0;
    rc = device_setup(&num_sms);
    if (rc != GSWA_OK) return rc;
    void *scratch = nullptr;
    rc = noalloc_scratch(&scratch);
    if (rc != GSWA_OK) return rc;
    return launch_full_decode(s, q, k, v, w_q, w_k, k_cache, v_cache, pos, y, scratch,
                              static_cast<cudaStream_t>(stream));
}

size_t gswa_workspace_bytes(int op, const gswa_shape_t *s)
{
    if (s == nullptr || s->B < 0 || s->T < 0 || s->Hkv <= 0 || s->D <= 0) return 0;
    switch (op) {
    case GSWA_OP_GSWA_FWD: return swa_fwd_ws(s);
    case GSWA_OP_FULL_FWD: return full_fwd_ws(s);
    case GSWA_OP_GSWA_BWD: return bwd_ws_layout(s, true).total;
    case GSWA_OP_FULL_BWD: return full_bwd_ws_layout(s).total;
    case GSWA_OP_FULL_DECODE: return s->cache_len > 0 ? full_decode_ws(s) : 0;
    default: return 0;
    }
}

int64_t gswa_kv_cache_bytes(int n_global_layers, int n_window_layers, int window, int Hkv, int D,
                            int bytes_per_elem, int64_t T)
{
    if (n_global_layers < 0 || n_window_layers < 0 || window < 0 || Hkv < 0 || D < 0 ||
        bytes_per_elem < 0 || T < 0)
        return -1;
    const int64_t per_token = 2LL * Hkv * D * bytes_per_elem;
    const int64_t swa_tokens = T < window ? T : window;
    return per_token * ((int64_t)n_global_layers * T + (int64_t)n_window_layers * swa_tokens);
}

int gswa_check_status(void *stream)
{
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return GSWA_ERR_LAUNCH;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, gswa::g_status, sizeof v) != cudaSuccess) return GSWA_ERR_LAUNCH;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(gswa::g_status, &zero, sizeof zero) != cudaSuccess) return GSWA_ERR_LAUNCH;
        return v == gswa::kStatusBadArg ? GSWA_ERR_INVALID_ARG
                                        : v == gswa::kStatusSetup ? GSWA_ERR_LAUNCH : GSWA_ERR_TIMEOUT;
    }
    return GSWA_OK;
}

int gswa_set_wait_limit_ns(uint64_t ns)
{
    const unsigned long long v = ns == 0 ? gswa::kWaitLimitNs : (unsigned long long)ns;
    if (cudaMemcpyToSymbol(gswa::g_wait_limit_ns, &v, sizeof v) != cudaSuccess) return GSWA_ERR_LAUNCH;
    return cudaDeviceSynchronize() == cudaSuccess ? GSWA_OK : GSWA_ERR_LAUNCH;
}

const char *gswa_strerror(int code)
{
    switch (code) {
    case GSWA_OK: return "ok";
    case GSWA_ERR_INVALID_ARG: return "invalid argument";
    case GSWA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case GSWA_ERR_MISALIGNED: return "misaligned pointer";
    case GSWA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case GSWA_ERR_LAUNCH: return "CUDA launch or runtime error";
    case GSWA_ERR_TIMEOUT: return "a bounded device wait timed out";
    case GSWA_ERR_UNIMPLEMENTED: return "not implemented";
    case GSWA_ERR_NO_DEVICE: return "no sm_100 device is current";
    case GSWA_ERR_SCRATCH_LIMIT: return "shape needs more than the fixed 36 MiB scratch of full_decode_noalloc";
    default: return "unknown error";
    }
}

}  // extern "C"
