// qk_prep.cuh -- stand-alone QK-RMSNorm + partial RoPE of a head tensor.
//
// ZGCM-1 §2.1 Figure 3 caption: RMS normalisation and partial RoPE act on the
// query/key branches.  out[b,t,h,:] = RoPE_{pos0+t}(RMSNorm(x[b,t,h,:]) * w),
// bf16 in, bf16 out (rounded once from f32).  Used for the keys of the full
// causal layers (a key tile is reused by every later query block, so it is
// prepared once rather than inside the attention loop) and to fill decode
// caches, which hold prepared keys.
//
// One warp per 32 consecutive rows: the rows are staged in shared memory with
// coalesced 16-byte loads, in the swizzled layout the attention prologue uses,
// and prep_row runs on them (one lane per row, cos/sin evaluated per pair).
#pragma once

#include "ptx.cuh"
#include "swa_fwd.cuh"

namespace gswa {
namespace prep {

constexpr int kWarps = 4;   // 4 x 8 KiB of static shared memory
constexpr uint32_t kRowsPerWarp = 32;
constexpr uint32_t kHalf = kRowsPerWarp * 128;      // 4096 B: 32 rows x 64 dims
constexpr uint32_t kWarpBytes = 2 * kHalf;          // 8192 B

struct Params {
    const __nv_bfloat16 *x;
    __nv_bfloat16 *out;
    const __nv_bfloat16 *w;
    long long rows;   // B * T * H
    int T, H;
    long long pos0;
    float eps;
    double theta[64];
};

// cos/sin of pair pp at a fixed position, evaluated directly.
template <int H>
struct RopeRow {
    int pos = 0;
    const double *theta = nullptr;
    __device__ __forceinline__ void get(int, int pp, float &c, float &sn) const
    {
        swa::rope_cs(theta[pp], pos, c, sn);
    }
};

template <int R>
__global__ void __launch_bounds__(kWarps * 32)
qk_prep_kernel(const __grid_constant__ Params p)
{
    __shared__ __align__(1024) uint8_t stage[kWarps * kWarpBytes];
    __shared__ __align__(16) float wsm[128];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x < 128) wsm[threadIdx.x] = __bfloat162float(p.w[threadIdx.x]);
    __syncthreads();
    const uint32_t tile = smem_u32(stage) + warp * kWarpBytes;
    const uint4 *src = reinterpret_cast<const uint4 *>(p.x);
    uint4 *dst = reinterpret_cast<uint4 *>(p.out);
    const long long ngroups = (p.rows + kRowsPerWarp - 1) / kRowsPerWarp;
    for (long long grp = (long long)blockIdx.x * kWarps + warp; grp < ngroups;
         grp += (long long)gridDim.x * kWarps) {
        const long long row0 = grp * kRowsPerWarp;
        const int nrows = (int)min((long long)kRowsPerWarp, p.rows - row0);
        // coalesced load: lane l takes 16-byte chunk l % 16 of row 2 i + l / 16
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
            const int rr = 2 * i + (lane >> 4), c = lane & 15;
            if (rr < nrows) sts128(tile + swa::chunk_off(rr, c, kHalf), src[(row0 + rr) * 16 + c]);
        }
        __syncwarp();
        if (lane < nrows) {
            const long long row = row0 + lane;
            RopeRow<R / 2> tab;
            tab.pos = (int)(p.pos0 + (row / p.H) % p.T);
            tab.theta = p.theta;
            swa::prep_row<R, false>(tile, kHalf, lane, wsm, p.eps, tab);
        }
        __syncwarp();
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
            const int rr = 2 * i + (lane >> 4), c = lane & 15;
            if (rr < nrows) dst[(row0 + rr) * 16 + c] = lds128(tile + swa::chunk_off(rr, c, kHalf));
        }
        __syncwarp();
    }
}

}  // namespace prep
}  // namespace gswa
