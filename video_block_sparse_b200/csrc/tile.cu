// Cube-major 4x4x4 tiling and its inverse (dataset card
// "wan2.2_production_values", section "Shapes"; untiling as an index gather
// per TensorRT-LLM PR #7).
//
// Pure data movement, HBM-bound: each CTA copies whole token rows (H*D bf16,
// 10 KiB at H=40, D=128) with 16-byte loads/stores, so every warp touches
// 512 contiguous bytes per instruction.  Algorithmic traffic per call:
//   tile:   read B*T*Hh*W rows, write B*S rows   (pads written as zeros)
//   untile: read B*T*Hh*W rows, write B*T*Hh*W rows
#include "internal.h"

namespace vsa {

CubeGeom make_geom(int T, int Hh, int W)
{
    CubeGeom g;
    g.T = T;
    g.Hh = Hh;
    g.W = W;
    g.nct = (T + 3) / 4;
    g.nch = (Hh + 3) / 4;
    g.ncw = (W + 3) / 4;
    g.nq = g.nct * g.nch * g.ncw;
    return g;
}

namespace {

// Raster index of the token held in slot r of cube c, or -1 for a pad slot.
__device__ __forceinline__ int64_t slot_source(const CubeGeom g, int c, int r)
{
    int cw = c % g.ncw;
    int ch = (c / g.ncw) % g.nch;
    int ct = c / (g.ncw * g.nch);
    int et = min(4, g.T - 4 * ct), eh = min(4, g.Hh - 4 * ch), ew = min(4, g.W - 4 * cw);
    if (r >= et * eh * ew) return -1;
    int lw = r % ew, lh = (r / ew) % eh, lt = r / (ew * eh);
    return ((int64_t)(4 * ct + lt) * g.Hh + (4 * ch + lh)) * g.W + (4 * cw + lw);
}

__device__ __forceinline__ int64_t raster_slot(const CubeGeom g, int64_t p)
{
    int w = (int)(p % g.W);
    int h = (int)((p / g.W) % g.Hh);
    int t = (int)(p / ((int64_t)g.W * g.Hh));
    int ct = t >> 2, ch = h >> 2, cw = w >> 2;
    int eh = min(4, g.Hh - 4 * ch), ew = min(4, g.W - 4 * cw);
    int c = (ct * g.nch + ch) * g.ncw + cw;
    return (int64_t)c * 64 + ((t - 4 * ct) * eh + (h - 4 * ch)) * ew + (w - 4 * cw);
}

// One destination row per loop trip; threads stride over its 16-byte chunks.
__global__ void __launch_bounds__(256) tile_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int B,
                                                   CubeGeom g, int row16)
{
    const int64_t S = 64LL * g.nq, L = (int64_t)g.T * g.Hh * g.W;
    const int64_t rows = (int64_t)B * S;
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
        int b = (int)(row / S);
        int s = (int)(row % S);
        int64_t p = slot_source(g, s >> 6, s & 63);
        uint4* d = dst + row * row16;
        if (p < 0) {
            for (int i = threadIdx.x; i < row16; i += blockDim.x) d[i] = make_uint4(0, 0, 0, 0);
        } else {
            const uint4* sp = src + ((int64_t)b * L + p) * row16;
            for (int i = threadIdx.x; i < row16; i += blockDim.x) d[i] = __ldg(sp + i);
        }
    }
}

__global__ void __launch_bounds__(256) untile_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int B,
                                                     CubeGeom g, int row16)
{
    const int64_t S = 64LL * g.nq, L = (int64_t)g.T * g.Hh * g.W;
    const int64_t rows = (int64_t)B * L;
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
        int b = (int)(row / L);
        int64_t p = row % L;
        const uint4* sp = src + ((int64_t)b * S + raster_slot(g, p)) * row16;
        uint4* d = dst + row * row16;
        for (int i = threadIdx.x; i < row16; i += blockDim.x) d[i] = __ldg(sp + i);
    }
}

int grid_for(int64_t rows)
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t g = (int64_t)sms * 8;  // 8 resident 256-thread CTAs per SM
    return (int)(rows < g ? rows : g);
}

}  // namespace

cudaError_t launch_tile(const uint16_t* x_grid, uint16_t* x_tiled, int B, const CubeGeom& g, int row_elems,
                        cudaStream_t s)
{
    int64_t rows = (int64_t)B * 64 * g.nq;
    int row16 = row_elems / 8;
    int threads = row16 >= 256 ? 256 : ((row16 + 31) / 32) * 32;
    tile_kernel<<<grid_for(rows), threads, 0, s>>>(reinterpret_cast<const uint4*>(x_grid),
                                                   reinterpret_cast<uint4*>(x_tiled), B, g, row16);
    return cudaGetLastError();
}

cudaError_t launch_untile(const uint16_t* x_tiled, uint16_t* x_grid, int B, const CubeGeom& g, int row_elems,
                          cudaStream_t s)
{
    int64_t rows = (int64_t)B * g.T * g.Hh * g.W;
    int row16 = row_elems / 8;
    int threads = row16 >= 256 ? 256 : ((row16 + 31) / 32) * 32;
    untile_kernel<<<grid_for(rows), threads, 0, s>>>(reinterpret_cast<const uint4*>(x_tiled),
                                                     reinterpret_cast<uint4*>(x_grid), B, g, row16);
    return cudaGetLastError();
}

}  // namespace vsa
