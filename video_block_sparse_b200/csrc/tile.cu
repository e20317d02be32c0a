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

// Mean of 8 FP64 column sums over n slots, rounded to bf16 (nearest even) in
// one step, packed in pairs; 0 for an empty cube.  The rounding is the one the
// routing uses (route.cu): the two files must agree bit for bit.
__device__ __forceinline__ uint16_t mean_bf16(double sum, int n)
{
    if (n == 0) return 0;
    const double x = sum / (double)n;
    const uint64_t u = (uint64_t)__double_as_longlong(x);
    const uint16_t sign = (uint16_t)((u >> 48) & 0x8000u);
    const uint64_t a = u & 0x7FFFFFFFFFFFFFFFull;
    if (a > 0x7FF0000000000000ull) return 0x7FC0;
    if (a == 0x7FF0000000000000ull) return sign | 0x7F80;
    const int e = (int)(a >> 52) - 1023;
    if (e >= -126) {
        const uint64_t lsb = (a >> 45) & 1ull;
        uint64_t r = a + ((1ull << 44) - 1ull) + lsb;
        r &= ~((1ull << 45) - 1ull);
        const int e2 = (int)(r >> 52) - 1023;
        if (e2 > 127) return sign | 0x7F80;
        return sign | (uint16_t)((uint32_t)(e2 + 127) << 7) | (uint16_t)((r >> 45) & 0x7Fu);
    }
    const double m = rint(__longlong_as_double((long long)a) * 0x1p133);
    return sign | (uint16_t)m;
}

__device__ __forceinline__ void add_bf16x8(double (&acc)[8], const uint4 w)
{
    const uint32_t p[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        acc[2 * e] += (double)__uint_as_float(p[e] << 16);
        acc[2 * e + 1] += (double)__uint_as_float(p[e] & 0xFFFF0000u);
    }
}

// Tiling of up to three tensors in one launch, one CTA per (cube, batch x
// column block, tensor): threads own 16-byte columns of the token rows and
// walk the cube's 64 slots, so a warp reads and writes 512 contiguous bytes
// per instruction; each thread keeps eight loads in flight.  The raster
// offsets of the cube's slots are computed once per CTA.  For a tensor with a
// means buffer the same pass also forms the cube mean: FP64 sums over slots
// 0 .. vbs[c] - 1 in slot order (pads count as zeros), divided by vbs[c] and
// rounded to bf16, into [B, H, Nq, D] -- the routing's means, without reading
// the tiled tensor again (for a sums buffer, the sum itself rounded to bf16:
// the summed values of proxy compensation).
constexpr int kTileCols = 320;  // 16-byte columns per CTA
constexpr int kTileUnroll = 8;

__global__ void __launch_bounds__(kTileCols) tile_cubes_kernel(TileJob job, const int32_t* __restrict__ vbs,
                                                               CubeGeom g, int B, int H, int D, int row16, int* err)
{
    __shared__ int64_t slot_off[64];  // raster row of slot r minus that of slot 0 (pads: unused)
    const int c = blockIdx.x, t = blockIdx.z;
    const int n_blk = (row16 + kTileCols - 1) / kTileCols;
    const int b = blockIdx.y / n_blk, col = (blockIdx.y % n_blk) * kTileCols + threadIdx.x;
    // selects, not an indexed parameter array (which would go through local memory)
    const uint4* __restrict__ src = t == 0 ? job.src[0] : (t == 1 ? job.src[1] : job.src[2]);
    uint4* __restrict__ dst = t == 0 ? job.dst[0] : (t == 1 ? job.dst[1] : job.dst[2]);
    uint16_t* __restrict__ xm = t == 0 ? job.means[0] : (t == 1 ? job.means[1] : job.means[2]);
    const int as_sum = t == 0 ? job.sums[0] : (t == 1 ? job.sums[1] : job.sums[2]);
    const int cw = c % g.ncw, ch = (c / g.ncw) % g.nch, ct = c / (g.ncw * g.nch);
    const int et = min(4, g.T - 4 * ct), eh = min(4, g.Hh - 4 * ch), ew = min(4, g.W - 4 * cw);
    const int n_real = et * eh * ew;
    if (threadIdx.x < 64) {
        const int r = threadIdx.x, lw = r % ew, lh = (r / ew) % eh, lt = r / (ew * eh);
        slot_off[r] = ((int64_t)lt * g.Hh + lh) * g.W + lw;
    }
    int n_mean = 0;
    if (xm != nullptr) {
        n_mean = __ldg(vbs + c);
        if (n_mean < 0 || n_mean > 64) {
            if (threadIdx.x == 0 && blockIdx.y == 0) atomicCAS(err, 0, (int)kErrVbs);
            n_mean = 0;
        }
    }
    __syncthreads();
    if (col >= row16) return;
    const int64_t L = (int64_t)g.T * g.Hh * g.W, S = 64LL * g.nq;
    const int64_t p0 = ((int64_t)(4 * ct) * g.Hh + 4 * ch) * g.W + 4 * cw;  // raster index of slot 0
    const uint4* sp = src + ((int64_t)b * L + p0) * row16 + col;
    uint4* dp = dst + ((int64_t)b * S + 64LL * c) * row16 + col;
    double acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0;
    for (int r0 = 0; r0 < 64; r0 += kTileUnroll) {
        uint4 w[kTileUnroll];
#pragma unroll
        for (int u = 0; u < kTileUnroll; ++u)
            w[u] = r0 + u < n_real ? __ldg(sp + slot_off[r0 + u] * row16) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < kTileUnroll; ++u) {
            dp[(int64_t)(r0 + u) * row16] = w[u];
            if (r0 + u < n_mean) add_bf16x8(acc, w[u]);
        }
    }
    if (xm != nullptr) {
        // the sum rounds as the mean of one (the division by 1 is exact); empty cubes give 0
        const int div = as_sum ? (n_mean > 0 ? 1 : 0) : n_mean;
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            o[e] = (uint32_t)mean_bf16(acc[2 * e], div) | ((uint32_t)mean_bf16(acc[2 * e + 1], div) << 16);
        const int h = (col * 8) / D, d = (col * 8) % D;
        *reinterpret_cast<uint4*>(xm + (((int64_t)b * H + h) * g.nq + c) * D + d) = make_uint4(o[0], o[1], o[2], o[3]);
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

cudaError_t launch_tile_cubes(const TileJob& job, int n_tensors, const int32_t* vbs, int B, const CubeGeom& g, int H,
                              int D, int* err, cudaStream_t s)
{
    const int row16 = H * D / 8;
    const int n_blk = (row16 + kTileCols - 1) / kTileCols;
    tile_cubes_kernel<<<dim3(g.nq, B * n_blk, n_tensors), kTileCols, 0, s>>>(job, vbs, g, B, H, D, row16, err);
    return cudaGetLastError();
}

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
