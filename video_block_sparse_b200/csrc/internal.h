// Internal launcher declarations shared by the CUDA translation units of
// libvsa.  Launchers assume arguments were validated by the C-ABI layer
// (api.cu) and only enqueue kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace vsa {

// device error codes latched in the library's error word
enum DeviceError : int {
    kErrNone = 0,
    kErrTopkIdx = 1,
    kErrVbs = 2,
    kErrWaitTimeout = 3,
    kErrPlan = 4,
};

struct CubeGeom {
    int T, Hh, W;     // latent grid extents
    int nct, nch, ncw;  // cubes per axis
    int nq;           // cube count
};

CubeGeom make_geom(int T, int Hh, int W);

// ---- tile.cu
struct TileJob {
    const uint4* src[3];   // raster tensors [B, T*Hh*W, H, D]
    uint4* dst[3];         // tiled tensors [B, 64*Nq, H, D]
    uint16_t* means[3];    // cube means [B, H, Nq, D] bf16, or nullptr
    int sums[3];           // 1: that buffer gets the cube sums instead of the means
};
cudaError_t launch_tile_cubes(const TileJob& job, int n_tensors, const int32_t* vbs, int B, const CubeGeom& g, int H,
                              int D, int* err, cudaStream_t s);
cudaError_t launch_tile(const uint16_t* x_grid, uint16_t* x_tiled, int B, const CubeGeom& g, int row_elems,
                        cudaStream_t s);
cudaError_t launch_untile(const uint16_t* x_tiled, uint16_t* x_grid, int B, const CubeGeom& g, int row_elems,
                          cudaStream_t s);

// ---- route.cu
size_t route_workspace_bytes(int B, int H, int nq, int D);
cudaError_t launch_route(const uint16_t* q, const uint16_t* k, const int32_t* vbs, int32_t* topk_idx, int B, int S,
                         int H, int nq, int topk, void* workspace, int* err, cudaStream_t s);
// vsa_route's argument checks other than the workspace (api.cu)
int route_check_args(const uint16_t* q, const uint16_t* k, const int32_t* vbs, const int32_t* topk_idx, int B, int S,
                     int H, int D, int Nq, int topk);
// scores and top-k from cube means qc, kc [B, H, Nq, 128] bf16
cudaError_t launch_score_topk(const uint16_t* qc, const uint16_t* kc, int32_t* topk_idx, int B, int H, int nq,
                              int topk, cudaStream_t s);

// ---- fwd_pair.cu (tcgen05 kernel, two query cubes per 128-row tile)
bool fwd_pair_supported(int nq, int topk);
// kc, vc: the proxies' mean keys and summed values [B, H, Nq, 128] (both NULL: no proxies)
cudaError_t launch_fwd_pair(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* topk_idx,
                            const int32_t* vbs, const int32_t* plan, const uint16_t* kc, const uint16_t* vc,
                            uint16_t* out, float* lse, int B, int S, int H, int nq, int topk, float sm_scale,
                            bool precise_p, int* err, cudaStream_t s);

// ---- plan.cu (pairing of query cubes by selection overlap)
size_t plan_workspace_bytes(int B, int H, int nq);
cudaError_t launch_stall_check(int* err, int* result, cudaStream_t s);
cudaError_t launch_plan(const int32_t* topk_idx, int32_t* plan, int B, int H, int nq, int topk, void* workspace,
                        int* err, cudaStream_t s);

}  // namespace vsa
