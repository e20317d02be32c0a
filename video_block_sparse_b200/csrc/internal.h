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
cudaError_t launch_tile(const uint16_t* x_grid, uint16_t* x_tiled, int B, const CubeGeom& g, int row_elems,
                        cudaStream_t s);
cudaError_t launch_untile(const uint16_t* x_tiled, uint16_t* x_grid, int B, const CubeGeom& g, int row_elems,
                          cudaStream_t s);

// ---- route.cu
size_t route_workspace_bytes(int B, int H, int nq, int D);
cudaError_t launch_route(const uint16_t* q, const uint16_t* k, const int32_t* vbs, int32_t* topk_idx, int B, int S,
                         int H, int nq, int topk, void* workspace, int* err, cudaStream_t s);

// ---- fwd_mma.cu (warp-level mma.sync kernel)
cudaError_t launch_fwd_mma(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* topk_idx,
                           const int32_t* vbs, uint16_t* out, float* lse, int B, int S, int H, int nq, int topk,
                           float sm_scale, bool precise_p, int* err, cudaStream_t s);

// ---- fwd_tc.cu (tcgen05 / TMEM / TMA kernel)
cudaError_t launch_fwd_tc(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* topk_idx,
                          const int32_t* vbs, uint16_t* out, float* lse, int B, int S, int H, int nq, int topk,
                          float sm_scale, bool precise_p, int* err, cudaStream_t s);

// ---- fwd_pair.cu (tcgen05 kernel, two query cubes per 128-row tile)
bool fwd_pair_supported(int nq, int topk);
// the variant with one MMA issuer shared by both tiles (fwd_pair_precise.cu); runs the precise mode
cudaError_t launch_fwd_pair_shared(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* topk_idx,
                                   const int32_t* vbs, const int32_t* plan, uint16_t* out, float* lse, int B, int S,
                                   int H, int nq, int topk, float sm_scale, bool precise_p, int* err, cudaStream_t s);
cudaError_t launch_fwd_pair(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* topk_idx,
                            const int32_t* vbs, const int32_t* plan, uint16_t* out, float* lse, int B, int S, int H,
                            int nq, int topk, float sm_scale, bool precise_p, int* err, cudaStream_t s);

// ---- plan.cu (pairing of query cubes by selection overlap)
size_t plan_workspace_bytes(int B, int H, int nq);
cudaError_t launch_stall_check(int* err, int* result, cudaStream_t s);
cudaError_t launch_plan(const int32_t* topk_idx, int32_t* plan, int B, int H, int nq, int topk, void* workspace,
                        int* err, cudaStream_t s);

}  // namespace vsa
