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
    kErrRoute = 5,  // a BSR row outside the index array or longer than 1024, or a bitmap row of more than 1024 cubes
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

// The forward's selections, row r = (b*H + h)*Nq + i for query cube i: fixed-length
// lists (topk_idx [B, H, Nq, topk]), BSR rows (indices[indptr[r] .. indptr[r+1]), nnz
// entries in all), or packed UInt32 bitmaps ([B, H, Nq, words], bit c % 32 of word c / 32
// selects cube c).
enum RouteKind : int { kRouteLists = 0, kRouteBsr = 1, kRouteMask = 2, kRouteAll = 3 };  // all: every KV cube
struct Routes {
    const int32_t* idx;     // lists: topk_idx; BSR: indices
    const int32_t* indptr;  // BSR: [B*H*Nq + 1]
    const uint32_t* mask;   // bitmaps
    int kind;
    int topk;   // lists: row length
    int nnz;    // BSR: entries of indices
    int words;  // bitmaps: words per row, ceil(Nq / 32)
};

// kc, vc: the proxies' mean keys and summed values [B, H, Nq, 128] (both NULL: no proxies)
// S_kv, nkv: the key/value sequence's tokens and cubes (the query sequence's for the fine
// stage); vbs NULL: every KV cube full but the last, which holds S_kv - 64 (nkv - 1) tokens
cudaError_t launch_fwd_pair(const uint16_t* q, const uint16_t* k, const uint16_t* v, const Routes& rt,
                            const int32_t* vbs, const int32_t* plan, const uint16_t* kc, const uint16_t* vc,
                            uint16_t* out, float* lse, int B, int S, int H, int nq, int S_kv, int nkv, float sm_scale,
                            bool precise_p, int* err, cudaStream_t s);

// ---- plan.cu (pairing of query cubes by selection overlap)
size_t plan_workspace_bytes(int B, int H, int nq);
cudaError_t launch_stall_check(int* err, int* result, cudaStream_t s);
cudaError_t launch_plan(const int32_t* topk_idx, int32_t* plan, int B, int H, int nq, int topk, void* workspace,
                        int* err, cudaStream_t s);

}  // namespace vsa
