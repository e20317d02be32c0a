// vsa_route_noalloc: the cube-mean routing of vsa_route with its scratch
// (the bf16 cube means of q and k) kept in a fixed array that is part of the
// library itself, for callers that cannot allocate device memory.
//
// Such callers include code that runs while a CUDA graph is being captured
// with a relaxed or thread-local capture mode forbidding cudaMalloc, plugins
// and runtimes that receive only pre-allocated input/output buffers from a
// host framework, and embedded deployments that pin every device allocation
// at start-up.  They still pass q, k, vbs and topk_idx; the library supplies
// the scratch.
//
// The array below is a file-scope __device__ variable: every GPU that loads
// this library's module holds kScratchBytes of it until the process exits.
// Host code cannot use the variable's name as a device address, so the first
// call on each device looks the address up with cudaGetSymbolAddress (with
// that device current) and caches it.  The cache slots are atomics: host
// threads making their first calls at the same time store the same address.
#include "vsa.h"

#include "internal.h"

#include <atomic>

namespace {

// 16 MiB: room for the means of B * H * Nq <= 32768 query/KV cubes
// (two bf16 [B, H, Nq, 128] arrays), e.g. the Wan2.2 832x480 shape
// (1 x 40 x 624).
constexpr size_t kScratchBytes = size_t(16) << 20;

static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];

}  // namespace

extern "C" {

VSA_API int vsa_route_noalloc(const vsa_bf16* q, const vsa_bf16* k, const int32_t* vbs, int32_t* topk_idx, int B,
                              int S, int H, int D, int Nq, int topk, cudaStream_t stream)
{
    // vsa_route's own checks first (arguments, then the device's architecture),
    // so that a bad call gets the same error as from vsa_route
    const int rc = vsa::route_check_args(q, k, vbs, topk_idx, B, S, H, D, Nq, topk);
    if (rc != VSA_OK) return rc;
    if (vsa_route_workspace_size(B, H, Nq, D) > kScratchBytes) return VSA_ERR_WORKSPACE;  // the array is too small
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return VSA_ERR_LAUNCH;
    void* scratch = g_scratch_addr[dev].load(std::memory_order_relaxed);
    if (scratch == nullptr) {
        if (cudaGetSymbolAddress(&scratch, g_route_scratch) != cudaSuccess || scratch == nullptr) return VSA_ERR_LAUNCH;
        g_scratch_addr[dev].store(scratch, std::memory_order_relaxed);
    }
    // vsa_route overwrites the whole scratch region it uses before reading it,
    // so no clearing is needed here.
    return vsa_route(q, k, vbs, topk_idx, B, S, H, D, Nq, topk, scratch, kScratchBytes, stream);
}

}  // extern "C"
