// C ABI of libvsa (declared in include/vsa.h): argument validation, the
// device error word, and dispatch to the kernel launchers.  Nothing here
// allocates memory or synchronises, except vsa_device_status.
#include "vsa.h"

#include "internal.h"

#include <atomic>
#include <climits>
#include <cstdint>

namespace {

// One error word per device; kernels latch the first error with atomicCAS.
__device__ int g_device_error;

// Per-device values looked up on first use.  Host threads may make their first
// calls at the same time: each slot is an atomic, and racing threads store the
// same value.
constexpr int kMaxDevices = 64;
std::atomic<int*> g_err_ptr[kMaxDevices];
std::atomic<int> g_sm_version[kMaxDevices];

int current_device(int* dev)
{
    if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= kMaxDevices) return VSA_ERR_LAUNCH;
    return VSA_OK;
}

int device_sm(int dev)
{
    int sm = g_sm_version[dev].load(std::memory_order_relaxed);
    if (sm == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return -1;
        sm = major * 10 + minor;
        g_sm_version[dev].store(sm, std::memory_order_relaxed);
    }
    return sm;
}

// Address of this device's error word (looked up once per device).
int device_error_word(int** out)
{
    int dev;
    if (current_device(&dev) != VSA_OK) return VSA_ERR_LAUNCH;
    int* p = g_err_ptr[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
        void* a = nullptr;
        if (cudaGetSymbolAddress(&a, g_device_error) != cudaSuccess || a == nullptr) return VSA_ERR_LAUNCH;
        p = static_cast<int*>(a);
        g_err_ptr[dev].store(p, std::memory_order_relaxed);
    }
    *out = p;
    return VSA_OK;
}

int check_arch()
{
    int dev;
    if (current_device(&dev) != VSA_OK) return VSA_ERR_LAUNCH;
    return device_sm(dev) == 100 ? VSA_OK : VSA_ERR_ARCH;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int launch_status(cudaError_t e) { return e == cudaSuccess ? VSA_OK : VSA_ERR_LAUNCH; }

// Shared checks of the attention-shaped calls.
int check_bshd(int B, int S, int H, int D, int Nq)
{
    if (B < 1 || H < 1 || Nq < 1 || D != 128) return VSA_ERR_ARG;
    if ((int64_t)Nq * 64 != (int64_t)S) return VSA_ERR_ARG;
    if ((int64_t)B * S * H * D > (int64_t)INT32_MAX * 8) return VSA_ERR_ARG;
    if ((int64_t)B * H * Nq > INT32_MAX) return VSA_ERR_ARG;
    return VSA_OK;
}

int fwd_dispatch(const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v, const vsa::Routes& rt,
                 const int32_t* vbs, const int32_t* plan, const vsa_bf16* kc, const vsa_bf16* vc, vsa_bf16* out,
                 float* lse, int B, int S, int H, int D, int Nq, float sm_scale, int flags, cudaStream_t stream);

}  // namespace

extern "C" {

const char* vsa_status_string(int status)
{
    switch (status) {
    case VSA_OK: return "VSA_OK";
    case VSA_ERR_ARG: return "VSA_ERR_ARG: size or count out of range";
    case VSA_ERR_NULL: return "VSA_ERR_NULL: required pointer is NULL";
    case VSA_ERR_ALIGN: return "VSA_ERR_ALIGN: pointer not 16-byte aligned";
    case VSA_ERR_WORKSPACE: return "VSA_ERR_WORKSPACE: workspace missing or too small";
    case VSA_ERR_ARCH: return "VSA_ERR_ARCH: device is not sm_100";
    case VSA_ERR_LAUNCH: return "VSA_ERR_LAUNCH: CUDA runtime error";
    case VSA_ERR_DEVICE: return "VSA_ERR_DEVICE: a kernel latched an error";
    default: return "unknown vsa status";
    }
}

int vsa_can_implement(int D, int sm_version) { return (D == 128 && sm_version == 100) ? 1 : 0; }

}  // extern "C"

namespace {

// Shared by every forward entry point: checks (sizes, then NULL pointers, then
// alignment, then the device), then the kernel.  rt: the selections in one of
// the three formats; kc and vc both NULL (plain) or both set (proxies).
int fwd_dispatch(const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v, const vsa::Routes& rt,
                 const int32_t* vbs, const int32_t* plan, const vsa_bf16* kc, const vsa_bf16* vc, vsa_bf16* out,
                 float* lse, int B, int S, int H, int D, int Nq, float sm_scale, int flags, cudaStream_t stream)
{
    int rc = check_bshd(B, S, H, D, Nq);
    if (rc != VSA_OK) return rc;
    const int64_t rows = (int64_t)B * H * Nq;
    if (rt.kind == vsa::kRouteLists) {
        if (rt.topk < 1 || (flags & ~VSA_FWD_PRECISE_P) != 0) return VSA_ERR_ARG;
        if (!vsa::fwd_pair_supported(Nq, rt.topk)) return VSA_ERR_ARG;
        if (rows * rt.topk > INT32_MAX) return VSA_ERR_ARG;
    } else {
        if ((flags & ~VSA_FWD_PRECISE_P) != 0 || !vsa::fwd_pair_supported(Nq, 1)) return VSA_ERR_ARG;
        if (rt.kind == vsa::kRouteBsr && (rt.nnz < 0 || rows + 1 > INT32_MAX)) return VSA_ERR_ARG;
        if (rt.kind == vsa::kRouteMask && rows * rt.words > INT32_MAX) return VSA_ERR_ARG;
    }
    const void* route_ptr = rt.kind == vsa::kRouteLists ? (const void*)rt.idx
                            : rt.kind == vsa::kRouteBsr ? (const void*)rt.indptr
                                                        : (const void*)rt.mask;
    if (!q || !k || !v || !route_ptr || !vbs || !out) return VSA_ERR_NULL;
    if (rt.kind == vsa::kRouteBsr && rt.nnz > 0 && !rt.idx) return VSA_ERR_NULL;
    if ((kc == nullptr) != (vc == nullptr)) return VSA_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(route_ptr) ||
        (rt.kind == vsa::kRouteBsr && rt.idx && !aligned16(rt.idx)) || !aligned16(vbs) || (lse && !aligned16(lse)) ||
        (plan && !aligned16(plan)) || (kc && !aligned16(kc)) || (vc && !aligned16(vc)))
        return VSA_ERR_ALIGN;
    if ((rc = check_arch()) != VSA_OK) return rc;
    int* err;
    if ((rc = device_error_word(&err)) != VSA_OK) return rc;
    const bool precise = (flags & VSA_FWD_PRECISE_P) != 0;
    return launch_status(vsa::launch_fwd_pair(q, k, v, rt, vbs, plan, kc, vc, out, lse, B, S, H, Nq, S, Nq, sm_scale,
                                              precise, err, stream));
}

vsa::Routes route_lists(const int32_t* topk_idx, int topk)
{
    vsa::Routes rt{};
    rt.idx = topk_idx;
    rt.kind = vsa::kRouteLists;
    rt.topk = topk;
    return rt;
}

}  // namespace

namespace vsa {

// The checks of vsa_route other than its workspace, in the same order.
int route_check_args(const uint16_t* q, const uint16_t* k, const int32_t* vbs, const int32_t* topk_idx, int B, int S,
                     int H, int D, int Nq, int topk)
{
    int rc = check_bshd(B, S, H, D, Nq);
    if (rc != VSA_OK) return rc;
    if (topk < 1 || topk > Nq || Nq > 4096) return VSA_ERR_ARG;
    if (!q || !k || !vbs || !topk_idx) return VSA_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(vbs) || !aligned16(topk_idx)) return VSA_ERR_ALIGN;
    return check_arch();
}

}  // namespace vsa

extern "C" {

int vsa_fwd_ex(const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v, const int32_t* topk_idx, const int32_t* vbs,
               vsa_bf16* out, float* lse, int B, int S, int H, int D, int Nq, int topk, float sm_scale, int flags,
               cudaStream_t stream)
{
    return fwd_dispatch(q, k, v, route_lists(topk_idx, topk), vbs, nullptr, nullptr, nullptr, out, lse, B, S, H, D, Nq,
                        sm_scale, flags, stream);
}

int vsa_fwd_planned(const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v, const int32_t* topk_idx,
                    const int32_t* vbs, const int32_t* plan, vsa_bf16* out, float* lse, int B, int S, int H, int D,
                    int Nq, int topk, float sm_scale, int flags, cudaStream_t stream)
{
    if (!plan) return VSA_ERR_NULL;
    return fwd_dispatch(q, k, v, route_lists(topk_idx, topk), vbs, plan, nullptr, nullptr, out, lse, B, S, H, D, Nq,
                        sm_scale, flags, stream);
}

int vsa_fwd_proxy(const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v, const int32_t* topk_idx,
                  const int32_t* vbs, const vsa_bf16* kc, const vsa_bf16* vc, const int32_t* plan, vsa_bf16* out,
                  float* lse, int B, int S, int H, int D, int Nq, int topk, float sm_scale, int flags,
                  cudaStream_t stream)
{
    if (!kc || !vc) return VSA_ERR_NULL;
    return fwd_dispatch(q, k, v, route_lists(topk_idx, topk), vbs, plan, kc, vc, out, lse, B, S, H, D, Nq, sm_scale,
                        flags, stream);
}

int vsa_fwd_bsr(const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v, const int32_t* block_indptr,
                const int32_t* block_indices, int nnz, const int32_t* vbs, const vsa_bf16* kc, const vsa_bf16* vc,
                const int32_t* plan, vsa_bf16* out, float* lse, int B, int S, int H, int D, int Nq, float sm_scale,
                int flags, cudaStream_t stream)
{
    vsa::Routes rt{};
    rt.idx = block_indices;
    rt.indptr = block_indptr;
    rt.kind = vsa::kRouteBsr;
    rt.nnz = nnz;
    return fwd_dispatch(q, k, v, rt, vbs, plan, kc, vc, out, lse, B, S, H, D, Nq, sm_scale, flags, stream);
}

int vsa_cross_attn(const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v, vsa_bf16* out, float* lse, int B, int S,
                   int S_kv, int H, int D, float sm_scale, int flags, cudaStream_t stream)
{
    if (S < 64 || S % 64 != 0) return VSA_ERR_ARG;
    int rc = check_bshd(B, S, H, D, S / 64);
    if (rc != VSA_OK) return rc;
    if ((flags & ~VSA_FWD_PRECISE_P) != 0 || !vsa::fwd_pair_supported(S / 64, 1)) return VSA_ERR_ARG;
    if (S_kv < 1 || S_kv > 64 * 1024 || (int64_t)B * S_kv * H * D > (int64_t)INT32_MAX * 8) return VSA_ERR_ARG;
    if (!q || !k || !v || !out) return VSA_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (lse && !aligned16(lse)))
        return VSA_ERR_ALIGN;
    if ((rc = check_arch()) != VSA_OK) return rc;
    int* err;
    if ((rc = device_error_word(&err)) != VSA_OK) return rc;
    vsa::Routes rt{};
    rt.kind = vsa::kRouteAll;
    const int nkv = (S_kv + 63) / 64;
    return launch_status(vsa::launch_fwd_pair(q, k, v, rt, nullptr, nullptr, nullptr, nullptr, out, lse, B, S, H, S / 64,
                                              S_kv, nkv, sm_scale, (flags & VSA_FWD_PRECISE_P) != 0, err, stream));
}

int vsa_fwd_bitmask(const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v, const uint32_t* mask,
                    const int32_t* vbs, const vsa_bf16* kc, const vsa_bf16* vc, const int32_t* plan, vsa_bf16* out,
                    float* lse, int B, int S, int H, int D, int Nq, float sm_scale, int flags, cudaStream_t stream)
{
    vsa::Routes rt{};
    rt.mask = mask;
    rt.kind = vsa::kRouteMask;
    rt.words = Nq > 0 ? (Nq + 31) / 32 : 0;
    return fwd_dispatch(q, k, v, rt, vbs, plan, kc, vc, out, lse, B, S, H, D, Nq, sm_scale, flags, stream);
}

int vsa_fwd(const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v, const int32_t* topk_idx, const int32_t* vbs,
            vsa_bf16* out, float* lse, int B, int S, int H, int D, int Nq, int topk, float sm_scale,
            cudaStream_t stream)
{
    return vsa_fwd_ex(q, k, v, topk_idx, vbs, out, lse, B, S, H, D, Nq, topk, sm_scale, VSA_FWD_DEFAULT, stream);
}

size_t vsa_route_workspace_size(int B, int H, int Nq, int D)
{
    if (B < 1 || H < 1 || Nq < 1 || D < 1) return 0;
    return vsa::route_workspace_bytes(B, H, Nq, D);
}

int vsa_route(const vsa_bf16* q, const vsa_bf16* k, const int32_t* vbs, int32_t* topk_idx, int B, int S, int H,
              int D, int Nq, int topk, void* workspace, size_t workspace_bytes, cudaStream_t stream)
{
    int rc = check_bshd(B, S, H, D, Nq);
    if (rc != VSA_OK) return rc;
    if (topk < 1 || topk > Nq || Nq > 4096) return VSA_ERR_ARG;
    if (!q || !k || !vbs || !topk_idx) return VSA_ERR_NULL;
    if (!workspace || workspace_bytes < vsa::route_workspace_bytes(B, H, Nq, D)) return VSA_ERR_WORKSPACE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(vbs) || !aligned16(topk_idx) || !aligned16(workspace))
        return VSA_ERR_ALIGN;
    if ((rc = check_arch()) != VSA_OK) return rc;
    int* err;
    if ((rc = device_error_word(&err)) != VSA_OK) return rc;
    return launch_status(vsa::launch_route(q, k, vbs, topk_idx, B, S, H, Nq, topk, workspace, err, stream));
}

size_t vsa_plan_workspace_size(int B, int H, int Nq, int topk)
{
    if (B < 1 || H < 1 || Nq < 1 || Nq > 8192 || topk < 1) return 0;
    return vsa::plan_workspace_bytes(B, H, Nq);
}

int vsa_plan(const int32_t* topk_idx, int32_t* plan, int B, int H, int Nq, int topk, void* workspace,
             size_t workspace_bytes, cudaStream_t stream)
{
    if (B < 1 || H < 1 || Nq < 1 || Nq > 8192 || topk < 1 || topk > Nq) return VSA_ERR_ARG;
    if ((int64_t)B * H * Nq * topk > INT32_MAX) return VSA_ERR_ARG;
    if (!topk_idx || !plan) return VSA_ERR_NULL;
    if (!workspace || workspace_bytes < vsa::plan_workspace_bytes(B, H, Nq)) return VSA_ERR_WORKSPACE;
    if (!aligned16(topk_idx) || !aligned16(plan) || !aligned16(workspace)) return VSA_ERR_ALIGN;
    int rc = check_arch();
    if (rc != VSA_OK) return rc;
    int* err;
    if ((rc = device_error_word(&err)) != VSA_OK) return rc;
    return launch_status(vsa::launch_plan(topk_idx, plan, B, H, Nq, topk, workspace, err, stream));
}

int vsa_cube_counts(int T, int Hh, int W, int32_t* vbs_host, int* Nq_out)
{
    if (T < 1 || Hh < 1 || W < 1) return VSA_ERR_ARG;
    const int64_t nq = (int64_t)((T + 3) / 4) * ((Hh + 3) / 4) * ((W + 3) / 4);
    if (nq > INT32_MAX / 64) return VSA_ERR_ARG;
    if (Nq_out) *Nq_out = (int)nq;
    if (!vbs_host) return VSA_OK;
    const vsa::CubeGeom g = vsa::make_geom(T, Hh, W);
    for (int ct = 0; ct < g.nct; ++ct)
        for (int ch = 0; ch < g.nch; ++ch)
            for (int cw = 0; cw < g.ncw; ++cw) {
                const int et = T - 4 * ct < 4 ? T - 4 * ct : 4;
                const int eh = Hh - 4 * ch < 4 ? Hh - 4 * ch : 4;
                const int ew = W - 4 * cw < 4 ? W - 4 * cw : 4;
                vbs_host[(ct * g.nch + ch) * g.ncw + cw] = et * eh * ew;
            }
    return VSA_OK;
}

// Sizes and the two pointers of a layout transform (no device query).
static int check_tile_pair(const void* a, const void* b, int B, int T, int Hh, int W, int H, int D)
{
    if (B < 1 || T < 1 || Hh < 1 || W < 1 || H < 1 || D < 1) return VSA_ERR_ARG;
    if (((int64_t)H * D) % 8 != 0 || (int64_t)H * D > INT32_MAX) return VSA_ERR_ARG;
    int nq = 0;
    if (vsa_cube_counts(T, Hh, W, nullptr, &nq) != VSA_OK) return VSA_ERR_ARG;
    if ((int64_t)B * 64 * nq * H * D > ((int64_t)1 << 40)) return VSA_ERR_ARG;
    if (!a || !b) return VSA_ERR_NULL;
    if (!aligned16(a) || !aligned16(b)) return VSA_ERR_ALIGN;
    return VSA_OK;
}

static int check_tile_args(const void* a, const void* b, int B, int T, int Hh, int W, int H, int D)
{
    const int rc = check_tile_pair(a, b, B, T, Hh, W, H, D);
    return rc != VSA_OK ? rc : check_arch();
}

int vsa_tile(const vsa_bf16* x_grid, vsa_bf16* x_tiled, int B, int T, int Hh, int W, int H, int D,
             cudaStream_t stream)
{
    int rc = check_tile_args(x_grid, x_tiled, B, T, Hh, W, H, D);
    if (rc != VSA_OK) return rc;
    return launch_status(vsa::launch_tile(x_grid, x_tiled, B, vsa::make_geom(T, Hh, W), H * D, stream));
}

int vsa_untile(const vsa_bf16* x_tiled, vsa_bf16* x_grid, int B, int T, int Hh, int W, int H, int D,
               cudaStream_t stream)
{
    int rc = check_tile_args(x_tiled, x_grid, B, T, Hh, W, H, D);
    if (rc != VSA_OK) return rc;
    return launch_status(vsa::launch_untile(x_tiled, x_grid, B, vsa::make_geom(T, Hh, W), H * D, stream));
}

int vsa_tile_qkv(const vsa_bf16* q_grid, const vsa_bf16* k_grid, const vsa_bf16* v_grid, vsa_bf16* q_tiled,
                 vsa_bf16* k_tiled, vsa_bf16* v_tiled, const int32_t* vbs, vsa_bf16* qc, vsa_bf16* kc, vsa_bf16* vc,
                 int B, int T, int Hh, int W, int H, int D, cudaStream_t stream)
{
    const bool means = qc != nullptr || kc != nullptr;
    if (means && (qc == nullptr || kc == nullptr)) return VSA_ERR_ARG;
    if ((means || vc != nullptr) && D != 128) return VSA_ERR_ARG;
    int rc;
    if ((rc = check_tile_pair(q_grid, q_tiled, B, T, Hh, W, H, D)) != VSA_OK) return rc;
    if ((rc = check_tile_pair(k_grid, k_tiled, B, T, Hh, W, H, D)) != VSA_OK) return rc;
    if ((rc = check_tile_pair(v_grid, v_tiled, B, T, Hh, W, H, D)) != VSA_OK) return rc;
    if (means || vc != nullptr) {
        if (!vbs) return VSA_ERR_NULL;
        if (!aligned16(vbs) || (means && (!aligned16(qc) || !aligned16(kc))) || (vc && !aligned16(vc)))
            return VSA_ERR_ALIGN;
    }
    if ((rc = check_arch()) != VSA_OK) return rc;
    int* err;
    if ((rc = device_error_word(&err)) != VSA_OK) return rc;
    vsa::TileJob job;
    const vsa_bf16* src[3] = {q_grid, k_grid, v_grid};
    vsa_bf16* dst[3] = {q_tiled, k_tiled, v_tiled};
    for (int t = 0; t < 3; ++t) {
        job.src[t] = reinterpret_cast<const uint4*>(src[t]);
        job.dst[t] = reinterpret_cast<uint4*>(dst[t]);
    }
    job.means[0] = qc;
    job.means[1] = kc;
    job.means[2] = vc;
    job.sums[0] = job.sums[1] = 0;
    job.sums[2] = 1;
    return launch_status(vsa::launch_tile_cubes(job, 3, vbs, B, vsa::make_geom(T, Hh, W), H, D, err, stream));
}

int vsa_route_means(const vsa_bf16* qc, const vsa_bf16* kc, int32_t* topk_idx, int B, int H, int D, int Nq, int topk,
                    cudaStream_t stream)
{
    if (B < 1 || H < 1 || Nq < 1 || D != 128) return VSA_ERR_ARG;
    if (topk < 1 || topk > Nq || Nq > 4096) return VSA_ERR_ARG;
    if ((int64_t)B * H * Nq * topk > INT32_MAX) return VSA_ERR_ARG;
    if (!qc || !kc || !topk_idx) return VSA_ERR_NULL;
    if (!aligned16(qc) || !aligned16(kc) || !aligned16(topk_idx)) return VSA_ERR_ALIGN;
    const int rc = check_arch();
    if (rc != VSA_OK) return rc;
    return launch_status(vsa::launch_score_topk(qc, kc, topk_idx, B, H, Nq, topk, stream));
}

int vsa_stall_check(int* result, cudaStream_t stream)
{
    if (result == nullptr) return VSA_ERR_NULL;
    int rc = check_arch();
    if (rc != VSA_OK) return rc;
    int* err;
    if ((rc = device_error_word(&err)) != VSA_OK) return rc;
    return launch_status(vsa::launch_stall_check(err, result, stream));
}

int vsa_device_status(cudaStream_t stream, int* detail)
{
    if (detail) *detail = 0;
    int* err;
    int rc = device_error_word(&err);
    if (rc != VSA_OK) return rc;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return VSA_ERR_LAUNCH;
    int h = 0;
    if (cudaMemcpy(&h, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return VSA_ERR_LAUNCH;
    if (h == 0) return VSA_OK;
    const int zero = 0;
    if (cudaMemcpy(err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return VSA_ERR_LAUNCH;
    if (detail) *detail = h;
    return VSA_ERR_DEVICE;
}

}  // extern "C"
