// Cube-mean q.k top-k routing (the VSA "predictor").
//
// "align VisualGen VSA with block-sparse FMHA" (TensorRT-LLM PR #7), review
// excerpts: a cube mean is the sum over the cube's valid tokens divided by the
// valid count and cast back to the tiled dtype.  "Video Sparse Attention
// Runner" (TensorRT-Edge docs): block means of K are rounded to bf16 before
// they are used to route.  The score of query cube i against KV cube j is the
// dot product of their bf16 means; each query cube keeps the topk best.
//
// The arithmetic is fixed so that the selection is exact and reproducible:
//   mean  = bf16_rne(fp64 sequential sum over u < vbs / vbs)   (0 when vbs = 0)
//   score = fp64 sequential sum over d = 0..D-1 of qc[d] * kc[d]
//           (each product of two bf16 values is exact in fp64)
//   order = score descending, cube index ascending, NaN counted as -inf
//
// Kernels:
//   cube_mean_kernel   one CTA per (cube, batch, tensor); threads own 8
//                      consecutive (h, d) columns and walk the cube's valid
//                      rows with 16-byte loads: HBM-bound, reads q and k once.
//   score_topk_kernel  one CTA per (QB query cubes, head, batch): streams the
//                      head's kc rows once, keeps QB score rows in shared
//                      memory as order-preserving 64-bit keys, then one warp
//                      per query cube selects the topk smallest keys exactly
//                      (radix select on 8-bit digits, ties by index) and
//                      sorts only the selected ones.
#include "internal.h"

namespace vsa {
namespace {

constexpr int kD = 128;

__device__ __forceinline__ double bf16_to_f64(uint32_t bits16) { return (double)__uint_as_float(bits16 << 16); }

// Nearest-even rounding of a double to bf16 bits, one rounding step.
// Normal range: drop the low 45 fraction bits of the binary64 pattern with
// round-half-even; below 2^-126 the bf16 grid is uniform with step 2^-133.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x)
{
    const uint64_t u = (uint64_t)__double_as_longlong(x);
    const uint16_t sign = (uint16_t)((u >> 48) & 0x8000u);
    const uint64_t a = u & 0x7FFFFFFFFFFFFFFFull;
    if (a > 0x7FF0000000000000ull) return 0x7FC0;           // NaN
    if (a == 0x7FF0000000000000ull) return sign | 0x7F80;   // inf
    const int e = (int)(a >> 52) - 1023;
    if (e >= -126) {
        const uint64_t lsb = (a >> 45) & 1ull;
        uint64_t r = a + ((1ull << 44) - 1ull) + lsb;
        r &= ~((1ull << 45) - 1ull);
        const int e2 = (int)(r >> 52) - 1023;
        if (e2 > 127) return sign | 0x7F80;
        return sign | (uint16_t)((uint32_t)(e2 + 127) << 7) | (uint16_t)((r >> 45) & 0x7Fu);
    }
    // |x| < 2^-126: multiples of 2^-133; the scaling by 2^133 is exact
    const double n = rint(__longlong_as_double((long long)a) * 0x1p133);
    return sign | (uint16_t)n;  // n <= 128; 128 encodes the smallest normal
}

// x [B, S, H, D] -> xc [B, H, Nq, D]; blockIdx = (cube, batch, tensor)
__global__ void __launch_bounds__(128) cube_mean_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                                                        const int32_t* __restrict__ vbs, uint16_t* __restrict__ qc,
                                                        uint16_t* __restrict__ kc, int S, int H, int nq, int* err)
{
    const int c = blockIdx.x, b = blockIdx.y;
    const uint16_t* x = blockIdx.z ? k : q;
    uint16_t* xc = blockIdx.z ? kc : qc;
    int n = __ldg(vbs + c);
    if (n < 0 || n > 64) {
        if (threadIdx.x == 0) atomicCAS(err, 0, (int)kErrVbs);
        n = 0;
    }
    const int row16 = H * kD / 8;
    const uint4* base = reinterpret_cast<const uint4*>(x + ((int64_t)b * S + 64LL * c) * H * kD);
    for (int ch = threadIdx.x; ch < row16; ch += blockDim.x) {
        double acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0;
        for (int u = 0; u < n; ++u) {
            uint4 w = __ldg(base + (int64_t)u * row16 + ch);
            uint32_t p[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[2 * e] += bf16_to_f64(p[e] & 0xFFFFu);
                acc[2 * e + 1] += bf16_to_f64(p[e] >> 16);
            }
        }
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            uint32_t lo = n ? f64_to_bf16_rne(acc[2 * e] / (double)n) : 0u;
            uint32_t hi = n ? f64_to_bf16_rne(acc[2 * e + 1] / (double)n) : 0u;
            o[e] = lo | (hi << 16);
        }
        const int h = (ch * 8) / kD, d = (ch * 8) % kD;
        *reinterpret_cast<uint4*>(xc + (((int64_t)b * H + h) * nq + c) * kD + d) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// Order-preserving key, inverted so that ascending key = descending score.
__device__ __forceinline__ uint64_t score_key(double s)
{
    uint64_t u = (uint64_t)__double_as_longlong(s);
    if (s != s) u = 0xFFF0000000000000ull;          // NaN ranks as -inf
    if (u == 0x8000000000000000ull) u = 0ull;       // -0 ranks as +0
    const uint64_t ord = (u >> 63) ? ~u : (u | 0x8000000000000000ull);
    return ~ord;
}

// Exact top-k of one row by radix selection on the 64-bit keys (ascending key
// = better), run by one warp: 8-bit digits from the most significant byte
// fix the threshold key T; the selection is every key < T plus the
// lowest-index entries equal to T; it is then sorted by (key, index).
__device__ void select_row(const uint64_t* __restrict__ keys, int n, int topk, int* hist, uint64_t* sel_k,
                           uint16_t* sel_i, int ns, int32_t* __restrict__ dst, int lane)
{
    uint64_t prefix = 0, pmask = 0;  // decided high bits of T and their mask
    int need = topk;                 // how many still to take at or above the current prefix
    bool done = false;
    for (int byte = 7; byte >= 0 && !done; --byte) {
        for (int b = lane; b < 256; b += 32) hist[b] = 0;
        __syncwarp();
        const int sh = 8 * byte;
        for (int j = lane; j < n; j += 32) {
            const uint64_t k = keys[j];
            if ((k & pmask) == prefix) atomicAdd(&hist[(int)((k >> sh) & 255u)], 1);
        }
        __syncwarp();
        // lane owns bins 8*lane .. 8*lane+7; exclusive prefix over lanes
        int c[8], tot = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            c[e] = hist[8 * lane + e];
            tot += c[e];
        }
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const int excl = incl - tot;
        // the bucket where the running count reaches `need`
        int found = -1, below = 0, cnt = 0;
        if (excl < need && need <= incl) {
            int run = excl;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (found < 0 && run + c[e] >= need) {
                    found = 8 * lane + e;
                    below = run;
                    cnt = c[e];
                }
                run += c[e];
            }
        }
        const uint32_t owner = __ballot_sync(0xffffffffu, found >= 0);
        const int src = __ffs(owner) - 1;
        found = __shfl_sync(0xffffffffu, found, src);
        below = __shfl_sync(0xffffffffu, below, src);
        cnt = __shfl_sync(0xffffffffu, cnt, src);
        prefix |= (uint64_t)found << sh;
        pmask |= (uint64_t)255u << sh;
        need -= below;
        if (cnt == need) done = true;  // the whole bucket is taken: no tie to break
        __syncwarp();
    }
    // gather: keys below the threshold prefix, plus `need` entries of the threshold
    // bucket in index order (all of it when done early)
    int taken_eq = 0, pos = 0;
    for (int base = 0; base < n; base += 32) {
        const int j = base + lane;
        uint64_t k = 0;
        bool lt = false, eq = false;
        if (j < n) {
            k = keys[j];
            const uint64_t hk = k & pmask;
            lt = hk < prefix;
            eq = hk == prefix;
        }
        const uint32_t meq = __ballot_sync(0xffffffffu, eq);
        const int eq_rank = taken_eq + __popc(meq & ((1u << lane) - 1u));
        const bool take = lt || (eq && eq_rank < need);
        const uint32_t mt = __ballot_sync(0xffffffffu, take);
        if (take) {
            const int p = pos + __popc(mt & ((1u << lane) - 1u));
            sel_k[p] = k;
            sel_i[p] = (uint16_t)j;
        }
        pos += __popc(mt);
        taken_eq += __popc(meq);
    }
    for (int p = pos + lane; p < ns; p += 32) {
        sel_k[p] = ~0ull;
        sel_i[p] = 0xFFFFu;
    }
    __syncwarp();
    // bitonic sort of the ns (power of two) selected entries by (key, index)
    for (int len = 2; len <= ns; len <<= 1) {
        for (int stride = len >> 1; stride > 0; stride >>= 1) {
            for (int a = lane; a < ns; a += 32) {
                const int q = a ^ stride;
                if (q > a) {
                    const uint64_t ka = sel_k[a], kq = sel_k[q];
                    const uint16_t ia = sel_i[a], iq = sel_i[q];
                    const bool a_after = (ka > kq) || (ka == kq && ia > iq);
                    const bool ascending = (a & len) == 0;
                    if (a_after == ascending) {
                        sel_k[a] = kq;
                        sel_k[q] = ka;
                        sel_i[a] = iq;
                        sel_i[q] = ia;
                    }
                }
            }
            __syncwarp();
        }
    }
    for (int t = lane; t < topk; t += 32) dst[t] = sel_i[t];
    __syncwarp();
}

// Scoring threads: kQH groups of query cubes x kKG groups of key cubes.  A
// thread keeps a kQT x kJT block of (query, key) sums in registers: every q
// element read from shared memory feeds kJT FMAs and every k element loaded
// feeds kQT, so shared-memory reads stay below the FP64 pipe's rate.  Every
// (query, key) sum still runs over d = 0..127 in order.
constexpr int kJT = 4;
constexpr int kKG = 160;  // key groups of kJT cubes (624 cubes: one pass)
template <int QB>
struct ScoreShape {
    static constexpr int kQT = QB < 4 ? QB : 4;  // query cubes per thread
    static constexpr int kQH = QB / kQT;         // query groups
    static constexpr int kThreads = kQH * kKG;
};

template <int QB>
__global__ void __launch_bounds__(ScoreShape<QB>::kThreads) score_topk_kernel(const uint16_t* __restrict__ qc,
                                                         const uint16_t* __restrict__ kc, int32_t* __restrict__ topk_idx,
                                                         int H, int nq, int ns, int topk, int sel_warps)
{
    extern __shared__ __align__(16) uint8_t smem[];
    double* qd = reinterpret_cast<double*>(smem);                          // [QB][D]
    uint64_t* keys = reinterpret_cast<uint64_t*>(qd + QB * kD);            // [QB][nq]
    uint64_t* sel_k = keys + (size_t)QB * nq;                                       // [sel_warps][ns]
    uint16_t* sel_i = reinterpret_cast<uint16_t*>(sel_k + (size_t)sel_warps * ns);  // [sel_warps][ns]
    int* hist = reinterpret_cast<int*>(sel_i + (size_t)sel_warps * ns);             // [sel_warps][256]

    const int i0 = blockIdx.x * QB, h = blockIdx.y, b = blockIdx.z;
    const int64_t head = (int64_t)b * H + h;
    for (int e = threadIdx.x; e < QB * kD; e += blockDim.x) {
        const int qi = i0 + e / kD;
        qd[e] = qi < nq ? bf16_to_f64(qc[(head * nq + qi) * kD + (e % kD)]) : 0.0;
    }
    __syncthreads();

    constexpr int kQT = ScoreShape<QB>::kQT;
    const int qg = threadIdx.x / kKG, kg = threadIdx.x % kKG;
    const double* qrow = qd + qg * kQT * kD;
    const uint4* krow = reinterpret_cast<const uint4*>(kc + head * nq * kD);
    for (int j0 = kg * kJT; j0 < nq; j0 += kKG * kJT) {
        double acc[kQT][kJT];
#pragma unroll
        for (int r = 0; r < kQT; ++r)
#pragma unroll
            for (int t = 0; t < kJT; ++t) acc[r][t] = 0.0;
        for (int ch = 0; ch < kD / 8; ++ch) {
            uint32_t p[kJT][4];
#pragma unroll
            for (int t = 0; t < kJT; ++t) {
                const uint4 w = j0 + t < nq ? __ldg(krow + (int64_t)(j0 + t) * (kD / 8) + ch) : make_uint4(0, 0, 0, 0);
                p[t][0] = w.x;
                p[t][1] = w.y;
                p[t][2] = w.z;
                p[t][3] = w.w;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                double kv[kJT];
#pragma unroll
                for (int t = 0; t < kJT; ++t)
                    kv[t] = bf16_to_f64((e & 1) ? (p[t][e >> 1] >> 16) : (p[t][e >> 1] & 0xFFFFu));
#pragma unroll
                for (int r = 0; r < kQT; ++r) {
                    const double qv = qrow[r * kD + ch * 8 + e];
#pragma unroll
                    for (int t = 0; t < kJT; ++t) acc[r][t] = __fma_rn(qv, kv[t], acc[r][t]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < kJT; ++t)
            if (j0 + t < nq)
#pragma unroll
                for (int r = 0; r < kQT; ++r) keys[(qg * kQT + r) * nq + j0 + t] = score_key(acc[r][t]);
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp >= sel_warps) return;
    for (int r = warp; r < QB; r += sel_warps) {
        const int qi = i0 + r;
        if (qi >= nq) continue;
        select_row(keys + (size_t)r * nq, nq, topk, hist + warp * 256, sel_k + (size_t)warp * ns,
                   sel_i + (size_t)warp * ns, ns, topk_idx + (head * nq + qi) * topk, lane);
    }
}

}  // namespace

size_t route_workspace_bytes(int B, int H, int nq, int D)
{
    return 2 * (size_t)B * H * nq * D * sizeof(uint16_t);
}

cudaError_t launch_score_topk(const uint16_t* qc, const uint16_t* kc, int32_t* topk_idx, int B, int H, int nq,
                              int topk, cudaStream_t s)
{
    int ns = 32;  // selection buffer: topk rounded up to a power of two
    while (ns < topk) ns <<= 1;
    // rows per CTA and selecting warps sized to the shared-memory budget
    auto smem_for = [&](int qb, int w) {
        return (size_t)qb * kD * 8 + (size_t)qb * nq * 8 + (size_t)w * ns * 10 + (size_t)w * 256 * 4;
    };
    const size_t budget = 200 * 1024;
    int qb = smem_for(8, 8) <= budget ? 8 : (smem_for(4, 1) <= budget ? 4 : 2);
    int w = qb;
    while (w > 1 && smem_for(qb, w) > budget) w >>= 1;
    const size_t smem = smem_for(qb, w);
    cudaError_t e;
    if (qb == 8) {
        auto kern = score_topk_kernel<8>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<dim3((nq + 7) / 8, H, B), ScoreShape<8>::kThreads, smem, s>>>(qc, kc, topk_idx, H, nq, ns, topk, w);
    } else if (qb == 4) {
        auto kern = score_topk_kernel<4>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<dim3((nq + 3) / 4, H, B), ScoreShape<4>::kThreads, smem, s>>>(qc, kc, topk_idx, H, nq, ns, topk, w);
    } else {
        auto kern = score_topk_kernel<2>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<dim3((nq + 1) / 2, H, B), ScoreShape<2>::kThreads, smem, s>>>(qc, kc, topk_idx, H, nq, ns, topk, w);
    }
    return cudaGetLastError();
}

cudaError_t launch_route(const uint16_t* q, const uint16_t* k, const int32_t* vbs, int32_t* topk_idx, int B, int S,
                         int H, int nq, int topk, void* workspace, int* err, cudaStream_t s)
{
    uint16_t* qc = static_cast<uint16_t*>(workspace);
    uint16_t* kc = qc + (size_t)B * H * nq * kD;
    cube_mean_kernel<<<dim3(nq, B, 2), 128, 0, s>>>(q, k, vbs, qc, kc, S, H, nq, err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_score_topk(qc, kc, topk_idx, B, H, nq, topk, s);
}

}  // namespace vsa
