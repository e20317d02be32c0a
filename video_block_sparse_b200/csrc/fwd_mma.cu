// VSA fine forward with warp-level tensor-core instructions (mma.sync
// m16n8k16, bf16 in, fp32 accumulate): the legacy tensor path.  It is the
// plain single-pass baseline that the tcgen05 kernel (fwd_tc.cu) is measured
// against.
//
// Dataset card "wan2.2_production_values", section "Operator contract":
// for query cube i of (b, h), attend to the first vbs[j] tokens of every cube
// j listed in topk_idx[b, h, i, :]; out = softmax(q k^T * sm_scale) v.
//
// One CTA (4 warps) per (b, h, query cube); warp w owns query rows
// 16w..16w+15.  Selected K/V cubes (64 x 128 bf16 each) are staged into
// shared memory with cp.async, double-buffered; rows at or beyond vbs[j] are
// zero-filled by the copy itself, so NaN/Inf in padded K/V never reaches an
// MMA.  Online softmax in base 2 with the running max guarded for rows that
// have seen no valid key yet.
#include "internal.h"

#include <cuda_bf16.h>

namespace vsa {
namespace {

constexpr int kD = 128;
constexpr int kRowBytes = kD * 2;          // 256 B per token row in shared memory
constexpr int kTileBytes = 64 * kRowBytes;  // 16 KiB per 64-token cube

// 16-byte chunk c (0..15) of row r, XOR-swizzled to spread ldmatrix rows
// over all banks.
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)(r * kRowBytes + ((c ^ (r & 7)) << 4)); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t p) { return __uint_as_float(p << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t p) { return __uint_as_float(p & 0xFFFF0000u); }

// Stage one 64 x 128 tile (rows = tokens) of a [B, S, H, D] tensor.  Rows at
// or beyond `valid` are zero-filled (no global read).
__device__ __forceinline__ void load_tile(uint32_t dst, const uint16_t* src_row0, int64_t row_stride, int valid)
{
#pragma unroll
    for (int it = 0; it < 8; ++it) {
        const int e = threadIdx.x + it * 128;  // 1024 chunks of 16 B
        const int r = e >> 4, c = e & 15;
        const uint16_t* src = src_row0 + r * row_stride + c * 8;
        cp_async16(dst + swz(r, c), src, r < valid ? 16 : 0);
    }
}

template <bool PRECISE>
__global__ void __launch_bounds__(128) fwd_mma_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                                                      const uint16_t* __restrict__ v,
                                                      const int32_t* __restrict__ topk_idx,
                                                      const int32_t* __restrict__ vbs, uint16_t* __restrict__ out,
                                                      float* __restrict__ lse, int S, int H, int nq, int topk,
                                                      float scale_log2, int* err)
{
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sq = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    const uint32_t sk[2] = {sq + kTileBytes, sq + 2 * kTileBytes};
    const uint32_t sv[2] = {sq + 3 * kTileBytes, sq + 4 * kTileBytes};

    const int item = blockIdx.x;  // ((b * H + h) * nq + i)
    const int i = item % nq;
    const int bh = item / nq;
    const int h = bh % H, b = bh / H;
    const int64_t rs = (int64_t)H * kD;  // token row stride in elements
    const uint16_t* qb = q + ((int64_t)b * S) * rs + (int64_t)h * kD;
    const uint16_t* kb = k + ((int64_t)b * S) * rs + (int64_t)h * kD;
    const uint16_t* vb = v + ((int64_t)b * S) * rs + (int64_t)h * kD;
    const int32_t* sel = topk_idx + (int64_t)item * topk;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    auto cube_of = [&](int t, int& j, int& n) {
        j = __ldg(sel + t);
        if (j < 0 || j >= nq) {
            if (threadIdx.x == 0) atomicCAS(err, 0, (int)kErrTopkIdx);
            j = 0;
            n = 0;
            return;
        }
        n = __ldg(vbs + j);
        if (n < 0 || n > 64) {
            if (threadIdx.x == 0) atomicCAS(err, 0, (int)kErrVbs);
            n = 0;
        }
    };

    load_tile(sq, qb + (int64_t)(64 * i) * rs, rs, 64);
    int j0, n0;
    cube_of(0, j0, n0);
    load_tile(sk[0], kb + (int64_t)(64 * j0) * rs, rs, n0);
    load_tile(sv[0], vb + (int64_t)(64 * j0) * rs, rs, n0);
    cp_async_commit();

    float o[16][4];
#pragma unroll
    for (int a = 0; a < 16; ++a)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[a][e] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};
    uint32_t qf[8][4];

    int n_cur = n0;
    for (int t = 0; t < topk; ++t) {
        int n_next = 0;
        if (t + 1 < topk) {
            int jn;
            cube_of(t + 1, jn, n_next);
            load_tile(sk[(t + 1) & 1], kb + (int64_t)(64 * jn) * rs, rs, n_next);
            load_tile(sv[(t + 1) & 1], vb + (int64_t)(64 * jn) * rs, rs, n_next);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        if (t == 0) {
            // Q fragments (A operand, rows 16w.., all 8 k-steps of 16)
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int mat = lane >> 3;
                const int r = warp * 16 + (mat & 1) * 8 + (lane & 7);
                const int c = ks * 2 + (mat >> 1);
                ldsm_x4(sq + swz(r, c), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
            }
        }
        const uint32_t kt = sk[t & 1], vt = sv[t & 1];
        if (n_cur > 0) {
            // S = Q K^T for this warp's 16 rows x 64 keys
            float s[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
                for (int np = 0; np < 4; ++np) {  // pairs of 8-key n-tiles
                    const int mat = lane >> 3;
                    const int r = np * 16 + (mat >> 1) * 8 + (lane & 7);
                    const int c = ks * 2 + (mat & 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kt + swz(r, c), b0, b1, b2, b3);
                    mma16816(s[2 * np], qf[ks], b0, b1);
                    mma16816(s[2 * np + 1], qf[ks], b2, b3);
                }
            }
            // scale to base 2, mask keys >= n_cur, row max
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = nt * 8 + (lane & 3) * 2 + (e & 1);
                    const float x = key < n_cur ? s[nt][e] * scale_log2 : -INFINITY;
                    s[nt][e] = x;
                    mx[e >> 1] = fmaxf(mx[e >> 1], x);
                }
            float alpha[2], m_use[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
                const float m_new = fmaxf(m_run[r], mx[r]);
                m_use[r] = m_new == -INFINITY ? 0.f : m_new;
                alpha[r] = exp2f(m_run[r] - m_use[r]);
                m_run[r] = m_new;
            }
            // P = exp2(x - m); l accumulates the fp32 weights
            uint32_t ph[8][2], pl[8][2];
            float ls[2] = {0.f, 0.f};
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                float p[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    p[e] = exp2f(s[nt][e] - m_use[e >> 1]);
                    ls[e >> 1] += p[e];
                }
                ph[nt][0] = pack_bf16(p[0], p[1]);
                ph[nt][1] = pack_bf16(p[2], p[3]);
                if (PRECISE) {
                    pl[nt][0] = pack_bf16(p[0] - bf16_lo(ph[nt][0]), p[1] - bf16_hi(ph[nt][0]));
                    pl[nt][1] = pack_bf16(p[2] - bf16_lo(ph[nt][1]), p[3] - bf16_hi(ph[nt][1]));
                }
            }
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                ls[r] += __shfl_xor_sync(0xffffffffu, ls[r], 1);
                ls[r] += __shfl_xor_sync(0xffffffffu, ls[r], 2);
                l_run[r] = l_run[r] * alpha[r] + ls[r];
            }
#pragma unroll
            for (int a = 0; a < 16; ++a) {
                o[a][0] *= alpha[0];
                o[a][1] *= alpha[0];
                o[a][2] *= alpha[1];
                o[a][3] *= alpha[1];
            }
            // O += P V over keys in steps of 16 (skip steps past the valid keys)
            const int ksteps = (n_cur + 15) >> 4;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                if (kk < ksteps) {
                    const uint32_t ah[4] = {ph[2 * kk][0], ph[2 * kk][1], ph[2 * kk + 1][0], ph[2 * kk + 1][1]};
                    uint32_t al[4];
                    if (PRECISE) {
                        al[0] = pl[2 * kk][0];
                        al[1] = pl[2 * kk][1];
                        al[2] = pl[2 * kk + 1][0];
                        al[3] = pl[2 * kk + 1][1];
                    }
#pragma unroll
                    for (int dp = 0; dp < 8; ++dp) {  // pairs of 8-wide d tiles
                        const int mat = lane >> 3;
                        const int r = kk * 16 + (mat & 1) * 8 + (lane & 7);
                        const int c = dp * 2 + (mat >> 1);
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4_t(vt + swz(r, c), b0, b1, b2, b3);
                        mma16816(o[2 * dp], ah, b0, b1);
                        mma16816(o[2 * dp + 1], ah, b2, b3);
                        if (PRECISE) {
                            mma16816(o[2 * dp], al, b0, b1);
                            mma16816(o[2 * dp + 1], al, b2, b3);
                        }
                    }
                }
            }
        }
        n_cur = n_next;
        __syncthreads();  // buffer (t & 1) is refilled by the next iteration's prefetch
    }

    // epilogue: o / l -> bf16; rows without any valid key give 0 and lse = -inf
    const int r0 = warp * 16 + (lane >> 2);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int row = r0 + 8 * r;
        const float inv = l_run[r] > 0.f ? 1.f / l_run[r] : 0.f;
        uint16_t* dst = out + ((int64_t)b * S + 64LL * i + row) * rs + (int64_t)h * kD;
#pragma unroll
        for (int a = 0; a < 16; ++a) {
            const int d = a * 8 + (lane & 3) * 2;
            *reinterpret_cast<uint32_t*>(dst + d) = pack_bf16(o[a][2 * r] * inv, o[a][2 * r + 1] * inv);
        }
        if (lse != nullptr && (lane & 3) == 0) {
            const float val = l_run[r] > 0.f ? (m_run[r] + __log2f(l_run[r])) * 0.69314718055994531f : -INFINITY;
            lse[((int64_t)b * H + h) * S + 64LL * i + row] = val;
        }
    }
}

}  // namespace

cudaError_t launch_fwd_mma(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* topk_idx,
                           const int32_t* vbs, uint16_t* out, float* lse, int B, int S, int H, int nq, int topk,
                           float sm_scale, bool precise_p, int* err, cudaStream_t s)
{
    const float scale_log2 = sm_scale * 1.4426950408889634f;
    const int smem = 5 * kTileBytes;
    const unsigned grid = (unsigned)((int64_t)B * H * nq);
    cudaError_t e;
    if (precise_p) {
        e = cudaFuncSetAttribute(fwd_mma_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        fwd_mma_kernel<true><<<grid, 128, smem, s>>>(q, k, v, topk_idx, vbs, out, lse, S, H, nq, topk, scale_log2, err);
    } else {
        e = cudaFuncSetAttribute(fwd_mma_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        fwd_mma_kernel<false><<<grid, 128, smem, s>>>(q, k, v, topk_idx, vbs, out, lse, S, H, nq, topk, scale_log2,
                                                      err);
    }
    return cudaGetLastError();
}

}  // namespace vsa
