// VSA fine forward on the Blackwell tensor cores (tcgen05 + TMEM + TMA).
//
// Dataset card "wan2.2_production_values", section "Operator contract": for
// query cube i of (batch b, head h) the keys are the first vbs[j] tokens of
// every cube j in topk_idx[b, h, i, :]; out = softmax(q k^T * sm_scale) v.
//
// Shape of the work on sm_100a.  A query cube has 64 rows and its own list
// of KV cubes, so the query side can only fill an MMA M of 64, which runs the
// tensor core at half rate.  The kernel therefore puts KEYS on the MMA M side
// ("keys on TMEM lanes"): one step takes two selected cubes (128 keys),
//     S^T[128 keys x 64 q]  = K_pair[128 x 128 d] . Q^T          (M=128, N=64)
//     O^T[128 d x 64 q]    += V_pair^T[128 d x 128 keys] . P^T   (M=128, N=64)
// both issued by one thread with tcgen05.mma (bf16 in, fp32 accumulate in
// TMEM).  K/V/Q tiles arrive by TMA (128-byte swizzle) into shared-memory
// rings; P^T is written to shared memory by the softmax threads.
//
// Roles (704 threads, one CTA per SM, persistent over (b, h, i) work items
// in head-major order so that the CTAs in flight share a head's K/V in L2):
//   warps 0-15  softmax in 4 groups of 4 warps; group g handles query columns
//               16g .. 16g+15; thread t of a group owns TMEM lane t = key t
//   warps 16-19 O correction and epilogue: thread owns TMEM lane d of O^T
//   warp 20     TMA producer (the warp stages selection lists, lane 0 copies)
//   warp 21     TMEM allocator and MMA issuer (one thread)
// (A warp reaches only the TMEM lanes 32 * (warp % 4) .. + 31.  Splitting the
// 64 query columns over four groups keeps each softmax thread's state small
// and gives every scheduler four independent softmax warps to interleave:
// the per-step softmax is a chain of dependent phases, so it is latency-bound.)
// The tensor core runs QK(g), PV(g-1), QK(g+1), PV(g), ...: the softmax of
// step g overlaps PV(g-1) and QK(g+1), and the O rescale for step g (waiting
// for PV(g-1)) overlaps QK(g+1).
//
// Softmax.  Logits are scaled to base 2 (x = s * sm_scale * log2 e); keys at
// or beyond vbs of their cube are set to -inf by selection, so NaN/Inf in
// padded K never propagates.  Each step computes the exact per-query maximum
// of its 128 keys (redux.sync per warp, then a shared-memory exchange).  The
// running offset m[q] is raised only when that maximum exceeds it by more
// than kTau = 8 (so P <= 2^8); only then are O and the partial sums rescaled.
// The output does not depend on which offset is used.  Each thread keeps its
// keys' weight sums per query in registers; the 128-lane sum runs once per
// work item.  PV k-steps beyond ceil16(vbs) of a cube are not issued; V rows
// between vbs and that boundary are zeroed in shared memory before P is
// published, so 0 * NaN cannot occur.
//
// Precise mode (VSA_FWD_PRECISE_P): P is carried as a bf16 pair hi + lo; the
// PV product then has N = 128 (hi and lo side by side) and O = O_hi + O_lo.
//
// Every wait on an mbarrier is bounded (~2 s of clock): on expiry the kernel
// latches kErrWaitTimeout and raises a CTA-wide abort flag; the roles leave
// their loops (the softmax warps together, at a step barrier), the producer
// and the MMA issuer wait (bounded) for their own copies and MMAs in flight,
// and TMEM is freed before exit.
#include "internal.h"
#include "sm100_ptx.cuh"

#include <cstddef>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

namespace vsa {
namespace {

using namespace ptx;

constexpr int kD = 128;
constexpr int kGroups = 4;                 // softmax warpgroups, each owning kCols query columns
constexpr int kCols = 64 / kGroups;
constexpr int kWarpCorr0 = 4 * kGroups;    // 16
constexpr int kWarpProducer = kWarpCorr0 + 4;
constexpr int kWarpMma = kWarpProducer + 1;
constexpr int kThreads = 32 * (kWarpMma + 1);  // 22 warps
constexpr float kTau = 8.0f;
constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 2 GHz

constexpr uint32_t kTileHalf = 64 * 128;        // 8 KiB: 64 rows x 64 bf16 (one TMA box)
constexpr uint32_t kQBytes = 2 * kTileHalf;     // Q cube: 2 column halves
constexpr uint32_t kCubeBytes = 2 * kTileHalf;  // one K or V cube (both column halves)
constexpr uint32_t kKVBytes = 4 * kTileHalf;    // K or V pair: 2 halves x 2 cubes
constexpr int kListChunk = 1024;                // selection-list entries staged per producer pass

struct Misc {
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[2], k_empty[2];
    uint64_t v_full[2], v_empty[2];
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full[2], p_empty[2];
    uint64_t a_full[2], c_full[2];
    uint64_t o_full[2], o_empty[2];
    uint64_t l_full[2];
    uint64_t drain;
    int32_t k_meta[2][2];  // valid counts of the two cubes in each K slot
    int32_t s_meta[2][2];  // valid counts of the pair whose S^T sits in each S buffer
    uint32_t tmem_base;
    int abort;
    int flags[2][4 * kGroups];  // softmax: per-step abort votes of the softmax warps
    int rflag[2][kGroups];      // softmax: per-step "offset raised" vote of each group
    int info[2][kGroups];       // per step and group: bit 0 rescale O, bit 1 the step has valid keys
    alignas(16) float m_sh[64];  // running offsets (base-2 units); read as float4
    alignas(16) float mu_sh[64]; // the offsets used for P (-inf replaced by 0)
    alignas(16) float alpha[2][64];
    alignas(16) float red_sh[kGroups][4][kCols];
    alignas(16) float lfin[2][64];
    alignas(16) float mfin[2][64];
    int32_t list_id[kListChunk];
    int32_t list_n[kListChunk];
};

// arrays read with 16-byte shared-memory loads must sit on 16-byte offsets
static_assert(offsetof(Misc, m_sh) % 16 == 0 && offsetof(Misc, mu_sh) % 16 == 0 && offsetof(Misc, alpha) % 16 == 0 &&
                  offsetof(Misc, red_sh) % 16 == 0 && offsetof(Misc, lfin) % 16 == 0 &&
                  offsetof(Misc, mfin) % 16 == 0,
              "float4 alignment of the softmax arrays");

template <bool PRECISE>
struct Layout {
    static constexpr int NQ = PRECISE ? 1 : 2;
    static constexpr int NK = 2;
    static constexpr int NV = 2;
    static constexpr uint32_t P_BYTES = PRECISE ? 32768 : 16384;
    static constexpr int PV_N = PRECISE ? 128 : 64;
    static constexpr uint32_t O_COLS = PRECISE ? 128 : 64;
    static constexpr uint32_t Q_OFF = 0;
    static constexpr uint32_t K_OFF = Q_OFF + NQ * kQBytes;
    static constexpr uint32_t V_OFF = K_OFF + NK * kKVBytes;
    static constexpr uint32_t P_OFF = V_OFF + NV * kKVBytes;
    static constexpr uint32_t TILE_BYTES = P_OFF + 2 * P_BYTES;
    static constexpr uint32_t MISC_BYTES = (sizeof(Misc) + 1023) / 1024 * 1024;
    static constexpr uint32_t SMEM_BYTES = MISC_BYTES + TILE_BYTES + 1024;  // + alignment slack
    static constexpr uint32_t S_COL0 = 0;    // TMEM: two S^T buffers of 64 columns
    static constexpr uint32_t O_COL0 = 128;  // then two O^T buffers
    static_assert(O_COL0 + 2 * O_COLS <= 512, "TMEM budget");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

__device__ __forceinline__ float4 lds128(const float* p) { return *reinterpret_cast<const float4*>(p); }

__device__ __forceinline__ bool aborted_flag(Misc& m) { return *reinterpret_cast<volatile int*>(&m.abort) != 0; }

// Bounded mbarrier wait that also gives up when another role aborted.  Each
// try_wait may suspend the thread (up to a 1 ms hint) until the phase
// completes, so waiting warps do not spin on the shared-memory pipe.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Misc& m, int* err)
{
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_sleep(bar, parity, 1000000u)) return true;
        {
            if (aborted_flag(m)) return false;
            if (clock64() - t0 > kWaitCycles) {
                atomicCAS(err, 0, (int)kErrWaitTimeout);
                *reinterpret_cast<volatile int*>(&m.abort) = 1;
                return false;
            }
        }
    }
}

// Warp-uniform bounded wait: true only if every lane saw the phase complete.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, Misc& m, int* err)
{
    const bool ok = wait_bar(bar, parity, m, err);
    return __all_sync(0xffffffffu, ok);
}

// Short bounded wait used while draining after an abort.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > kWaitCycles / 4) return;
}

// Valid-token count of list entry t (0 past topk and for invalid entries,
// which also latch an error).
__device__ __forceinline__ int cube_count(const int32_t* sel, int t, int topk, int nq, const int32_t* vbs, int& j,
                                          int* err)
{
    j = 0;
    if (t >= topk) return 0;
    j = __ldg(sel + t);
    if (j < 0 || j >= nq) {
        atomicCAS(err, 0, (int)kErrTopkIdx);
        j = 0;
        return 0;
    }
    const int n = __ldg(vbs + j);
    if (n < 0 || n > 64) {
        atomicCAS(err, 0, (int)kErrVbs);
        return 0;
    }
    return n;
}



__device__ __forceinline__ float redux_max(float v)
{
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v) : "memory");
    return r;
}

__device__ __forceinline__ float redux_min(float v)
{
    float r;
    asm volatile("redux.sync.min.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v) : "memory");
    return r;
}

// 32 consecutive 32-bit TMEM columns of this thread's lane, one wait.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    tmem_ld16(taddr, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
    tmem_ld16(taddr + 16, *reinterpret_cast<uint32_t(*)[16]>(&r[16]));
    tmem_ld_wait();
}


template <bool PRECISE, bool NEG>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, const int32_t* __restrict__ topk_idx,
                  const int32_t* __restrict__ vbs, uint16_t* __restrict__ out, float* __restrict__ lse, int S, int H,
                  int nq, int topk, int n_items, float scale_log2, int* err)
{
    using L = Layout<PRECISE>;
    extern __shared__ uint8_t smem_raw[];
    Misc& m = *reinterpret_cast<Misc*>(smem_raw);
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t tiles = (raw_addr + L::MISC_BYTES + 1023u) & ~1023u;  // 1 KiB aligned for 128B swizzle
    uint8_t* tiles_ptr = smem_raw + (tiles - raw_addr);

    const int warp = threadIdx.x >> 5;
    const uint32_t lane = threadIdx.x & 31;
    const int nsteps = (topk + 1) >> 1;

    // ------------------------------------------------------------ set-up
    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&m.q_full[s], 1);
            mbar_init(&m.q_empty[s], 1);
            mbar_init(&m.k_full[s], 1);
            mbar_init(&m.k_empty[s], 1);
            mbar_init(&m.v_full[s], 1);
            mbar_init(&m.v_empty[s], 1);
            mbar_init(&m.s_full[s], 2);   // MMA thread (metadata) + MMA completion
            mbar_init(&m.s_empty[s], 4 * kGroups);  // softmax warps
            mbar_init(&m.p_full[s], 4 * kGroups);   // softmax warps
            mbar_init(&m.p_empty[s], 1);  // PV completion
            mbar_init(&m.a_full[s], kGroups);  // thread 0 of each softmax group
            mbar_init(&m.c_full[s], 4);   // correction warps
            mbar_init(&m.o_full[s], 1);   // last PV of an item
            mbar_init(&m.o_empty[s], 4);  // correction warps, epilogue done
            mbar_init(&m.l_full[s], kGroups);  // thread 0 of each softmax group
        }
        mbar_init(&m.drain, 1);
        m.abort = 0;
        for (int q = 0; q < 64; ++q) m.m_sh[q] = -INFINITY;
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(&m.tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == kWarpProducer && lane == 0) {
        prefetch_tmap(&tmq);
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = m.tmem_base;

    if (warp == kWarpProducer) {
        // -------------------------------------------------------- TMA producer
        int g = 0, n = 0;
        int armed_k[2] = {-1, -1}, armed_v[2] = {-1, -1}, armed_q[2] = {-1, -1};
        bool aborted = false;
        for (int item = blockIdx.x; item < n_items && !aborted; item += gridDim.x, ++n) {
            const int i = item % nq, bh = item / nq;
            const int h = bh % H, b = bh / H;
            const int tok0 = b * S;
            const int32_t* sel = topk_idx + (int64_t)item * topk;
            if (lane == 0) {
                const int qs = n % L::NQ;
                if (wait_bar(&m.q_empty[qs], ((n / L::NQ) & 1) ^ 1, m, err)) {
                    mbar_expect_tx(&m.q_full[qs], kQBytes);
                    armed_q[qs] = (n / L::NQ) & 1;
                    uint8_t* qdst = tiles_ptr + L::Q_OFF + qs * kQBytes;
                    tma_load_3d(&tmq, &m.q_full[qs], qdst, 0, h, tok0 + 64 * i);
                    tma_load_3d(&tmq, &m.q_full[qs], qdst + kTileHalf, 64, h, tok0 + 64 * i);
                } else {
                    aborted = true;
                }
            }
            aborted = __shfl_sync(0xffffffffu, aborted, 0);
            for (int c0 = 0; c0 < topk && !aborted; c0 += kListChunk) {
                const int cn = min(kListChunk, topk - c0);
                __syncwarp();
                for (int e = lane; e < cn; e += 32) {
                    int j;
                    m.list_n[e] = cube_count(sel, c0 + e, topk, nq, vbs, j, err);
                    m.list_id[e] = j;
                }
                __syncwarp();
                if (lane == 0) {
                    for (int e = 0; e < cn; e += 2, ++g) {
                        const int n0 = m.list_n[e], j0 = m.list_id[e];
                        const int n1 = e + 1 < cn ? m.list_n[e + 1] : 0, j1 = e + 1 < cn ? m.list_id[e + 1] : 0;
                        const uint32_t bytes = kCubeBytes * ((n0 > 0) + (n1 > 0));
                        const int ks = g % L::NK, vs = g % L::NV;
                        if (!wait_bar(&m.k_empty[ks], ((g / L::NK) & 1) ^ 1, m, err)) { aborted = true; break; }
                        m.k_meta[ks][0] = n0;
                        m.k_meta[ks][1] = n1;
                        mbar_expect_tx(&m.k_full[ks], bytes);
                        armed_k[ks] = (g / L::NK) & 1;
                        uint8_t* kdst = tiles_ptr + L::K_OFF + ks * kKVBytes;
                        if (n0 > 0) {
                            tma_load_3d(&tmk, &m.k_full[ks], kdst, 0, h, tok0 + 64 * j0);
                            tma_load_3d(&tmk, &m.k_full[ks], kdst + 2 * kTileHalf, 64, h, tok0 + 64 * j0);
                        }
                        if (n1 > 0) {
                            tma_load_3d(&tmk, &m.k_full[ks], kdst + kTileHalf, 0, h, tok0 + 64 * j1);
                            tma_load_3d(&tmk, &m.k_full[ks], kdst + 3 * kTileHalf, 64, h, tok0 + 64 * j1);
                        }
                        if (!wait_bar(&m.v_empty[vs], ((g / L::NV) & 1) ^ 1, m, err)) { aborted = true; break; }
                        mbar_expect_tx(&m.v_full[vs], bytes);
                        armed_v[vs] = (g / L::NV) & 1;
                        uint8_t* vdst = tiles_ptr + L::V_OFF + vs * kKVBytes;
                        if (n0 > 0) {
                            tma_load_3d(&tmv, &m.v_full[vs], vdst, 0, h, tok0 + 64 * j0);
                            tma_load_3d(&tmv, &m.v_full[vs], vdst + 2 * kTileHalf, 64, h, tok0 + 64 * j0);
                        }
                        if (n1 > 0) {
                            tma_load_3d(&tmv, &m.v_full[vs], vdst + kTileHalf, 0, h, tok0 + 64 * j1);
                            tma_load_3d(&tmv, &m.v_full[vs], vdst + 3 * kTileHalf, 64, h, tok0 + 64 * j1);
                        }
                    }
                }
                aborted = __shfl_sync(0xffffffffu, aborted, 0);
                g = __shfl_sync(0xffffffffu, g, 0);
            }
        }
        if (aborted && lane == 0) {
            // copies issued by this thread must land before the CTA's shared memory goes away
            for (int s = 0; s < 2; ++s) {
                if (armed_q[s] >= 0) drain_wait(&m.q_full[s], armed_q[s]);
                if (armed_k[s] >= 0) drain_wait(&m.k_full[s], armed_k[s]);
                if (armed_v[s] >= 0) drain_wait(&m.v_full[s], armed_v[s]);
            }
        }
    } else if (warp == kWarpMma) {
        // -------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 64, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, L::PV_N, true, true);
            const uint32_t q_base = tiles + L::Q_OFF, k_base = tiles + L::K_OFF;
            const uint32_t v_base = tiles + L::V_OFF, p_base = tiles + L::P_OFF;
            int g = 0, n = 0;
            bool aborted = false;
            for (int item = blockIdx.x; item < n_items && !aborted; item += gridDim.x, ++n) {
                const int qs = n % L::NQ, os = n & 1;
                const uint32_t o_tmem = tbase + L::O_COL0 + os * L::O_COLS;
                if (!wait_bar(&m.o_empty[os], ((n >> 1) & 1) ^ 1, m, err)) { aborted = true; break; }
                if (!wait_bar(&m.q_full[qs], (n / L::NQ) & 1, m, err)) { aborted = true; break; }
                bool o_init = false;
                auto issue_pv = [&](int gs) -> bool {
                    const int vs = gs % L::NV, ps = gs & 1;
                    if (!wait_bar(&m.v_full[vs], (gs / L::NV) & 1, m, err)) return false;
                    if (!wait_bar(&m.p_full[ps], (gs >> 1) & 1, m, err)) return false;
                    if (!wait_bar(&m.c_full[ps], (gs >> 1) & 1, m, err)) return false;
                    tc_fence_after();
                    const int cnt[2] = {m.s_meta[ps][0], m.s_meta[ps][1]};
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const int nk = (cnt[c] + 15) >> 4;
                        for (int kk = 0; kk < nk; ++kk) {
                            const int kstep = 4 * c + kk;
                            const uint64_t a = smem_desc_sw128(v_base + vs * kKVBytes + kstep * 2048, 16384, 1024);
                            const uint64_t bdesc =
                                smem_desc_sw128(p_base + ps * L::P_BYTES + kstep * 2048, 16384, 1024);
                            umma_ss(o_tmem, a, bdesc, idesc_pv, o_init ? 1u : 0u);
                            o_init = true;
                        }
                    }
                    umma_commit(&m.v_empty[vs]);
                    umma_commit(&m.p_empty[ps]);
                    return true;
                };
                for (int p = 0; p < nsteps; ++p, ++g) {
                    const int ks = g % L::NK, ss = g & 1;
                    if (!wait_bar(&m.k_full[ks], (g / L::NK) & 1, m, err)) { aborted = true; break; }
                    if (!wait_bar(&m.s_empty[ss], ((g >> 1) & 1) ^ 1, m, err)) { aborted = true; break; }
                    m.s_meta[ss][0] = m.k_meta[ks][0];
                    m.s_meta[ss][1] = m.k_meta[ks][1];
                    mbar_arrive(&m.s_full[ss]);  // publishes s_meta (release)
                    tc_fence_after();
                    const uint32_t s_tmem = tbase + L::S_COL0 + ss * 64;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk & 3) * 32u;
                        const uint64_t a = smem_desc_sw128(k_base + ks * kKVBytes + (kk >> 2) * (2 * kTileHalf) + off,
                                                           16, 1024);
                        const uint64_t bdesc = smem_desc_sw128(q_base + qs * kQBytes + (kk >> 2) * kTileHalf + off,
                                                               16, 1024);
                        umma_ss(s_tmem, a, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&m.s_full[ss]);
                    umma_commit(&m.k_empty[ks]);
                    if (p == nsteps - 1) umma_commit(&m.q_empty[qs]);
                    if (p > 0 && !issue_pv(g - 1)) { aborted = true; break; }
                }
                if (aborted) break;
                if (!issue_pv(g - 1)) { aborted = true; break; }
                umma_commit(&m.o_full[os]);
            }
            if (aborted) {
                umma_commit(&m.drain);
                drain_wait(&m.drain, 0);
            }
        }
    } else if (warp < kWarpCorr0) {
        // -------------------------------------------------------- softmax (warps 0-15)
        const int grp = warp >> 2;           // query columns q0 .. q0 + kCols - 1
        const int wq = warp & 3;             // warp within the group == TMEM lane quarter
        const int t = threadIdx.x & 127;     // TMEM lane == key of the pair
        const uint32_t bar_id = 1 + grp;     // named barrier of the group
        const int q0 = kCols * grp;
        const uint32_t lane_base = tbase + ((uint32_t)(wq * 32) << 16);
        const uint32_t p_base = tiles + L::P_OFF;
        const uint32_t v_base = tiles + L::V_OFF;
        int g = 0, n = 0;
        float lsum[kCols];
        for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++n) {
#pragma unroll
            for (int q = 0; q < kCols; ++q) lsum[q] = 0.f;
            for (int p = 0; p < nsteps; ++p, ++g) {
                const int ss = g & 1;
                wait_bar(&m.s_full[ss], (g >> 1) & 1, m, err);  // an abort is acted on at the step barrier
                __syncwarp();
                const int n0 = m.s_meta[ss][0], n1 = m.s_meta[ss][1];
                const int my_n = t < 64 ? n0 : n1;
                const bool valid = (t & 63) < my_n;
                tc_fence_after();
                uint32_t r[kCols];  // raw scores of key t for this group's queries
                tmem_ld16(lane_base + L::S_COL0 + ss * 64 + q0, r);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&m.s_empty[ss]);  // S buffer may be overwritten

                // pass 1: per-query extreme of the raw scores over the 128 keys (max for
                // a positive scale, min for a negative one: NEG); masked keys take the
                // neutral value, so garbage never takes part
                {
                    const bool all_valid = __all_sync(0xffffffffu, valid);  // warp-uniform
                    const float neutral = NEG ? INFINITY : -INFINITY;
#pragma unroll
                    for (int q4 = 0; q4 < kCols / 4; ++q4) {
                        float w[4];
                        if (all_valid) {
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                w[e] = NEG ? redux_min(__uint_as_float(r[4 * q4 + e])) : redux_max(__uint_as_float(r[4 * q4 + e]));
                        } else {
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float v = valid ? __uint_as_float(r[4 * q4 + e]) : neutral;
                                w[e] = NEG ? redux_min(v) : redux_max(v);
                            }
                        }
                        if (lane == 0)
                            asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(&m.red_sh[grp][wq][4 * q4])),
                                         "f"(w[0]), "f"(w[1]), "f"(w[2]), "f"(w[3])
                                         : "memory");
                    }
                }
                if (lane == 0) m.flags[g & 1][warp] = aborted_flag(m) ? 1 : 0;
                named_bar_sync(bar_id, 128);
                {
                    const int* f = &m.flags[g & 1][4 * grp];
                    if ((f[0] | f[1] | f[2] | f[3]) != 0) goto softmax_exit;  // the same decision in the group
                }
                if (wq == 0) {
                    bool raise = false;
                    if (lane < kCols) {
                        const int q = q0 + lane;
                        const float e0 = m.red_sh[grp][0][lane], e1 = m.red_sh[grp][1][lane];
                        const float e2 = m.red_sh[grp][2][lane], e3 = m.red_sh[grp][3][lane];
                        const float ext = NEG ? fminf(fminf(e0, e1), fminf(e2, e3)) : fmaxf(fmaxf(e0, e1), fmaxf(e2, e3));
                        const float step = isinf(ext) ? -INFINITY : ext * scale_log2;  // no valid key: -inf
                        const float m_old = m.m_sh[q];
                        raise = step > m_old + kTau;  // false when step is -inf
                        const float m_new = raise ? step : m_old;
                        m.m_sh[q] = m_new;
                        m.mu_sh[q] = m_new == -INFINITY ? 0.f : m_new;
                        m.alpha[g & 1][q] = raise ? (m_old == -INFINITY ? 0.f : ex2(m_old - m_new)) : 1.f;
                    }
                    const bool any_raise = __any_sync(0xffffffffu, raise);
                    if (lane == 0) {
                        m.rflag[g & 1][grp] = any_raise ? 1 : 0;
                        m.info[g & 1][grp] = (any_raise ? 1 : 0) | ((n0 + n1) > 0 ? 2 : 0);
                    }
                }
                named_bar_sync(bar_id, 128);
                const bool resc = m.rflag[g & 1][grp] != 0;
                if (t == 0) mbar_arrive(&m.a_full[g & 1]);

                // pass 2: P = exp2(x - m) -> this group's columns of P^T row t
                // (MN-major, 128B swizzle: 16-byte chunk c of row t at c ^ (t & 7))
                const int ps = g & 1;
                wait_bar(&m.p_empty[ps], ((g >> 1) & 1) ^ 1, m, err);
                __syncwarp();
                if (resc) {
#pragma unroll
                    for (int q4 = 0; q4 < kCols / 4; ++q4) {
                        const float4 al = lds128(&m.alpha[g & 1][q0 + 4 * q4]);
                        lsum[4 * q4] *= al.x;
                        lsum[4 * q4 + 1] *= al.y;
                        lsum[4 * q4 + 2] *= al.z;
                        lsum[4 * q4 + 3] *= al.w;
                    }
                }
                const uint32_t prow = p_base + ps * L::P_BYTES + t * 128;
                if (valid) {
#pragma unroll
                    for (int c = 0; c < kCols / 8; ++c) {  // 8 queries = one 16-byte chunk of the row
                        const int c8 = q0 / 8 + c;
                        const float4 mA = lds128(&m.mu_sh[8 * c8]);
                        const float4 mB = lds128(&m.mu_sh[8 * c8 + 4]);
                        const float mu[8] = {mA.x, mA.y, mA.z, mA.w, mB.x, mB.y, mB.z, mB.w};
                        float pv[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            pv[e] = ex2(fmaf(__uint_as_float(r[8 * c + e]), scale_log2, -mu[e]));
                            lsum[8 * c + e] += pv[e];
                        }
                        const uint32_t h0 = pack_bf16(pv[0], pv[1]), h1 = pack_bf16(pv[2], pv[3]);
                        const uint32_t h2 = pack_bf16(pv[4], pv[5]), h3 = pack_bf16(pv[6], pv[7]);
                        const uint32_t addr = prow + (((uint32_t)c8 ^ (t & 7)) << 4);
                        sts128(addr, h0, h1, h2, h3);
                        if (PRECISE) {
                            const uint32_t hh[4] = {h0, h1, h2, h3};
                            uint32_t lo[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float a0 = __uint_as_float(hh[e] << 16);
                                const float a1 = __uint_as_float(hh[e] & 0xFFFF0000u);
                                lo[e] = pack_bf16(pv[2 * e] - a0, pv[2 * e + 1] - a1);
                            }
                            sts128(addr + 16384, lo[0], lo[1], lo[2], lo[3]);
                        }
                    }
                } else {
                    // a masked key: its weights are exactly zero (its scores are never read)
#pragma unroll
                    for (int c = 0; c < kCols / 8; ++c) {
                        const uint32_t addr = prow + (((uint32_t)(q0 / 8 + c) ^ (t & 7)) << 4);
                        sts128(addr, 0, 0, 0, 0);
                        if (PRECISE) sts128(addr + 16384, 0, 0, 0, 0);
                    }
                }
                // V rows between vbs and the next multiple of 16 are read by the last
                // issued k-step of their cube: group 0 zeroes key t's row (both halves).
                const int vs = g % L::NV;
                const bool zero_row = grp == 0 && !valid && (t & 63) < ((my_n + 15) & ~15);
                if (__any_sync(0xffffffffu, zero_row)) {
                    wait_bar(&m.v_full[vs], (g / L::NV) & 1, m, err);  // V must have landed
                    __syncwarp();
                }
                if (zero_row) {
#pragma unroll
                    for (int half = 0; half < 2; ++half)
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            sts128(v_base + vs * kKVBytes + half * 2 * kTileHalf + t * 128 + c * 16, 0, 0, 0, 0);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&m.p_full[ps]);
            }

            // item end: per-query weight sums and offsets for the epilogue.  Butterfly
            // over the warp: afterwards lanes l and l + 16 hold the sum of query q0 + (l & 15).
            {
#pragma unroll
                for (int w = kCols / 2, bit = kCols / 2; w >= 1; w >>= 1, bit >>= 1) {
                    const bool up = lane & bit;
#pragma unroll
                    for (int q = 0; q < kCols / 2; ++q) {
                        if (q < w) {
                            const float send = up ? lsum[q] : lsum[q + w];
                            const float keep = up ? lsum[q + w] : lsum[q];
                            lsum[q] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
                        }
                    }
                }
                lsum[0] += __shfl_xor_sync(0xffffffffu, lsum[0], 16);
                if (lane < kCols) m.red_sh[grp][wq][lane] = lsum[0];
                named_bar_sync(bar_id, 128);
                if (wq == 0 && lane < kCols) {
                    const int q = q0 + lane;
                    m.lfin[n & 1][q] = m.red_sh[grp][0][lane] + m.red_sh[grp][1][lane] + m.red_sh[grp][2][lane] +
                                       m.red_sh[grp][3][lane];
                    m.mfin[n & 1][q] = m.m_sh[q];
                    m.m_sh[q] = -INFINITY;  // the next item starts afresh
                }
                named_bar_sync(bar_id, 128);
                if (t == 0) mbar_arrive(&m.l_full[n & 1]);
            }
        }
    softmax_exit:;
    } else if (warp < kWarpProducer) {
        // -------------------------------------------------------- correction + epilogue (warps 16-19)
        const int d = threadIdx.x - 32 * kWarpCorr0;  // TMEM lane of O^T == head-dim index
        const uint32_t lane_base = tbase + ((uint32_t)((warp - kWarpCorr0) * 32) << 16);
        int g = 0, n = 0;
        for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++n) {
            const int i = item % nq, bh = item / nq;
            const int h = bh % H, b = bh / H;
            const int os = n & 1;
            const uint32_t o_col = lane_base + L::O_COL0 + os * L::O_COLS;
            bool o_valid = false;
            for (int p = 0; p < nsteps; ++p, ++g) {
                if (!wait_warp(&m.a_full[g & 1], (g >> 1) & 1, m, err)) goto corr_exit;
                int info = 0;
#pragma unroll
                for (int gi = 0; gi < kGroups; ++gi) info |= m.info[g & 1][gi];
                if ((info & 1) && o_valid) {
                    // every PV issued so far must be complete before O is rescaled
                    if (!wait_warp(&m.p_empty[(g - 1) & 1], ((g - 1) >> 1) & 1, m, err)) goto corr_exit;
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < (PRECISE ? 8 : 4); ++c) {  // 16 columns at a time
                        uint32_t r[16];
                        const uint32_t addr = o_col + 16 * c;
                        tmem_ld16(addr, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            const float4 al = lds128(&m.alpha[g & 1][(16 * c + 4 * q4) & 63]);
                            r[4 * q4] = __float_as_uint(__uint_as_float(r[4 * q4]) * al.x);
                            r[4 * q4 + 1] = __float_as_uint(__uint_as_float(r[4 * q4 + 1]) * al.y);
                            r[4 * q4 + 2] = __float_as_uint(__uint_as_float(r[4 * q4 + 2]) * al.z);
                            r[4 * q4 + 3] = __float_as_uint(__uint_as_float(r[4 * q4 + 3]) * al.w);
                        }
                        tmem_st16(addr, r);
                    }
                    tmem_st_wait();
                }
                if (info & 2) o_valid = true;
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&m.c_full[g & 1]);
            }
            // epilogue: out[b, 64 i + q, h, d] = O^T[d][q] / l[q]; lse from (m, l)
            if (!wait_warp(&m.l_full[os], (n >> 1) & 1, m, err)) goto corr_exit;
            if (!wait_warp(&m.o_full[os], (n >> 1) & 1, m, err)) goto corr_exit;
            tc_fence_after();
            if (lse != nullptr && d < 64) {
                const float l = m.lfin[os][d];
                lse[((int64_t)b * H + h) * S + 64LL * i + d] =
                    l > 0.f ? (m.mfin[os][d] + __log2f(l)) * 0.69314718055994531f : -INFINITY;
            }
            uint16_t* dst = out + ((int64_t)b * S + 64LL * i) * H * kD + (int64_t)h * kD + d;
#pragma unroll
            for (int c = 0; c < 4; ++c) {  // 16 queries at a time
                uint32_t r[16];
                tmem_ld16(o_col + 16 * c, r);
                tmem_ld_wait();
                float o[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) o[q] = __uint_as_float(r[q]);
                if (PRECISE) {
                    tmem_ld16(o_col + 64 + 16 * c, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 16; ++q) o[q] += __uint_as_float(r[q]);
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const float4 l4 = lds128(&m.lfin[os][16 * c + 4 * q4]);
                    const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int q = 16 * c + 4 * q4 + e;
                        const float val = lv[e] > 0.f ? o[4 * q4 + e] / lv[e] : 0.f;
                        __nv_bfloat16 bv = __float2bfloat16_rn(val);
                        dst[(int64_t)q * H * kD] = *reinterpret_cast<uint16_t*>(&bv);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&m.o_empty[os]);
        }
    corr_exit:;
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) tmem_dealloc(tbase, 512);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// [B*S tokens][H][D] bf16 viewed as a 3-D tensor; box = 64 d x 1 head x 64 tokens.
bool make_map(CUtensorMap* map, const void* base, int64_t tokens, int H)
{
    auto enc = encode_fn();
    if (enc == nullptr) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)tokens};
    const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2};
    const cuuint32_t box[3] = {64, 1, 64};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool PRECISE, bool NEG>
cudaError_t launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const int32_t* topk_idx,
                   const int32_t* vbs, uint16_t* out, float* lse, int B, int S, int H, int nq, int topk,
                   float scale_log2, int* err, cudaStream_t s)
{
    using L = Layout<PRECISE>;
    auto kern = fwd_tc_kernel<PRECISE, NEG>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int n_items = B * H * nq;
    const int grid = n_items < sms ? n_items : sms;
    kern<<<grid, kThreads, L::SMEM_BYTES, s>>>(mq, mk, mv, topk_idx, vbs, out, lse, S, H, nq, topk, n_items,
                                               scale_log2, err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_tc(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* topk_idx,
                          const int32_t* vbs, uint16_t* out, float* lse, int B, int S, int H, int nq, int topk,
                          float sm_scale, bool precise_p, int* err, cudaStream_t s)
{
    CUtensorMap mq, mk, mv;
    const int64_t tokens = (int64_t)B * S;
    if (!make_map(&mq, q, tokens, H) || !make_map(&mk, k, tokens, H) || !make_map(&mv, v, tokens, H))
        return cudaErrorInvalidValue;
    const float scale_log2 = sm_scale * 1.4426950408889634f;
    const bool neg = scale_log2 < 0.f;
    if (precise_p)
        return neg ? launch<true, true>(mq, mk, mv, topk_idx, vbs, out, lse, B, S, H, nq, topk, scale_log2, err, s)
                   : launch<true, false>(mq, mk, mv, topk_idx, vbs, out, lse, B, S, H, nq, topk, scale_log2, err, s);
    return neg ? launch<false, true>(mq, mk, mv, topk_idx, vbs, out, lse, B, S, H, nq, topk, scale_log2, err, s)
               : launch<false, false>(mq, mk, mv, topk_idx, vbs, out, lse, B, S, H, nq, topk, scale_log2, err, s);
}

}  // namespace vsa
