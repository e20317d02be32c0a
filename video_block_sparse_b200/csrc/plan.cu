// Tile plan for the paired forward kernel: which two query cubes of a
// (batch, head) share one 128-row tile.
//
// The paired kernel walks the union of the two cubes' selection lists and
// loads a KV cube that both select once for both.  Its cost (tensor work and
// L2->SM gather traffic) therefore falls with the overlap of the two lists.
// The plan pairs query cubes whose lists overlap most:
//
//   1. bits   : one Nq-bit membership bitmap per selection list;
//   2. cand   : for every query cube i, the kCand cubes j != i with the
//               largest overlap |L_i ∩ L_j| (popcount of the bitmaps' AND),
//               ties broken by the smaller j;
//   3. match  : rounds of mutual proposals: every unpaired cube proposes to
//               its first still-unpaired candidate; two cubes that propose
//               to each other are paired.  Rounds repeat until none pairs.
//               Refills: while two or more cubes are unpaired, their
//               candidates are recomputed among the unpaired cubes (same
//               rule) and the rounds run again, until a refill pairs none.
//               Without the refills ~55 of 624 cubes per head at Wan 832x480
//               ended up paired in index order, whatever their overlap, and
//               the CTAs that drew those tiles set the forward's end.
//               Cubes left over are paired in index order (the last one
//               alone if their number is odd).  Tiles are emitted in order
//               of their smaller cube index, as (smaller, larger) or (i, -1).
//
// Every step is integer work with fixed tie rules, so the plan is
// deterministic and reproducible.  The plan changes only which cubes share
// a tile: the attention result does not depend on it.
#include "internal.h"

#include <cstdint>

namespace vsa {
namespace {

constexpr int kCand = 8;
constexpr int kMaxRounds = 64;
constexpr int kMaxRefills = 64;

// One warp per (bh, i) list: clear the bitmap row, then set the listed bits.
__global__ void plan_bits_kernel(const int32_t* __restrict__ topk_idx, uint32_t* __restrict__ bits, int n_lists,
                                 int nq, int topk, int words, int* err)
{
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= n_lists) return;
    uint32_t* row = bits + (int64_t)warp * words;
    for (int w = lane; w < words; w += 32) row[w] = 0u;
    __syncwarp();
    const int32_t* list = topk_idx + (int64_t)warp * topk;
    for (int t = lane; t < topk; t += 32) {
        const int j = __ldg(list + t);
        if (j < 0 || j >= nq) {
            atomicCAS(err, 0, (int)kErrTopkIdx);
            continue;
        }
        atomicOr(row + (j >> 5), 1u << (j & 31));
    }
}

// Insert (ov, j) into a descending top-kCand list kept in registers; ties by smaller j.
__device__ __forceinline__ void cand_insert(int (&co)[kCand], int (&cj)[kCand], int ov, int j)
{
    if (ov < co[kCand - 1] || (ov == co[kCand - 1] && j > cj[kCand - 1])) return;
    int p = kCand - 1;
    while (p > 0 && (ov > co[p - 1] || (ov == co[p - 1] && j < cj[p - 1]))) {
        co[p] = co[p - 1];
        cj[p] = cj[p - 1];
        --p;
    }
    co[p] = ov;
    cj[p] = j;
}

// Merge the 32 lanes' candidate lists (each sorted, larger overlap first, ties by
// the smaller cube): kCand rounds of a warp-wide (max ov, min j) pick; lane 0
// writes the winners (-1 where there are fewer than kCand), and their overlaps
// if out_o is given.
__device__ void warp_merge_cand(const int (&co)[kCand], const int (&cj)[kCand], int lane, int32_t* out_j,
                                int32_t* out_o)
{
    int head = 0;
    for (int c = 0; c < kCand; ++c) {
        int ov = -1, j = 0x7fffffff;
#pragma unroll
        for (int q = 0; q < kCand; ++q)
            if (q == head) {
                ov = co[q];
                j = cj[q];
            }
        // key: larger ov first, then smaller j
        for (int s = 16; s >= 1; s >>= 1) {
            const int ov2 = __shfl_xor_sync(0xffffffffu, ov, s);
            const int j2 = __shfl_xor_sync(0xffffffffu, j, s);
            if (ov2 > ov || (ov2 == ov && j2 < j)) {
                ov = ov2;
                j = j2;
            }
        }
        // the owner of the winner advances its head
        bool mine = false;
#pragma unroll
        for (int q = 0; q < kCand; ++q)
            if (q == head && cj[q] == j && co[q] == ov) mine = true;
        if (mine) ++head;
        if (lane == 0) {
            out_j[c] = ov >= 0 ? j : -1;
            if (out_o != nullptr) out_o[c] = ov;
        }
    }
}

// CTA = (bh, 32 consecutive rows); warp w handles row i0 + w.  Column
// bitmaps are staged through shared memory in chunks, each row padded with
// zero words to ws words (a multiple of 4 with ws / 4 odd), so that the
// 16-byte loads of 32 lanes reading 32 different rows hit distinct banks in
// every quarter warp.
__global__ void __launch_bounds__(1024) plan_cand_kernel(const uint32_t* __restrict__ bits, int32_t* __restrict__ cand,
                                                         int32_t* __restrict__ cand_ov, int nq, int words, int ws,
                                                         int chunk_rows)
{
    extern __shared__ uint4 sh4[];
    uint32_t* sh = reinterpret_cast<uint32_t*>(sh4);
    const int rb = (nq + 31) / 32;
    const int bh = blockIdx.x / rb, i0 = (blockIdx.x % rb) * 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t* bbh = bits + (int64_t)bh * nq * words;
    uint32_t* rows = sh;                     // 32 x ws: this CTA's rows
    uint32_t* cols = sh + 32 * ws;           // chunk_rows x ws: current column chunk
    for (int e = threadIdx.x; e < 32 * ws; e += blockDim.x) {
        const int r = e / ws, w = e - r * ws;
        rows[e] = i0 + r < nq && w < words ? bbh[(int64_t)(i0 + r) * words + w] : 0u;
    }
    const int i = i0 + warp;
    int co[kCand], cj[kCand];
#pragma unroll
    for (int c = 0; c < kCand; ++c) {
        co[c] = -1;
        cj[c] = 0x7fffffff;
    }
    for (int c0 = 0; c0 < nq; c0 += chunk_rows) {
        const int cn = min(chunk_rows, nq - c0);
        __syncthreads();
        for (int e = threadIdx.x; e < cn * ws; e += blockDim.x) {
            const int r = e / ws, w = e - r * ws;
            cols[e] = w < words ? bbh[(int64_t)(c0 + r) * words + w] : 0u;
        }
        __syncthreads();
        if (i < nq) {
            const uint4* ri = reinterpret_cast<const uint4*>(rows + warp * ws);
            for (int jj = lane; jj < cn; jj += 32) {
                const int j = c0 + jj;
                if (j == i) continue;
                const uint4* rj = reinterpret_cast<const uint4*>(cols + jj * ws);
                int ov = 0;
                for (int w = 0; w < ws / 4; ++w) {
                    const uint4 a = ri[w], b = rj[w];
                    ov += __popc(a.x & b.x) + __popc(a.y & b.y) + __popc(a.z & b.z) + __popc(a.w & b.w);
                }
                cand_insert(co, cj, ov, j);
            }
        }
    }
    if (i >= nq) return;
    warp_merge_cand(co, cj, lane, cand + ((int64_t)bh * nq + i) * kCand, cand_ov + ((int64_t)bh * nq + i) * kCand);
}

// One CTA per (bh): proposal rounds over the candidate lists; refills while
// two or more cubes are unpaired (their candidates recomputed among the
// unpaired cubes, then the rounds again); leftovers in index order; then the
// tiles in order of their smaller cube.
__global__ void __launch_bounds__(1024) plan_match_kernel(int32_t* cand, const uint32_t* __restrict__ bits,
                                                          int32_t* __restrict__ plan, int nq, int words)
{
    extern __shared__ int32_t smi[];
    int32_t* partner = smi;       // nq: paired cube, -1 unpaired
    int32_t* prop = smi + nq;     // nq: this round's proposal
    __shared__ int n_unpaired;
    __shared__ int nleft;
    const int bh = blockIdx.x;
    // candidate lists: written by plan_cand_kernel, rewritten here by the refills
    // (plain loads: the read-only path must not serve them)
    int32_t* cb = cand + (int64_t)bh * nq * kCand;
    const uint32_t* bbh = bits + (int64_t)bh * nq * words;
    for (int i = threadIdx.x; i < nq; i += blockDim.x) partner[i] = -1;
    __syncthreads();
    for (int refill = 0; refill <= kMaxRefills; ++refill) {
        if (refill > 0) {
            int mine = 0;
            for (int i = threadIdx.x; i < nq; i += blockDim.x) mine += partner[i] < 0 ? 1 : 0;
            if (threadIdx.x == 0) n_unpaired = 0;
            __syncthreads();
            if (mine > 0) atomicAdd(&n_unpaired, mine);
            __syncthreads();
            if (n_unpaired < 2) break;  // the same value in every thread
            // each unpaired cube's kCand candidates among the unpaired cubes
            // (largest overlap first, ties by the smaller index, as plan_cand_kernel):
            // one warp per unpaired cube, its lanes over the other unpaired cubes
            const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
            for (int i = warp; i < nq; i += (int)(blockDim.x >> 5)) {
                if (partner[i] >= 0) continue;  // warp-uniform
                int co[kCand], cj[kCand];
#pragma unroll
                for (int c = 0; c < kCand; ++c) {
                    co[c] = -1;
                    cj[c] = 0x7fffffff;
                }
                const uint32_t* bi = bbh + (int64_t)i * words;
                for (int j = lane; j < nq; j += 32) {
                    if (j == i || partner[j] >= 0) continue;
                    const uint32_t* bj = bbh + (int64_t)j * words;
                    int ov = 0;
                    for (int w = 0; w < words; ++w) ov += __popc(__ldg(bi + w) & __ldg(bj + w));
                    cand_insert(co, cj, ov, j);
                }
                warp_merge_cand(co, cj, lane, cb + (int64_t)i * kCand, nullptr);
            }
            __syncthreads();
        }
        bool paired_any = false;
        for (int round = 0; round < kMaxRounds; ++round) {
            for (int i = threadIdx.x; i < nq; i += blockDim.x) {
                int p = -1;
                if (partner[i] < 0) {
                    for (int c = 0; c < kCand; ++c) {
                        const int j = cb[(int64_t)i * kCand + c];
                        if (j >= 0 && partner[j] < 0) {
                            p = j;
                            break;
                        }
                    }
                }
                prop[i] = p;
            }
            __syncthreads();
            int mine = 0;
            for (int i = threadIdx.x; i < nq; i += blockDim.x) {
                const int j = prop[i];
                if (j >= 0 && prop[j] == i) {
                    partner[i] = j;  // the mirror thread sets partner[j]
                    mine = 1;
                }
            }
            if (!__syncthreads_or(mine)) break;  // a barrier too: the next round reads partner
            paired_any = true;
        }
        if (!paired_any) break;  // the same in every thread
    }
    // leftovers: pair in index order (one warp, ballot-based)
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int pending = -1;  // warp-uniform: a leftover waiting for its mate
        for (int base = 0; base < nq; base += 32) {
            const int i = base + lane;
            const bool left = i < nq && partner[i] < 0;
            uint32_t mask = __ballot_sync(0xffffffffu, left);
            while (mask) {
                const int l = __ffs(mask) - 1;
                mask &= mask - 1;
                const int c = base + l;
                if (pending < 0) {
                    pending = c;
                } else {
                    if (lane == 0) {
                        partner[pending] = c;
                        partner[c] = pending;
                    }
                    pending = -1;
                }
            }
            __syncwarp();
        }
        if (lane == 0) nleft = pending;  // the odd one out (or -1)
    }
    __syncthreads();
    // emit: a tile per cube i with partner > i, or the single leftover
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int pos = 0;
        int32_t* pb = plan + (int64_t)bh * ((nq + 1) / 2) * 2;
        for (int base = 0; base < nq; base += 32) {
            const int i = base + lane;
            const bool lead = i < nq && (partner[i] > i || i == nleft);
            const uint32_t mask = __ballot_sync(0xffffffffu, lead);
            if (lead) {
                const int p = pos + __popc(mask & ((1u << lane) - 1u));
                pb[2 * p] = i;
                pb[2 * p + 1] = i == nleft ? -1 : partner[i];
            }
            pos += __popc(mask);
        }
    }
}

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

size_t plan_workspace_bytes(int B, int H, int nq)
{
    const size_t words = (size_t)(nq + 31) / 32;
    const size_t lists = (size_t)B * H * nq;
    return align256(lists * words * 4) + 2 * align256(lists * kCand * 4);
}

cudaError_t launch_plan(const int32_t* topk_idx, int32_t* plan, int B, int H, int nq, int topk, void* workspace,
                        int* err, cudaStream_t s)
{
    const int words = (nq + 31) / 32;
    const int64_t lists = (int64_t)B * H * nq;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint32_t* bits = reinterpret_cast<uint32_t*>(ws);
    int32_t* cand = reinterpret_cast<int32_t*>(ws + align256((size_t)lists * words * 4));
    int32_t* cand_ov = cand + align256((size_t)lists * kCand * 4) / 4;

    const int warps_per_block = 8;
    plan_bits_kernel<<<(unsigned)((lists + warps_per_block - 1) / warps_per_block), 32 * warps_per_block, 0, s>>>(
        topk_idx, bits, (int)lists, nq, topk, words, err);

    // padded row stride (a multiple of 4 words, stride / 4 odd); column chunk: up to
    // 32 KiB of bitmaps, plus this CTA's 32 rows
    int stride = (words + 3) / 4 * 4;
    if (((stride / 4) & 1) == 0) stride += 4;
    int chunk_rows = (32 * 1024) / (stride * 4);
    if (chunk_rows > 512) chunk_rows = 512;
    if (chunk_rows < 1) chunk_rows = 1;
    const size_t smem_c = (size_t)(32 + chunk_rows) * stride * 4;
    cudaError_t e = cudaFuncSetAttribute(plan_cand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_c);
    if (e != cudaSuccess) return e;
    const int rb = (nq + 31) / 32;
    plan_cand_kernel<<<(unsigned)(B * H * rb), 1024, smem_c, s>>>(bits, cand, cand_ov, nq, words, stride, chunk_rows);

    const size_t smem_m = (size_t)2 * nq * 4;
    e = cudaFuncSetAttribute(plan_match_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_m);
    if (e != cudaSuccess) return e;
    plan_match_kernel<<<(unsigned)(B * H), 1024, smem_m, s>>>(cand, bits, plan, nq, words);
    return cudaGetLastError();
}

}  // namespace vsa
