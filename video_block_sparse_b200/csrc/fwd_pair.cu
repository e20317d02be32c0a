// VSA fine forward on the Blackwell tensor cores: two query cubes per
// 128-row tile, queries on TMEM lanes, two tiles in flight per CTA, each tile
// ("slot") with its own producer, MMA issuer and correction warps.
//
// Dataset card "wan2.2_production_values", section "Operator contract": for
// query cube i of (batch b, head h) the keys are the first vbs[j] tokens of
// every cube j in topk_idx[b, h, i, :]; out = softmax(q k^T * sm_scale) v.
//
// Shape of the work on sm_100a.  A query cube has only 64 rows, and an MMA
// with M = 64 runs the tensor core at half rate, so two query cubes (i1 rows
// 0-63, i2 rows 64-127) of the same (b, h) share one 128-row tile that walks
// the union of their selection lists, two KV cubes (128 keys) per step:
//     S[128 q x 128 keys]  = Q_tile[128 x 128 d] . K_pair^T       (M=128, N=128)
//     O[128 q x 128 d]    += P[128 x 128 keys] . V_pair[128 keys x 128 d]
// both tcgen05.mma (bf16 in, fp32 accumulate in TMEM); P is written over S
// in TMEM as bf16 and is the A operand of the second product.  A KV cube
// that only one of the two query cubes selected has weight 0 for the other
// cube's rows.  Cubes both lists name are walked first and loaded once for
// both; vsa_plan pairs query cubes whose lists overlap most.
//
// Each softmax thread owns one query row (one TMEM lane): row maximum and row
// sum are thread-local.  Two tiles are in flight per CTA.  A slot's chain is
// strictly serial (QK -> softmax -> PV -> next QK, S/P reuse), so the slots
// are made fully independent: each has its own Q, K and V buffers, its own
// producer warp, MMA-issuing warp and correction warps, and the tensor core
// takes whichever slot's products are ready.  No warp ever waits on the other
// slot's progress.
//
// Roles (640 threads, one persistent CTA per SM):
//   warps 0-3 / 4-7    softmax + epilogue of slot 0 / 1 (thread = row = lane)
//   warps 8-11 / 12-15 O correction of slot 0 / 1: rescale the rows whose
//                      running offset rose (thread = row)
//   warp 16 / 18       TMA producer of slot 0 / 1: builds each tile's step list
//                      (shared cubes first) and streams its Q, K and V tiles
//   warp 17 / 19       MMA issuer of slot 0 / 1 (the whole warp runs the
//                      schedule, one elected lane issues); zeroes V pad rows
//                      inside a partial k-step before the product.  Warp 17
//                      also owns the TMEM allocation.
//
// Softmax.  Logits in base 2 (x = s * sm_scale * log2 e).  Keys at or beyond
// vbs of their cube and cubes the row's query cube did not select are
// replaced by -inf (a select: NaN/Inf there never propagates).  The running
// offset of a row is raised only when the step maximum exceeds it by more
// than kTau (so P <= 2^kTau); only then are the row of O and the row sum
// rescaled.  PV k-steps (16 keys) beyond ceil16(vbs) of a cube are not issued;
// V rows between vbs and that boundary are zeroed before the product, so
// 0 * NaN cannot occur.
//
// Every mbarrier wait is bounded (~2 s of clock): on expiry the kernel
// latches kErrWaitTimeout and raises a CTA-wide abort flag; every role leaves
// its loop, producers and MMA issuers wait (bounded) for their own copies and
// products in flight, and TMEM is freed before exit.
#include "fwd_pair_common.cuh"

namespace vsa {
namespace {

using namespace ptx;

constexpr int kThreads = 640;

// Pairs (bit c: columns 2c, 2c+1 of each 32-column chunk) whose exp2 runs on
// the FMA pipe instead of the multi-function unit.
#ifndef VSA_POLY_PAIRS
#define VSA_POLY_PAIRS 0x5252
#endif
constexpr uint32_t kPolyPairs = VSA_POLY_PAIRS;
constexpr int kWarpCorr0 = 8;  // warps 8-11 correct slot 0, 12-15 slot 1
constexpr int kWarpRole0 = 16; // warp 16 + 2x: producer of slot x, 17 + 2x: MMA issuer of slot x

struct SlotBars {
    uint64_t q_full, q_empty;  // Q tile landed / last QK of the tile done
    uint64_t k_full, k_empty;  // K pair landed / QK done
    uint64_t v_full, v_empty;  // V pair landed / PV done
    uint64_t s_full;           // step word published + QK done (2 arrivals)
    uint64_t a_full;           // offsets decided (128 softmax threads)
    uint64_t p_full;           // P written and O corrected (128 softmax + 128 correction threads)
    uint64_t o_full;           // last PV of a tile done
    uint64_t drain;
};

struct Misc {
    SlotBars bar[2];
    uint32_t k_meta[2];  // step word of the K pair in each slot's K buffer
    uint32_t s_meta[2];  // step word of the S in each slot
    uint32_t tmem_base;
    int abort;
    alignas(16) float alpha[2][128];  // per slot, row: O rescale factor of the current step
    int rflag[2][4];                  // per slot, warp: some row of the warp rescales
    uint32_t bits1[2][kMaxNq / 32];   // per slot: membership bitmap of list 1
    uint32_t bits2[2][kMaxNq / 32];   //                           and of list 2
    int32_t list1[2][kMaxTopk];       // per slot: the two selection lists
    int32_t list2[2][kMaxTopk];
};

struct Layout {
    static constexpr uint32_t Q_OFF = 0;                       // Q tile of slot x at Q_OFF + x * 32 KiB
    static constexpr uint32_t K_OFF = Q_OFF + 2 * kTileBytes;  // K pair of slot x
    static constexpr uint32_t V_OFF = K_OFF + 2 * kTileBytes;  // V pair of slot x
    static constexpr uint32_t TILE_BYTES = V_OFF + 2 * kTileBytes;
    static constexpr uint32_t MISC_BYTES = (sizeof(Misc) + 1023) / 1024 * 1024;
    static constexpr uint32_t SMEM_BYTES = MISC_BYTES + TILE_BYTES + 1024;  // + alignment slack
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// TMEM columns of slot x: S/P at 256x, O at 256x + 128.
__device__ __forceinline__ uint32_t s_col(int x) { return 256u * x; }
__device__ __forceinline__ uint32_t o_col(int x) { return 256u * x + 128u; }

template <bool NEG>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_pair_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv, const int32_t* __restrict__ topk_idx,
                    const int32_t* __restrict__ vbs, const int32_t* __restrict__ plan, uint16_t* __restrict__ out,
                    float* __restrict__ lse, int S, int H, int nq, int topk, int tiles_per_bh, int n_tiles,
                    float scale_log2, int* err)
{
    using L = Layout;
    extern __shared__ uint8_t smem_raw[];
    Misc& m = *reinterpret_cast<Misc*>(smem_raw);
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t tiles = (raw_addr + L::MISC_BYTES + 1023u) & ~1023u;  // 1 KiB aligned for 128B swizzle
    uint8_t* tiles_ptr = smem_raw + (tiles - raw_addr);

    const int warp = threadIdx.x >> 5;
    const uint32_t lane = threadIdx.x & 31;
    const int my_tiles = n_tiles > (int)blockIdx.x ? (n_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

    // ------------------------------------------------------------ set-up
    if (threadIdx.x == 0) {
        for (int x = 0; x < 2; ++x) {
            SlotBars& sb = m.bar[x];
            mbar_init(&sb.q_full, 1);
            mbar_init(&sb.q_empty, 1);
            mbar_init(&sb.k_full, 1);
            mbar_init(&sb.k_empty, 1);
            mbar_init(&sb.v_full, 1);
            mbar_init(&sb.v_empty, 1);
            mbar_init(&sb.s_full, 2);    // MMA warp (step word) + QK completion
            mbar_init(&sb.a_full, 128);  // every softmax thread of the slot
            mbar_init(&sb.p_full, 256);  // every softmax and every correction thread of the slot
            mbar_init(&sb.o_full, 1);
            mbar_init(&sb.drain, 1);
        }
        m.abort = 0;
        fence_mbar_init();
    }
    if (warp == kWarpRole0 + 1) {
        tmem_alloc(&m.tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == kWarpRole0 && lane == 0) {
        prefetch_tmap(&tmq);
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = m.tmem_base;

    if (warp >= kWarpRole0) {
        const int x = (warp - kWarpRole0) >> 1;
        SlotBars& sb = m.bar[x];
        uint8_t* qdst = tiles_ptr + L::Q_OFF + x * kTileBytes;
        uint8_t* kdst = tiles_ptr + L::K_OFF + x * kTileBytes;
        uint8_t* vdst = tiles_ptr + L::V_OFF + x * kTileBytes;
        if (((warp - kWarpRole0) & 1) == 0) {
            // ---------------------------------------------------- TMA producer of slot x
            ListGen gen;
            int qn = 0, kc = 0;
            int armed_q = -1, armed_k = -1, armed_v = -1;
            bool aborted = false;
            for (int n = x; n < my_tiles && !aborted; n += 2) {
                const TileRef t =
                    checked_tile(blockIdx.x + n * gridDim.x, H, nq, tiles_per_bh, plan, lane == 0 ? err : nullptr);
                gen_start(gen, t, topk_idx, vbs, H, nq, topk, m.list1[x], m.list2[x], m.bits1[x], m.bits2[x], err,
                          lane);
                const int tok0 = t.b * S;
                if (lane == 0) {
                    if (wait_bar(&sb.q_empty, (qn & 1) ^ 1, &m.abort, err)) {
                        mbar_expect_tx(&sb.q_full, 2 * kHalfBox * ((t.i1 >= 0) + (t.i2 >= 0)));
                        armed_q = qn & 1;
                        if (t.i1 >= 0) load_cube(&tmq, &sb.q_full, qdst, 0, t.h, tok0 + 64 * t.i1);
                        if (t.i2 >= 0) load_cube(&tmq, &sb.q_full, qdst, 1, t.h, tok0 + 64 * t.i2);
                    } else {
                        aborted = true;
                    }
                }
                aborted = __shfl_sync(0xffffffffu, aborted, 0);
                ++qn;
                bool first = true;
                while (!aborted) {
                    const Entry ea = gen.next;
                    Entry eb{0, 0, 0};
                    if (ea.mem != 0) {
                        gen.next = gen_pull(gen, m.list1[x], m.list2[x], m.bits1[x], m.bits2[x], vbs, lane);
                        eb = gen.next;
                        if (eb.mem != 0) gen.next = gen_pull(gen, m.list1[x], m.list2[x], m.bits1[x], m.bits2[x], vbs, lane);
                    }
                    const bool last = gen.next.mem == 0;
                    StepMeta meta;
                    meta.ja = ea.j;
                    meta.jb = eb.j;
                    meta.na = ea.n;
                    meta.nb = eb.n;
                    meta.ma = ea.mem;
                    meta.mb = eb.mem;
                    meta.flags = (first ? 1 : 0) | (last ? 2 : 0);
                    first = false;
                    const uint32_t bytes = 2 * kHalfBox * ((meta.na > 0) + (meta.nb > 0));
                    if (lane == 0) {
                        // K pair of the step: the buffer is free once the previous QK finished
                        if (wait_bar(&sb.k_empty, (kc & 1) ^ 1, &m.abort, err)) {
                            m.k_meta[x] = step_word(meta);
                            mbar_expect_tx(&sb.k_full, bytes);
                            armed_k = kc & 1;
                            if (meta.na > 0) load_cube(&tmk, &sb.k_full, kdst, 0, t.h, tok0 + 64 * meta.ja);
                            if (meta.nb > 0) load_cube(&tmk, &sb.k_full, kdst, 1, t.h, tok0 + 64 * meta.jb);
                        } else {
                            aborted = true;
                        }
                        // V pair of the step: free once the previous PV finished
                        if (!aborted && wait_bar(&sb.v_empty, (kc & 1) ^ 1, &m.abort, err)) {
                            mbar_expect_tx(&sb.v_full, bytes);
                            armed_v = kc & 1;
                            if (meta.na > 0) load_cube(&tmv, &sb.v_full, vdst, 0, t.h, tok0 + 64 * meta.ja);
                            if (meta.nb > 0) load_cube(&tmv, &sb.v_full, vdst, 1, t.h, tok0 + 64 * meta.jb);
                        } else {
                            aborted = true;
                        }
                    }
                    aborted = __shfl_sync(0xffffffffu, aborted, 0);
                    ++kc;
                    if (last) break;
                }
            }
            if (aborted && lane == 0) {
                // copies issued by this thread must land before the CTA's shared memory goes away
                if (armed_q >= 0) drain_wait(&sb.q_full, armed_q);
                if (armed_k >= 0) drain_wait(&sb.k_full, armed_k);
                if (armed_v >= 0) drain_wait(&sb.v_full, armed_v);
            }
        } else {
            // ---------------------------------------------------- MMA issuer of slot x
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, false, true);
            // operand descriptors built once; a k-step adds its byte offset / 16
            const uint64_t d_hi = smem_desc_sw128(0, 0, 1024);
            const uint32_t ql = (uint32_t)smem_desc_sw128(smem_u32(qdst), 16, 1024);
            const uint32_t kl = (uint32_t)smem_desc_sw128(smem_u32(kdst), 16, 1024);
            const uint32_t vl = (uint32_t)smem_desc_sw128(smem_u32(vdst), 2 * kHalfBox, 1024);
            const uint32_t s_tmem = tbase + s_col(x), o_tmem = tbase + o_col(x);
            int qn = 0, kc = 0;
            bool aborted = false;
            for (int n = x; n < my_tiles && !aborted; n += 2) {
                if (!wait_warp(&sb.q_full, qn & 1, &m.abort, err)) { aborted = true; break; }
                ++qn;
                bool o_init = false;
                for (;;) {
                    // ---- S = Q . K^T
                    if (!wait_warp(&sb.k_full, kc & 1, &m.abort, err)) { aborted = true; break; }
                    const uint32_t meta = m.k_meta[x];
                    __syncwarp();
                    if (lane == 0) {
                        m.s_meta[x] = meta;
                        mbar_arrive(&sb.s_full);  // publishes the step word (release)
                    }
                    __syncwarp();
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = ((kk >> 2) * (2 * kHalfBox) + (kk & 3) * 32u) >> 4;
                        umma_ss_elect(s_tmem, d_hi | (ql + off), d_hi | (kl + off), idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    umma_commit_elect(&sb.s_full);
                    umma_commit_elect(&sb.k_empty);
                    const bool last = (sw_flags(meta) & 2) != 0;
                    if (last) umma_commit_elect(&sb.q_empty);
                    // ---- O += P . V
                    if (!wait_warp(&sb.p_full, kc & 1, &m.abort, err)) { aborted = true; break; }
                    if (!wait_warp(&sb.v_full, kc & 1, &m.abort, err)) { aborted = true; break; }
                    const int na = sw_na(meta), nb = sw_nb(meta);
                    const int za = (na & 15) ? 16 - (na & 15) : 0, zb = (nb & 15) ? 16 - (nb & 15) : 0;
                    if (za + zb > 0) {
                        // V rows between vbs and the next multiple of 16 are read by the last
                        // k-step of their cube: zero them (both d halves) before the product
                        const uint32_t vb = smem_u32(vdst);
                        for (int w = lane; w < (za + zb) * 16; w += 32) {
                            const int zr = w >> 4, chunk = w & 15;
                            const int row = zr < za ? na + zr : 64 + nb + (zr - za);
                            sts128(vb + (chunk >> 3) * (2 * kHalfBox) + row * 128 + (chunk & 7) * 16, 0u, 0u, 0u, 0u);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                    }
                    tc_fence_after();
                    // k-steps (16 keys) 0..ceil16(na)-1 of half 0 and 4..4+ceil16(nb)-1 of half 1
                    const uint32_t kmask = ((1u << ((na + 15) >> 4)) - 1u) | (((1u << ((nb + 15) >> 4)) - 1u) << 4);
                    uint32_t acc = o_init ? 1u : 0u;
#pragma unroll
                    for (int kstep = 0; kstep < 8; ++kstep) {
                        if (kmask & (1u << kstep)) {
                            umma_ts_elect(o_tmem, s_tmem + kstep * 8, d_hi | (vl + ((kstep * 2048) >> 4)), idesc_pv, acc);
                            acc = 1u;
                        }
                    }
                    o_init = o_init || kmask != 0;
                    umma_commit_elect(&sb.v_empty);
                    if (last) umma_commit_elect(&sb.o_full);
                    ++kc;
                    if (last) break;
                }
            }
            if (aborted) {
                umma_commit_elect(&sb.drain);
                if (lane == 0) drain_wait(&sb.drain, 0);
                __syncwarp();
            }
        }
    } else if (warp >= kWarpCorr0) {
        // -------------------------------------------------------- O correction of slot x
        const int x = (warp - kWarpCorr0) >> 2, wq = warp & 3;
        const int r = 32 * wq + (int)lane;
        SlotBars& sb = m.bar[x];
        const uint32_t oa = tbase + ((uint32_t)(32 * wq) << 16) + o_col(x);
        int g = 0;
        for (int n = x; n < my_tiles; n += 2) {
            for (;;) {
                if (!wait_warp(&sb.a_full, g & 1, &m.abort, err)) goto corr_exit;
                const uint32_t meta = m.s_meta[x];
                tc_fence_after();
                if (!(sw_flags(meta) & 1) && m.rflag[x][wq] != 0) {
                    // O row r *= alpha (1 for rows whose offset stayed); the previous
                    // P.V of the slot finished before this step's S was published
                    const float a = m.alpha[x][r];
#pragma unroll 1
                    for (int c4 = 0; c4 < 4; ++c4) {
                        uint32_t o[32];
                        tmem_ld32(oa + 32 * c4, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * a);
                        tmem_st32(oa + 32 * c4, o);
                    }
                    tmem_st_wait();
                }
                tc_fence_before();
                mbar_arrive(&sb.p_full);
                ++g;
                if (sw_flags(meta) & 2) break;
            }
        }
    corr_exit:;
    } else {
        // -------------------------------------------------------- softmax + epilogue of slot x
        const int x = warp >> 2, wq = warp & 3;
        const int r = 32 * wq + (int)lane;  // query row of the tile == TMEM lane
        const int qbit = r >> 6;            // 0: query cube i1, 1: i2
        SlotBars& sb = m.bar[x];
        const uint32_t lane_base = tbase + ((uint32_t)(32 * wq) << 16);
        const uint32_t s_addr = lane_base + s_col(x), o_addr = lane_base + o_col(x);
        constexpr float kNeutral = NEG ? INFINITY : -INFINITY;  // a masked logit
        int g = 0, tc = 0;
        float m_run = -INFINITY, l_run = 0.f;
        for (int n = x; n < my_tiles; n += 2, ++tc) {
            const TileRef t = checked_tile(blockIdx.x + n * gridDim.x, H, nq, tiles_per_bh, plan, nullptr);
            for (;;) {
                if (!wait_warp_inl(&sb.s_full, g & 1, &m.abort, err)) goto softmax_exit;
                const uint32_t meta = m.s_meta[x];
                const int na = sw_na(meta), nb = sw_nb(meta), ma = sw_ma(meta), mb = sw_mb(meta), flags = sw_flags(meta);
                const int myn0 = ((ma >> qbit) & 1) ? na : 0, myn1 = ((mb >> qbit) & 1) ? nb : 0;
                if (flags & 1) {
                    m_run = -INFINITY;
                    l_run = 0.f;
                }
                tc_fence_after();
                // pass 1: row extreme over the selected keys, one 32-column TMEM load at a
                // time (small loop bodies keep the hot code in the instruction cache)
                float e4[4] = {kNeutral, kNeutral, kNeutral, kNeutral};
#pragma unroll 1
                for (int ch = 0; ch < 4; ++ch) {
                    const int nv = ch < 2 ? myn0 : myn1;
                    const int cb = (ch & 1) * 32;  // first column of the chunk in its 64-key half
                    if (nv <= cb) continue;        // no selected key in this chunk
                    float sc[32];
                    tmem_ld32(s_addr + 32 * ch, reinterpret_cast<uint32_t*>(sc));
                    tmem_ld_wait();
                    if (nv < cb + 32) {
#pragma unroll
                        for (int c = 0; c < 32; ++c) sc[c] = cb + c < nv ? sc[c] : kNeutral;
                    }
#pragma unroll
                    for (int c = 0; c < 32; c += 8) {
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            e4[u] = NEG ? min3(e4[u], sc[c + 2 * u], sc[c + 2 * u + 1])
                                        : max3(e4[u], sc[c + 2 * u], sc[c + 2 * u + 1]);
                    }
                }
                const float ext = NEG ? min3(fminf(e4[0], e4[1]), e4[2], e4[3]) : max3(fmaxf(e4[0], e4[1]), e4[2], e4[3]);
                const bool any_valid = (myn0 | myn1) != 0;
                const float m_step = any_valid ? ext * scale_log2 : -INFINITY;  // base-2 units
                const bool raise = m_step > m_run + kTau;                    // false for -inf
                float alpha = 1.f;
                if (raise) {
                    alpha = m_run == -INFINITY ? 0.f : ex2(m_run - m_step);
                    m_run = m_step;
                    l_run *= alpha;
                }
                m.alpha[x][r] = alpha;
                const bool warp_raise = __any_sync(0xffffffffu, raise && !(flags & 1));
                if (lane == 0) m.rflag[x][wq] = warp_raise ? 1 : 0;
                mbar_arrive(&sb.a_full);

                // pass 2: P = exp2(x - m) as bf16 pairs over S's first 64 columns; the
                // chunk's P lands on columns whose logits were already consumed
                const float mu = m_run == -INFINITY ? 0.f : m_run;
                float ls0 = 0.f, ls1 = 0.f;
#pragma unroll 1
                for (int ch = 0; ch < 4; ++ch) {
                    const int nv = ch < 2 ? myn0 : myn1;
                    const int cb = (ch & 1) * 32;
                    uint32_t pk[16];
                    if (nv <= cb) {
#pragma unroll
                        for (int c = 0; c < 16; ++c) pk[c] = 0u;
                    } else {
                        float sc[32];
                        tmem_ld32(s_addr + 32 * ch, reinterpret_cast<uint32_t*>(sc));
                        tmem_ld_wait();
                        if (nv < cb + 32) {
#pragma unroll
                            for (int c = 0; c < 32; ++c) sc[c] = cb + c < nv ? sc[c] : kNeutral;
                        }
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            float x0, x1, p0, p1;
                            ffma2(x0, x1, sc[2 * c], sc[2 * c + 1], scale_log2, scale_log2, -mu, -mu);
                            if ((kPolyPairs >> c) & 1) {
                                // weights below 2^-125 (masked keys included) become 2^-125
                                const float2 pp = ex2_fma2(make_float2(fmaxf(x0, -125.f), fmaxf(x1, -125.f)));
                                p0 = pp.x;
                                p1 = pp.y;
                            } else {
                                p0 = ex2(x0);
                                p1 = ex2(x1);
                            }
                            fadd2(ls0, ls1, p0, p1);
                            pk[c] = pack_bf16(p0, p1);
                        }
                    }
                    tmem_st16(s_addr + 16 * ch, pk);
                }
                l_run += ls0 + ls1;
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&sb.p_full);
                ++g;
                if (flags & 2) break;
            }

            // ---- epilogue: out[b, 64 i + (r % 64), h, :] = O[r, :] / l; lse = (m + log2 l) ln 2
            if (!wait_warp_inl(&sb.o_full, tc & 1, &m.abort, err)) goto softmax_exit;
            tc_fence_after();
            {
                const int cube = qbit == 0 ? t.i1 : t.i2;
                const float inv = l_run > 0.f ? __frcp_rn(l_run) : 0.f;
                const int64_t token = (int64_t)t.b * S + 64LL * cube + (r & 63);
                uint16_t* dst = out + (token * H + t.h) * kD;
#pragma unroll 1
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint32_t o[32];
                    tmem_ld32(o_addr + 32 * c4, o);
                    tmem_ld_wait();
                    if (cube >= 0) {
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                w[e] = pack_bf16(__uint_as_float(o[8 * v + 2 * e]) * inv,
                                                 __uint_as_float(o[8 * v + 2 * e + 1]) * inv);
                            st_global_v4(dst + 32 * c4 + 8 * v, w[0], w[1], w[2], w[3]);
                        }
                    }
                }
                if (lse != nullptr && cube >= 0)
                    lse[((int64_t)t.b * H + t.h) * S + 64LL * cube + (r & 63)] =
                        l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
            }
            tc_fence_before();
        }
    softmax_exit:;
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpRole0 + 1) tmem_dealloc(tbase, 512);
}

template <bool NEG>
cudaError_t launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const int32_t* topk_idx,
                   const int32_t* vbs, const int32_t* plan, uint16_t* out, float* lse, int B, int S, int H, int nq,
                   int topk, float scale_log2, int* err, cudaStream_t s)
{
    auto kern = fwd_pair_kernel<NEG>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Layout::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int tiles_per_bh = (nq + 1) / 2;
    const int n_tiles = B * H * tiles_per_bh;
    const int grid = n_tiles < sms ? n_tiles : sms;
    kern<<<grid, kThreads, Layout::SMEM_BYTES, s>>>(mq, mk, mv, topk_idx, vbs, plan, out, lse, S, H, nq, topk,
                                                    tiles_per_bh, n_tiles, scale_log2, err);
    return cudaGetLastError();
}

}  // namespace

bool fwd_pair_supported(int nq, int topk) { return nq <= kMaxNq && topk <= kMaxTopk; }

cudaError_t launch_fwd_pair(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* topk_idx,
                            const int32_t* vbs, const int32_t* plan, uint16_t* out, float* lse, int B, int S, int H,
                            int nq, int topk, float sm_scale, bool precise_p, int* err, cudaStream_t s)
{
    if (precise_p)
        return launch_fwd_pair_shared(q, k, v, topk_idx, vbs, plan, out, lse, B, S, H, nq, topk, sm_scale, true, err, s);
    CUtensorMap mq, mk, mv;
    const int64_t tokens = (int64_t)B * S;
    if (!make_map(&mq, q, tokens, H) || !make_map(&mk, k, tokens, H) || !make_map(&mv, v, tokens, H))
        return cudaErrorInvalidValue;
    const float scale_log2 = sm_scale * 1.4426950408889634f;
    return scale_log2 < 0.f
               ? launch<true>(mq, mk, mv, topk_idx, vbs, plan, out, lse, B, S, H, nq, topk, scale_log2, err, s)
               : launch<false>(mq, mk, mv, topk_idx, vbs, plan, out, lse, B, S, H, nq, topk, scale_log2, err, s);
}

}  // namespace vsa
