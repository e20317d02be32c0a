// VSA fine forward on the Blackwell tensor cores, queries on TMEM lanes,
// two query cubes per 128-row tile: the variant with one MMA issuer and one
// producer shared by both tiles in flight.  The library runs it for the
// precise-weight mode (its softmax keeps a whole 128-column row of S in
// registers, which the 640-thread per-slot kernel of fwd_pair.cu cannot);
// the default mode runs fwd_pair.cu.
//
// Dataset card "wan2.2_production_values", section "Operator contract": for
// query cube i of (batch b, head h) the keys are the first vbs[j] tokens of
// every cube j in topk_idx[b, h, i, :]; out = softmax(q k^T * sm_scale) v.
//
// Shape of the work on sm_100a.  A query cube has only 64 rows, and an MMA
// with M = 64 runs the tensor core at half rate.  This kernel stacks TWO
// query cubes (i1 rows 0-63, i2 rows 64-127) of the same (b, h) into one
// 128-row tile and walks the union of their two selection lists, two KV
// cubes (128 keys) per step:
//     S[128 q x 128 keys]  = Q_tile[128 x 128 d] . K_pair^T         (M=128, N=128)
//     O[128 q x 128 d]    += P[128 x 128 keys] . V_pair[128 keys x 128 d]
// Both are tcgen05.mma (bf16 in, fp32 accumulate in TMEM); P stays in TMEM
// (bf16, written over S) and is the A operand of the second product.  A KV
// cube that only one of the two query cubes selected is masked (weight 0)
// for the other cube's rows.  Cubes both lists name are walked first, so a
// tile whose query cubes select similar cubes (the pairing that vsa_plan
// chooses) loads each shared K/V cube once for both: the L2->SM traffic of
// the gather and the tensor work both drop with the overlap of the paired
// lists.
//
// Each thread of a softmax warp owns one query row (one TMEM lane), so the
// row maximum and the row sum are thread-local: no cross-lane reduction.
//
// Two tiles are in flight per CTA (slots A and B), each with its own S/P
// (128 TMEM columns) and O (128 columns); the tensor core alternates
//     QK_A(s)  PV_B(s-1)  QK_B(s)  PV_A(s)  QK_A(s+1) ...
// so the softmax of one slot overlaps the products of the other.
//
// Roles (512 threads = 4 warpgroups, one persistent CTA per SM):
//   WG0 (warps 0-3)   softmax + epilogue of slot A (thread = row = TMEM lane)
//   WG1 (warps 4-7)   softmax + epilogue of slot B
//   WG2 (warps 8-11)  O correction of both slots (rescale rows whose offset
//                     rose), zeroing of V pad rows inside a partial k-step, and
//                     the check that the step's V pair has landed
//   WG3 warp 12       TMA producer: builds each tile's step list (shared
//                     cubes first) and streams Q, K and V tiles
//       warp 13       TMEM allocator and MMA issuer (one thread)
//       warps 14-15   idle
//
// Softmax.  Logits are taken in base 2 (x = s * sm_scale * log2 e).  Keys at
// or beyond vbs of their cube, and cubes the row's query cube did not
// select, are replaced by -inf (a select, so NaN/Inf there never
// propagates).  The running offset m of a row is raised only when the
// step's maximum exceeds it by more than kTau (so P <= 2^kTau); only then
// are O's row and the row sum rescaled.  The result does not depend on the
// offsets used.  PV k-steps (16 keys) beyond ceil16(vbs) of a cube are not
// issued; V rows between vbs and that boundary are zeroed in shared memory
// before the product, so 0 * NaN cannot occur.
//
// Precise mode (VSA_FWD_PRECISE_P): P is carried as a bf16 pair hi + lo in
// the two halves of the S columns, and the P.V product runs twice.
//
// Every mbarrier wait is bounded (~2 s of clock): on expiry the kernel
// latches kErrWaitTimeout, raises a CTA-wide abort flag, every role leaves
// its loop, the producer and the MMA issuer wait (bounded) for their own
// copies and products in flight, and TMEM is freed before exit.
#include "fwd_pair_common.cuh"

namespace vsa {
namespace {

using namespace ptx;

constexpr int kThreads = 512;
constexpr int kWarpProducer = 12;
constexpr int kWarpMma = 13;
constexpr int kNK = 2;  // K ring slots
constexpr int kNV = 2;  // V ring slots

struct Misc {
    uint64_t q_full[2], q_empty[2];        // per slot
    uint64_t k_full[kNK], k_empty[kNK];
    uint64_t v_full[kNV], v_empty[kNV];
    uint64_t s_full[2];                    // per slot: QK done (count 2: MMA meta + commit)
    uint64_t p_full[2];                    // per slot: P in TMEM, O corrected, V landed and its pads
                                           // zeroed (every softmax and correction thread)
    uint64_t a_full[2];                    // per slot: offsets decided (every softmax thread)
    uint64_t o_full[2];                    // per slot: last PV of a tile done (commit)
    uint64_t drain;
    uint32_t k_meta[kNK];                  // step word of the K pair in each K slot
    uint32_t s_meta[2];                    // step word whose S sits in each slot
    uint32_t tmem_base;
    int abort;
    alignas(16) float alpha[2][128];       // per slot, row: O rescale factor of the current step
    int rflag[2][4];                       // per slot, warp: some row of the warp rescales
    uint32_t bits1[2][kMaxNq / 32];        // per slot: membership bitmap of list 1
    uint32_t bits2[2][kMaxNq / 32];        //                           and of list 2
    int32_t list1[2][kMaxTopk];            // per slot: the two selection lists
    int32_t list2[2][kMaxTopk];
};

template <bool PRECISE>
struct Layout {
    static constexpr uint32_t Q_OFF = 0;                         // two Q tiles (slots A, B)
    static constexpr uint32_t K_OFF = Q_OFF + 2 * kTileBytes;
    static constexpr uint32_t V_OFF = K_OFF + kNK * kTileBytes;
    static constexpr uint32_t TILE_BYTES = V_OFF + kNV * kTileBytes;
    static constexpr uint32_t MISC_BYTES = (sizeof(Misc) + 1023) / 1024 * 1024;
    static constexpr uint32_t SMEM_BYTES = MISC_BYTES + TILE_BYTES + 1024;  // + alignment slack
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// TMEM columns of slot x: S/P at 256x, O at 256x + 128.
__device__ __forceinline__ uint32_t s_col(int x) { return 256u * x; }
__device__ __forceinline__ uint32_t o_col(int x) { return 256u * x + 128u; }

template <bool PRECISE, bool NEG>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_pair_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv, const int32_t* __restrict__ topk_idx,
                    const int32_t* __restrict__ vbs, const int32_t* __restrict__ plan, uint16_t* __restrict__ out,
                    float* __restrict__ lse, int S, int H, int nq, int topk, int tiles_per_bh, int n_tiles,
                    float scale_log2, int* err)
{
    using L = Layout<PRECISE>;
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
            mbar_init(&m.q_full[x], 1);
            mbar_init(&m.q_empty[x], 1);
            mbar_init(&m.s_full[x], 2);    // MMA thread (metadata) + QK completion
            mbar_init(&m.p_full[x], 256);  // every softmax thread of the slot + every correction thread
            mbar_init(&m.a_full[x], 128);
            mbar_init(&m.o_full[x], 1);
        }
        for (int i = 0; i < kNK; ++i) {
            mbar_init(&m.k_full[i], 1);
            mbar_init(&m.k_empty[i], 1);
        }
        for (int i = 0; i < kNV; ++i) {
            mbar_init(&m.v_full[i], 1);
            mbar_init(&m.v_empty[i], 1);
        }
        mbar_init(&m.drain, 1);
        m.abort = 0;
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

    // Registers: the softmax warpgroups hold a 128-column row of S per thread.
    // Each warpgroup sets its budget before it splits into roles, so that the
    // code of every role is dominated by its warpgroup's setmaxnreg.
    if (warp >= 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 72;" ::: "memory");
    if (warp == kWarpProducer) {
        // -------------------------------------------------------- TMA producer
        ListGen gen[2];
        int tn[2] = {0, 1};
        bool active[2] = {my_tiles > 0, my_tiles > 1};
        bool need_start[2] = {true, true};
        bool pend_v[2] = {false, false};
        StepMeta pend[2];
        int h_of[2] = {0, 0}, tok0_of[2] = {0, 0};
        int ku = 0, vu = 0, qn[2] = {0, 0};
        int armed_q[2] = {-1, -1}, armed_k[kNK], armed_v[kNV];
        for (int i = 0; i < kNK; ++i) armed_k[i] = -1;
        for (int i = 0; i < kNV; ++i) armed_v[i] = -1;
        bool aborted = false;
        while (!aborted) {
#pragma unroll 1
            for (int e = 0; e < 4 && !aborted; ++e) {
                const int x = (e == 0 || e == 3) ? 0 : 1;
                if (e == 0 || e == 2) {
                    // ---- K pair of slot x's next step (and Q at a tile start)
                    if (!active[x]) continue;
                    bool first = false;
                    if (need_start[x]) {
                        const TileRef t =
                            checked_tile(blockIdx.x + tn[x] * gridDim.x, H, nq, tiles_per_bh, plan, lane == 0 ? err : nullptr);
                        gen_start(gen[x], t, topk_idx, vbs, H, nq, topk, m.list1[x], m.list2[x], m.bits1[x],
                                  m.bits2[x], err, lane);
                        h_of[x] = t.h;
                        tok0_of[x] = t.b * S;
                        if (lane == 0) {
                            if (wait_bar(&m.q_empty[x], (qn[x] & 1) ^ 1, &m.abort, err)) {
                                const uint32_t bytes = 2 * kHalfBox * ((t.i1 >= 0) + (t.i2 >= 0));
                                mbar_expect_tx(&m.q_full[x], bytes);
                                armed_q[x] = qn[x] & 1;
                                uint8_t* qdst = tiles_ptr + L::Q_OFF + x * kTileBytes;
                                if (t.i1 >= 0) load_cube(&tmq, &m.q_full[x], qdst, 0, t.h, t.b * S + 64 * t.i1);
                                if (t.i2 >= 0) load_cube(&tmq, &m.q_full[x], qdst, 1, t.h, t.b * S + 64 * t.i2);
                            } else {
                                aborted = true;
                            }
                        }
                        aborted = __shfl_sync(0xffffffffu, aborted, 0);
                        if (aborted) break;
                        ++qn[x];
                        need_start[x] = false;
                        first = true;
                    }
                    ListGen& G = gen[x];
                    const Entry ea = G.next;
                    Entry eb{0, 0, 0};
                    if (ea.mem != 0) {
                        G.next = gen_pull(G, m.list1[x], m.list2[x], m.bits1[x], m.bits2[x], vbs, lane);
                        eb = G.next;
                        if (eb.mem != 0) G.next = gen_pull(G, m.list1[x], m.list2[x], m.bits1[x], m.bits2[x], vbs, lane);
                    }
                    const bool last = G.next.mem == 0;
                    StepMeta meta;
                    meta.ja = ea.j;
                    meta.jb = eb.j;
                    meta.na = ea.n;
                    meta.nb = eb.n;
                    meta.ma = ea.mem;
                    meta.mb = eb.mem;
                    meta.flags = (first ? 1 : 0) | (last ? 2 : 0);
                    meta.vslot = 0;
                    meta.vpar = 0;
                    if (lane == 0) {
                        const int ks = ku % kNK;
                        if (wait_bar(&m.k_empty[ks], ((ku / kNK) & 1) ^ 1, &m.abort, err)) {
                            m.k_meta[ks] = step_word(meta);
                            const uint32_t bytes = 2 * kHalfBox * ((meta.na > 0) + (meta.nb > 0));
                            mbar_expect_tx(&m.k_full[ks], bytes);
                            armed_k[ks] = (ku / kNK) & 1;
                            uint8_t* kdst = tiles_ptr + L::K_OFF + ks * kTileBytes;
                            if (meta.na > 0) load_cube(&tmk, &m.k_full[ks], kdst, 0, h_of[x], tok0_of[x] + 64 * meta.ja);
                            if (meta.nb > 0) load_cube(&tmk, &m.k_full[ks], kdst, 1, h_of[x], tok0_of[x] + 64 * meta.jb);
                        } else {
                            aborted = true;
                        }
                    }
                    aborted = __shfl_sync(0xffffffffu, aborted, 0);
                    ++ku;
                    pend[x] = meta;
                    pend_v[x] = true;
                    if (last) {
                        tn[x] += 2;
                        need_start[x] = true;
                        active[x] = tn[x] < my_tiles;
                    }
                } else {
                    // ---- V pair of slot x's pending step
                    if (!pend_v[x]) continue;
                    if (lane == 0) {
                        const int vs = vu % kNV;
                        if (wait_bar(&m.v_empty[vs], ((vu / kNV) & 1) ^ 1, &m.abort, err)) {
                            const StepMeta& p = pend[x];
                            const uint32_t bytes = 2 * kHalfBox * ((p.na > 0) + (p.nb > 0));
                            mbar_expect_tx(&m.v_full[vs], bytes);
                            armed_v[vs] = (vu / kNV) & 1;
                            uint8_t* vdst = tiles_ptr + L::V_OFF + vs * kTileBytes;
                            if (p.na > 0) load_cube(&tmv, &m.v_full[vs], vdst, 0, h_of[x], tok0_of[x] + 64 * p.ja);
                            if (p.nb > 0) load_cube(&tmv, &m.v_full[vs], vdst, 1, h_of[x], tok0_of[x] + 64 * p.jb);
                        } else {
                            aborted = true;
                        }
                    }
                    aborted = __shfl_sync(0xffffffffu, aborted, 0);
                    ++vu;
                    pend_v[x] = false;
                }
            }
            if (!active[0] && !active[1] && !pend_v[0] && !pend_v[1]) break;
        }
        if (aborted && lane == 0) {
            // copies issued by this thread must land before the CTA's shared memory goes away
            for (int x = 0; x < 2; ++x)
                if (armed_q[x] >= 0) drain_wait(&m.q_full[x], armed_q[x]);
            for (int i = 0; i < kNK; ++i)
                if (armed_k[i] >= 0) drain_wait(&m.k_full[i], armed_k[i]);
            for (int i = 0; i < kNV; ++i)
                if (armed_v[i] >= 0) drain_wait(&m.v_full[i], armed_v[i]);
        }
    } else if (warp == kWarpMma) {
        // -------------------------------------------------------- MMA issuer
        // The whole warp runs the schedule (every value below is warp-uniform);
        // each tcgen05.mma / commit is issued by one elected lane.
        constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, false, true);
        // Descriptors of every operand tile, built once; a k-step only adds its
        // byte offset / 16 to the start-address field (no carry: smem < 256 KiB).
        const uint64_t d_hi = smem_desc_sw128(0, 0, 1024);  // SBO, version, swizzle: shared by all
        const uint32_t q_lo0 = (uint32_t)smem_desc_sw128(tiles + L::Q_OFF, 16, 1024);
        const uint32_t k_lo0 = (uint32_t)smem_desc_sw128(tiles + L::K_OFF, 16, 1024);
        const uint32_t v_lo0 = (uint32_t)smem_desc_sw128(tiles + L::V_OFF, 2 * kHalfBox, 1024);
        int tn[2] = {0, 1}, g[2] = {0, 0}, qn[2] = {0, 0};
        bool active[2] = {my_tiles > 0, my_tiles > 1};
        bool pending[2] = {false, false}, new_tile[2] = {true, true}, o_init[2] = {false, false};
        uint32_t cur[2] = {0u, 0u};
        int ku = 0, vu = 0;
        bool aborted = false;
        while (!aborted) {
#pragma unroll
            for (int e = 0; e < 4 && !aborted; ++e) {
                const int x = (e == 0 || e == 3) ? 0 : 1;
                if (e == 0 || e == 2) {
                    // ---- S_x = Q_x . K^T
                    if (!active[x]) continue;
                    if (new_tile[x]) {
                        if (!wait_warp(&m.q_full[x], qn[x] & 1, &m.abort, err)) { aborted = true; break; }
                        ++qn[x];
                        new_tile[x] = false;
                        o_init[x] = false;
                    }
                    const int ks = ku % kNK;
                    if (!wait_warp(&m.k_full[ks], (ku / kNK) & 1, &m.abort, err)) { aborted = true; break; }
                    const int vidx = vu + (pending[x ^ 1] ? 1 : 0);  // V uses before this step's PV
                    const uint32_t meta =
                        m.k_meta[ks] | ((uint32_t)(vidx % kNV) << 20) | ((uint32_t)((vidx / kNV) & 1) << 21);
                    __syncwarp();
                    if (lane == 0) {
                        m.s_meta[x] = meta;
                        mbar_arrive(&m.s_full[x]);  // publishes s_meta (release)
                    }
                    __syncwarp();
                    tc_fence_after();
                    const uint32_t ql = q_lo0 + x * (kTileBytes >> 4), kl = k_lo0 + ks * (kTileBytes >> 4);
                    const uint32_t s_tmem = tbase + s_col(x);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = ((kk >> 2) * (2 * kHalfBox) + (kk & 3) * 32u) >> 4;
                        umma_ss_elect(s_tmem, d_hi | (ql + off), d_hi | (kl + off), idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    umma_commit_elect(&m.s_full[x]);
                    umma_commit_elect(&m.k_empty[ks]);
                    ++ku;
                    cur[x] = meta;
                    pending[x] = true;
                    if (sw_flags(meta) & 2) {
                        umma_commit_elect(&m.q_empty[x]);
                        tn[x] += 2;
                        new_tile[x] = true;
                        active[x] = tn[x] < my_tiles;
                    }
                } else {
                    // ---- O_x += P_x . V
                    if (!pending[x]) continue;
                    const uint32_t c = cur[x];
                    // one wait: P written, O corrected, V landed (the correction waited for it)
                    if (!wait_warp(&m.p_full[x], g[x] & 1, &m.abort, err)) { aborted = true; break; }
                    tc_fence_after();
                    const uint32_t vl = v_lo0 + sw_vslot(c) * (kTileBytes >> 4);
                    const uint32_t p_tmem = tbase + s_col(x), o_tmem = tbase + o_col(x);
                    // k-steps (16 keys) 0..ceil16(na)-1 of half 0 and 4..4+ceil16(nb)-1 of half 1
                    const uint32_t kmask =
                        ((1u << ((sw_na(c) + 15) >> 4)) - 1u) | (((1u << ((sw_nb(c) + 15) >> 4)) - 1u) << 4);
                    uint32_t acc = o_init[x] ? 1u : 0u;
#pragma unroll
                    for (int kstep = 0; kstep < 8; ++kstep) {
                        const uint32_t on = (kmask >> kstep) & 1u;  // warp-uniform, no branch
                        const uint64_t bd = d_hi | (vl + ((kstep * 2048) >> 4));
                        umma_ts_elect_if(o_tmem, p_tmem + kstep * 8, bd, idesc_pv, acc, on);
                        acc |= on;
                        if (PRECISE) umma_ts_elect_if(o_tmem, p_tmem + 64 + kstep * 8, bd, idesc_pv, 1u, on);
                    }
                    o_init[x] = o_init[x] || kmask != 0;
                    umma_commit_elect(&m.v_empty[sw_vslot(c)]);
                    if (sw_flags(c) & 2) umma_commit_elect(&m.o_full[x]);
                    ++vu;
                    ++g[x];
                    pending[x] = false;
                }
            }
            if (!active[0] && !active[1] && !pending[0] && !pending[1]) break;
        }
        if (aborted) {
            umma_commit_elect(&m.drain);
            if (lane == 0) drain_wait(&m.drain, 0);
            __syncwarp();
        }
    } else if (warp < kWarpProducer) {
        // -------------------------------------------------------- correction (warps 8-11)
        const int wq = warp & 3;
        const int r = 32 * wq + (int)lane;
        const uint32_t lane_base = tbase + ((uint32_t)(32 * wq) << 16);
        int tn[2] = {0, 1}, g[2] = {0, 0};
        bool active[2] = {my_tiles > 0, my_tiles > 1};
        bool pending[2] = {false, false};
        for (;;) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int x = (e == 0 || e == 3) ? 0 : 1;
                if (e == 0 || e == 2) {
                    pending[x] = active[x];  // the MMA issues QK_x here
                    continue;
                }
                if (!pending[x]) continue;
                if (!wait_warp(&m.a_full[x], g[x] & 1, &m.abort, err)) goto corr_exit;
                const uint32_t meta = m.s_meta[x];
                tc_fence_after();
                if (!(sw_flags(meta) & 1) && m.rflag[x][wq] != 0) {
                    // O row r *= alpha (1 for rows whose offset stayed)
                    const float a = m.alpha[x][r];
                    const uint32_t oa = lane_base + o_col(x);
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
                // V rows between vbs and the next multiple of 16 are read by the last
                // k-step of their cube: zero them (both d halves) before the product
                const int mna = sw_na(meta), mnb = sw_nb(meta);
                const int za = (mna & 15) ? 16 - (mna & 15) : 0;
                const int zb = (mnb & 15) ? 16 - (mnb & 15) : 0;
                if (!wait_warp(&m.v_full[sw_vslot(meta)], sw_vpar(meta), &m.abort, err)) goto corr_exit;
                if (za + zb > 0) {
                    const uint32_t vb = tiles + L::V_OFF + sw_vslot(meta) * kTileBytes;
                    for (int w = r; w < (za + zb) * 16; w += 128) {
                        const int zr = w >> 4, chunk = w & 15;
                        const int row = zr < za ? mna + zr : 64 + mnb + (zr - za);
                        sts128(vb + (chunk >> 3) * (2 * kHalfBox) + row * 128 + (chunk & 7) * 16, 0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();
                }
                tc_fence_before();
                mbar_arrive(&m.p_full[x]);
                ++g[x];
                pending[x] = false;
                if (sw_flags(meta) & 2) {
                    tn[x] += 2;
                    active[x] = tn[x] < my_tiles;
                }
            }
            if (!active[0] && !active[1] && !pending[0] && !pending[1]) break;
        }
    corr_exit:;
    }
    } else {
        // -------------------------------------------------------- softmax + epilogue (warps 0-7)
        asm volatile("setmaxnreg.inc.sync.aligned.u32 184;" ::: "memory");
        const int x = warp >> 2, wq = warp & 3;
        const int r = 32 * wq + (int)lane;  // query row of the tile == TMEM lane
        const int qbit = r >> 6;            // 0: query cube i1, 1: i2
        const uint32_t lane_base = tbase + ((uint32_t)(32 * wq) << 16);
        const uint32_t s_addr = lane_base + s_col(x), o_addr = lane_base + o_col(x);
        constexpr float kNeutral = NEG ? INFINITY : -INFINITY;  // a masked logit
        int g = 0, tc = 0;
        float m_run = -INFINITY, l_run = 0.f;
        for (int n = x; n < my_tiles; n += 2, ++tc) {
            const TileRef t = checked_tile(blockIdx.x + n * gridDim.x, H, nq, tiles_per_bh, plan, nullptr);
            for (;;) {
                if (!wait_warp_inl(&m.s_full[x], g & 1, &m.abort, err)) goto softmax_exit;
                const uint32_t meta = m.s_meta[x];
                const int na = sw_na(meta), nb = sw_nb(meta), ma = sw_ma(meta), mb = sw_mb(meta), flags = sw_flags(meta);
                const int myn[2] = {((ma >> qbit) & 1) ? na : 0, ((mb >> qbit) & 1) ? nb : 0};
                if (flags & 1) {
                    m_run = -INFINITY;
                    l_run = 0.f;
                }
                tc_fence_after();
                if constexpr (!PRECISE) {
                    // pass 1: row extreme over the selected keys, one 32-column TMEM load
                    // at a time (small loop bodies keep the hot code in the instruction cache)
                    float e4[4] = {kNeutral, kNeutral, kNeutral, kNeutral};
#pragma unroll 1
                    for (int ch = 0; ch < 4; ++ch) {
                        const int nv = ch < 2 ? myn[0] : myn[1];
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
                    const bool any_valid = (myn[0] | myn[1]) != 0;
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
                    mbar_arrive(&m.a_full[x]);

                    // pass 2: P = exp2(x - m) as bf16 pairs over S's first 64 columns; the
                    // chunk's P lands on columns whose logits were already consumed
                    const float mu = m_run == -INFINITY ? 0.f : m_run;
                    float ls0 = 0.f, ls1 = 0.f;
#pragma unroll 1
                    for (int ch = 0; ch < 4; ++ch) {
                        const int nv = ch < 2 ? myn[0] : myn[1];
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
                                float x0, x1;
                                ffma2(x0, x1, sc[2 * c], sc[2 * c + 1], scale_log2, scale_log2, -mu, -mu);
                                const float p0 = ex2(x0), p1 = ex2(x1);
                                fadd2(ls0, ls1, p0, p1);
                                pk[c] = pack_bf16(p0, p1);
                            }
                        }
                        tmem_st16(s_addr + 16 * ch, pk);
                    }
                    l_run += ls0 + ls1;
                } else {
                float s[128];
                tmem_ld32(s_addr, reinterpret_cast<uint32_t*>(&s[0]));
                tmem_ld32(s_addr + 32, reinterpret_cast<uint32_t*>(&s[32]));
                tmem_ld32(s_addr + 64, reinterpret_cast<uint32_t*>(&s[64]));
                tmem_ld32(s_addr + 96, reinterpret_cast<uint32_t*>(&s[96]));
                tmem_ld_wait();

                // keys outside the row's selection take the neutral value (a select:
                // NaN/Inf from unselected or padded keys never propagates)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int nv = myn[hf];
                    if (nv < 64) {
#pragma unroll
                        for (int c = 0; c < 64; ++c) s[64 * hf + c] = c < nv ? s[64 * hf + c] : kNeutral;
                    }
                }
                // row extreme of the raw logits (max for a positive scale, min for a negative one)
                float e4[4] = {kNeutral, kNeutral, kNeutral, kNeutral};
#pragma unroll
                for (int c = 0; c < 128; c += 8) {
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        e4[u] = NEG ? min3(e4[u], s[c + 2 * u], s[c + 2 * u + 1])
                                    : max3(e4[u], s[c + 2 * u], s[c + 2 * u + 1]);
                }
                const float ext = NEG ? min3(fminf(e4[0], e4[1]), e4[2], e4[3]) : max3(fmaxf(e4[0], e4[1]), e4[2], e4[3]);
                const bool any_valid = (myn[0] | myn[1]) != 0;
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
                mbar_arrive(&m.a_full[x]);

                // P = exp2(x - m) as bf16 pairs over S's first 64 columns (hi part
                // of the precise mode; its lo part goes to columns 64-127)
                const float mu = m_run == -INFINITY ? 0.f : m_run;
                float ls[4] = {0.f, 0.f, 0.f, 0.f};
                // 16 columns of P (32 keys) per TMEM store; S is already in registers,
                // so writing P over S's leading columns is safe
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    uint32_t pk[16];
                    uint32_t pl[16];
                    if (myn[ch >> 1] == 0) {
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            pk[c] = 0u;
                            pl[c] = 0u;
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            const float p0 = ex2(fmaf(s[32 * ch + 2 * c], scale_log2, -mu));
                            const float p1 = ex2(fmaf(s[32 * ch + 2 * c + 1], scale_log2, -mu));
                            ls[c & 3] += p0 + p1;
                            const uint32_t hb = pack_bf16(p0, p1);
                            pk[c] = hb;
                            if (PRECISE) {
                                const float a0 = __uint_as_float(hb << 16), a1 = __uint_as_float(hb & 0xFFFF0000u);
                                pl[c] = pack_bf16(p0 - a0, p1 - a1);
                            }
                        }
                    }
                    tmem_st16(s_addr + 16 * ch, pk);
                    if (PRECISE) tmem_st16(s_addr + 64 + 16 * ch, pl);
                }
                l_run += (ls[0] + ls[1]) + (ls[2] + ls[3]);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&m.p_full[x]);
                ++g;
                if (flags & 2) break;
            }

            // ---- epilogue: out[b, 64 i + (r % 64), h, :] = O[r, :] / l; lse = (m + log2 l) ln 2
            if (!wait_warp_inl(&m.o_full[x], tc & 1, &m.abort, err)) goto softmax_exit;
            tc_fence_after();
            {
                const int cube = qbit == 0 ? t.i1 : t.i2;
                const float inv = l_run > 0.f ? __frcp_rn(l_run) : 0.f;
                const int64_t token = (int64_t)t.b * S + 64LL * cube + (r & 63);
                uint16_t* dst = out + (token * H + t.h) * kD;
#pragma unroll
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
    if (warp == kWarpMma) tmem_dealloc(tbase, 512);
}

template <bool PRECISE, bool NEG>
cudaError_t launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const int32_t* topk_idx,
                   const int32_t* vbs, const int32_t* plan, uint16_t* out, float* lse, int B, int S, int H, int nq,
                   int topk, float scale_log2, int* err, cudaStream_t s)
{
    using L = Layout<PRECISE>;
    auto kern = fwd_pair_kernel<PRECISE, NEG>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int tiles_per_bh = (nq + 1) / 2;
    const int n_tiles = B * H * tiles_per_bh;
    const int grid = n_tiles < sms ? n_tiles : sms;
    kern<<<grid, kThreads, L::SMEM_BYTES, s>>>(mq, mk, mv, topk_idx, vbs, plan, out, lse, S, H, nq, topk,
                                               tiles_per_bh, n_tiles, scale_log2, err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_pair_shared(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* topk_idx,
                            const int32_t* vbs, const int32_t* plan, uint16_t* out, float* lse, int B, int S, int H,
                            int nq, int topk, float sm_scale, bool precise_p, int* err, cudaStream_t s)
{
    CUtensorMap mq, mk, mv;
    const int64_t tokens = (int64_t)B * S;
    if (!make_map(&mq, q, tokens, H) || !make_map(&mk, k, tokens, H) || !make_map(&mv, v, tokens, H))
        return cudaErrorInvalidValue;
    const float scale_log2 = sm_scale * 1.4426950408889634f;
    const bool neg = scale_log2 < 0.f;
    if (precise_p)
        return neg ? launch<true, true>(mq, mk, mv, topk_idx, vbs, plan, out, lse, B, S, H, nq, topk, scale_log2, err, s)
                   : launch<true, false>(mq, mk, mv, topk_idx, vbs, plan, out, lse, B, S, H, nq, topk, scale_log2, err, s);
    return neg ? launch<false, true>(mq, mk, mv, topk_idx, vbs, plan, out, lse, B, S, H, nq, topk, scale_log2, err, s)
               : launch<false, false>(mq, mk, mv, topk_idx, vbs, plan, out, lse, B, S, H, nq, topk, scale_log2, err, s);
}

}  // namespace vsa
