// VSA fine forward on the Blackwell tensor cores: two query cubes per
// 128-row tile, queries on TMEM lanes, the logits of three steps in flight.
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
// cube's rows.  A cube both lists name is loaded once for both; vsa_plan
// pairs query cubes whose lists overlap most.
//
// Proxy compensation (vsa_fwd_proxy; TensorRT-LLM PR #7, the embedded FlashInfer
// PR "support proxy-compensated block-sparse attention"): after a tile's
// selected cubes come ceil(Nq / 128) proxy steps whose keys are the cubes'
// mean keys and whose values are their summed values; a row uses the proxy of
// every cube with valid tokens that its query cube did not select, with its
// weight counted vbs[j] times in the row sum.  PROXY is a template parameter:
// the plain kernels hold none of it.
//
// Pipeline.  TMEM holds three S/P buffers (columns 0, 128, 256) and O
// (columns 384-511).  Step g uses buffer g % 3, and the two MMA issuers run
// the products in the order  ..., PV(g), QK(g + 3), PV(g + 1), QK(g + 4), ...
// so the logits of the next two steps are ready while the softmax of step g
// runs; the softmax, not the QK -> softmax -> PV chain, sets the pace, and the
// tensor core sees one PV and one QK per softmax step.  Steps run on across
// tile boundaries; the tile's offsets and sums restart at its first step.
//
// Roles (640 threads, one persistent CTA per SM):
//   warps 0-11  softmax: warp w owns TMEM lanes 32 (w % 4) .. +31 (query rows,
//               all 128 columns) and the steps g with g % 3 == w / 4, so each
//               SMSP runs three softmax warps on three consecutive steps
//   warps 12-15 O correction and epilogue (thread = row): rescale the rows
//               whose running offset rose, once the previous PV has finished;
//               at a tile's end, O / l -> out and the log-sum-exp -> lse
//   warp 16     TMA producer of Q and K: builds each tile's step list (list 1,
//               then list 2's other cubes) over the tile's list 1, from lists
//               copied in one tile ahead, streams Q
//               (one buffer; loaded after the tile's first K pair) and K pairs
//               (ring of 3) and posts each step's V pair to warp 18
//   warp 17     PV MMA issuer (the whole warp runs the schedule, one elected
//               lane issues); zeroes V pad rows inside a partial k-step before
//               the product; owns the TMEM allocation
//   warp 18     TMA producer of V pairs (ring of 2: a V pair is needed only
//               after its step's softmax, so it has two steps to land)
//   warp 19     QK MMA issuer
//
// Softmax.  Logits in base 2 (x = s * sm_scale * log2 e).  Keys at or beyond
// vbs of their cube and cubes the row's query cube did not select are
// replaced by -inf (a select: NaN/Inf there never propagates).  The running
// offset of a row is raised only when the step maximum exceeds it by more
// than kTau (so P <= 2^kTau); only then are the row of O and the row sums
// rescaled.  PV k-steps (16 keys) beyond ceil16(vbs) of a cube are not issued;
// V rows between vbs and that boundary are zeroed before the product, so
// 0 * NaN cannot occur.
//
// Every mbarrier wait is bounded (~2 s of clock): on expiry the kernel
// latches kErrWaitTimeout and raises a CTA-wide abort flag; every role leaves
// its loop, the producer and the MMA issuer wait (bounded) for their own
// copies and products in flight, and TMEM is freed before exit.
#include "fwd_pair_common.cuh"

namespace vsa {
namespace {

using namespace ptx;

constexpr int kWarpCorr0 = 12;  // warps 0-11: softmax, three per SMSP; 12-15: correction and epilogue
constexpr int kWarpProd = 16;
constexpr int kWarpMma = 17;
constexpr int kWarpVProd = 18;
constexpr int kWarpQk = 19;  // kWarpMma issues the PV products, kWarpQk the QK products
constexpr int kThreads = 20 * 32;
constexpr int kVReq = 4;  // ring of V load requests from the K producer to the V producer
constexpr int kSBuf = 3;  // S/P buffers in TMEM
constexpr int kKBuf = 3;  // K ring depth
constexpr int kVBuf = 2;  // V ring depth
constexpr uint32_t kOCol = 384;
constexpr uint32_t kFinal = 1u << 22;  // step word: last step of the CTA's last tile
constexpr uint32_t kProxyStep = 1u << 23;  // step word: the keys are proxies of omitted cubes

// Pairs (bit c: columns 2c, 2c+1 of each 32-column chunk) whose exp2 runs on
// the FMA pipe instead of the multi-function unit.  None by default: with three
// softmax warps per SMSP the exp pass is bound by latency and instruction issue,
// not by the multi-function unit, and the FMA-pipe exp2 costs eight more
// instructions a pair (Wan 832x480: 5.94 ms without, 6.16 ms with 6 of 16 pairs).
#ifndef VSA_POLY_PAIRS
#define VSA_POLY_PAIRS 0
#endif
constexpr uint32_t kPolyPairs = VSA_POLY_PAIRS;

struct Bars {
    uint64_t q_full, q_empty;                // Q tile landed / last QK of the tile done
    uint64_t k_full[kKBuf], k_empty[kKBuf];  // K pair landed / its QK done
    uint64_t v_full[kVBuf], v_empty[kVBuf];  // V pair landed / its PV done
    uint64_t s_full[kSBuf];  // step word published + QK done (2 arrivals)
    uint64_t a_full[kSBuf];  // offsets decided (the 128 threads of the step's softmax warps)
    uint64_t p_full[kSBuf];  // P written (128 softmax threads) and O corrected (128)
    uint64_t pv_done[2];     // PV of step j done: pv_done[j & 1]
    uint64_t o_full;         // last PV of a tile done
    uint64_t l_full[2];      // tile parity: row sums and offsets written (128)
    uint64_t l_empty[2];     // tile parity: the epilogue has read them (128)
    uint64_t dec[kSBuf][4];   // [step % 3][lane quarter]: offsets after the step decided (32)
    uint64_t lsum[kSBuf][4];  // [step % 3][lane quarter]: row sums after the step written (32)
    uint64_t vr_full[kVReq], vr_empty[kVReq];  // V load request posted / taken
    uint64_t pv_issued[kSBuf];  // PV of the step in S buffer b issued (after a tcgen05 before-fence)
    uint64_t drain[2];
};

struct Misc {
    Bars bar;
    int4 vreq[kVReq];        // V load request: first token of cube a (-1: none), of cube b, head, step word
    uint32_t v_meta[kVBuf];  // step word of the V pair in each V buffer
    uint32_t k_meta[kKBuf];  // step word of the K pair in each K buffer
    uint32_t s_meta[kSBuf];  // step word of each S buffer
    // proxy steps: which of the step's 128 proxy keys each query cube may use
    // ([cube][key half][32-key word]) and the first proxy key's cube index
    uint32_t k_pmask[kKBuf][8];
    int k_pbase[kKBuf];
    uint32_t s_pmask[kSBuf][8];
    int s_pbase[kSBuf];
    uint32_t tmem_base;
    int abort;
    int end_g;  // the CTA's last step, once its softmax is done (the other softmax warps stop there)
    alignas(16) float alpha[kSBuf][128];  // per S buffer, row: O rescale factor of that step
    int rflag[kSBuf][4];                  // per S buffer, lane quarter: some row rescales
    float m_state[2][128];                // [step parity][row]: offset after the step's decision
    float l_state[2][128];                // [step parity][row]: row sum after the step
    int n_state[2][4];                    // [step parity][lane quarter]: tiles finished after the step
    float lfin[2][128];                   // [tile parity][row]: row sum at the tile's end
    float mfin[2][128];                   // [tile parity][row]: running offset at the tile's end
    uint32_t bits1[kMaxNq / 32];          // membership bitmaps of the tile's two lists
    uint32_t bits2[kMaxNq / 32];
    int32_t list1[2][kMaxTopk];           // [tile parity]: the tile's two selection lists
    int32_t list2[2][kMaxTopk];           // (the next tile's are copied in while this one runs)
    alignas(16) uint8_t vbs8[kMaxNq];     // the valid counts (255: out of range)
};

struct Layout {
    static constexpr uint32_t Q_OFF = 0;                           // Q tile
    static constexpr uint32_t K_OFF = Q_OFF + kTileBytes;          // K ring
    static constexpr uint32_t V_OFF = K_OFF + kKBuf * kTileBytes;  // V ring
    static constexpr uint32_t TILE_BYTES = V_OFF + kVBuf * kTileBytes;
    static constexpr uint32_t MISC_BYTES = (sizeof(Misc) + 1023) / 1024 * 1024;
    static constexpr uint32_t SMEM_BYTES = MISC_BYTES + TILE_BYTES + 1024;  // + alignment slack
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <bool B>
struct Flag {
    static constexpr bool value = B;
};

// PROXY: the kernel runs the proxy steps after each tile's selected cubes.  It is a
// template parameter so that the plain kernels hold none of that code: as a run-time
// flag it cost the plain forward 25-40 % (its branches and instructions sat in the
// producer's and the softmax's per-step paths, whose issue slots the softmax needs).
template <bool NEG, bool PRECISE, bool PROXY>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_pair_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmkc,
                    const __grid_constant__ CUtensorMap tmvc, const Routes rt,
                    const int32_t* __restrict__ vbs, const int32_t* __restrict__ plan, uint16_t* __restrict__ out,
                    float* __restrict__ lse, int S, int H, int nq, int S_kv, int nkv, int tiles_per_bh, int n_tiles,
                    float scale_log2, int* err)
{
    using L = Layout;
    extern __shared__ uint8_t smem_raw[];
    Misc& m = *reinterpret_cast<Misc*>(smem_raw);
    Bars& bb = m.bar;
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t tiles = (raw_addr + L::MISC_BYTES + 1023u) & ~1023u;  // 1 KiB aligned for 128B swizzle
    uint8_t* tiles_ptr = smem_raw + (tiles - raw_addr);

    // Values that are the same in every lane (the warp index, a step word read from
    // shared memory) go through a shuffle from lane 0: the compiler then knows them
    // to be warp-uniform, and branches on them need no divergence handling around
    // the warp-collective tcgen05 loads and stores they contain (Wan 832x480 forward
    // 4.75 -> 4.67 ms).
    const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0);
    const uint32_t lane = threadIdx.x & 31;
    const int my_tiles = n_tiles > (int)blockIdx.x ? (n_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

    // ------------------------------------------------------------ set-up
    if (threadIdx.x == 0) {
        mbar_init(&bb.q_full, 1);
        mbar_init(&bb.q_empty, 1);
        for (int i = 0; i < kKBuf; ++i) {
            mbar_init(&bb.k_full[i], 1);
            mbar_init(&bb.k_empty[i], 1);
        }
        for (int i = 0; i < kVBuf; ++i) {
            mbar_init(&bb.v_full[i], 1);
            mbar_init(&bb.v_empty[i], 1);
        }
        for (int i = 0; i < kSBuf; ++i) {
            mbar_init(&bb.s_full[i], 2);    // MMA warp (step word) + QK completion
            mbar_init(&bb.a_full[i], 128);  // the four softmax warps of the step
            mbar_init(&bb.p_full[i], 256);  // those and every correction thread
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bb.pv_done[i], 1);
            mbar_init(&bb.l_full[i], 128);
            mbar_init(&bb.l_empty[i], 128);
        }
        for (int i = 0; i < kVReq; ++i) {
            mbar_init(&bb.vr_full[i], 1);
            mbar_init(&bb.vr_empty[i], 1);
        }
        for (int i = 0; i < kSBuf; ++i)
            for (int j = 0; j < 4; ++j) {
                mbar_init(&bb.dec[i][j], 32);
                mbar_init(&bb.lsum[i][j], 32);
            }
        mbar_init(&bb.o_full, 1);
        for (int i = 0; i < kSBuf; ++i) mbar_init(&bb.pv_issued[i], 1);
        mbar_init(&bb.drain[0], 1);
        mbar_init(&bb.drain[1], 1);
        m.abort = 0;
        m.end_g = 0x7fffffff;
        fence_mbar_init();
    }
    vbs_stage(vbs, nkv, S_kv, m.vbs8, err);
    if (warp == kWarpMma) {
        tmem_alloc(&m.tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == kWarpProd && lane == 0) {
        prefetch_tmap(&tmq);
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
        if (PROXY) {
            prefetch_tmap(&tmkc);
            prefetch_tmap(&tmvc);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = m.tmem_base;

    if (warp == kWarpProd) {
        // ------------------------------------------------------------ TMA producer of Q and K
        // (it posts each step's V pair to the V producer, so that K loads never wait
        // behind a V buffer)
        int kc = 0;
        int armed_q = -1, armed_k = -1, armed_kb = 0;
        const uint64_t l2_keep = PROXY ? l2_policy_evict_last() : 0ull;
        bool aborted = false;
        uint8_t* qdst = tiles_ptr + L::Q_OFF;
        TileRef t_next;
        if (my_tiles > 0) {
            t_next = checked_tile(blockIdx.x, H, nq, tiles_per_bh, plan, lane == 0 ? err : nullptr);
            lists_fetch(t_next, rt, H, nq, m.list1[0], m.list2[0], err, lane);
        }
        for (int n = 0; n < my_tiles && !aborted; ++n) {
            const TileRef t = t_next;
            int32_t* l1 = m.list1[n & 1];
            int32_t* l2 = m.list2[n & 1];
            const int n_ent = rt.kind == kRouteMask  ? steps_build_mask(t, nkv, l1, l2, m.bits1, m.bits2, err, lane)
                              : rt.kind == kRouteAll ? steps_build_all(t, nkv, l1, lane)
                                                     : steps_build(t, nkv, l1, l2, m.bits1, m.bits2, err, lane);
            const uint16_t* ent = reinterpret_cast<const uint16_t*>(l1);  // written over list 1
            const int tok0 = t.b * S;        // the tile's query tokens
            const int tok0kv = t.b * S_kv;   // its key / value tokens
            // proxy mode: after the selected cubes, ceil(nq / 128) steps over the proxy keys
            // (cube j's mean key and summed value), 128 cubes per step; a tile without
            // entries then has no plain step (else it takes one empty step)
            const int n_proxy = PROXY ? (nkv + 127) / 128 : 0;
            const int n_plain = PROXY ? (n_ent + 1) / 2 : max(1, (n_ent + 1) / 2);
            const int n_steps = n_plain + n_proxy;
            // Step s of the tile: its K pair (rows ka, kb of head kh of map kmap; -1: none),
            // its V request, and with the tile's first step the tile's Q and the next tile's
            // lists.  Inlined at two sites, each with a fixed map.
            auto issue = [&](int s, const CUtensorMap* kmap, int kh, int ka, int kb2, int vh, uint32_t word,
                             const uint32_t* pmw, int pbase) {
                const uint32_t bytes = 2 * kHalfBox * ((ka >= 0) + (kb2 >= 0));
                const int kb = kc % kKBuf, vr = kc % kVReq;
                if (lane == 0) {
                    // K pair of the step: its buffer is free once the QK two steps back finished
                    if (wait_bar(&bb.k_empty[kb], ((kc / kKBuf) & 1) ^ 1, &m.abort, err)) {
                        if (pmw != nullptr) {
#pragma unroll
                            for (int w = 0; w < 8; ++w) m.k_pmask[kb][w] = pmw[w];
                            m.k_pbase[kb] = pbase;
                        }
                        m.k_meta[kb] = word;  // published, with the masks, by the expect-tx arrival
                        mbar_expect_tx(&bb.k_full[kb], bytes);
                        armed_k = (kc / kKBuf) & 1;
                        armed_kb = kb;
                        uint8_t* kdst = tiles_ptr + L::K_OFF + kb * kTileBytes;
                        if (pmw != nullptr) {  // mean keys: every tile of the head reads them
                            if (ka >= 0) load_cube_keep(kmap, &bb.k_full[kb], kdst, 0, kh, ka, l2_keep);
                            if (kb2 >= 0) load_cube_keep(kmap, &bb.k_full[kb], kdst, 1, kh, kb2, l2_keep);
                        } else {
                            if (ka >= 0) load_cube(kmap, &bb.k_full[kb], kdst, 0, kh, ka);
                            if (kb2 >= 0) load_cube(kmap, &bb.k_full[kb], kdst, 1, kh, kb2);
                        }
                    } else {
                        aborted = true;
                    }
                    // the step's V pair, for the V producer (same rows as the K pair)
                    if (!aborted && wait_bar(&bb.vr_empty[vr], ((kc / kVReq) & 1) ^ 1, &m.abort, err)) {
                        m.vreq[vr] = make_int4(ka, kb2, vh, (int)word);
                        mbar_arrive(&bb.vr_full[vr]);
                    } else {
                        aborted = true;
                    }
                    // the tile's Q, once the previous tile's last QK has released the buffer
                    if (!aborted && s == 0) {
                        if (wait_bar(&bb.q_empty, (n & 1) ^ 1, &m.abort, err)) {
                            mbar_expect_tx(&bb.q_full, 2 * kHalfBox * ((t.i1 >= 0) + (t.i2 >= 0)));
                            armed_q = n & 1;
                            if (t.i1 >= 0) load_cube(&tmq, &bb.q_full, qdst, 0, t.h, tok0 + 64 * t.i1);
                            if (t.i2 >= 0) load_cube(&tmq, &bb.q_full, qdst, 1, t.h, tok0 + 64 * t.i2);
                        } else {
                            aborted = true;
                        }
                    }
                }
                if (s == 0 && n + 1 < my_tiles) {
                    // the next tile, once this one's first loads are out: its lists copied
                    // into the other list buffer and its Q cubes prefetched into L2
                    t_next = checked_tile(blockIdx.x + (n + 1) * gridDim.x, H, nq, tiles_per_bh, plan,
                                          lane == 0 ? err : nullptr);
                    lists_fetch(t_next, rt, H, nq, m.list1[(n + 1) & 1], m.list2[(n + 1) & 1], err, lane);
                    if (lane == 0) {
                        for (int q2 = 0; q2 < 2; ++q2) {
                            const int i = q2 == 0 ? t_next.i1 : t_next.i2;
                            if (i < 0) continue;
                            tma_prefetch_3d(&tmq, 0, t_next.h, t_next.b * S + 64 * i);
                            tma_prefetch_3d(&tmq, 64, t_next.h, t_next.b * S + 64 * i);
                        }
                    }
                }
                aborted = __shfl_sync(0xffffffffu, aborted, 0);
                ++kc;
            };
            // the selected cubes, two entries a step (one 32-bit load: 2 s is even)
            for (int s = 0; s < n_plain && !aborted; ++s) {
                const uint32_t pair = 2 * s < n_ent ? *reinterpret_cast<const uint32_t*>(ent + 2 * s) : 0u;
                const uint32_t ea = pair & 0xffffu;
                const uint32_t eb = 2 * s + 1 < n_ent ? pair >> 16 : 0u;
                const int ja = (int)(ea & 0x1fffu), jb = (int)(eb & 0x1fffu);
                StepMeta meta;
                meta.ma = (int)(ea >> 14);
                meta.mb = (int)(eb >> 14);
                const int va = m.vbs8[ja], vb = m.vbs8[jb];  // 255: an invalid count, no tokens
                meta.na = meta.ma != 0 && va <= 64 ? va : 0;
                meta.nb = meta.mb != 0 && vb <= 64 ? vb : 0;
                const bool last = s + 1 == n_steps;
                meta.flags = (s == 0 ? 1 : 0) | (last ? 2 : 0);
                const uint32_t word = step_word(meta) | (last && n == my_tiles - 1 ? kFinal : 0u);
                issue(s, &tmk, t.h, meta.na > 0 ? tok0kv + 64 * ja : -1, meta.nb > 0 ? tok0kv + 64 * jb : -1, t.h, word,
                      nullptr, 0);
            }
            if constexpr (PROXY) {
                // proxy keys pbase .. pbase + 127 (rows of the [B*H*nq, D] means and sums): key
                // j may be used by query cube q iff cube j has valid tokens and q did not
                // select it (no double count)
                const int cubes_here = (t.i1 >= 0 ? 1 : 0) | (t.i2 >= 0 ? 2 : 0);
                for (int pc = 0; pc < n_proxy && !aborted; ++pc) {
                    const int s = n_plain + pc, pbase = 128 * pc;
                    StepMeta meta;
                    meta.na = min(64, nkv - pbase);
                    meta.nb = min(64, max(0, nkv - pbase - 64));
                    meta.ma = cubes_here;
                    meta.mb = meta.nb > 0 ? cubes_here : 0;
                    uint32_t pm = 0;  // lane w < 8: mask word w, [cube][key half][32-key word]
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const int j = pbase + 32 * w + (int)lane;
                        const int nj = j < nkv ? (int)m.vbs8[j] : 0;
                        const uint32_t valid = __ballot_sync(0xffffffffu, nj >= 1 && nj <= 64);
                        const int word = (pbase >> 5) + w;
                        const bool in_range = pbase + 32 * w < nkv;
                        const uint32_t m1 = t.i1 >= 0 && in_range ? valid & ~m.bits1[word] : 0u;
                        const uint32_t m2 = t.i2 >= 0 && in_range ? valid & ~m.bits2[word] : 0u;
                        if ((int)lane == w) pm = m1;
                        if ((int)lane == 4 + w) pm = m2;
                    }
                    uint32_t pmw[8];  // in every lane (lane 0 stores them with the K pair)
#pragma unroll
                    for (int w = 0; w < 8; ++w) pmw[w] = __shfl_sync(0xffffffffu, pm, w);
                    const bool last = s + 1 == n_steps;
                    meta.flags = (s == 0 ? 1 : 0) | (last ? 2 : 0);
                    const uint32_t word =
                        step_word(meta) | (last && n == my_tiles - 1 ? kFinal : 0u) | kProxyStep;
                    const int row = (t.b * H + t.h) * nkv + pbase;
                    issue(s, &tmkc, 0, row, meta.nb > 0 ? row + 64 : -1, 0, word, pmw, pbase);
                }
            }
        }
        cp_async_wait_all();  // a list copy still in flight after an abort
        if (aborted && lane == 0) {
            // copies issued by this thread must land before the CTA's shared memory goes away
            if (armed_q >= 0) drain_wait(&bb.q_full, armed_q);
            if (armed_k >= 0) drain_wait(&bb.k_full[armed_kb], armed_k);
        }
    } else if (warp == kWarpVProd) {
        // ------------------------------------------------------------ TMA producer of V
        int armed_v = -1, armed_vb = 0;
        const uint64_t l2_keep = PROXY ? l2_policy_evict_last() : 0ull;
        for (int vc = 0; my_tiles > 0 && lane == 0; ++vc) {
            const int vr = vc % kVReq, vb = vc % kVBuf;
            if (!wait_bar(&bb.vr_full[vr], (vc / kVReq) & 1, &m.abort, err)) break;
            const int4 rq = m.vreq[vr];
            mbar_arrive(&bb.vr_empty[vr]);
            // the V buffer is free once the PV two steps back finished
            if (!wait_bar(&bb.v_empty[vb], ((vc / kVBuf) & 1) ^ 1, &m.abort, err)) break;
            m.v_meta[vb] = (uint32_t)rq.w;  // published by the arrival below
            mbar_expect_tx(&bb.v_full[vb], 2 * kHalfBox * ((rq.x >= 0) + (rq.y >= 0)));
            armed_v = (vc / kVBuf) & 1;
            armed_vb = vb;
            uint8_t* vdst = tiles_ptr + L::V_OFF + vb * kTileBytes;
            if (PROXY && ((uint32_t)rq.w & kProxyStep)) {
                // summed values: every tile of the head reads them, so they stay in L2
                if (rq.x >= 0) load_cube_keep(&tmvc, &bb.v_full[vb], vdst, 0, rq.z, rq.x, l2_keep);
                if (rq.y >= 0) load_cube_keep(&tmvc, &bb.v_full[vb], vdst, 1, rq.z, rq.y, l2_keep);
            } else {
                if (rq.x >= 0) load_cube(&tmv, &bb.v_full[vb], vdst, 0, rq.z, rq.x);
                if (rq.y >= 0) load_cube(&tmv, &bb.v_full[vb], vdst, 1, rq.z, rq.y);
            }
            if ((uint32_t)rq.w & kFinal) break;  // the CTA's last step
        }
        if (lane == 0 && armed_v >= 0 && aborted_flag(&m.abort)) drain_wait(&bb.v_full[armed_vb], armed_v);
        __syncwarp();
    } else if (warp == kWarpMma || warp == kWarpQk) {
        // ------------------------------------------------------------ MMA issuers
        // Two warps feed the tensor core: warp kWarpQk issues the QK products, warp
        // kWarpMma the PV products.  While one is blocked issuing a group (the
        // tensor core's queue is short), the other does the barrier checks for
        // its next group, so the groups reach the tensor core back to back.  The
        // order QK(j) after PV(j - 3) (they share S buffer j % 3) is kept by
        // barrier pv_issued: the PV warp arrives after issuing PV(j) (after a
        // tcgen05 before-fence), the QK warp waits for it before QK(j + 3).  In each
        // warp the whole warp runs the schedule and one elected lane issues, with no
        // branch around an elect: conditions go into the issue predicate.
        constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, false, true);
        // operand descriptors built once; a k-step adds its byte offset / 16
        const uint64_t d_hi = smem_desc_sw128(0, 0, 1024);
        bool aborted = false;
        if (warp == kWarpQk) {
            const uint32_t ql = (uint32_t)smem_desc_sw128(tiles + L::Q_OFF, 16, 1024);
            const uint32_t kl0 = (uint32_t)smem_desc_sw128(tiles + L::K_OFF, 16, 1024);
            int qn = 0;
            for (int j = 0; my_tiles > 0; ++j) {
                const int kb = j % kKBuf, sb = j % kSBuf;
                if (!wait_warp(&bb.k_full[kb], (j / kKBuf) & 1, &m.abort, err)) { aborted = true; break; }
                const uint32_t meta = m.k_meta[kb];
                if (sw_flags(meta) & 1) {
                    if (!wait_warp(&bb.q_full, qn & 1, &m.abort, err)) { aborted = true; break; }
                    ++qn;
                }
                // S buffer sb is free once PV(j - 3) has been issued
                if (j >= kSBuf && !wait_warp(&bb.pv_issued[sb], ((j - kSBuf) / kSBuf) & 1, &m.abort, err)) {
                    aborted = true;
                    break;
                }
                if (PROXY && (meta & kProxyStep)) {
                    // every lane stores the same words, so the elected arrival publishes them
#pragma unroll
                    for (int w = 0; w < 8; ++w) m.s_pmask[sb][w] = m.k_pmask[kb][w];
                    m.s_pbase[sb] = m.k_pbase[kb];
                }
                m.s_meta[sb] = meta;                // every lane stores the same word
                mbar_arrive_elect(&bb.s_full[sb]);  // publishes it (release)
                tc_fence_after();
                const uint32_t kl = kl0 + ((uint32_t)kb * kTileBytes >> 4);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = ((kk >> 2) * (2 * kHalfBox) + (kk & 3) * 32u) >> 4;
                    umma_ss_elect(tbase + 128u * sb, d_hi | (ql + off), d_hi | (kl + off), idesc_qk, kk > 0 ? 1u : 0u);
                }
                umma_commit_elect(&bb.s_full[sb]);
                umma_commit_elect(&bb.k_empty[kb]);
                umma_commit_elect_if(&bb.q_empty, sw_flags(meta) & 2);
                if (meta & kFinal) break;
            }
        } else {
            const uint32_t vl0 = (uint32_t)smem_desc_sw128(tiles + L::V_OFF, 2 * kHalfBox, 1024);
            const uint32_t o_tmem = tbase + kOCol;
            bool o_init = false;
            for (int j = 0; my_tiles > 0; ++j) {
                const int sb = j % kSBuf, vb = j % kVBuf;
                const uint32_t par = (j / kSBuf) & 1;
                if (!wait_warp(&bb.v_full[vb], (j / kVBuf) & 1, &m.abort, err)) { aborted = true; break; }
                // everything that needs only the V pair is done before waiting for P
                const uint32_t meta = m.v_meta[vb];
                const int na = sw_na(meta), nb = sw_nb(meta);
                const uint32_t vl = vl0 + ((uint32_t)vb * kTileBytes >> 4);
                const int za = (na & 15) ? 16 - (na & 15) : 0, zb = (nb & 15) ? 16 - (nb & 15) : 0;
                if (za + zb > 0) {
                    // V rows between vbs and the next multiple of 16 are read by the last
                    // k-step of their cube: zero them (both d halves) before the product
                    const uint32_t vbase = tiles + L::V_OFF + vb * kTileBytes;
                    for (int w = lane; w < (za + zb) * 16; w += 32) {
                        const int zr = w >> 4, chunk = w & 15;
                        const int row = zr < za ? na + zr : 64 + nb + (zr - za);
                        sts128(vbase + (chunk >> 3) * (2 * kHalfBox) + row * 128 + (chunk & 7) * 16, 0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                if (!wait_warp(&bb.p_full[sb], par, &m.abort, err)) { aborted = true; break; }
                tc_fence_after();
                // k-steps (16 keys) 0..ceil16(na)-1 of half 0 and 4..4+ceil16(nb)-1 of half 1; the
                // bf16 P of key half h sits in the first 32 columns of that half's 64 (precise
                // mode: the high and low parts of 32-key chunk c in columns 32 c .. +15, +16 .. +31)
                const uint32_t kmask = ((1u << ((na + 15) >> 4)) - 1u) | (((1u << ((nb + 15) >> 4)) - 1u) << 4);
                const uint32_t p_tmem = tbase + 128u * sb;
                if (sw_flags(meta) & 1) o_init = false;
                uint32_t acc = o_init ? 1u : 0u;
#pragma unroll
                for (int kstep = 0; kstep < 8; ++kstep) {
                    const uint32_t on = (kmask >> kstep) & 1u;  // warp-uniform, no branch
                    const uint64_t vdesc = d_hi | (vl + ((kstep * 2048) >> 4));
                    if (PRECISE) {
                        // the weights of keys 16 kstep .. +15: high bf16 part, then the low part
                        const uint32_t a_col = 32u * (kstep >> 1) + 8u * (kstep & 1);
                        umma_ts_elect_if(o_tmem, p_tmem + a_col, vdesc, idesc_pv, acc, on);
                        acc |= on;
                        umma_ts_elect_if(o_tmem, p_tmem + a_col + 16u, vdesc, idesc_pv, acc, on);
                    } else {
                        const uint32_t a_col = kstep < 4 ? 8u * kstep : 64u + 8u * (kstep - 4);
                        umma_ts_elect_if(o_tmem, p_tmem + a_col, vdesc, idesc_pv, acc, on);
                    }
                    acc |= on;
                }
                o_init = o_init || kmask != 0;
                // PV(j) is in the tensor core's queue: S buffer sb may be written again (the
                // QK issuer's products go after it; the commits below track this warp's only)
                tc_fence_before();
                mbar_arrive_elect(&bb.pv_issued[sb]);
                umma_commit_elect(&bb.v_empty[vb]);
                umma_commit_elect(&bb.pv_done[j & 1]);
                umma_commit_elect_if(&bb.o_full, sw_flags(meta) & 2);
                if (meta & kFinal) break;
            }
        }
        if (aborted) {
            umma_commit_elect(&bb.drain[warp == kWarpQk ? 1 : 0]);
            if (lane == 0) drain_wait(&bb.drain[warp == kWarpQk ? 1 : 0], 0);
            __syncwarp();
        }
    } else if (warp >= kWarpCorr0) {
        // ------------------------------------------------------------ O correction and epilogue
        const int wq = warp & 3;
        const int r = 32 * wq + (int)lane;
        const int qbit = r >> 6;
        const uint32_t oa = tbase + ((uint32_t)(32 * wq) << 16) + kOCol;
        int g = 0;
        bool released = false;    // this tile's first step was handled by the previous tile's epilogue
        uint32_t released_meta = 0;  // and this was its step word
        for (int n = 0; n < my_tiles; ++n) {
            for (;;) {
                const int b = g % kSBuf;
                if (released) {  // a first step: no rescale, its arrival made already
                    released = false;
                    ++g;
                    if (sw_flags(released_meta) & 2) break;
                    continue;
                }
                if (!wait_warp(&bb.a_full[b], (g / kSBuf) & 1, &m.abort, err)) goto corr_exit;
                const uint32_t meta = m.s_meta[b];
                const int rescale = __shfl_sync(0xffffffffu, !(sw_flags(meta) & 1) && m.rflag[b][wq] != 0, 0);
                if (rescale) {
                    // O row r *= alpha (1 for rows whose offset stayed), once the
                    // previous step's PV has finished
                    const int jp = g - 1;
                    if (!wait_warp(&bb.pv_done[jp & 1], (jp >> 1) & 1, &m.abort, err)) goto corr_exit;
                    tc_fence_after();
                    const float a = m.alpha[b][r];
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
                mbar_arrive(&bb.p_full[b]);
                ++g;
                if (sw_flags(meta) & 2) break;
            }

            // ---- epilogue: out[b, 64 i + (r % 64), h, :] = O[r, :] / l; lse = (m + log2 l) ln 2
            if (!wait_warp(&bb.o_full, n & 1, &m.abort, err)) goto corr_exit;
            if (!wait_warp(&bb.l_full[n & 1], (n >> 1) & 1, &m.abort, err)) goto corr_exit;
            tc_fence_after();
            {
                const TileRef t = checked_tile(blockIdx.x + n * gridDim.x, H, nq, tiles_per_bh, plan, nullptr);
                const float l = m.lfin[n & 1][r];
                const float m_row = m.mfin[n & 1][r];
                mbar_arrive(&bb.l_empty[n & 1]);
                const int cube = qbit == 0 ? t.i1 : t.i2;
                const bool has = l > 0.f;
                const float inv = has ? __frcp_rn(l) : 0.f;
                const int64_t token = (int64_t)t.b * S + 64LL * cube + (r & 63);
                uint16_t* dst = out + (token * H + t.h) * kD;
                // read and round the whole row
                uint32_t pk[4][16];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint32_t o[32];
                    tmem_ld32(oa + 32 * c4, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[c4][e] = has ? pack_bf16(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv)
                                        : 0u;
                }
                if (cube >= 0) {
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4)
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            st_global_v4(dst + 32 * c4 + 8 * v, pk[c4][4 * v], pk[c4][4 * v + 1], pk[c4][4 * v + 2],
                                         pk[c4][4 * v + 3]);
                }
                if (lse != nullptr && cube >= 0)
                    lse[((int64_t)t.b * H + t.h) * S + 64LL * cube + (r & 63)] =
                        has ? (m_row + __log2f(l)) * 0.69314718055994531f : -INFINITY;
                // The next tile's first step (a first step, which never rescales) is handled
                // here, so that its product, which overwrites O (read above), need not wait
                // for this warp's next pass.  Every product of this tile has completed
                // (o_full), so the arrival can only count toward that step's phase.  Its
                // offsets are waited for first: until this arrival no product of that step
                // can be issued, so no later step can complete a_full of its buffer again
                // before this wait (a release ahead of the wait let the softmax lap this warp
                // on that ring when tiles are four steps long).
                if (n + 1 < my_tiles) {
                    const int b1 = g % kSBuf;
                    if (!wait_warp(&bb.a_full[b1], (g / kSBuf) & 1, &m.abort, err)) goto corr_exit;
                    released_meta = __shfl_sync(0xffffffffu, m.s_meta[b1], 0);
                    tc_fence_before();
                    mbar_arrive(&bb.p_full[b1]);
                    released = true;
                }
            }
            tc_fence_before();
        }
    corr_exit:;
    } else {
        // ------------------------------------------------------------ softmax: steps in turn
        //
        // Warp w owns TMEM lanes 32 (w % 4) .. +31 (query rows, thread = row) and
        // the steps g with g % 3 == w / 4, all 128 columns.  The three warps of a
        // lane quarter share an SMSP and work on three consecutive steps at once
        // (one per S buffer), so the SMSP's exp2 units always have work while
        // any one warp waits for TMEM or a barrier.  A row's running offset and
        // running sum pass from step to step through shared memory (dec: offset
        // and tile count after the decision of step g; lsum: row sum after step g).
        // Those barriers come in three sets by step % 3: the warp of step g waits
        // for step g - 1 only after its own step g - 3, which waited for g - 4,
        // so a barrier is never two phases behind its waiter.
        const int wq = warp & 3, par = warp >> 2;
        const int r = 32 * wq + (int)lane;  // query row of the tile == TMEM lane
        const int qbit = wq >> 1;           // 0: query cube i1, 1: i2 (rows r >> 6)
        const uint32_t lane_base = tbase + ((uint32_t)(32 * wq) << 16);
        constexpr float kNeutral = NEG ? INFINITY : -INFINITY;  // a masked logit
        for (int g = par;; g += kSBuf) {
            const int b = g % kSBuf;
            const uint32_t spar = (g / kSBuf) & 1;
            int n_before = 0;
            float m_prev = -INFINITY;
            if (my_tiles == 0) break;
            if (!wait_warp(&bb.s_full[b], spar, &m.abort, err)) goto softmax_exit;
            if (g > *reinterpret_cast<volatile int*>(&m.end_g)) break;  // past the CTA's last step
            const uint32_t meta = __shfl_sync(0xffffffffu, m.s_meta[b], 0);  // warp-uniform
            tc_fence_after();
            const int na = sw_na(meta), nb = sw_nb(meta), flags = sw_flags(meta);
            const int nv0 = ((sw_ma(meta) >> qbit) & 1) ? na : 0;  // valid keys of each half
            const int nv1 = ((sw_mb(meta) >> qbit) & 1) ? nb : 0;  // for this row (warp-uniform)
            const uint32_t s_addr = lane_base + 128u * b;
            // proxy step: the keys are mean keys of cubes pbase .. pbase + 127; chunk ch's
            // mask word (which of them this row's query cube may use) and their token counts
            const bool pstep = PROXY && (meta & kProxyStep) != 0;
            const uint32_t* pmask = m.s_pmask[b] + 4 * qbit;
            const int pbase = pstep ? m.s_pbase[b] : 0;

            // pass 1: extreme of the selected logits, one 32-column chunk at a time
            // (chunk ch: columns 32 ch .. +31, key half ch / 2).  Both passes come in two
            // instantiations: a proxy step masks by its bits, a plain step only its ragged
            // tail, and plain steps run none of the proxy code.
            auto pass1 = [&](auto px) -> float {
                constexpr bool PX = decltype(px)::value;
                float e4[4] = {kNeutral, kNeutral, kNeutral, kNeutral};
#pragma unroll 1
                for (int ch = 0; ch < 4; ++ch) {
                    const int nv = (ch < 2 ? nv0 : nv1) - 32 * (ch & 1);  // valid columns of the chunk
                    if (nv <= 0) continue;
                    float sc[32];
                    tmem_ld32(s_addr + 32 * ch, reinterpret_cast<uint32_t*>(sc));
                    tmem_ld_wait();
                    if constexpr (PX) {
                        const uint32_t mw = pmask[ch];
#pragma unroll
                        for (int c = 0; c < 32; ++c) sc[c] = (mw >> c) & 1u ? sc[c] : kNeutral;
                    } else if (nv < 32) {
#pragma unroll
                        for (int c = 0; c < 32; ++c) sc[c] = c < nv ? sc[c] : kNeutral;
                    }
#pragma unroll
                    for (int c = 0; c < 32; c += 8) {
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            e4[u] = NEG ? min3(e4[u], sc[c + 2 * u], sc[c + 2 * u + 1])
                                        : max3(e4[u], sc[c + 2 * u], sc[c + 2 * u + 1]);
                    }
                }
                return NEG ? min3(fminf(e4[0], e4[1]), e4[2], e4[3]) : max3(fmaxf(e4[0], e4[1]), e4[2], e4[3]);
            };
            const float ext = PROXY && pstep ? pass1(Flag<PROXY>{}) : pass1(Flag<false>{});

            // decision: the row's offset after this step (lazy: raised by more than kTau only)
            if (g > 0) {
                if (!wait_warp(&bb.dec[(g - 1) % kSBuf][wq], ((g - 1) / kSBuf) & 1, &m.abort, err))
                    goto softmax_exit;
                n_before = m.n_state[(g - 1) & 1][wq];
                m_prev = m.m_state[(g - 1) & 1][r];
            }
            if (flags & 1) m_prev = -INFINITY;  // a tile's first step starts afresh
            const float m_step = (nv0 | nv1) != 0 ? ext * scale_log2 : -INFINITY;  // base-2 units
            const bool raise = m_step > m_prev + kTau;                            // false for -inf
            const float m_run = raise ? m_step : m_prev;
            // alpha scales O and the running sum; 0 at a tile's first step (nothing before)
            const float alpha = (flags & 1) ? 0.f : (raise ? (m_prev == -INFINITY ? 0.f : ex2(m_prev - m_step)) : 1.f);
            const int n_after = n_before + ((flags & 2) ? 1 : 0);
            m.alpha[b][r] = alpha;
            m.m_state[g & 1][r] = m_run;
            const bool warp_raise = __any_sync(0xffffffffu, raise && !(flags & 1));
            if (lane == 0) {
                m.rflag[b][wq] = warp_raise ? 1 : 0;
                m.n_state[g & 1][wq] = n_after;
            }
            mbar_arrive(&bb.a_full[b]);
            mbar_arrive(&bb.dec[b][wq]);

            // pass 2: P = exp2(x - m) as bf16 pairs; chunk ch's P goes to columns
            // 64 (ch / 2) + 16 (ch % 2): each half's P fills the half's first 32
            // columns, over logits already consumed.  Precise mode: P = hi + lo, two
            // bf16 parts (lo = bf16(P - hi), so hi + lo is within 2^-17 of P) in the
            // chunk's own columns 32 ch .. +15 and +16 .. +31
            const float mu = m_run == -INFINITY ? 0.f : m_run;
            auto pass2 = [&](auto px) -> float2 {
                constexpr bool PX = decltype(px)::value;
                float ls0 = 0.f, ls1 = 0.f;
#pragma unroll 1
                for (int ch = 0; ch < 4; ++ch) {
                    const int nv = (ch < 2 ? nv0 : nv1) - 32 * (ch & 1);
                    uint32_t pk[16], pl[16];
                    if (nv > 0) {
                        float sc[32];
                        tmem_ld32(s_addr + 32 * ch, reinterpret_cast<uint32_t*>(sc));
                        tmem_ld_wait();
                        if constexpr (PX) {
                            const uint32_t mw = pmask[ch];
#pragma unroll
                            for (int c = 0; c < 32; ++c) sc[c] = (mw >> c) & 1u ? sc[c] : kNeutral;
                        } else if (nv < 32) {
#pragma unroll
                            for (int c = 0; c < 32; ++c) sc[c] = c < nv ? sc[c] : kNeutral;
                        }
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            float x0, x1, p0, p1;
                            ffma2(x0, x1, sc[2 * c], sc[2 * c + 1], scale_log2, scale_log2, -mu, -mu);
                            if ((kPolyPairs >> (c & 15)) & 1) {
                                // weights below 2^-125 (masked keys included) become 2^-125
                                const float2 pp = ex2_fma2(make_float2(fmaxf(x0, -125.f), fmaxf(x1, -125.f)));
                                p0 = pp.x;
                                p1 = pp.y;
                            } else {
                                p0 = ex2(x0);
                                p1 = ex2(x1);
                            }
                            pk[c] = pack_bf16(p0, p1);
                            if (PRECISE) {
                                const float h0 = __uint_as_float(pk[c] << 16), h1 = __uint_as_float(pk[c] & 0xffff0000u);
                                pl[c] = pack_bf16(p0 - h0, p1 - h1);  // the differences are exact in fp32
                                fadd2(ls0, ls1, p0, p1);
                            } else {
                                // the row sum adds the bf16 weights the P.V product sees, so that
                                // numerator and denominator carry the same rounding
                                add_bf16x2_f32(ls0, ls1, pk[c]);
                            }
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 16; ++c) pk[c] = pl[c] = 0u;
                    }
                    if (PRECISE) {
                        tmem_st16(s_addr + 32 * ch, pk);
                        tmem_st16(s_addr + 32 * ch + 16, pl);
                    } else {
                        tmem_st16(s_addr + 64 * (ch >> 1) + 16 * (ch & 1), pk);
                    }
                    if (PX && nv > 0) {
                        // a proxy stands for vbs[j] tokens: the loop above added its weight once,
                        // this adds it vbs[j] - 1 more times (its summed value enters P.V once)
                        const uint4 wa = *reinterpret_cast<const uint4*>(m.vbs8 + pbase + 32 * ch);
                        const uint4 wb = *reinterpret_cast<const uint4*>(m.vbs8 + pbase + 32 * ch + 16);
                        const uint32_t wn[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            // the counts as floats: byte k of the word under the exponent of 2^23
                            const uint32_t w = wn[c >> 1], k = 2 * (c & 1);
                            float n0 = __uint_as_float(__byte_perm(w, 0x4B000000u, k | 0x7540u));
                            float n1 = __uint_as_float(__byte_perm(w, 0x4B000000u, (k + 1) | 0x7540u));
                            fadd2(n0, n1, -8388609.f, -8388609.f);  // vbs[j] - 1
                            float h0 = __uint_as_float(pk[c] << 16), h1 = __uint_as_float(pk[c] & 0xffff0000u);
                            if (PRECISE)  // the weight is hi + lo
                                fadd2(h0, h1, __uint_as_float(pl[c] << 16), __uint_as_float(pl[c] & 0xffff0000u));
                            ffma2(ls0, ls1, h0, h1, n0, n1, ls0, ls1);
                        }
                    }
                }
                return make_float2(ls0, ls1);
            };
            const float2 lsum = PROXY && pstep ? pass2(Flag<PROXY>{}) : pass2(Flag<false>{});
            const float ls0 = lsum.x, ls1 = lsum.y;
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bb.p_full[b]);

            // running row sum: l(g) = l(g - 1) * alpha(g) + sum of P(g)
            float l_prev = 0.f;
            if (g > 0) {
                if (!wait_warp(&bb.lsum[(g - 1) % kSBuf][wq], ((g - 1) / kSBuf) & 1, &m.abort, err))
                    goto softmax_exit;
                if (!(flags & 1)) l_prev = m.l_state[(g - 1) & 1][r];
            }
            const float l_run = l_prev * alpha + (ls0 + ls1);
            m.l_state[g & 1][r] = l_run;
            mbar_arrive(&bb.lsum[b][wq]);
            if (flags & 2) {
                // the tile's row sum and offset for the epilogue (ring of two tiles)
                const int n = n_before;
                if (!wait_warp(&bb.l_empty[n & 1], ((n >> 1) & 1) ^ 1, &m.abort, err)) goto softmax_exit;
                m.lfin[n & 1][r] = l_run;
                m.mfin[n & 1][r] = m_run;
                mbar_arrive(&bb.l_full[n & 1]);
            }
            if (meta & kFinal) {
                // no step g + 1 or g + 2 will come: complete their s_full phases (two
                // arrivals each) so that the warps waiting for them wake up, see
                // end_g and stop.  Those warps have consumed their previous phase of
                // those barriers: they decided steps g - 2 and g - 1 before this one.
                if (wq == 0 && lane == 0) {
                    m.end_g = g;
                    for (int e = 1; e <= 2; ++e) {
                        mbar_arrive(&bb.s_full[(g + e) % kSBuf]);
                        mbar_arrive(&bb.s_full[(g + e) % kSBuf]);
                    }
                }
                break;
            }
        }
    softmax_exit:;
    }

    // ------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) tmem_dealloc(tbase, 512);
}

// The maps of one forward call: q, k, v ([B*S tokens][H][D]) and, for proxy
// compensation, the mean keys and summed values ([B*H*Nq rows][1][D]).
struct FwdMaps {
    CUtensorMap q, k, v, kc, vc;
};

template <bool NEG, bool PRECISE, bool PROXY>
cudaError_t launch(const FwdMaps& mp, const Routes& rt, const int32_t* vbs, const int32_t* plan, uint16_t* out,
                   float* lse, int B, int S, int H, int nq, int S_kv, int nkv, float scale_log2, int* err,
                   cudaStream_t s)
{
    auto kern = fwd_pair_kernel<NEG, PRECISE, PROXY>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Layout::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int tiles_per_bh = (nq + 1) / 2;
    const int n_tiles = B * H * tiles_per_bh;
    const int grid = n_tiles < sms ? n_tiles : sms;
    kern<<<grid, kThreads, Layout::SMEM_BYTES, s>>>(mp.q, mp.k, mp.v, mp.kc, mp.vc, rt, vbs, plan, out, lse,
                                                    S, H, nq, S_kv, nkv, tiles_per_bh, n_tiles, scale_log2, err);
    return cudaGetLastError();
}

}  // namespace

bool fwd_pair_supported(int nq, int topk) { return nq <= kMaxNq && topk <= kMaxTopk; }

cudaError_t launch_fwd_pair(const uint16_t* q, const uint16_t* k, const uint16_t* v, const Routes& rt,
                            const int32_t* vbs, const int32_t* plan, const uint16_t* kc, const uint16_t* vc,
                            uint16_t* out, float* lse, int B, int S, int H, int nq, int S_kv, int nkv, float sm_scale,
                            bool precise_p, int* err, cudaStream_t s)
{
    FwdMaps mp;
    const int64_t tokens = (int64_t)B * S, kv_tokens = (int64_t)B * S_kv;
    if (!make_map(&mp.q, q, tokens, H) || !make_map(&mp.k, k, kv_tokens, H) || !make_map(&mp.v, v, kv_tokens, H))
        return cudaErrorInvalidValue;
    const bool proxy = kc != nullptr && vc != nullptr;
    if (proxy) {
        const int64_t rows = (int64_t)B * H * nkv;
        if (!make_map(&mp.kc, kc, rows, 1) || !make_map(&mp.vc, vc, rows, 1)) return cudaErrorInvalidValue;
    } else {
        mp.kc = mp.k;  // not read
        mp.vc = mp.v;
    }
    const float scale_log2 = sm_scale * 1.4426950408889634f;
    // one kernel per (sign of the scale, weight precision, proxy steps)
    using Launch = cudaError_t (*)(const FwdMaps&, const Routes&, const int32_t*, const int32_t*, uint16_t*, float*, int,
                                   int, int, int, int, int, float, int*, cudaStream_t);
    static constexpr Launch table[8] = {
        launch<false, false, false>, launch<true, false, false>, launch<false, true, false>, launch<true, true, false>,
        launch<false, false, true>,  launch<true, false, true>,  launch<false, true, true>,  launch<true, true, true>};
    const int which = (scale_log2 < 0.f ? 1 : 0) | (precise_p ? 2 : 0) | (proxy ? 4 : 0);
    return table[which](mp, rt, vbs, plan, out, lse, B, S, H, nq, S_kv, nkv, scale_log2, err, s);
}

}  // namespace vsa
