// Device helpers of the paired-tile forward kernel (fwd_pair.cu): step descriptors, bounded mbarrier waits, tcgen05 /
// TMEM wrappers, packed fp32 pair arithmetic, the tile list generator (the
// union of two selection lists, shared cubes first) and the TMA tensor maps.
// Everything lives in an anonymous namespace: each kernel file gets its own
// copy.
#pragma once

#include "internal.h"
#include "exp2_poly.h"
#include "sm100_ptx.cuh"

#include <cstddef>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

namespace vsa {
namespace {

using namespace ptx;

constexpr int kD = 128;
constexpr float kTau = 8.0f;
constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 2 GHz

constexpr uint32_t kHalfBox = 64 * 128;        // 8 KiB: 64 rows x 64 bf16 (one TMA box)
constexpr uint32_t kTileBytes = 4 * kHalfBox;  // 128 rows x 128 d: Q tile, K pair or V pair (32 KiB)

constexpr int kMaxTopk = 1024;  // per-slot list staging in shared memory
constexpr int kMaxNq = 8192;    // per-slot membership bitmaps in shared memory

// Per-step description, produced by the producer warp with each K pair.
struct StepMeta {
    int32_t na, nb;   // valid keys of key halves 0 (keys 0-63) and 1 (64-127); 0: nothing loaded
    int32_t ma, mb;   // membership: bit 0 = query cube i1 selects it, bit 1 = i2
    int32_t flags;    // bit 0 first step of the tile, bit 1 last step
};

// The fields the other roles need, packed in one 32-bit word in shared memory:
// na [0,7) nb [7,14) ma [14,16) mb [16,18) flags [18,20); the kernel adds its
// own flags above bit 21.
__device__ __forceinline__ uint32_t step_word(const StepMeta& s)
{
    return (uint32_t)s.na | ((uint32_t)s.nb << 7) | ((uint32_t)s.ma << 14) | ((uint32_t)s.mb << 16) |
           ((uint32_t)s.flags << 18);
}
__device__ __forceinline__ int sw_na(uint32_t w) { return (int)(w & 127u); }
__device__ __forceinline__ int sw_nb(uint32_t w) { return (int)((w >> 7) & 127u); }
__device__ __forceinline__ int sw_ma(uint32_t w) { return (int)((w >> 14) & 3u); }
__device__ __forceinline__ int sw_mb(uint32_t w) { return (int)((w >> 16) & 3u); }
__device__ __forceinline__ int sw_flags(uint32_t w) { return (int)((w >> 18) & 3u); }


__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Adding kRound = 1.5 * 2^23 to a float of magnitude below 2^22 rounds it to
// an integer n (the sum has unit spacing) and leaves n, in two's complement,
// in the sum's low mantissa bits; kRound's own low 9 bits are zero.
constexpr float kRound = 12582912.f;

// 2^x for a pair of exponents x in [-125, 126] on the FMA pipe.  The
// multi-function unit's exp2 rate (16 per clock per SM) equals the tensor
// cores' rate at this tile shape, so a share of the exponentials is evaluated
// here instead:
//   t = x + kRound = kRound + n,  n = round(x);   f = x - n in [-1/2, 1/2] (exact)
//   2^f ~ 1 + f (C1 + C2 f + C3 f^2), the fit of exp2_poly.h (relative error
//   1.0e-4, exact at f = 0), and 2^x = 2^f with n added to its exponent
//   field: n << 23 is t's bit pattern shifted left by 23.
__device__ __forceinline__ float2 ex2_fma2(float2 x)
{
    const float2 t = __fadd2_rn(x, make_float2(kRound, kRound));
    const float2 n = __fadd2_rn(t, make_float2(-kRound, -kRound));
    const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
    float2 p = __ffma2_rn(make_float2(VSA_EXP2_C3, VSA_EXP2_C3), f, make_float2(VSA_EXP2_C2, VSA_EXP2_C2));
    p = __ffma2_rn(p, f, make_float2(VSA_EXP2_C1, VSA_EXP2_C1));
    p = __ffma2_rn(p, f, make_float2(1.f, 1.f));
    return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float max3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ float min3(float a, float b, float c)
{
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// tcgen05.mma / commit issued by one elected lane of a converged warp: the
// operands are warp-uniform values, the predicate picks a single issuer.
__device__ __forceinline__ void umma_ss_elect(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_ts_elect(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The same, issued only when `issue` is nonzero: the condition is folded into
// the issue predicate, so the warp runs no branch around the warp-wide elect
// (a branch per MMA doubled the issue interval of the PV group, ~100 -> ~46
// cycles per MMA when removed).
__device__ __forceinline__ void umma_ts_elect_if(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate, uint32_t issue)
{
    asm volatile(
        "{\n\t.reg .pred p, e, q;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.ne.b32 q, %5, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "and.pred e, e, q;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(issue)
        : "memory");
}

__device__ __forceinline__ void umma_commit_elect(uint64_t* bar)
{
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
            smem_u32(bar))
        : "memory");
}

// Commit issued by one elected lane only when `issue` is nonzero (no branch).
__device__ __forceinline__ void umma_commit_elect_if(uint64_t* bar, uint32_t issue)
{
    asm volatile(
        "{\n\t.reg .pred e, q;\n\t"
        "setp.ne.b32 q, %1, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "and.pred e, e, q;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar)),
        "r"(issue)
        : "memory");
}

// mbarrier arrival by one elected lane of a converged warp (no branch).
__device__ __forceinline__ void mbar_arrive_elect(uint64_t* bar)
{
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e mbarrier.arrive.shared::cta.b64 _, [%0];\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

// Packed pair arithmetic (one instruction for two fp32 lanes on sm_100).
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0, float c1)
{
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

__device__ __forceinline__ void fadd2(float& d0, float& d1, float a0, float a1)
{
    asm("{\n\t.reg .b64 ra, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rd, {%0, %1};\n\t"
        "add.rn.f32x2 rd, rd, ra;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(a0), "f"(a1));
}

// d0 += the low bf16 of w, d1 += its high bf16: each widened exactly and added
// with one fp32 rounding (the same sums as unpacking to fp32 first, in fewer
// instructions).
__device__ __forceinline__ void add_bf16x2_f32(float& d0, float& d1, uint32_t w)
{
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "mov.b32 {lo, hi}, %2;\n\t"
        "add.rn.f32.bf16 %0, lo, %0;\n\t"
        "add.rn.f32.bf16 %1, hi, %1;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "r"(w));
}


__device__ __forceinline__ bool aborted_flag(int* abort) { return *reinterpret_cast<volatile int*>(abort) != 0; }

// Bounded mbarrier wait that also gives up when another role aborted.  The
// slow path is a real call: it is reached from many sites, and inlining it
// everywhere would bloat the instruction footprint of the hot loops.
__device__ __noinline__ bool wait_bar_slow(uint64_t* bar, uint32_t parity, int* abort, int* err)
{
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 1000000u)) return true;
        if (aborted_flag(abort)) return false;
        if (clock64() - t0 > kWaitCycles) {
            atomicCAS(err, 0, (int)kErrWaitTimeout);
            *reinterpret_cast<volatile int*>(abort) = 1;
            return false;
        }
    }
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, int* abort, int* err)
{
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bar_slow(bar, parity, abort, err);
}

// The same wait fully inlined, for the softmax warps: code that runs under a
// raised setmaxnreg budget makes no calls.
__device__ __forceinline__ bool wait_bar_inl(uint64_t* bar, uint32_t parity, int* abort, int* err)
{
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 1000000u)) return true;
        if (aborted_flag(abort)) return false;
        if (clock64() - t0 > kWaitCycles) {
            atomicCAS(err, 0, (int)kErrWaitTimeout);
            *reinterpret_cast<volatile int*>(abort) = 1;
            return false;
        }
    }
}

// Warp-uniform bounded wait: true only if every lane saw the phase complete.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, int* abort, int* err)
{
    const bool ok = wait_bar(bar, parity, abort, err);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ bool wait_warp_inl(uint64_t* bar, uint32_t parity, int* abort, int* err)
{
    const bool ok = wait_bar_inl(bar, parity, abort, err);
    return __all_sync(0xffffffffu, ok);
}

// Short bounded wait used while draining after an abort.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity)
{
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > kWaitCycles / 4) return;
}


// 32x32b TMEM load of 32 consecutive columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32"
        " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
        " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32"
        " [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16,"
        " %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]), "r"(r[32])
        : "memory");
}

__device__ __forceinline__ void st_global_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

// The CTA's tiles are t = blockIdx.x + n * gridDim.x; tile n goes to slot n & 1.
struct TileRef {
    int b, h, i1, i2;  // i2 = -1: a single query cube (rows 64-127 unused)
    int len1, len2;    // the rows' lengths as copied in (entries, or words of a bitmap row)
};

__device__ __forceinline__ TileRef tile_ref(int t, int H, int nq, int tiles_per_bh, const int32_t* plan)
{
    TileRef r;
    r.len1 = r.len2 = 0;
    const int bh = t / tiles_per_bh, p = t - bh * tiles_per_bh;
    r.b = bh / H;
    r.h = bh - r.b * H;
    if (plan != nullptr) {
        r.i1 = __ldg(plan + 2 * (int64_t)t);
        r.i2 = __ldg(plan + 2 * (int64_t)t + 1);
    } else {
        r.i1 = 2 * p;
        r.i2 = 2 * p + 1 < nq ? 2 * p + 1 : -1;
    }
    return r;
}

// ------------------------------------------------------------------ step lists
//
// A tile's keys are the union of its two selection lists, as 16-bit entries
// (cube j in bits 0-12, membership in bits 14-15: 1 = query cube i1, 2 = i2,
// 3 = both), in this order: every entry of list 1 (membership 3 when list 2
// names the same cube), then the entries of list 2 that list 1 does not name.
// A list that names a cube twice disables the sharing (list 1's entries are
// all membership 1 and list 2's all membership 2), which keeps every
// multiplicity.  A cube without valid tokens stays in the list; its half of
// a step is empty.
__device__ __forceinline__ bool test_bit(const uint32_t* bits, int j) { return (bits[j >> 5] >> (j & 31)) & 1u; }

// The valid counts of the nkv KV cubes as bytes in shared memory; a count
// outside [0, 64] latches an error and is kept as 255, which the kernel treats
// as an empty cube.  vbs NULL: every cube full but the last, which holds the
// S_kv - 64 (nkv - 1) tokens left.
__device__ __forceinline__ void vbs_stage(const int32_t* __restrict__ vbs, int nkv, int S_kv, uint8_t* vbs8, int* err)
{
    for (int c = threadIdx.x; c < nkv; c += blockDim.x) {
        const int n = vbs != nullptr ? __ldg(vbs + c) : min(64, S_kv - 64 * c);
        const bool bad = n < 0 || n > 64;
        if (bad) atomicCAS(err, 0, (int)kErrVbs);
        vbs8[c] = (uint8_t)(bad ? 255 : n);
    }
}

// Copy a tile's two rows of the selection into shared memory asynchronously
// (cp.async, one 4-byte word per lane and pass) and set their lengths in t
// (entries, or words of a bitmap row); the build waits for them.  Run one tile
// ahead, so that the copies overlap the previous tile's steps.  A BSR row that
// does not lie within the index array latches an error and is taken as empty;
// one longer than kMaxTopk latches an error and is cut to its first kMaxTopk.
__device__ __forceinline__ void lists_fetch(TileRef& t, const Routes& rt, int H, int nq, int32_t* l1, int32_t* l2,
                                            int* err, uint32_t lane)
{
    for (int s = 0; s < 2; ++s) {
        const int i = s == 0 ? t.i1 : t.i2;
        int len = 0;
        if (i >= 0) {
            const int64_t r = ((int64_t)t.b * H + t.h) * nq + i;
            const int32_t* src;
            if (rt.kind == kRouteBsr) {
                const int a = __ldg(rt.indptr + r), e = __ldg(rt.indptr + r + 1);
                const bool inside = a >= 0 && e >= a && e <= rt.nnz;
                len = inside ? min(e - a, kMaxTopk) : 0;
                if ((!inside || e - a > kMaxTopk) && lane == 0) atomicCAS(err, 0, (int)kErrRoute);
                src = rt.idx + (inside ? a : 0);
            } else if (rt.kind == kRouteMask) {
                len = rt.words;
                src = reinterpret_cast<const int32_t*>(rt.mask + r * rt.words);
            } else if (rt.kind == kRouteAll) {
                len = 0;  // nothing to copy: every KV cube
                src = nullptr;
            } else {
                len = rt.topk;
                src = rt.idx + r * rt.topk;
            }
            int32_t* dst = s == 0 ? l1 : l2;
            for (int e = lane; e < len; e += 32) cp_async4(dst + e, src + e);
        }
        if (s == 0)
            t.len1 = len;
        else
            t.len2 = len;
    }
    cp_async_commit();
}

// Build a tile's membership bitmaps and its entry list from its two selection
// lists (fetched by lists_fetch), by the whole producer warp.  Shared memory is
// busy with the tensor core's operands and the TMA copies while this runs, so
// the work is laid out for few round trips: up to kBuildBatch windows of both
// lists at once, the first batch kept in registers from the bitmap pass to the
// emission.  The entries are written over list 1 (each batch of it is read
// before any entry lands on it: after windows 0 .. w at most 32 (w + 1) entries
// exist, which end within their bytes).  Invalid cube ids latch an error and
// are dropped.  Returns the number of entries (warp-uniform).
constexpr int kBuildBatch = 4;

__device__ int steps_build(const TileRef& t, int nq, int32_t* l1, int32_t* l2, uint32_t* b1, uint32_t* b2,
                           int* err, uint32_t lane)
{
    const int words = (nq + 31) >> 5;
    for (int w = lane; w < words; w += 32) {
        b1[w] = 0u;
        b2[w] = 0u;
    }
    const int len1 = t.len1, len2 = t.len2;
    cp_async_wait_all();
    __syncwarp();
    // bitmaps by shared-memory ORs; a list names a cube twice iff one of its ORs
    // finds the bit already set
    bool dup = false;
    int j0[2][kBuildBatch];  // the first batch (-1: none or invalid)
    for (int base = 0; base < max(len1, len2); base += 32 * kBuildBatch) {
        int j[2][kBuildBatch];
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int u = 0; u < kBuildBatch; ++u) {
                const int e = base + 32 * u + (int)lane;
                j[s][u] = e < (s == 0 ? len1 : len2) ? (s == 0 ? l1 : l2)[e] : -1;
            }
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int u = 0; u < kBuildBatch; ++u) {
                const int e = base + 32 * u + (int)lane;
                if (e >= (s == 0 ? len1 : len2)) continue;
                const int jj = j[s][u];
                if (jj < 0 || jj >= nq) {
                    atomicCAS(err, 0, (int)kErrTopkIdx);
                    (s == 0 ? l1 : l2)[e] = -1;
                    j[s][u] = -1;
                } else {
                    const uint32_t bit = 1u << (jj & 31);
                    dup |= (atomicOr(&(s == 0 ? b1 : b2)[jj >> 5], bit) & bit) != 0u;
                }
            }
        if (base == 0) {
#pragma unroll
            for (int s = 0; s < 2; ++s)
#pragma unroll
                for (int u = 0; u < kBuildBatch; ++u) j0[s][u] = j[s][u];
        }
    }
    __syncwarp();
    const bool share = !__any_sync(0xffffffffu, dup) && len1 > 0 && len2 > 0;
    uint16_t* ent = reinterpret_cast<uint16_t*>(l1);
    const uint32_t lt = (1u << lane) - 1u;  // lanes below this one
    int count = 0;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
        const int len = s == 0 ? len1 : len2;
        const int32_t* lst = s == 0 ? l1 : l2;
        for (int base = 0; base < len; base += 32 * kBuildBatch) {
            bool q[kBuildBatch];
            uint32_t code[kBuildBatch];
#pragma unroll
            for (int u = 0; u < kBuildBatch; ++u) {
                const int e = base + 32 * u + (int)lane;
                const int jj = base == 0 ? j0[s][u] : (e < len ? lst[e] : -1);
                q[u] = jj >= 0;
                uint32_t mem = s == 0 ? 1u : 2u;
                if (q[u] && share) {
                    const bool other = test_bit(s == 0 ? b2 : b1, jj);
                    if (s == 0 && other) mem = 3u;  // both select it: walked with list 1
                    if (s == 1 && other) q[u] = false;
                }
                code[u] = (uint32_t)jj | (mem << 14);
            }
            __syncwarp();  // the batch is read before entries land on list 1
#pragma unroll
            for (int u = 0; u < kBuildBatch; ++u) {
                const uint32_t mask = __ballot_sync(0xffffffffu, q[u]);
                if (q[u]) ent[count + __popc(mask & lt)] = (uint16_t)code[u];
                count += __popc(mask);
            }
        }
    }
    __syncwarp();
    return count;
}

// Inclusive prefix sum of x over the warp's lanes.
__device__ __forceinline__ int warp_incl_sum(int x, uint32_t lane)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if ((int)lane >= o) x += y;
    }
    return x;
}

// The same for bitmap rows (copied in by lists_fetch): the rows become the
// membership bitmaps (bits at cubes >= nq cleared; a row of more than
// kMaxTopk cubes latches an error and keeps its first kMaxTopk), then the
// entries are written over list 1 in the order of steps_build with each
// list in ascending cube order: row 1's cubes (membership 3 where row 2 has
// the cube too), then row 2's others.
__device__ int steps_build_mask(const TileRef& t, int nq, int32_t* l1, int32_t* l2, uint32_t* b1, uint32_t* b2,
                                int* err, uint32_t lane)
{
    const int words = (nq + 31) >> 5;
    const uint32_t last = (nq & 31) ? (1u << (nq & 31)) - 1u : 0xffffffffu;
    cp_async_wait_all();
    __syncwarp();
    for (int s = 0; s < 2; ++s) {
        const int len = s == 0 ? t.len1 : t.len2;
        const uint32_t* src = reinterpret_cast<const uint32_t*>(s == 0 ? l1 : l2);
        uint32_t* dst = s == 0 ? b1 : b2;
        int seen = 0;  // cubes in the words before this pass's
        for (int base = 0; base < words; base += 32) {
            const int w = base + (int)lane;
            uint32_t m = w < len ? src[w] : 0u;
            if (w == words - 1) m &= last;
            const int c = __popc(m);
            const int incl = warp_incl_sum(c, lane);
            const int before = seen + incl - c;
            if (before + c > kMaxTopk) {
                atomicCAS(err, 0, (int)kErrRoute);
                uint32_t keep = 0u;  // the lowest kMaxTopk - before of its cubes
                for (int n = max(0, kMaxTopk - before); n > 0 && m != 0u; --n) {
                    const uint32_t lo = m & (0u - m);
                    keep |= lo;
                    m ^= lo;
                }
                m = keep;
            }
            seen += __shfl_sync(0xffffffffu, incl, 31);
            if (w < words) dst[w] = m;
        }
    }
    __syncwarp();
    uint16_t* ent = reinterpret_cast<uint16_t*>(l1);  // the row of list 1 is in b1 now
    int count = 0;
    for (int s = 0; s < 2; ++s) {
        for (int base = 0; base < words; base += 32) {
            const int w = base + (int)lane;
            uint32_t m = 0u, both = 0u;
            if (w < words) {
                const uint32_t x1 = b1[w], x2 = b2[w];
                m = s == 0 ? x1 : (x2 & ~x1);
                both = s == 0 ? (x1 & x2) : 0u;
            }
            const int c = __popc(m);
            const int incl = warp_incl_sum(c, lane);
            int pos = count + incl - c;
            while (m != 0u) {
                const int bit = __ffs((int)m) - 1;
                const uint32_t mem = s == 1 ? 2u : (((both >> bit) & 1u) ? 3u : 1u);
                ent[pos++] = (uint16_t)((uint32_t)(32 * w + bit) | (mem << 14));
                m &= m - 1u;
            }
            count += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
    __syncwarp();
    return count;
}

// The step list of a tile that attends to every one of the nkv KV cubes (both
// query cubes, cube order).
__device__ int steps_build_all(const TileRef& t, int nkv, int32_t* l1, uint32_t lane)
{
    cp_async_wait_all();
    __syncwarp();
    const uint32_t mem = (t.i1 >= 0 ? 1u : 0u) | (t.i2 >= 0 ? 2u : 0u);
    uint16_t* ent = reinterpret_cast<uint16_t*>(l1);
    for (int j = (int)lane; j < nkv; j += 32) ent[j] = (uint16_t)((uint32_t)j | (mem << 14));
    __syncwarp();
    return nkv;
}

// A tile with an out-of-range plan entry latches an error; the bad cube is dropped.
__device__ __forceinline__ TileRef checked_tile(int t, int H, int nq, int tiles_per_bh, const int32_t* plan, int* err)
{
    TileRef r = tile_ref(t, H, nq, tiles_per_bh, plan);
    if (r.i1 < 0 || r.i1 >= nq) {
        if (err != nullptr) atomicCAS(err, 0, (int)kErrPlan);
        r.i1 = -1;
    }
    if (r.i2 < -1 || r.i2 >= nq) {
        if (err != nullptr) atomicCAS(err, 0, (int)kErrPlan);
        r.i2 = -1;
    }
    return r;
}

// TMA copy of one 64-token cube (both 64-wide d halves) into rows 64*part of a 128-row tile.
__device__ __forceinline__ void load_cube(const CUtensorMap* map, uint64_t* bar, uint8_t* dst, int part, int h,
                                          int tok)
{
    tma_load_3d(map, bar, dst + part * kHalfBox, 0, h, tok);
    tma_load_3d(map, bar, dst + 2 * kHalfBox + part * kHalfBox, 64, h, tok);
}

// The same with an L2 cache policy.
__device__ __forceinline__ void load_cube_keep(const CUtensorMap* map, uint64_t* bar, uint8_t* dst, int part, int h,
                                               int tok, uint64_t policy)
{
    tma_load_3d_hint(map, bar, dst + part * kHalfBox, 0, h, tok, policy);
    tma_load_3d_hint(map, bar, dst + 2 * kHalfBox + part * kHalfBox, 64, h, tok, policy);
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


}  // namespace
}  // namespace vsa
