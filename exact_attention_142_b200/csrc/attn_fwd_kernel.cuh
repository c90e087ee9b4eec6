// attn_fwd_kernel.cuh -- fused exact attention forward for sm_100a.
//
// A CTA computes pairs of 128-row query tiles that read the same key/value
// head, streaming 128-key blocks of K and V through a shared-memory ring.  It
// is persistent: after its own pair it takes over the pairs of CTAs that have
// not started (cluster launch control; see UnitSource).
//
//   warps 0-3  softmax for query tile 0 (one thread per query row)
//   warps 4-7  softmax for query tile 1
//   warp  8    producer: the schedule, TMA loads of Q (once per pair) and of
//              the K/V ring
//   warp  9    MMA issuer: tcgen05 S = Q K^T (both operands in shared memory)
//              and O += P V (P read from tensor memory)
//   (both run converged over all 32 lanes; one elected lane issues)
//   warps 10-11 spare (complete the third warpgroup)
// Registers move from the third warpgroup to the two softmax warpgroups with
// setmaxnreg (the whole score row of a query lives in one thread).
//
// Tensor memory (512 columns, fp32): S0 [0,128), S1 [128,256), O0 [256,384),
// O1 [384,512).  Each softmax thread loads its whole score row, writes the
// bf16 weights P back into the upper half of the same S columns, and the PV
// product reads them from there.
//
// Algorithm ("FlashAttention", ozercemkelahmet.com/tools/flashattention,
// "How it works"): Step 1 tiles along the sequence, Step 2 scores per tile on
// chip, Step 3 online softmax with a running maximum and running sum whose old
// values are rescaled when the maximum grows, Step 4 the output accumulated
// with the same correction and divided by the final sum once, Step 5 the
// per-row log-sum-exp saved, Step 6 whole key blocks outside the causal or
// sliding-window band skipped and the boundary blocks masked element-wise,
// Step 7 the work spread over (query block, batch, head), Step 8 16-bit
// operands with fp32 accumulation and fp32 statistics.
//
// The running maximum is allowed to lag the true maximum by up to 2^8 in the
// exponent (the correction of O is skipped until the growth exceeds that).
// This stays exact: every weight and the sum use the same reference maximum,
// so the final division cancels it.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "attn.h"
#include "exp2_poly.cuh"
#include "ptx.cuh"

namespace attn {

// Device status word (one per device); see attn_device_status().  All kernels
// are compiled in one translation unit, which owns this definition.
__device__ int g_attn_status = 0;

constexpr int kBM = 128;        // query rows per tile
constexpr int kBN = 128;        // keys per block
constexpr int kThreads = 384;   // 8 softmax warps + producer + MMA + 2 spare
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO0 = 256;
constexpr uint32_t kPOffset = 64;      // P columns inside an S region
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kLn2 = 0.693147180559945309f;
constexpr float kLog2e = 1.442695040888963407f;
// Register split after launch (384 threads x 168 = 64512 registers):
// 128 x (216 + 216 + 72) = 64512.
constexpr uint32_t kRegsSoftmax = 216;
// Readers of the unit queue: the MMA warp and the eight softmax warps.
constexpr uint32_t kUnitReaders = 9;
constexpr uint32_t kRegsOther = 72;

// One in kPolyPeriod groups of four weights takes its exponential from the
// FMA-pipe polynomial instead of the MUFU unit (whose rate equals the tensor
// core's at d = 128 and would otherwise be the bottleneck).
constexpr int kPolyPeriod = 8;

// P is handed to the P V product in kPParts parts of 128 / kPParts keys: the
// product of one part overlaps the exponentials of the next.
constexpr int kPParts = 2;

enum : int { kPairHeads = 0, kPairRows = 1 };

// 2^x for a pair of arguments x <= 8 on the FMA/ALU pipes:
// n = rint(x) via the 1.5 * 2^23 rounding constant, f = x - n in [-1/2, 1/2]
// (exact), 2^f by the fitted cubic, times 2^n built in the exponent field.
// Arguments are clamped below at -127, where the bits of 2^n, (n + 127) << 23,
// are all zero: the result is exactly 0 for x < -126.5, and in particular for
// -inf, so a masked key weighs exactly 0 here as it does on the MUFU path.
__device__ __forceinline__ void exp2_poly_pair(float x0, float x1, float& y0, float& y1) {
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
    const uint64_t x = ptx::f2_pack(fmaxf(x0, -127.0f), fmaxf(x1, -127.0f));
    const uint64_t t = ptx::fadd2(x, ptx::f2_pack(kRound, kRound));
    const uint64_t n = ptx::fadd2(t, ptx::f2_pack(-kRound, -kRound));
    const uint64_t f = ptx::ffma2(n, ptx::f2_pack(-1.0f, -1.0f), x);
    uint64_t p = ptx::ffma2(f, ptx::f2_pack(exp2poly::kC3, exp2poly::kC3),
                            ptx::f2_pack(exp2poly::kC2, exp2poly::kC2));
    p = ptx::ffma2(p, f, ptx::f2_pack(exp2poly::kC1, exp2poly::kC1));
    p = ptx::ffma2(p, f, ptx::f2_pack(1.0f, 1.0f));
    float t0, t1;
    ptx::f2_unpack(t, t0, t1);
    // the low bits of t hold n; shifted by 23 they are n in the exponent field,
    // and adding the bits of 1.0f biases it: the bits of 2^n (0 for n = -127)
    const float s0 = __int_as_float((__float_as_int(t0) << 23) + 0x3f800000);
    const float s1 = __int_as_float((__float_as_int(t1) << 23) + 0x3f800000);
    ptx::f2_unpack(ptx::fmul2(p, ptx::f2_pack(s0, s1)), y0, y1);
}

struct FwdParams {
    void* o;
    float* lse;
    const int32_t* cu_seqlens;  // nullptr in dense mode
    int B, Hq, Hkv;
    int N;             // dense: sequence length; packed: total tokens
    int group;         // Hq / Hkv
    int left, right;   // -1 = unlimited; causal is already folded into right = 0
    int pair_mode;     // kPairHeads: heads (2p, 2p+1) of one row block
                       // kPairRows : row blocks (2p, 2p+1) of one head
    int n_row_blocks;  // ceil(max sequence length / 128)
    float scale_log2;  // scale * log2(e)
    float scale;
    unsigned long long wait_limit_ns;
};

template <int D, int STAGES>
struct SmemLayout {
    static constexpr uint32_t kTileBytes = kBM * D * 2;  // one Q, K or V tile (bf16)
    static constexpr uint32_t kBoxBytes = 128 * 128;     // one TMA box: 128 rows x 128 bytes
    static constexpr uint32_t kQ0 = 0;
    static constexpr uint32_t kQ1 = kTileBytes;
    static constexpr uint32_t kKV = 2 * kTileBytes;
    // Output staging: 4 KB per softmax warp (32 rows x 64 bf16 columns).
    static constexpr uint32_t kStg = kKV + STAGES * kTileBytes;
    static constexpr uint32_t kBar = kStg + 8 * 4096;
    // q_full, kv_full[S], kv_empty[S], s_full[2], p_ready[2], o_done[2], mma_final,
    // q_empty, o_free[2], clc, unit_full[2], unit_empty[2], p_part[2][kPParts - 1]
    static constexpr uint32_t kNumBars = 16 + 2 * (kPParts - 1) + 2 * STAGES;
    static constexpr uint32_t kMisc = kBar + kNumBars * 8;  // tmem address, abort flag
    static constexpr uint32_t kClcResp = kMisc + 16;        // launch-control response (16 B)
    static constexpr uint32_t kUnitQ = kClcResp + 16;       // unit queue: two ints
    static constexpr uint32_t kBytes = kUnitQ + 16;
    static constexpr uint32_t kDynamicBytes = kBytes + 1024;  // room to align the base to 1 KB
    static_assert(kClcResp % 16 == 0, "the launch-control response needs 16-byte alignment");

    static __device__ __forceinline__ uint32_t bar_q(uint32_t base) { return base + kBar; }
    static __device__ __forceinline__ uint32_t bar_kv_full(uint32_t base, int s) {
        return base + kBar + 8u * (1 + s);
    }
    static __device__ __forceinline__ uint32_t bar_kv_empty(uint32_t base, int s) {
        return base + kBar + 8u * (1 + STAGES + s);
    }
    static __device__ __forceinline__ uint32_t bar_s_full(uint32_t base, int x) {
        return base + kBar + 8u * (1 + 2 * STAGES + x);
    }
    static __device__ __forceinline__ uint32_t bar_p_ready(uint32_t base, int x) {
        return base + kBar + 8u * (3 + 2 * STAGES + x);
    }
    static __device__ __forceinline__ uint32_t bar_o_done(uint32_t base, int x) {
        return base + kBar + 8u * (5 + 2 * STAGES + x);
    }
    static __device__ __forceinline__ uint32_t bar_mma_final(uint32_t base) {
        return base + kBar + 8u * (7 + 2 * STAGES);
    }
    static __device__ __forceinline__ uint32_t bar_q_empty(uint32_t base) {
        return base + kBar + 8u * (8 + 2 * STAGES);
    }
    static __device__ __forceinline__ uint32_t bar_o_free(uint32_t base, int x) {
        return base + kBar + 8u * (9 + 2 * STAGES + x);
    }
    static __device__ __forceinline__ uint32_t bar_clc(uint32_t base) {
        return base + kBar + 8u * (11 + 2 * STAGES);
    }
    static __device__ __forceinline__ uint32_t bar_unit_full(uint32_t base, int slot) {
        return base + kBar + 8u * (12 + 2 * STAGES + slot);
    }
    static __device__ __forceinline__ uint32_t bar_unit_empty(uint32_t base, int slot) {
        return base + kBar + 8u * (14 + 2 * STAGES + slot);
    }
    static __device__ __forceinline__ uint32_t bar_p_part(uint32_t base, int x, int k) {
        return base + kBar + 8u * (16 + 2 * STAGES + (kPParts - 1) * x + k);
    }
};


// Wait for an mbarrier phase with a time limit.  On expiry the block-wide
// abort flag is raised and the device status word records the timeout; once
// the flag is up every other bounded wait of the block returns at once.
__device__ __forceinline__ bool bounded_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             unsigned long long limit_ns) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::global_timer_ns();
    while (true) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (ptx::global_timer_ns() - t0 > limit_ns) {
            *abort_flag = 1;
            atomicCAS(&g_attn_status, 0, ATTN_ERR_DEVICE_TIMEOUT);
            return false;
        }
    }
}

// Teardown wait for work already in flight (TMA copies, MMAs): ignores the
// abort flag but is still bounded.
__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity,
                                           unsigned long long limit_ns) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::global_timer_ns();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::global_timer_ns() - t0 > limit_ns) {
            atomicCAS(&g_attn_status, 0, ATTN_ERR_DEVICE_TIMEOUT);
            return false;
        }
    }
    return true;
}

// bounded_wait by every lane of a warp, with a warp-uniform outcome.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long limit_ns) {
    return __all_sync(0xffffffffu, bounded_wait(bar, parity, abort_flag, limit_ns));
}

// Entry n of the CTA's unit queue (filled by the producer warp): the next tile
// pair with rows to compute, or -1 once the grid's work is exhausted (or the
// block aborted).  Called by a whole warp; lane 0 releases the slot.
// Only n mod 4 matters (slot and phase).
template <class L>
__device__ __forceinline__ int unit_take(uint32_t sbase, uint32_t n, volatile int* abort_flag,
                                         unsigned long long limit_ns) {
    const int slot = n & 1;
    if (!warp_wait(L::bar_unit_full(sbase, slot), (n >> 1) & 1, abort_flag, limit_ns)) return -1;
    const int u = ptx::ld_volatile_smem(sbase + L::kUnitQ + 4 * slot);
    __syncwarp();
    if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(L::bar_unit_empty(sbase, slot));
    return u;
}

// The two query tiles of one CTA and the key blocks each of them needs.
struct TilePair {
    int b, start, len, g;
    int h[2];
    int r0[2];
    int lo[2], hi[2];  // key-block range [lo, hi); empty when the tile is inactive
    bool active[2];
    bool bad;          // packed boundaries inconsistent with the launch (pair skipped)
    int ulo, uhi;      // union of the two ranges
};

__device__ __forceinline__ TilePair decode_pair(int u, const FwdParams& p) {
    TilePair w;
    int t[2];
    if (p.pair_mode == kPairHeads) {
        const int hp_count = p.Hq / 2;
        const int per_t = p.B * hp_count;
        const int tb = p.n_row_blocks - 1 - u / per_t;  // heaviest (latest) rows first
        const int rem = u % per_t;
        w.b = rem / hp_count;
        const int hp = rem % hp_count;
        w.h[0] = 2 * hp;
        w.h[1] = 2 * hp + 1;
        t[0] = t[1] = tb;
    } else {
        const int np = (p.n_row_blocks + 1) / 2;
        const int per_t = p.B * p.Hq;
        const int tp = np - 1 - u / per_t;
        const int rem = u % per_t;
        w.b = rem / p.Hq;
        w.h[0] = w.h[1] = rem % p.Hq;
        t[0] = 2 * tp;
        t[1] = 2 * tp + 1;
    }
    w.bad = false;
    if (p.cu_seqlens) {
        // The boundaries must lie inside [0, N], must not decrease, and the
        // sequence must fit the row blocks the launch was sized for
        // (max_seqlen).  Otherwise the pair has no rows: nothing of it is read
        // or written, and the producer reports the inconsistency.
        const int s0 = p.cu_seqlens[w.b];
        const int s1 = p.cu_seqlens[w.b + 1];
        w.bad = s0 < 0 || s1 < s0 || s1 > p.N || (long long)(s1 - s0) > (long long)p.n_row_blocks * kBM;
        w.start = w.bad ? 0 : s0;
        w.len = w.bad ? 0 : s1 - s0;
    } else {
        w.start = w.b * p.N;
        w.len = p.N;
    }
    w.g = w.h[0] / p.group;
    w.ulo = 0x7fffffff;
    w.uhi = 0;
    for (int x = 0; x < 2; ++x) {
        w.r0[x] = t[x] * kBM;
        w.active[x] = w.r0[x] < w.len;
        if (w.active[x]) {
            const long long kv_lo = p.left >= 0 ? (long long)w.r0[x] - p.left : 0;
            const long long kv_hi =
                p.right >= 0 ? (long long)w.r0[x] + kBM + p.right : (long long)w.len;
            const long long lo_c = kv_lo < 0 ? 0 : kv_lo;
            const long long hi_c = kv_hi > w.len ? w.len : kv_hi;
            w.lo[x] = (int)(lo_c / kBN);
            w.hi[x] = (int)((hi_c + kBN - 1) / kBN);
            if (w.lo[x] < w.ulo) w.ulo = w.lo[x];
            if (w.hi[x] > w.uhi) w.uhi = w.hi[x];
        } else {
            w.lo[x] = w.hi[x] = 0;
        }
    }
    if (w.uhi <= w.ulo) w.ulo = w.uhi = 0;
    return w;
}

__device__ __forceinline__ bool tile_active_at(const TilePair& w, int x, int j) {
    return w.active[x] && j >= w.lo[x] && j < w.hi[x];
}

// ---------------------------------------------------------------- schedule
// Persistent, varlen-aware schedule.  The grid holds one CTA per tile pair in
// heaviest-first order.  A running CTA starts with its own pair; when the
// producer has issued every load of a pair it takes the next pending pair by
// cancelling the launch of a CTA that has not started (cluster launch
// control), skipping pairs with no rows (packed sequences shorter than the
// longest, and sequences whose boundaries do not fit the launch, which it
// reports in the status word), and passes it to the MMA and softmax warps through a two-entry
// queue in shared memory.  Pairs are thus handed out greedily in the same
// order as by the hardware's block scheduler, while the next pair's Q load
// and first products overlap the previous pair's epilogue.
//
// UnitSource is the producer warp's side.  L provides bar_clc, kClcResp,
// kUnitQ, bar_unit_full and bar_unit_empty.
template <class L>
struct UnitSource {
    uint32_t sbase;
    int cand;          // next pair to examine (-1: ask the hardware)
    int requests;      // launch-control requests answered
    int published;     // unit queue entries written
    bool pending;      // a request whose answer has not been seen
    bool more;         // false after a request that cancelled nothing

    __device__ __forceinline__ explicit UnitSource(uint32_t base)
        : sbase(base), cand(blockIdx.x), requests(0), published(0), pending(false), more(true) {}

    // The next pair with rows, or -1 (the grid is exhausted, or a wait timed
    // out: then ok is cleared).  Called by the whole warp.
    __device__ __forceinline__ int next(const FwdParams& p, volatile int* abort_flag, bool& ok) {
        const uint32_t resp = sbase + L::kClcResp;
        while (true) {
            if (cand >= 0) {
                const TilePair w = decode_pair(cand, p);
                const int u = cand;
                cand = -1;
                if (w.bad && (threadIdx.x & 31) == 0) atomicCAS(&g_attn_status, 0, ATTN_ERR_SEQLENS);
                if (w.active[0] || w.active[1]) return u;
            }
            if (!more) return -1;
            ptx::fence_proxy_async_smem();  // the last response was read before it is rewritten
            __syncwarp();
            ptx::clc_try_cancel_elect(resp, L::bar_clc(sbase));
            pending = true;
            if (!warp_wait(L::bar_clc(sbase), requests & 1, abort_flag, p.wait_limit_ns)) {
                ok = false;
                return -1;
            }
            pending = false;
            ++requests;
            cand = ptx::clc_query_x(resp);
            if (cand < 0) more = false;
        }
    }

    // Hands pair u (or -1: no more work) to the MMA and softmax warps.
    __device__ __forceinline__ bool publish(int u, volatile int* abort_flag, unsigned long long lim) {
        const int slot = published & 1;
        if (!warp_wait(L::bar_unit_empty(sbase, slot), ((published >> 1) & 1) ^ 1, abort_flag, lim))
            return false;
        if ((threadIdx.x & 31) == 0) ptx::st_volatile_smem(sbase + L::kUnitQ + 4 * slot, u);
        __syncwarp();
        if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(L::bar_unit_full(sbase, slot));
        ++published;
        return true;
    }

    // A request still in flight must land before the block exits.
    __device__ __forceinline__ void drain(unsigned long long lim) {
        if (pending) drain_wait(L::bar_clc(sbase), requests & 1, lim);
    }
};

// Initialises the schedule's barriers (one thread).
template <class L>
__device__ __forceinline__ void init_schedule_barriers(uint32_t sbase) {
    ptx::mbar_init(L::bar_q_empty(sbase), 1);
    for (int x = 0; x < 2; ++x) ptx::mbar_init(L::bar_o_free(sbase, x), 128);
    ptx::mbar_init(L::bar_clc(sbase), 1);
    for (int x = 0; x < 2; ++x)
        for (int k = 0; k < kPParts - 1; ++k) ptx::mbar_init(L::bar_p_part(sbase, x, k), 128);
    for (int slot = 0; slot < 2; ++slot) {
        ptx::mbar_init(L::bar_unit_full(sbase, slot), 1);
        ptx::mbar_init(L::bar_unit_empty(sbase, slot), kUnitReaders);
    }
}

// ---------------------------------------------------------------- producer
template <int D, int STAGES>
__device__ __forceinline__ void producer_role(const FwdParams& p, const CUtensorMap* tm_q,
                                              const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                              uint32_t sbase, volatile int* abort_flag) {
    using L = SmemLayout<D, STAGES>;
    constexpr int kBoxes = D / 64;
    const unsigned long long lim = p.wait_limit_ns;
    const uint64_t pol_q = ptx::policy_evict_first();
    const uint64_t pol_kv = ptx::policy_evict_last();
    UnitSource<L> src(sbase);
    int issued = 0;  // K/V ring loads
    int units = 0;   // pairs whose Q was loaded
    bool ok = true;
    int u = src.next(p, abort_flag, ok);
    while (ok) {
        if (!(ok = src.publish(u, abort_flag, lim)) || u < 0) break;
        const TilePair w = decode_pair(u, p);
        // the previous pair's score products have finished reading Q
        if (units > 0 && !(ok = warp_wait(L::bar_q_empty(sbase), (units - 1) & 1, abort_flag, lim))) break;
        ptx::mbar_arrive_expect_tx_elect(L::bar_q(sbase), 2 * L::kTileBytes);
        for (int x = 0; x < 2; ++x) {
#pragma unroll
            for (int bx = 0; bx < kBoxes; ++bx)
                ptx::tma_load_2d_elect(sbase + (x ? L::kQ1 : L::kQ0) + bx * L::kBoxBytes, tm_q, L::bar_q(sbase),
                                       w.h[x] * D + bx * 64, w.start + w.r0[x], pol_q);
        }
        ++units;
        for (int j = w.ulo; j < w.uhi && ok; ++j) {
            for (int kv = 0; kv < 2; ++kv) {
                const int s = issued % STAGES;
                const uint32_t ph = (issued / STAGES) & 1;
                if (!(ok = warp_wait(L::bar_kv_empty(sbase, s), ph ^ 1, abort_flag, lim))) break;
                ptx::mbar_arrive_expect_tx_elect(L::bar_kv_full(sbase, s), L::kTileBytes);
#pragma unroll
                for (int bx = 0; bx < kBoxes; ++bx)
                    ptx::tma_load_2d_elect(sbase + L::kKV + s * L::kTileBytes + bx * L::kBoxBytes, kv ? tm_v : tm_k,
                                           L::bar_kv_full(sbase, s), w.g * D + bx * 64, w.start + j * kBN, pol_kv);
                ++issued;
            }
        }
        if (ok) u = src.next(p, abort_flag, ok);
    }
    // Every copy and request issued must have landed before the block may exit.
    src.drain(lim);
    if (units > 0) drain_wait(L::bar_q(sbase), (units - 1) & 1, lim);
    const int first = issued > STAGES ? issued - STAGES : 0;
    for (int i = first; i < issued; ++i) drain_wait(L::bar_kv_full(sbase, i % STAGES), (i / STAGES) & 1, lim);
}

// ---------------------------------------------------------------- O stores
// Writes one softmax warp's 32 rows of O (d fp32 columns of tensor memory at
// t_o, this thread's row in its lane, times inv, rounded to bf16) to
// o[start + row][h][:].  They pass through the warp's 4 KB staging area (stg,
// 1 KB aligned), 64 columns at a time: each thread writes its row's 128 bytes
// there with the 16-byte chunks rotated by the row (chunk c of row r at
// c ^ (r mod 8): conflict-free, and the 128-byte swizzle of a TMA box).  When
// all 32 rows lie inside the sequence, one lane stores the staging area as a
// 32 x 64 box through tm_o (the copy engine writes O; no load/store-unit
// traffic) and waits until the copy has read it before the next 64 columns
// are staged.  Otherwise (a warp that reaches past a packed sequence's end, or
// no map) each of the warp's eight store instructions writes four whole
// 128-byte row segments, and rows at or past len are skipped.
template <int D>
__device__ __forceinline__ void store_o_rows(const FwdParams& p, uint32_t stg, int lane, uint32_t t_o, float inv,
                                             int rbase, int len, int start, int h, const CUtensorMap* tm_o) {
    const bool box = tm_o != nullptr && rbase + 32 <= len;
#pragma unroll
    for (int hf = 0; hf < D / 64; ++hf) {
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            uint32_t o[32];
            ptx::tmem_ld32_sync(t_o + hf * 64 + cc * 32, o);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int ch = cc * 4 + c;
                ptx::st_shared_v4(stg + lane * 128 + ((ch ^ (lane & 7)) << 4),
                                  ptx::pack_bf16x2(__uint_as_float(o[8 * c + 0]) * inv, __uint_as_float(o[8 * c + 1]) * inv),
                                  ptx::pack_bf16x2(__uint_as_float(o[8 * c + 2]) * inv, __uint_as_float(o[8 * c + 3]) * inv),
                                  ptx::pack_bf16x2(__uint_as_float(o[8 * c + 4]) * inv, __uint_as_float(o[8 * c + 5]) * inv),
                                  ptx::pack_bf16x2(__uint_as_float(o[8 * c + 6]) * inv, __uint_as_float(o[8 * c + 7]) * inv));
            }
        }
        if (box) {
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                ptx::tma_store_2d(tm_o, stg, h * D + hf * 64, start + rbase);
                ptx::bulk_commit_group();
                ptx::bulk_wait_group_read0();
            }
            __syncwarp();
            continue;
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = 4 * i + (lane >> 3);
            const int ch = lane & 7;
            uint32_t a, b, c, d;
            ptx::ld_shared_v4(stg + r * 128 + ((ch ^ (r & 7)) << 4), a, b, c, d);
            if (rbase + r < len) {
                uint8_t* dst = reinterpret_cast<uint8_t*>(p.o) +
                               ((size_t)(start + rbase + r) * p.Hq + h) * (size_t)D * 2 + hf * 128 + ch * 16;
                ptx::st_global_v4(dst, a, b, c, d);
            }
        }
        __syncwarp();  // the staging area is rewritten for the next 64 columns
    }
}

// ---------------------------------------------------------------- MMA issuer
template <int D, int STAGES>
__device__ __forceinline__ void issue_qk(uint32_t tmem, uint32_t sbase, int x, int slot) {
    using L = SmemLayout<D, STAGES>;
    constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(kBM, kBN, false, false);
    const uint32_t qa = sbase + (x ? L::kQ1 : L::kQ0);
    const uint32_t ka = sbase + L::kKV + slot * L::kTileBytes;
    const uint32_t d_tmem = tmem + (x ? 128u : 0u);
    // K-major, 128-byte swizzle: 16 elements (32 bytes) per step inside a
    // 64-element box, the next box 16 KB further.  A step's descriptor is the
    // tile's plus the byte offset / 16 (the 14-bit start-address field cannot
    // carry: shared addresses stay below 256 KB).  All steps go out from one
    // elected lane.
    static_assert(L::kBoxBytes == 16384, "the step offsets assume 16 KB boxes");
    const uint64_t qd = ptx::smem_desc_sw128(qa, 16, 1024);
    const uint64_t kd = ptx::smem_desc_sw128(ka, 16, 1024);
    if constexpr (D == 128)
        ptx::mma_ss_kmajor8_elect(d_tmem, qd, kd, kIdesc, 0u);
    else
        ptx::mma_ss_kmajor4_elect(d_tmem, qd, kd, kIdesc, 0u);
}

// Keys [128 part / kPParts, 128 (part + 1) / kPParts) of the block.
template <int D, int STAGES>
__device__ __forceinline__ void issue_pv(uint32_t tmem, uint32_t sbase, int x, int slot, int part,
                                         bool accumulate) {
    using L = SmemLayout<D, STAGES>;
    // B = V is [keys, d] with d contiguous: MN-major operand.  Swizzle atoms of
    // 8 keys x 64 values are 1 KB apart along the keys (SBO) and the second
    // 64-value half of d sits one 16 KB box further (LBO).
    constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(kBM, D, false, true);
    const uint32_t va = sbase + L::kKV + slot * L::kTileBytes;
    const uint32_t p_tmem = tmem + (x ? 128u : 0u) + kPOffset;
    const uint32_t d_tmem = tmem + kTmemO0 + (x ? 128u : 0u);
    constexpr int kSteps = kBN / 16 / kPParts;  // K = 16 keys per instruction
    static_assert(kSteps == 4, "one four-step group per part");
    // Step kk reads P columns +8 kk and the V rows 16 kk.. (2 KB further each).
    const int kk0 = part * kSteps;
    ptx::mma_ts_mnmajor4_elect(d_tmem, p_tmem + kk0 * 8,
                               ptx::smem_desc_sw128(va, L::kBoxBytes, 1024) + ((kk0 * 2048) >> 4), kIdesc,
                               accumulate ? 1u : 0u);
}

// The MMA warp's loop over the pairs of its CTA.  qk(x, slot) issues the score
// product of tile x from ring slot `slot`; issue(x, slot, part, accumulate) the
// P V product of key part `part`.  Shared by the bf16 and the e4m3 kernels.
template <class L, int STAGES, class IssueQK, class IssuePV>
__device__ __forceinline__ void mma_loop(const FwdParams& p, uint32_t sbase, volatile int* abort_flag,
                                         IssueQK&& qk, IssuePV&& issue) {
    const unsigned long long lim = p.wait_limit_ns;
    // Phase bits, kept in one word (this warp runs with few registers):
    enum : uint32_t {
        kPc = 1u,          // << x: parity of the P hand-offs consumed for tile x
        kPending = 4u,     // << x: O of tile x handed to an epilogue not yet released
        kFreed = 16u,      // << x: parity of the o_free phases consumed for tile x
        kFirst = 64u,      // << x: the next PV of tile x starts a fresh accumulator
        kQ = 256u,         // parity of the Q loads consumed
        kUnitShift = 9u,   // bits 9-10: unit queue index mod 4
    };
    static_assert(kPParts == 2, "the P V product is handed over in two parts");
    uint32_t f = 0;
    // Ring position of the next key tile (slot and barrier phase), advanced
    // one slot at a time: no division on this warp's path.
    int ks = 0;
    uint32_t kph = 0;
    auto adv = [](int& slot, uint32_t& ph) {
        if (++slot == STAGES) {
            slot = 0;
            ph ^= 1u;
        }
    };
    bool ok = true;
    // P V of tile x in two parts: each waits for the softmax's hand-off of its
    // half of the weights (p_part, then p_ready); before the first P V of a
    // pair the first part also waits for the previous pair's epilogue to have
    // read O (o_free).  Every hand-off barrier completes once per key block.
    // `after_first` runs between the two parts (commits that may block on a
    // full tensor-core queue go there, behind products already queued).
    auto pv = [&](int x, int slot, bool last, auto&& after_first) -> bool {
        if (!warp_wait(L::bar_p_part(sbase, x, 0), (f >> x) & 1u, abort_flag, lim)) return false;
        if ((f & (kFirst << x)) && (f & (kPending << x))) {
            if (!warp_wait(L::bar_o_free(sbase, x), (f >> (4 + x)) & 1u, abort_flag, lim)) return false;
            f ^= (kFreed << x) | (kPending << x);
        }
        ptx::tc_fence_after_sync();
        issue(x, slot, 0, !(f & (kFirst << x)));
        after_first();
        if (!warp_wait(L::bar_p_ready(sbase, x), (f >> x) & 1u, abort_flag, lim)) return false;
        ptx::tc_fence_after_sync();
        issue(x, slot, 1, true);
        f &= ~(kFirst << x);
        f ^= kPc << x;
        if (last) {
            ptx::tc_commit_elect(L::bar_o_done(sbase, x));
            f |= kPending << x;
        }
        return true;
    };
    auto nothing = [] {};
    // Two ring tiles awaited together: both probes, one vote; the bounded wait
    // only when one of them is not there yet.
    auto kv_wait2 = [&](int s0, uint32_t ph0, int s1, uint32_t ph1) -> bool {
        const bool a = ptx::mbar_try_wait(L::bar_kv_full(sbase, s0), ph0);
        const bool b = ptx::mbar_try_wait(L::bar_kv_full(sbase, s1), ph1);
        if (__all_sync(0xffffffffu, a && b)) {
            ptx::tc_fence_after_sync();
            return true;
        }
        const bool r = warp_wait(L::bar_kv_full(sbase, s0), ph0, abort_flag, lim) &&
                       warp_wait(L::bar_kv_full(sbase, s1), ph1, abort_flag, lim);
        ptx::tc_fence_after_sync();
        return r;
    };
    while (ok) {
        const int u = unit_take<L>(sbase, (f >> kUnitShift) & 3u, abort_flag, lim);
        f = (f & ~(3u << kUnitShift)) | ((((f >> kUnitShift) + 1u) & 3u) << kUnitShift);
        if (u < 0) break;
        const TilePair w = decode_pair(u, p);
        const int lo0 = w.lo[0], hi0 = w.hi[0], lo1 = w.lo[1], hi1 = w.hi[1];  // empty when inactive
        if (!(ok = warp_wait(L::bar_q(sbase), (f & kQ) ? 1u : 0u, abort_flag, lim))) break;
        f ^= kQ;
        f |= kFirst | (kFirst << 1);
        ptx::tc_fence_after_sync();
        if (w.uhi <= w.ulo) {
            ptx::tc_commit_elect(L::bar_q_empty(sbase));  // no products: Q is free
            continue;
        }
        // Issue order per key block j:  PV1(j-1), S1(j), PV0(j), S0(j+1), with
        // S0 of the pair's first block before the loop.  Each softmax group
        // then has the two products of the other tile to hide its
        // exponentials behind, and each tile's P V product is followed at once
        // by its next score product.  This warp's waits and commits sit where
        // a score product (512 tensor cycles) has just been queued: the value
        // tile of block j and the key tile of block j+1 are awaited together
        // after S1(j), and the key tile's release goes out behind PV0(j).  S_x(j) overwrites the P_x(j-1) columns only after
        // PV_x(j-1) was issued; tcgen05 MMAs from one thread execute in order.
        if (!(ok = warp_wait(L::bar_kv_full(sbase, ks), kph, abort_flag, lim))) break;
        ptx::tc_fence_after_sync();
        if (w.ulo >= lo0 && w.ulo < hi0) {
            qk(0, ks);
            ptx::tc_commit_elect(L::bar_s_full(sbase, 0));
        }
        int pvs = 0;  // ring slot of the previous block's value tile
        for (int j = w.ulo; j < w.uhi; ++j) {
            int vs = ks;
            uint32_t vph = kph;
            adv(vs, vph);
            int nks = vs;
            uint32_t nph = vph;
            adv(nks, nph);
            const bool more = j + 1 < w.uhi;
            if (j > w.ulo) {
                if (j - 1 >= lo1 && j - 1 < hi1 && !(ok = pv(1, pvs, j - 1 == hi1 - 1, nothing))) break;
                ptx::tc_commit_elect(L::bar_kv_empty(sbase, pvs));
            }
            if (j >= lo1 && j < hi1) {
                qk(1, ks);
                ptx::tc_commit_elect(L::bar_s_full(sbase, 1));
            }
            // value tile j and key tile j+1 (loaded well ahead): one wait for both,
            // while the score product just issued keeps the tensor pipe busy
            if (!(ok = kv_wait2(vs, vph, more ? nks : vs, more ? nph : vph))) break;
            // the key tile of block j is free once both score products are out
            const int kslot = ks;
            auto release_k = [&] {
                ptx::tc_commit_elect(L::bar_kv_empty(sbase, kslot));
                if (j == w.uhi - 1) ptx::tc_commit_elect(L::bar_q_empty(sbase));  // last score products issued
            };
            if (j >= lo0 && j < hi0) {
                if (!(ok = pv(0, vs, j == hi0 - 1, release_k))) break;
            } else {
                release_k();
            }
            if (more && j + 1 >= lo0 && j + 1 < hi0) {
                qk(0, nks);
                ptx::tc_commit_elect(L::bar_s_full(sbase, 0));
            }
            pvs = vs;
            ks = nks;
            kph = nph;
        }
        if (!ok) break;
        const int j = w.uhi - 1;
        if (j >= lo1 && j < hi1 && !(ok = pv(1, pvs, true, nothing))) break;
        ptx::tc_commit_elect(L::bar_kv_empty(sbase, pvs));
    }
    // All MMAs must be complete before tensor memory is released.
    ptx::tc_commit_elect(L::bar_mma_final(sbase));
    drain_wait(L::bar_mma_final(sbase), 0, lim);
}

template <int D, int STAGES>
__device__ __forceinline__ void mma_role(const FwdParams& p, uint32_t tmem, uint32_t sbase,
                                         volatile int* abort_flag) {
    mma_loop<SmemLayout<D, STAGES>, STAGES>(
        p, sbase, abort_flag, [&](int x, int slot) { issue_qk<D, STAGES>(tmem, sbase, x, slot); },
        [&](int x, int slot, int part, bool acc) { issue_pv<D, STAGES>(tmem, sbase, x, slot, part, acc); });
}

// ---------------------------------------------------------------- softmax
// ACC = false: O (bf16) and LSE are written.  ACC = true: this call's result is
// merged into an fp32 accumulator (o as float [tokens, Hq, d], lse holding the
// accumulator's log-sum-exp) by the online-softmax rule (Step 3 applied to two
// partial results; "Long context beyond a single GPU").
template <int D, int STAGES, bool ACC>
__device__ __forceinline__ bool softmax_unit(const TilePair& w, const FwdParams& p, int x,
                                             int warp_in_group, int lane, uint32_t tmem,
                                             uint32_t sbase, volatile int* abort_flag, uint32_t& phases, int u,
                                             const CUtensorMap* tm_o) {
    using L = SmemLayout<D, STAGES>;
    const int r0 = x ? w.r0[1] : w.r0[0];
    const int blk_lo = x ? w.lo[1] : w.lo[0];
    const int blk_hi = x ? w.hi[1] : w.hi[0];
    const unsigned long long lim = p.wait_limit_ns;
    const int row = r0 + warp_in_group * 32 + lane;  // row within the sequence
    const uint32_t lane_off = static_cast<uint32_t>(warp_in_group * 32) << 16;
    const uint32_t t_s = tmem + lane_off + (x ? 128u : 0u);
    const uint32_t t_p = t_s + kPOffset;
    const uint32_t t_o = tmem + lane_off + kTmemO0 + (x ? 128u : 0u);
    const float sl2 = p.scale_log2;

    // Visible keys of this row: [key_lo, key_hi] (inclusive), inside the sequence.
    const int key_lo = p.left >= 0 ? (row - p.left > 0 ? row - p.left : 0) : 0;
    long long khi = p.right >= 0 ? (long long)row + p.right : (long long)w.len - 1;
    if (khi > (long long)w.len - 1) khi = (long long)w.len - 1;
    const int key_hi = (int)khi;
    // A block needs no element mask when every (row, key) pair of the tile is visible.
    const int tile_last_row = r0 + kBM - 1;

    float m_ref = -INFINITY;  // reference maximum, log2 units (score * scale * log2 e)
    float l_sum = 0.0f;       // running sum of the fp32 weights 2^(x - m_ref)  -> LSE
    float l_bf = 0.0f;        // running sum of the same weights rounded to bf16 -> O
    bool ok = true;

    for (int j = blk_lo; j < blk_hi; ++j) {
        ok = __all_sync(0xffffffffu, bounded_wait(L::bar_s_full(sbase, x), phases & 1u, abort_flag, lim));
        if (!ok) break;
        phases ^= 1u;
        ptx::tc_fence_after_sync();
        uint32_t s[128];
        ptx::tmem_ld128_sync(t_s, s);

        const int k0 = j * kBN;
        const bool full_block =
            (k0 + kBN <= w.len) && (p.left < 0 || (long long)k0 >= (long long)tile_last_row - p.left) &&
            (p.right < 0 || (long long)k0 + kBN - 1 <= (long long)r0 + p.right);
        if (!full_block) {
            const int c_lo = key_lo - k0, c_hi = key_hi - k0;
#pragma unroll
            for (int c = 0; c < 128; ++c)
                if (c < c_lo || c > c_hi) s[c] = __float_as_uint(-INFINITY);
        }
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
            mx0 = ptx::fmax3(mx0, __uint_as_float(s[c + 0]), __uint_as_float(s[c + 1]));
            mx1 = ptx::fmax3(mx1, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
            mx2 = ptx::fmax3(mx2, __uint_as_float(s[c + 4]), __uint_as_float(s[c + 5]));
            mx3 = ptx::fmax3(mx3, __uint_as_float(s[c + 6]), __uint_as_float(s[c + 7]));
        }
        const float m_blk = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;

        // Online softmax (Step 3): move the reference maximum only when the
        // block's maximum exceeds it by more than the threshold.
        float alpha = 1.0f;
        bool rescale_o = false;
        if (m_blk > m_ref + kRescaleThreshold) {
            alpha = ptx::ex2_approx(m_ref - m_blk);
            rescale_o = (m_ref != -INFINITY);
            l_sum *= alpha;
            l_bf *= alpha;
            m_ref = m_blk;
        }
        // Step 4: the partial output takes the same correction.  The previous
        // PV product of this tile is complete: it was issued before this S.
        if (__any_sync(0xffffffffu, rescale_o)) {
            const float a = rescale_o ? alpha : 1.0f;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                ptx::tmem_ld32_sync(t_o + cc * 32, o);
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * a);
                ptx::tmem_st32(t_o + cc * 32, o);
            }
        }

        const float neg_m = (m_ref == -INFINITY) ? 0.0f : -m_ref;
        const uint64_t sl2_2 = ptx::f2_pack(sl2, sl2);
        const uint64_t negm_2 = ptx::f2_pack(neg_m, neg_m);
        // The PV product multiplies the bf16-rounded weights, so O is divided by
        // the sum of exactly those (a normalised convex combination of V); the
        // LSE uses the sum of the unrounded fp32 weights.
        uint64_t sum_a = 0, sum_b = 0;  // fp32 weights, packed pairs
        float rb0 = 0.f, rb1 = 0.f, rb2 = 0.f, rb3 = 0.f;  // bf16-rounded weights
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
                const int c = q * 32 + 2 * i;
                float x0, x1, x2, x3;
                ptx::f2_unpack(ptx::ffma2(ptx::f2_pack(__uint_as_float(s[c + 0]), __uint_as_float(s[c + 1])),
                                          sl2_2, negm_2), x0, x1);
                ptx::f2_unpack(ptx::ffma2(ptx::f2_pack(__uint_as_float(s[c + 2]), __uint_as_float(s[c + 3])),
                                          sl2_2, negm_2), x2, x3);
                float p0, p1, p2, p3;
                if ((i / 2) % kPolyPeriod == kPolyPeriod - 1) {
                    exp2_poly_pair(x0, x1, p0, p1);
                    exp2_poly_pair(x2, x3, p2, p3);
                } else {
                    p0 = ptx::ex2_approx(x0);
                    p1 = ptx::ex2_approx(x1);
                    p2 = ptx::ex2_approx(x2);
                    p3 = ptx::ex2_approx(x3);
                }
                sum_a = ptx::fadd2(sum_a, ptx::f2_pack(p0, p1));
                sum_b = ptx::fadd2(sum_b, ptx::f2_pack(p2, p3));
                pk[i] = ptx::pack_bf16x2(p0, p1);
                pk[i + 1] = ptx::pack_bf16x2(p2, p3);
                if ((i / 2) % 2 == 0) {
                    rb0 = ptx::add_bf16x2_to_f32(rb0, pk[i]);
                    rb1 = ptx::add_bf16x2_to_f32(rb1, pk[i + 1]);
                } else {
                    rb2 = ptx::add_bf16x2_to_f32(rb2, pk[i]);
                    rb3 = ptx::add_bf16x2_to_f32(rb3, pk[i + 1]);
                }
            }
            ptx::tmem_st16(t_p + q * 16, pk);
            if ((q + 1) % (4 / kPParts) == 0 && q < 3) {  // a part of P is complete
                ptx::tmem_wait_st();
                ptx::tc_fence_before_sync();
                ptx::mbar_arrive(L::bar_p_part(sbase, x, q / (4 / kPParts)));
            }
        }
        {
            float a0, a1, b0, b1;
            ptx::f2_unpack(sum_a, a0, a1);
            ptx::f2_unpack(sum_b, b0, b1);
            l_sum += (a0 + a1) + (b0 + b1);
            l_bf += (rb0 + rb1) + (rb2 + rb3);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before_sync();
        ptx::mbar_arrive(L::bar_p_ready(sbase, x));
    }

    if (!ok) return false;
    // Epilogue (Step 4 and 5): wait for the last PV product, divide once by the
    // sum, round to bf16, and store O and the log-sum-exp.
    ok = __all_sync(0xffffffffu, bounded_wait(L::bar_o_done(sbase, x), (phases >> 1) & 1u, abort_flag, lim));
    if (!ok) return false;
    ptx::tc_fence_after_sync();
    // The pair's indices again (recomputed rather than kept live through the loop).
    int u_again = u;
    asm volatile("" : "+r"(u_again));
    const TilePair we = decode_pair(u_again, p);
    const int h = x ? we.h[1] : we.h[0];
    const bool store = row < we.len;
    if constexpr (ACC) {
        const size_t idx = p.cu_seqlens ? (size_t)h * p.N + we.start + (store ? row : 0)
                                        : ((size_t)we.b * p.Hq + h) * p.N + (store ? row : 0);
        // both log-sum-exps in log2 units; weights relative to the larger one
        const float lse_new = l_sum > 0.0f ? m_ref + ptx::lg2_approx(l_sum) : -INFINITY;
        const float lse_old = store ? p.lse[idx] * kLog2e : -INFINITY;
        const bool has_old = lse_old != -INFINITY;  // an empty row's o_acc is not read
        const float mx = fmaxf(lse_old, lse_new);
        const float mu = mx == -INFINITY ? 0.0f : mx;
        const float w_old = ptx::ex2_approx(lse_old - mu);
        const float w_new = ptx::ex2_approx(lse_new - mu);
        const float den = w_old + w_new;
        const float inv_den = den > 0.0f ? 1.0f / den : 0.0f;
        const float a_old = w_old * inv_den;
        const float a_new = l_bf > 0.0f ? w_new * inv_den / l_bf : 0.0f;
        float* acc = static_cast<float*>(p.o) + ((size_t)(we.start + (store ? row : 0)) * p.Hq + h) * (size_t)D;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            ptx::tmem_ld32_sync(t_o + cc * 32, o);
            if (store) {
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    float4* ap = reinterpret_cast<float4*>(acc + cc * 32 + v * 4);
                    float4 a = has_old ? *ap : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    a.x = fmaf(a_old, a.x, a_new * __uint_as_float(o[4 * v + 0]));
                    a.y = fmaf(a_old, a.y, a_new * __uint_as_float(o[4 * v + 1]));
                    a.z = fmaf(a_old, a.z, a_new * __uint_as_float(o[4 * v + 2]));
                    a.w = fmaf(a_old, a.w, a_new * __uint_as_float(o[4 * v + 3]));
                    *ap = a;
                }
            }
        }
        if (store) p.lse[idx] = den > 0.0f ? (mu + ptx::lg2_approx(den)) * kLn2 : -INFINITY;
        ptx::tc_fence_before_sync();
        ptx::mbar_arrive(L::bar_o_free(sbase, x));
        return true;
    }
    const float inv = l_bf > 0.0f ? 1.0f / l_bf : 0.0f;
    store_o_rows<D>(p, sbase + L::kStg + (uint32_t)(x * 4 + warp_in_group) * 4096u, lane, t_o, inv,
                    r0 + warp_in_group * 32, we.len, we.start, h, tm_o);
    if (store) {
        const float lse = l_sum > 0.0f ? (m_ref + ptx::lg2_approx(l_sum)) * kLn2 : -INFINITY;
        const size_t idx = p.cu_seqlens ? (size_t)h * p.N + we.start + row
                                        : ((size_t)we.b * p.Hq + h) * p.N + row;
        p.lse[idx] = lse;
    }
    // O has been read: the next unit's first PV of this tile may overwrite it
    ptx::tc_fence_before_sync();
    ptx::mbar_arrive(L::bar_o_free(sbase, x));
    return true;
}

// The units of this CTA for one tile of the pair (tiles with no rows skipped).
template <int D, int STAGES, bool ACC>
__device__ __forceinline__ void softmax_role(const FwdParams& p, int x, int warp_in_group, int lane,
                                             uint32_t tmem, uint32_t sbase, volatile int* abort_flag,
                                             const CUtensorMap* tm_o) {
    // bit 0: s_full parity, bit 1: o_done parity, bits 2-3: unit queue index mod 4
    uint32_t phases = 0;
    while (true) {
        const int u = unit_take<SmemLayout<D, STAGES>>(sbase, phases >> 2, abort_flag, p.wait_limit_ns);
        phases = (phases + 4u) & 15u;
        if (u < 0) break;
        const TilePair w = decode_pair(u, p);
        if (!(x ? w.active[1] : w.active[0])) continue;
        if (!softmax_unit<D, STAGES, ACC>(w, p, x, warp_in_group, lane, tmem, sbase, abort_flag, phases, u, tm_o))
            break;
        phases ^= 2u;
    }
    if (lane == 0) ptx::bulk_wait_group0();  // this warp's output copies are complete
}

// ---------------------------------------------------------------- kernel
template <int D, int STAGES, bool ACC = false>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const FwdParams p) {
    using L = SmemLayout<D, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = ptx::smem_addr(smem);
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x % 32;

    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

    if (warp == kWarpProducer && lane == 0) {
        ptx::mbar_init(L::bar_q(sbase), 1);
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(L::bar_kv_full(sbase, s), 1);
            ptx::mbar_init(L::bar_kv_empty(sbase, s), 1);
        }
        for (int x = 0; x < 2; ++x) {
            ptx::mbar_init(L::bar_s_full(sbase, x), 1);
            ptx::mbar_init(L::bar_p_ready(sbase, x), 128);
            ptx::mbar_init(L::bar_o_done(sbase, x), 1);
        }
        ptx::mbar_init(L::bar_mma_final(sbase), 1);
        init_schedule_barriers<L>(sbase);
        *abort_flag = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tensormap(&tm_q);
        ptx::prefetch_tensormap(&tm_k);
        ptx::prefetch_tensormap(&tm_v);
        ptx::prefetch_tensormap(&tm_o);
    }
    if (warp == kWarpMma) {
        ptx::tmem_alloc(ptx::smem_addr(tmem_slot), kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp < 8) {
        ptx::setmaxnreg_inc<kRegsSoftmax>();
        softmax_role<D, STAGES, ACC>(p, warp / 4, warp % 4, lane, tmem, sbase, abort_flag, ACC ? nullptr : &tm_o);
    } else {
        ptx::setmaxnreg_dec<kRegsOther>();
        if (warp == kWarpProducer) {
            producer_role<D, STAGES>(p, &tm_q, &tm_k, &tm_v, sbase, abort_flag);
        } else if (warp == kWarpMma) {
            mma_role<D, STAGES>(p, tmem, sbase, abort_flag);
        }
    }

    ptx::tc_fence_before_sync();
    __syncthreads();
    if (warp == kWarpMma) {
        ptx::tc_fence_after_sync();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

// A block that waits on a barrier nothing will signal: proves that bounded
// waits give up, record the timeout and return without faulting the GPU.
__global__ void selftest_bounded_wait_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        ptx::mbar_init(ptx::smem_addr(&bar), 1);
        abort_flag = 0;
        ptx::fence_mbar_init();
    }
    __syncthreads();
    bounded_wait(ptx::smem_addr(&bar), 0, &abort_flag, limit_ns);
    __syncthreads();
}

}  // namespace attn
