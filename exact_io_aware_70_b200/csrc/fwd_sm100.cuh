// fwd_sm100.cuh -- exact attention forward (prefill) for B200, sm_100a.
//
// What it computes: O = softmax(scale * Q K^T [+ bottom-right causal mask]) V
// and the per-row LSE, per (batch, head). The method is the one the pages
// describe: tiles of Q, K and V are staged on chip, the score tile S and the
// probability tile P never leave the SM, and a running row max m and row sum l
// rescale the partial output by exp(m_old - m_new) whenever a new K/V tile
// raises the max ("Describe Flash Attention at a high level" (mantramindai),
// "The two ideas"; "How FlashAttention Speeds Up the Attention Layer"
// (hassanahmed.net), tiling and online-softmax paragraphs; the QK^T, softmax
// and .V steps fused into one kernel as in "flashattention-memory-bound"
// (appliedaiprep), "A strong answer").
//
// How it maps onto a B200 SM (this design is ours; the pages' A100/H100
// kernels are prior art only):
//   * Persistent grid, one CTA per SM. A work unit is (batch*head, 256 query
//     rows) = two 128-row Q tiles. CTAs take units from a device counter as
//     they become free (a dynamic queue), in an order that groups the heads so
//     that the K/V of the heads in flight stays in L2 and that goes
//     heaviest-first inside a group (longest-first balance of the causal
//     triangle); see fwd_fetch_unit.
//   * Warp 8 is the TMA producer (lane 0 issues): Q tiles once per unit,
//     then K_j and V_j tiles into a ring of shared-memory slots, 128-byte
//     swizzled, completion counted on mbarriers.
//   * Lane 0 of warp 9 issues the tcgen05.mma products (head dim 128), or
//     lane 0 of warp 9 those of Q tile 0 and lane 0 of warp 10 those of Q tile
//     1 (head dim 64, fwd_mma_split), with shared-memory descriptors
//     precomputed per tile and advanced by constant offsets: S_t = Q_t K_j^T
//     into tensor memory (fp32, 128x128), and O_t += P_t V_j with P_t read
//     straight from tensor memory (bf16). The issuing thread blocks while the
//     tensor core's queue is full, so it spends about as long on a product as
//     the tensor core does (64 cycles for 128x128x16, measured; a 128x64x16
//     product still takes about 56), and every commit and wait on its path
//     delays the next product.
//   * 384 threads = 3 warpgroups; warps 10-11 only complete the third
//     warpgroup (warp 10 lane 0 issues tile 1's products at head dim 64) so
//     it can shrink its register budget (setmaxnreg) in favour of the two
//     softmax warpgroups.
//   * Warps 0-3 and 4-7 are the softmax groups of Q tile 0 and Q tile 1, one
//     thread per query row (= TMEM lane). While one group exponentiates its
//     tile, the tensor core works on the other tile's products (ping-pong).
//     Each group also rescales its O tile in tensor memory when its running max
//     grows by more than 2^8 (lazy rescaling: exact, since every p and l uses
//     the same stale reference max), and runs the epilogue (O / l -> bf16
//     through a per-warp shared-memory staging block: row-contiguous warp
//     stores at head dim 128, one TMA tile store per warp at head dim 64;
//     LSE = ln 2 * (m + log2 l)).
//   * Exponentials are base 2 with log2(e) folded into the scale, computed
//     with MUFU ex2 on pairs prepared by sm_100's packed f32x2 FMA; the row
//     max uses the three-input max. A fraction of the pairs can instead be
//     exponentiated on the FMA pipe (exp2_poly_pair, kPolyEvery<D, FP8>). For
//     bf16 inputs it is slower at every fraction tried (the MMA pipe, not the
//     exponentials, sets the pace: a copy of the kernel without exponentials
//     runs at the same speed), so it is off; for e4m3 inputs, whose products
//     take half the tensor cycles, one pair in four is faster. A masked
//     (-inf) score comes out of the polynomial as about 2^-125 rather than 0:
//     negligible next to the row sum (at least 1 once a row has seen a
//     visible key), and rows with
//     no visible key at all are set to O = 0, LSE = -inf in the epilogue.
//   * P_t is handed to the MMA warp once per step (EATTN_SPLIT_P=1 hands it
//     over in two halves so the first half of O_t += P_t V_j can start early;
//     that costs the MMA issuer one more barrier check per tile and step and
//     measured slower). K_j and V_j complete on one barrier, and each Q tile is
//     released to the producer right after its last S product of the unit.
//   * Tensor memory columns, head dim 128: S0 [0,128), S1 [128,256), O0
//     [256,384), O1 [384,512), P_t over S_t's first 64 columns; S_t(j+1)
//     overwrites P_t(j), so it is issued after P_t(j) V. Head dim 64: tile t
//     owns [256t, 256t+256): S_t, then P_t in its own 64 columns, then O_t;
//     S_t(j+1) is computed as soon as the softmax group has read S_t(j) into
//     registers, while it still exponentiates it (fwd_mma_split).
//   * Epilogue: O / l in bf16 goes through a 2 KB shared-memory block per
//     warp so that each global store instruction writes whole rows' 64-byte
//     pieces (full 32-byte sectors) rather than one 16-byte piece of 32 rows.
//   * The same kernel serves e4m3 inputs (FP8 = true): tiles of one swizzle
//     panel (16 KB of 128-byte rows at d=128, an 8-slot K/V ring; 8 KB of
//     64-byte rows with the 64-byte swizzle at d=64, 16 slots), both products as
//     kind::f8f6f4 MMAs (K = 32), P rounded to e4m3 and packed four to a TMEM
//     column, per-head descale factors folded into the exponent scale and the
//     epilogue (see FwdTraits for the exponent shift that keeps P normal).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx_sm100.cuh"
#include "tmem_wide.cuh"

namespace eattn {


struct FwdParams {
    uint16_t* o;        // bf16 [BH, Nq, D]
    float* lse;         // fp32 [BH, Nq]
    // e4m3 inputs only: per (batch*head) factors that turn the stored codes
    // into values (x = descale * code); null for bf16 inputs
    const float* q_descale;
    const float* k_descale;
    const float* v_descale;
    int BH;             // batch * heads
    int Nq, Nkv;
    int num_qb;         // ceil(Nq / 256)
    int num_units;      // BH * num_qb
    int group_heads;    // heads per group of the unit order (see fwd_unit)
    int dynamic_units;  // 1: units come from the device counter; 0: static snake deal
    int queue_slot;     // which entry of g_fwd_queues this launch counts its units in
    float scale_log2;   // scale * log2(e)
};

#ifndef EATTN_KV_SLOTS_D128
#define EATTN_KV_SLOTS_D128 4
#endif
// 1: K_j and V_j complete on K_j's full barrier (one wait per K/V pair for
//    the MMA issuer); 0: each tile has its own full barrier.
// 1: TMA loads carry L2 policies: K/V tiles (re-read by every query block of
//    their head) evict-last, Q tiles (read by one CTA) evict-first.
#ifndef EATTN_FWD_L2_HINTS
#define EATTN_FWD_L2_HINTS 1
#endif
#ifndef EATTN_KV_PAIR_BARRIER
#define EATTN_KV_PAIR_BARRIER 1
#endif
// 1: P is released to the MMA issuer in two halves (p_lo, p_hi); 0: once.
#ifndef EATTN_SPLIT_P
#define EATTN_SPLIT_P 0
#endif

// 1: at head dim 64 the score products rotate over three TMEM buffers and run
//    one step ahead of the softmax (fwd_mma_ahead); 0: two fixed buffers.
#ifndef EATTN_SBUFS_AHEAD
#define EATTN_SBUFS_AHEAD 1
#endif
// 1: (bf16) P is stored to TMEM once per tile (64 columns) after both halves'
//    exponentials, instead of once per half
#ifndef EATTN_P_STORE_ONCE
#define EATTN_P_STORE_ONCE 0
#endif
// 1: at head dim 64 each Q tile has its own MMA-issuing thread and its own
//    tensor-memory columns for S, P and O (fwd_mma_split), so the two tiles'
//    chains of products no longer wait on each other; 0: one issuing thread
//    for both tiles.
#ifndef EATTN_SPLIT_ISSUE
#define EATTN_SPLIT_ISSUE 1
#endif
// 1: (bf16 inputs) the softmax groups signal "P handed over", "S read" and
//    "O free" with one barrier arrival per warp (after a warp-level sync)
//    rather than one per thread; 0: every thread arrives. (For e4m3 inputs
//    the per-warp form made the compiler spill and measured 5% slower.)
#ifndef EATTN_WARP_ARRIVE
#define EATTN_WARP_ARRIVE 1
#endif
// 1: two sets of Q tiles where shared memory allows (see FwdTraits::kQBufs).
//    With one issuing thread it measured slower on gpt2_1k (45.1 against
//    43.0 us), so there it is off; the split issue always uses two sets.
#ifndef EATTN_Q_DOUBLE
#define EATTN_Q_DOUBLE 0
#endif
// 1: the epilogue's O stores go through shared memory as row-contiguous
//    64-byte pieces (full sectors); 0: each thread stores its own row.
#ifndef EATTN_STAGE_O
#define EATTN_STAGE_O 1
#endif
// 1: at head dim 64 each softmax warp writes its 32 rows x 64 columns of O
//    into a 4 KB staging block in the 128-byte swizzle and one lane stores the
//    block with a TMA tile store (the copy engine writes O while the warp goes
//    on to the next unit; the warp waits only before it reuses the block);
//    0: the warp stores the staged rows itself (fwd_store_chunk), as it always
//    does at head dim 128, where the TMA store measured 0.6% slower (8K, 16K)
//    against 3% faster on gpt2_1k at head dim 64.
#ifndef EATTN_TMA_STORE_O
#define EATTN_TMA_STORE_O 1
#endif

// FP8 = true: Q, K, V are e4m3 codes with per-(batch*head) descale factors;
// S and P V run as tcgen05.mma kind::f8f6f4 (K = 32 per instruction), P is
// rounded to e4m3 in tensor memory. At head dim 64 an e4m3 row is 64 bytes,
// so those tiles use the 64-byte swizzle (8-row atoms of 512 bytes).
template <int D, bool FP8 = false>
struct FwdTraits {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int kElemBytes = FP8 ? 1 : 2;
    static constexpr int kRows = 128;                     // rows of a Q, K or V tile
    // bytes of one row within a swizzle panel: 128 (128-byte swizzle), or 64
    // for e4m3 at head dim 64 (64-byte swizzle)
    static constexpr int kRowBytes = D * kElemBytes < 128 ? D * kElemBytes : 128;
    static constexpr bool kSwizzle64 = kRowBytes == 64;
    static constexpr int kAtomBytes = 8 * kRowBytes;      // 8-row swizzle atom (descriptor SBO)
    static constexpr int kPanelBytes = 128 * kRowBytes;   // 128 rows of one swizzle panel
    static constexpr int kPanelElems = kRowBytes / kElemBytes;  // elements of a row in one panel
    static constexpr int kPanels = D * kElemBytes / kRowBytes;
    static constexpr int kTileBytes = kPanels * kPanelBytes;
    static constexpr int kKSteps = D * kElemBytes / 32;   // 32-byte K steps of S = Q K^T
    static constexpr int kPvSteps = FP8 ? 4 : 8;          // MMAs of P V per 128 keys
    static constexpr int kPvRowBytes = (FP8 ? 32 : 16) * kRowBytes;   // V bytes one P V MMA consumes
    // e4m3 P: exponents are taken against (reference max - kShift), so a row's
    // largest values of P lie in [2^6, 2^8] and e4m3's subnormal range (below
    // 2^-6) only holds values under 2^-12 of the row maximum; the lazy-rescale
    // threshold is lowered so P never exceeds 2^8 (< 448, the e4m3 maximum).
    // The shift cancels in O = acc / l and is taken out of the LSE.
    static constexpr float kShift = FP8 ? 6.0f : 0.0f;
    static constexpr float kLazy = FP8 ? 2.0f : 8.0f;
    static constexpr int kSlots =
        FP8 ? (D == 128 ? 8 : 16) : ((D == 128) ? EATTN_KV_SLOTS_D128 : 8);   // K/V ring depth
    static_assert(kSlots >= 2, "the ring holds K_j and V_j at once");
    static_assert(!EATTN_KV_PAIR_BARRIER || kSlots % 2 == 0, "K/V pairs need an even ring");
    static constexpr int kThreads = 384;                  // 3 warpgroups
    // Registers: the launch gives every thread kLaunchRegs (the build checks
    // ptxas reports exactly that); the softmax warpgroups then grow to
    // kSoftmaxRegs and the producer/MMA warpgroup shrinks to kOtherRegs.
    // 2 * 128 * kSoftmaxRegs + 128 * kOtherRegs must not exceed 384 * kLaunchRegs.
    static constexpr int kLaunchRegs = 168;
    static constexpr int kSoftmaxRegs = 192;
    static constexpr int kOtherRegs = 120;
    static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs <= kThreads * kLaunchRegs,
                  "register split exceeds the launch allocation");
    static constexpr int kNumBars = 2 * kSlots + 27;   // FwdBars<kSlots>::kCount
    // One MMA-issuing thread per Q tile (head dim 64: 2 x (128 S + 64 P + D O)
    // columns fit in the 512).
    static constexpr bool kSplit = EATTN_SPLIT_ISSUE && 2 * (128 + 64 + D) <= 512;
    // epilogue staging per softmax warp: 32 rows x 64 bytes (32 bf16 columns), or
    // 32 rows x 128 bytes (a 64-column TMA store box) with kTmaStoreO
    static constexpr bool kTmaStoreO = EATTN_TMA_STORE_O && D == 64;
    static constexpr int kStageWarpBytes = kTmaStoreO ? 32 * 128 : 32 * 64;
    static constexpr int kStageBytes = EATTN_STAGE_O ? 8 * kStageWarpBytes : 0;
    // Q tiles: two (one unit's), or four where shared memory allows (head dim
    // 64, and e4m3 inputs), so that the next unit's Q is loaded while this
    // unit still runs instead of after its last S product
    static constexpr int kQBufs =
        ((EATTN_Q_DOUBLE || kSplit) &&
         1024 + (4 + kSlots) * kTileBytes + kStageBytes + kNumBars * 8 + 32 <= 232448) ? 4 : 2;
    static constexpr int kSmemBytes =
        1024 + (kQBufs + kSlots) * kTileBytes + kStageBytes + kNumBars * 8 + 16 + 16;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static constexpr uint32_t kTmemCols = 512;
    // Score buffers of 128 fp32 columns. With two (head dim 128: 2 x 128 + 2 x
    // 128 O columns fill the 512) tile t always uses buffer t, so S_t(j+1) can
    // only be computed once P_t(j) V has been issued (it overwrites P_t(j)).
    // With three (head dim 64: 3 x 128 + 2 x 64 = 512) the S products rotate
    // over the buffers in issue order and S_t(j+1) is computed ahead, while
    // the softmax still works on S_t(j) (see fwd_mma).
    // With one issuing thread per tile (kSplit) tile t has its own S buffer at
    // column 256 t, P (bf16 pairs or e4m3 quads) at 256 t + 128 instead of
    // over S, and O at 256 t + 192: S_t(j+1) may then be computed as soon as
    // the softmax has read S_t(j), while it still works on it.
    static constexpr int kSBufs = (!kSplit && EATTN_SBUFS_AHEAD && 3 * 128 + 2 * D <= 512) ? 3 : 2;
    static constexpr uint32_t kColS0 = 0, kColS1 = kSplit ? 256 : 128;
    static constexpr uint32_t kColP0 = kSplit ? 128 : kColS0, kColP1 = kSplit ? 384 : kColS1;
    static constexpr uint32_t kColO0 = kSplit ? 192 : 128 * kSBufs;
    static constexpr uint32_t kColO1 = kSplit ? 448 : 128 * kSBufs + D;
    // readers of a unit-ring entry: the MMA issuer(s) and one lane of each softmax warp
    static constexpr int kUnitReaders = kSplit ? 10 : 9;
    // arrivals of one softmax warpgroup on p_lo/p_hi, o_free and (kSplit) "S free"
    static constexpr bool kWarpArrive = EATTN_WARP_ARRIVE && !FP8;
    static constexpr int kArrivals = kWarpArrive ? 4 : 128;
};

// One exponent pair in every kPolyEvery<D, FP8> goes to the FMA-pipe polynomial
// (0: none, the measured-best setting for both head dims).
#ifndef EATTN_POLY_EVERY_D128
#define EATTN_POLY_EVERY_D128 0
#endif
#ifndef EATTN_POLY_EVERY_D64
#define EATTN_POLY_EVERY_D64 0
#endif
// e4m3 inputs halve the tensor-core time per tile while the exponentials stay,
// so there the FMA-pipe polynomial has idle cycles to use: one pair in four
// measured best on B200 (8K causal: 1158 -> 1289 TFLOP/s; one in 2, 3 and 6
// in between).
#ifndef EATTN_POLY_EVERY_FP8
#define EATTN_POLY_EVERY_FP8 4
#endif
template <int D, bool FP8 = false>
constexpr int kPolyEvery =
    FP8 ? EATTN_POLY_EVERY_FP8 : ((D == 128) ? EATTN_POLY_EVERY_D128 : EATTN_POLY_EVERY_D64);

// Work units are handed out dynamically: each CTA's producer takes the next
// index from a device counter (p.queue[0], one atomicAdd per unit) and passes
// it to the MMA and softmax roles through a two-entry ring in shared memory.
// Index u maps to a unit in this order: the heads are taken in groups of
// p.group_heads (the host sizes a group so that its K and V fit comfortably
// in L2), and inside a group the query blocks go heaviest first (latest block
// first under the causal mask), the group's heads interleaved. So the CTAs in
// flight share the K/V tiles of a few heads, which stay in L2 instead of being
// re-read from DRAM, and each group ends with its lightest units, which keeps
// the SMs balanced as a longest-first schedule would.
// g_fwd_queues[2 * slot] counts units handed out, g_fwd_queues[2 * slot + 1]
// the CTAs that have finished; both are zero when a launch starts, and the
// launch's last CTA sets them back to zero.
constexpr int kFwdQueueSlots = 64;
__device__ int g_fwd_queues[2 * kFwdQueueSlots];

// The unit a CTA's producer publishes as its round-th unit. Dynamic: the next
// index of the device counter. Static (used when the K/V of all heads fit in
// L2, where grouping gains nothing and the counter's latency would only
// delay each unit): a snake deal of the same order -- CTA i takes index
// r * G + i in even rounds and r * G + G - 1 - i in odd ones (G = grid size),
// which balances the heaviest-first order about as well as longest-first
// greedy.
__device__ __forceinline__ int fwd_fetch_unit(const FwdParams& p, uint32_t round) {
    long long u;
    if (p.dynamic_units) {
        u = atomicAdd(&g_fwd_queues[2 * p.queue_slot], 1);
    } else {
        const int g = gridDim.x, i = blockIdx.x;
        u = (long long)round * g + ((round & 1) ? (g - 1 - i) : i);
    }
    return u < p.num_units ? (int)u : -1;
}

struct FwdUnit {
    int bh, qb;
    int n[2];   // K/V tiles visible to Q tile 0 / Q tile 1 (0: tile has no work)
    int nmax;
};

template <bool CAUSAL>
__device__ __forceinline__ FwdUnit fwd_unit(int u, const FwdParams& p) {
    FwdUnit x;
    if (p.group_heads >= p.BH) {   // one group: plain heaviest-first order
        x.qb = p.num_qb - 1 - u / p.BH;
        x.bh = u % p.BH;
    } else {
        const int per_group = p.group_heads * p.num_qb;
        const int g = u / per_group;
        const int r = u - g * per_group;
        const int heads = min(p.group_heads, p.BH - g * p.group_heads);   // the last group may be short
        x.qb = p.num_qb - 1 - r / heads;   // heaviest (latest) query blocks first
        x.bh = g * p.group_heads + r % heads;
    }
    dcheck(x.qb >= 0 && x.bh < p.BH);
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const long long r0 = (long long)x.qb * 256 + t * 128;
        int n = 0;
        if (r0 < p.Nq) {
            long long kv_end = p.Nkv;
            if (CAUSAL) {
                const long long r1 = min(r0 + 127, (long long)p.Nq - 1);
                kv_end = min(kv_end, r1 + ((long long)p.Nkv - p.Nq) + 1);
            }
            n = kv_end <= 0 ? 0 : (int)((kv_end + 127) / 128);
        }
        x.n[t] = n;
    }
    x.nmax = max(x.n[0], x.n[1]);
    return x;
}

// Position of S_t(i) among the unit's score products in issue order: all
// products of index i' < i (tile 0's before tile 1's at each index), then
// S_0(i) before S_1(i).
__device__ __forceinline__ int fwd_s_pos(const FwdUnit& x, int t, int i) {
    return min(i, x.n[0]) + min(i, x.n[1]) + ((t == 1 && i < x.n[0]) ? 1 : 0);
}

// mbarrier addresses, all derived from one shared-memory base address so that
// only a single register is live across the roles. Layout (8 bytes each):
// kv_full[S], kv_empty[S], then 2 each of q_full, q_empty, s_full, p_lo, p_hi,
// o_final, o_free, then drain, then 2 each of unit_full, unit_empty, s_full_b,
// pv_done, and of q_full, q_empty for the second set of Q tiles.
template <int S>
struct FwdBars {
    uint32_t base;
    __device__ __forceinline__ uint32_t kv_full(uint32_t i) const { return base + 8 * i; }
    __device__ __forceinline__ uint32_t kv_empty(uint32_t i) const { return base + 8 * (S + i); }
    // Q tile slot qi = 2 * set + t (set 1 exists only with four Q tiles)
    __device__ __forceinline__ uint32_t q_full(int qi) const {
        return base + 8 * (qi < 2 ? 2 * S + qi : 2 * S + 23 + (qi - 2));
    }
    __device__ __forceinline__ uint32_t q_empty(int qi) const {
        return base + 8 * (qi < 2 ? 2 * S + 2 + qi : 2 * S + 25 + (qi - 2));
    }
    __device__ __forceinline__ uint32_t s_full(int t) const { return base + 8 * (2 * S + 4 + t); }
    __device__ __forceinline__ uint32_t p_lo(int t) const { return base + 8 * (2 * S + 6 + t); }
    __device__ __forceinline__ uint32_t p_hi(int t) const { return base + 8 * (2 * S + 8 + t); }
    __device__ __forceinline__ uint32_t o_final(int t) const { return base + 8 * (2 * S + 10 + t); }
    __device__ __forceinline__ uint32_t o_free(int t) const { return base + 8 * (2 * S + 12 + t); }
    __device__ __forceinline__ uint32_t drain() const { return base + 8 * (2 * S + 14); }
    __device__ __forceinline__ uint32_t unit_full(int i) const { return base + 8 * (2 * S + 15 + i); }
    __device__ __forceinline__ uint32_t unit_empty(int i) const { return base + 8 * (2 * S + 17 + i); }
    // three score buffers only: S_t products alternate between s_full(t) and
    // s_full_b(t) (one may complete before the softmax has seen the other);
    // pv_done(t) completes with every P_t V product. With one issuer per tile
    // s_full_b(t) is instead "S_t free": the softmax group has read S_t.
    __device__ __forceinline__ uint32_t s_full_b(int t) const { return base + 8 * (2 * S + 19 + t); }
    __device__ __forceinline__ uint32_t pv_done(int t) const { return base + 8 * (2 * S + 21 + t); }
    // barrier and parity of tile t's c-th score product (c counted over the CTA's life)
    template <int kSBufs>
    __device__ __forceinline__ uint32_t s_bar(int t, uint32_t c) const {
        return (kSBufs == 3 && (c & 1)) ? s_full_b(t) : s_full(t);
    }
    template <int kSBufs>
    static __device__ __forceinline__ uint32_t s_parity(uint32_t c) {
        return kSBufs == 3 ? (c >> 1) & 1 : c & 1;
    }
    static constexpr int kCount = 2 * S + 27;
    // shared-memory words after the barriers: TMEM base, abort flag, unit ring[2]
    __device__ __forceinline__ volatile int* unit_slot(int i) const {
        return reinterpret_cast<volatile int*>(unit_ring_ptr) + i;
    }
    uint8_t* unit_ring_ptr;
};

// Next unit for a consumer role. Dynamic deal: waits for ring entry k, reads
// it and releases the entry (the MMA issuer and lane 0 of each softmax warp
// count as its readers). Static deal: the k-th unit of the snake deal. Returns
// false on a failed wait; *u = -1 marks the end.
template <int S>
__device__ __forceinline__ bool fwd_next_unit(const FwdParams& p, const FwdBars<S>& b, uint32_t k,
                                              bool arrive, volatile int* abort_flag, int* u) {
    // the static deal needs no hand-over: every role computes the same sequence
    if (!p.dynamic_units) {
        *u = fwd_fetch_unit(p, k);
        return true;
    }
    const int slot = k & 1;
    if (!mbar_wait(b.unit_full(slot), (k >> 1) & 1, abort_flag, &g_attn_status)) return false;
    *u = *b.unit_slot(slot);
    if (arrive) mbar_arrive(b.unit_empty(slot));
    return true;
}

// Bounded wait executed by a whole warp; the outcome is made warp-uniform.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    bool ok = mbar_wait(bar, parity, abort_flag, &g_attn_status);
    return __all_sync(0xffffffffu, ok);
}

// The producer and MMA roles run either on one lane (EATTN_WARP_ISSUE 0: the
// other 31 lanes go straight to the final barrier) or on the whole warp with
// converged control flow and only lane 0 issuing (EATTN_WARP_ISSUE 1).
#ifndef EATTN_WARP_ISSUE
#define EATTN_WARP_ISSUE 0
#endif
__device__ __forceinline__ bool role_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
#if EATTN_WARP_ISSUE
    return warp_wait(bar, parity, abort_flag);
#else
    return mbar_wait(bar, parity, abort_flag, &g_attn_status);
#endif
}

// ----------------------------------------------------------- TMA producer --
// Run by the whole producer warp with converged control flow; lane 0 issues.
template <int D, bool CAUSAL, bool FP8>
__device__ void fwd_producer(const FwdParams& p, const CUtensorMap* tq, const CUtensorMap* tk,
                             const CUtensorMap* tv, uint32_t sQ, uint32_t sKV,
                             const FwdBars<FwdTraits<D, FP8>::kSlots>& b, uint32_t leader,
                             volatile int* abort_flag) {
    using T = FwdTraits<D, FP8>;
    const uint64_t pol_q = l2_policy_evict_first();
    const uint64_t pol_kv = l2_policy_evict_last();
    uint32_t kv_iter = 0;
    uint32_t q_issued[4] = {0, 0, 0, 0};
    int u = fwd_fetch_unit(p, 0);
    for (uint32_t k = 0;; ++k) {
        // dynamic deal: publish unit u (or the end) in ring entry k once its last
        // readers are done (the static deal needs no hand-over)
        if (p.dynamic_units) {
            const int slot = k & 1;
            if (k >= 2 && !role_wait(b.unit_empty(slot), ((k >> 1) - 1) & 1, abort_flag))
                goto fail;
            *b.unit_slot(slot) = u;
            mbar_arrive(b.unit_full(slot));
        }
        if (u < 0) break;
        const FwdUnit x = fwd_unit<CAUSAL>(u, p);
        const int qset = T::kQBufs == 4 ? (int)(k & 1) : 0;
        for (int t = 0; t < 2; ++t) {
            const int qi = 2 * qset + t;
            if (q_issued[qi] > 0 &&
                !role_wait(b.q_empty(qi), (q_issued[qi] - 1) & 1, abort_flag))
                goto fail;
            mbar_arrive_expect_tx_w(b.q_full(qi), T::kTileBytes, leader);
#pragma unroll
            for (int pn = 0; pn < T::kPanels; ++pn)
                if (EATTN_FWD_L2_HINTS)
                    tma_load_3d_hint_w(sQ + qi * T::kTileBytes + pn * T::kPanelBytes, tq,
                                       b.q_full(qi), pn * T::kPanelElems, x.qb * 256 + t * 128,
                                       x.bh, pol_q, leader);
                else
                    tma_load_3d_w(sQ + qi * T::kTileBytes + pn * T::kPanelBytes, tq,
                                  b.q_full(qi), pn * T::kPanelElems, x.qb * 256 + t * 128, x.bh,
                                  leader);
            ++q_issued[qi];
        }
        u = fwd_fetch_unit(p, k + 1);   // the next unit, fetched while this one's tiles stream in
        for (int j = 0; j < x.nmax; ++j) {
#pragma unroll
            for (int which = 0; which < 2; ++which) {   // K_j, then V_j
                const uint32_t slot = kv_iter % T::kSlots;
                const uint32_t round = kv_iter / T::kSlots;
                if (round > 0 && !role_wait(b.kv_empty(slot), (round - 1) & 1, abort_flag))
                    goto fail;
                // with pair barriers, V_j's copy completes on K_j's barrier (slot - 1)
                const uint32_t fbar =
                    b.kv_full(EATTN_KV_PAIR_BARRIER && which ? slot - 1 : slot);
                if (!EATTN_KV_PAIR_BARRIER)
                    mbar_arrive_expect_tx_w(fbar, T::kTileBytes, leader);
                else if (which == 0)
                    mbar_arrive_expect_tx_w(fbar, 2 * T::kTileBytes, leader);
#pragma unroll
                for (int pn = 0; pn < T::kPanels; ++pn)
                    if (EATTN_FWD_L2_HINTS)
                        tma_load_3d_hint_w(sKV + slot * T::kTileBytes + pn * T::kPanelBytes,
                                           which ? tv : tk, fbar, pn * T::kPanelElems, j * 128,
                                           x.bh, pol_kv, leader);
                    else
                        tma_load_3d_w(sKV + slot * T::kTileBytes + pn * T::kPanelBytes,
                                      which ? tv : tk, fbar, pn * T::kPanelElems, j * 128, x.bh,
                                      leader);
                ++kv_iter;
            }
        }
    }
    return;
fail: {
    // Give up: wait (bounded, ignoring the abort flag) for the copies still in
    // flight so none lands in shared memory after the CTA has exited.
    volatile int no_abort = 0;
    const uint32_t first = kv_iter > (uint32_t)T::kSlots ? kv_iter - T::kSlots : 0;
    for (uint32_t i = first; i < kv_iter; ++i)
        if (!EATTN_KV_PAIR_BARRIER || (i % 2) == 0)
            mbar_wait(b.kv_full(i % T::kSlots), (i / T::kSlots) & 1, &no_abort, &g_attn_status);
    for (int qi = 0; qi < T::kQBufs; ++qi)
        if (q_issued[qi] > 0)
            mbar_wait(b.q_full(qi), (q_issued[qi] - 1) & 1, &no_abort, &g_attn_status);
}
}

// ------------------------------------------------------------ MMA issuer --
// Shared-memory descriptor of a tile in the traits' swizzle: 128-byte (layout
// type 2, 1024-byte atoms) or 64-byte (layout type 4, 512-byte atoms).
template <class T>
__device__ __forceinline__ uint64_t fwd_sdesc(uint32_t saddr, uint32_t lbo_bytes) {
    uint64_t d = sdesc_sw128(saddr, lbo_bytes, T::kAtomBytes);
    if (T::kSwizzle64) d = (d & ~(uint64_t(7) << 61)) | (uint64_t(4) << 61);
    return d;
}

// Descriptor bases are computed once; an operand at byte offset `off` from a
// base is the base plus off >> 4 (the start-address field never overflows:
// shared memory addresses are below 2^18).
template <int D, bool FP8>
__device__ __forceinline__ void fwd_issue_s(uint32_t tmem_s, uint64_t dq, uint64_t dk,
                                            uint32_t leader) {
    using T = FwdTraits<D, FP8>;
    constexpr uint32_t idesc =
        FP8 ? idesc_e4m3_f32(128, 128, false) : idesc_bf16_f32(128, 128, false);
#pragma unroll
    for (int kk = 0; kk < T::kKSteps; ++kk) {
        // one MMA consumes 32 bytes of every row (16 bf16 or 32 e4m3 elements)
        const uint64_t off = ((kk / 4) * T::kPanelBytes + (kk % 4) * 32) >> 4;
        if (FP8)
            mma_f8_ss_w(tmem_s, dq + off, dk + off, idesc, kk > 0 ? 1u : 0u, leader);
        else
            mma_bf16_ss_w(tmem_s, dq + off, dk + off, idesc, kk > 0 ? 1u : 0u, leader);
    }
}

template <int D, bool FP8>
__device__ __forceinline__ void fwd_issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint64_t dv,
                                             bool accumulate, int half, uint32_t leader) {
    using T = FwdTraits<D, FP8>;
    constexpr uint32_t idesc = FP8 ? idesc_e4m3_f32(128, D, true) : idesc_bf16_f32(128, D, true);
    constexpr int kHalfSteps = T::kPvSteps / 2;
#pragma unroll
    for (int kk = kHalfSteps * half; kk < kHalfSteps * (half + 1); ++kk) {
        // P: 8 TMEM columns per MMA (16 keys as bf16 pairs, or 32 keys as
        // e4m3 quads). V: the same keys' rows, 8-row swizzle atoms of 1024
        // bytes; bf16 V's two 64-column panels are kPanelBytes apart (the
        // descriptor's leading-dimension offset).
        if (FP8)
            mma_f8_ts_w(tmem_o, tmem_p + kk * 8, dv + ((kk * T::kPvRowBytes) >> 4), idesc,
                        (accumulate || kk > 0) ? 1u : 0u, leader);
        else
            mma_bf16_ts_w(tmem_o, tmem_p + kk * 8, dv + ((kk * T::kPvRowBytes) >> 4), idesc,
                          (accumulate || kk > 0) ? 1u : 0u, leader);
    }
}

// Three score buffers (head dim 64). Per K/V step j the issue order is
//   S_0(j+1), P_0(j) V_j, S_1(j+1), P_1(j) V_j,
// every score product going to buffer (products issued so far) mod 3. The
// buffer S_t(j+1) overwrites last held the product issued three before it,
// whose P V has always been issued by then (S_1(j) at the end of step j-1 for
// S_0(j+1); S_0(j) just before for S_1(j+1); earlier still when a tile has
// fewer steps, and all of the previous unit's), and tensor-core operations
// run in issue order. So S_t(j+1) is computed while the softmax group still
// works on S_t(j), and the group finds it ready when it hands over P_t(j).
template <int D, bool CAUSAL, bool FP8>
__device__ void fwd_mma_ahead(const FwdParams& p, uint32_t tbase, uint32_t sQ, uint32_t sKV,
                              const FwdBars<FwdTraits<D, FP8>::kSlots>& b, uint32_t leader,
                              volatile int* abort_flag) {
    using T = FwdTraits<D, FP8>;
    static_assert(T::kSBufs == 3, "three score buffers");
    static_assert(!EATTN_SPLIT_P, "P is handed over once per step here");
    constexpr uint64_t kTileStep = T::kTileBytes >> 4;
    const uint64_t dq0 = fwd_sdesc<T>(sQ, 16);
    const uint64_t dk0 = fwd_sdesc<T>(sKV, 16);                       // K-major K tile
    const uint64_t dv0 = fwd_sdesc<T>(sKV, T::kPanelBytes);           // MN-major V tile
    const uint32_t colO[2] = {T::kColO0, T::kColO1};
    uint32_t kv_iter = 0, s_issued = 0;
    uint32_t q_use[2] = {0, 0};     // units that used Q set 0 / set 1
    uint32_t o_use[2] = {0, 0}, p_cnt[2] = {0, 0}, s_cnt[2] = {0, 0};
    uint32_t cur_col[2] = {0, 0};   // buffer holding S_t(j) / P_t(j)
    for (uint32_t k = 0;; ++k) {
        int u;
        if (!fwd_next_unit(p, b, k, true, abort_flag, &u)) goto done;
        if (u < 0) break;
        {
            const FwdUnit x = fwd_unit<CAUSAL>(u, p);
            const int qset = T::kQBufs == 4 ? (int)(k & 1) : 0;
            if (!role_wait(b.q_full(2 * qset), q_use[qset] & 1, abort_flag)) goto done;
            if (!role_wait(b.q_full(2 * qset + 1), q_use[qset] & 1, abort_flag)) goto done;
            tc_fence_after_sync();
            // S_t(i) into the next buffer in rotation; Q_t is released after its last product
            auto issue_s = [&](int t, int i, uint32_t kslot) {
                const uint32_t col = (s_issued++ % 3) * 128;
                fwd_issue_s<D, FP8>(tbase + col, dq0 + (2 * qset + t) * kTileStep,
                                    dk0 + kslot * kTileStep, leader);
                mma_commit_w(b.template s_bar<3>(t, s_cnt[t]++), leader);
                if (i == x.n[t] - 1) mma_commit_w(b.q_empty(2 * qset + t), leader);
                return col;
            };
            if (x.nmax > 0) {
                uint32_t kslot = kv_iter % T::kSlots;
                if (!role_wait(b.kv_full(kslot), (kv_iter / T::kSlots) & 1, abort_flag)) goto done;
                tc_fence_after_sync();
                for (int t = 0; t < 2; ++t)
                    if (x.n[t] > 0) cur_col[t] = issue_s(t, 0, kslot);
                mma_commit_w(b.kv_empty(kslot), leader);
                ++kv_iter;
                for (int j = 0; j < x.nmax; ++j) {
                    const uint32_t vslot = kv_iter % T::kSlots;   // V_j arrived with K_j
                    ++kv_iter;
                    const bool has_next = j + 1 < x.nmax;
                    kslot = kv_iter % T::kSlots;
                    if (has_next) {
                        if (!role_wait(b.kv_full(kslot), (kv_iter / T::kSlots) & 1, abort_flag))
                            goto done;
                        tc_fence_after_sync();
                    }
                    for (int t = 0; t < 2; ++t) {
                        uint32_t next_col = cur_col[t];
                        if (j + 1 < x.n[t]) next_col = issue_s(t, j + 1, kslot);
                        if (j < x.n[t]) {
                            // P_t hand-overs alternate between two barriers: the group may
                            // release P_t(j+1) before this wait for P_t(j) has run, since
                            // S_t(j+1) is already issued; P_t(j+2) it may not.
                            if (!role_wait((p_cnt[t] & 1) ? b.p_lo(t) : b.p_hi(t),
                                           (p_cnt[t] >> 1) & 1, abort_flag))
                                goto done;
                            ++p_cnt[t];
                            if (j == 0 && o_use[t] > 0 &&
                                !role_wait(b.o_free(t), (o_use[t] - 1) & 1, abort_flag))
                                goto done;
                            tc_fence_after_sync();
                            fwd_issue_pv<D, FP8>(tbase + colO[t], tbase + cur_col[t],
                                                 dv0 + vslot * kTileStep, j > 0, 0, leader);
                            fwd_issue_pv<D, FP8>(tbase + colO[t], tbase + cur_col[t],
                                                 dv0 + vslot * kTileStep, true, 1, leader);
                            mma_commit_w(b.pv_done(t), leader);
                            if (j == x.n[t] - 1) mma_commit_w(b.o_final(t), leader);
                        }
                        cur_col[t] = next_col;
                    }
                    mma_commit_w(b.kv_empty(vslot), leader);
                    if (has_next) {
                        mma_commit_w(b.kv_empty(kslot), leader);
                        ++kv_iter;
                    }
                }
            }
            // Q tiles without any S product in this unit are released here
            for (int t = 0; t < 2; ++t)
                if (x.n[t] == 0) mma_commit_w(b.q_empty(2 * qset + t), leader);
            ++q_use[qset];
            for (int t = 0; t < 2; ++t)
                if (x.n[t] > 0) ++o_use[t];
        }
    }
done: {
    // Every MMA issued so far must finish before tensor memory is released.
    volatile int no_abort = 0;
    mma_commit_w(b.drain(), leader);
    mbar_wait(b.drain(), 0, &no_abort, &g_attn_status);
}
}

// One issuing thread per Q tile (FwdTraits::kSplit): this thread issues
// every product of tile t. Per K/V step j of a unit the order is
//   S_t(j) (once the softmax group has read S_t(j-1)), then P_t(j-1) V_{j-1},
// so S_t(j) is computed while the group still exponentiates S_t(j-1), and
// P_t(j-1) V waits only for this tile's own hand-over, never for the other
// tile's. K and V slots are released by both issuers (kv_empty counts two
// arrivals); a tile with fewer steps than the unit still waits for each K/V
// pair, in order, and releases it at once.
template <int D, bool CAUSAL, bool FP8>
__device__ void fwd_mma_split(const FwdParams& p, uint32_t tbase, uint32_t sQ, uint32_t sKV,
                              const FwdBars<FwdTraits<D, FP8>::kSlots>& b, uint32_t leader,
                              volatile int* abort_flag, int t) {
    using T = FwdTraits<D, FP8>;
    static_assert(T::kSplit && !EATTN_SPLIT_P && EATTN_KV_PAIR_BARRIER, "split issue layout");
    constexpr uint64_t kTileStep = T::kTileBytes >> 4;
    const uint64_t dq0 = fwd_sdesc<T>(sQ, 16);
    const uint64_t dk0 = fwd_sdesc<T>(sKV, 16);                       // K-major K tile
    const uint64_t dv0 = fwd_sdesc<T>(sKV, T::kPanelBytes);           // MN-major V tile
    const uint32_t tS = tbase + (t ? T::kColS1 : T::kColS0);
    const uint32_t tP = tbase + (t ? T::kColP1 : T::kColP0);
    const uint32_t tO = tbase + (t ? T::kColO1 : T::kColO0);
    uint32_t kv_iter = 0;           // K and V tiles of all units so far (two per step)
    uint32_t q_use[2] = {0, 0};     // units that used Q set 0 / set 1
    uint32_t o_use = 0, s_cnt = 0, p_cnt = 0;
    for (uint32_t k = 0;; ++k) {
        int u;
        if (!fwd_next_unit(p, b, k, true, abort_flag, &u)) goto done;
        if (u < 0) break;
        {
            const FwdUnit x = fwd_unit<CAUSAL>(u, p);
            const int n = x.n[t];
            const int qi = 2 * (T::kQBufs == 4 ? (int)(k & 1) : 0) + t;
            const uint32_t qset = qi >> 1;
            if (!role_wait(b.q_full(qi), q_use[qset] & 1, abort_flag)) goto done;
            ++q_use[qset];
            if (n == 0) mma_commit_w(b.q_empty(qi), leader);
            // P_t(i) V_i, V_i in ring slot vslot
            auto issue_pv = [&](int i, uint32_t vslot) -> bool {
                if (!role_wait(b.p_hi(t), p_cnt & 1, abort_flag)) return false;
                ++p_cnt;
                if (i == 0 && o_use > 0 && !role_wait(b.o_free(t), (o_use - 1) & 1, abort_flag))
                    return false;
                tc_fence_after_sync();
                fwd_issue_pv<D, FP8>(tO, tP, dv0 + vslot * kTileStep, i > 0, 0, leader);
                fwd_issue_pv<D, FP8>(tO, tP, dv0 + vslot * kTileStep, true, 1, leader);
                mma_commit_w(b.pv_done(t), leader);
                if (i == n - 1) mma_commit_w(b.o_final(t), leader);
                mma_commit_w(b.kv_empty(vslot), leader);
                return true;
            };
            uint32_t prev_vslot = 0;
            for (int j = 0; j < x.nmax; ++j) {
                const uint32_t kslot = kv_iter % T::kSlots;
                const uint32_t vslot = (kv_iter + 1) % T::kSlots;
                if (!role_wait(b.kv_full(kslot), (kv_iter / T::kSlots) & 1, abort_flag)) goto done;
                kv_iter += 2;
                if (j < n) {
                    // S_t(j) overwrites S_t(j-1): wait until the softmax group has read it
                    if (s_cnt > 0 && !role_wait(b.s_full_b(t), (s_cnt - 1) & 1, abort_flag))
                        goto done;
                    tc_fence_after_sync();
                    fwd_issue_s<D, FP8>(tS, dq0 + qi * kTileStep, dk0 + kslot * kTileStep, leader);
                    mma_commit_w(b.s_full(t), leader);
                    ++s_cnt;
                    if (j == n - 1) mma_commit_w(b.q_empty(qi), leader);
                    mma_commit_w(b.kv_empty(kslot), leader);
                } else if (leader) {
                    mbar_arrive(b.kv_empty(kslot));   // this tile does not read K_j
                }
                if (j >= 1) {
                    if (j - 1 < n) {
                        if (!issue_pv(j - 1, prev_vslot)) goto done;
                    } else if (leader) {
                        mbar_arrive(b.kv_empty(prev_vslot));
                    }
                }
                prev_vslot = vslot;
            }
            if (x.nmax > 0) {
                if (x.nmax - 1 < n) {
                    if (!issue_pv(x.nmax - 1, prev_vslot)) goto done;
                } else if (leader) {
                    mbar_arrive(b.kv_empty(prev_vslot));
                }
            }
            if (n > 0) ++o_use;
        }
    }
done: {
    // Every MMA this thread issued must finish before tensor memory is released
    // (the drain barrier counts one arrival per issuing thread).
    volatile int no_abort = 0;
    mma_commit_w(b.drain(), leader);
    mbar_wait(b.drain(), 0, &no_abort, &g_attn_status);
}
}

// Run by the whole MMA warp with converged control flow; lane 0 issues.
template <int D, bool CAUSAL, bool FP8>
__device__ void fwd_mma(const FwdParams& p, uint32_t tbase, uint32_t sQ, uint32_t sKV,
                        const FwdBars<FwdTraits<D, FP8>::kSlots>& b, uint32_t leader,
                        volatile int* abort_flag) {
    using T = FwdTraits<D, FP8>;
    constexpr uint64_t kTileStep = T::kTileBytes >> 4;
    const uint64_t dq0 = fwd_sdesc<T>(sQ, 16);
    const uint64_t dk0 = fwd_sdesc<T>(sKV, 16);                       // K-major K tile
    const uint64_t dv0 = fwd_sdesc<T>(sKV, T::kPanelBytes);           // MN-major V tile
    const uint32_t colS[2] = {T::kColS0, T::kColS1};
    const uint32_t colO[2] = {T::kColO0, T::kColO1};
    uint32_t kv_iter = 0;
    uint32_t q_use[2] = {0, 0};     // units that used Q set 0 / set 1
    uint32_t o_use[2] = {0, 0}, p_phase[2] = {0, 0};
    for (uint32_t k = 0;; ++k) {
        int u;
        if (!fwd_next_unit(p, b, k, true, abort_flag, &u)) goto done;
        if (u < 0) break;
        const FwdUnit x = fwd_unit<CAUSAL>(u, p);
        const int qset = T::kQBufs == 4 ? (int)(k & 1) : 0;
        const uint64_t dqs = dq0 + 2 * qset * kTileStep;
        if (!role_wait(b.q_full(2 * qset), q_use[qset] & 1, abort_flag)) goto done;
        if (!role_wait(b.q_full(2 * qset + 1), q_use[qset] & 1, abort_flag)) goto done;
        tc_fence_after_sync();
        if (x.nmax > 0) {
            uint32_t kslot = kv_iter % T::kSlots;
            if (!role_wait(b.kv_full(kslot), (kv_iter / T::kSlots) & 1, abort_flag)) goto done;
            tc_fence_after_sync();
            for (int t = 0; t < 2; ++t)
                if (x.n[t] > 0) {
                    fwd_issue_s<D, FP8>(tbase + colS[t], dqs + t * kTileStep, dk0 + kslot * kTileStep,
                                   leader);
                    mma_commit_w(b.s_full(t), leader);
                    // Q_t's last use in this unit: let the producer refill it now
                    if (x.n[t] == 1) mma_commit_w(b.q_empty(2 * qset + t), leader);
                }
            mma_commit_w(b.kv_empty(kslot), leader);
            ++kv_iter;
            for (int j = 0; j < x.nmax; ++j) {
                const uint32_t vslot = kv_iter % T::kSlots;
                if (!EATTN_KV_PAIR_BARRIER) {   // else V_j arrived with K_j
                    if (!role_wait(b.kv_full(vslot), (kv_iter / T::kSlots) & 1, abort_flag))
                        goto done;
                    tc_fence_after_sync();
                }
                ++kv_iter;
                const bool has_next = j + 1 < x.nmax;
                kslot = kv_iter % T::kSlots;
                const uint32_t kpar = (kv_iter / T::kSlots) & 1;
                for (int t = 0; t < 2; ++t) {
                    if (j < x.n[t]) {
                        if (!role_wait(EATTN_SPLIT_P ? b.p_lo(t) : b.p_hi(t), p_phase[t], abort_flag))
                            goto done;
                        if (j == 0 && o_use[t] > 0 &&
                            !role_wait(b.o_free(t), (o_use[t] - 1) & 1, abort_flag))
                            goto done;
                        tc_fence_after_sync();
                        fwd_issue_pv<D, FP8>(tbase + colO[t], tbase + colS[t], dv0 + vslot * kTileStep,
                                        j > 0, 0, leader);
                        if (EATTN_SPLIT_P) {
                            if (!role_wait(b.p_hi(t), p_phase[t], abort_flag)) goto done;
                            tc_fence_after_sync();
                        }
                        fwd_issue_pv<D, FP8>(tbase + colO[t], tbase + colS[t], dv0 + vslot * kTileStep,
                                        true, 1, leader);
                        p_phase[t] ^= 1;
                        if (j == x.n[t] - 1) mma_commit_w(b.o_final(t), leader);
                    }
                    if (t == 0 && has_next) {
                        if (!role_wait(b.kv_full(kslot), kpar, abort_flag)) goto done;
                        tc_fence_after_sync();
                    }
                    if (t == 1) mma_commit_w(b.kv_empty(vslot), leader);
                    if (j + 1 < x.n[t]) {
                        fwd_issue_s<D, FP8>(tbase + colS[t], dqs + t * kTileStep,
                                       dk0 + kslot * kTileStep, leader);
                        mma_commit_w(b.s_full(t), leader);
                        if (j + 2 == x.n[t]) mma_commit_w(b.q_empty(2 * qset + t), leader);
                    }
                }
                if (has_next) {
                    mma_commit_w(b.kv_empty(kslot), leader);
                    ++kv_iter;
                }
            }
        }
        // Q tiles without any S product in this unit are released here
        for (int t = 0; t < 2; ++t)
            if (x.n[t] == 0) mma_commit_w(b.q_empty(2 * qset + t), leader);
        ++q_use[qset];
        for (int t = 0; t < 2; ++t)
            if (x.n[t] > 0) ++o_use[t];
    }
done: {
    // Every MMA issued so far must finish before tensor memory is released.
    volatile int no_abort = 0;
    mma_commit_w(b.drain(), leader);
    mbar_wait(b.drain(), 0, &no_abort, &g_attn_status);
}
}

// --------------------------------------------------------------- softmax --
// Arrival of a softmax warp on a barrier the MMA issuer waits for, after this
// thread's tensor-memory accesses (made complete by the caller's tcgen05
// wait) are ordered before it. Counts FwdTraits::kArrivals per warpgroup.
template <bool kPerWarp>
__device__ __forceinline__ void softmax_arrive(uint32_t bar, int lane) {
    tc_fence_before_sync();
    if (kPerWarp) {
        __syncwarp();
        if (lane == 0) mbar_arrive(bar);
    } else {
        mbar_arrive(bar);
    }
}



// TMA tile store shared -> global of one 3-D box ({x, y, z} element
// coordinates, x a multiple of 64 bf16, never negative), tracked by this
// thread's bulk async-group; rows past the map's extent are not written.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int x, int y,
                                             int z) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(src)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// this thread's bulk stores have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// this thread's bulk stores are complete
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// generic-proxy shared-memory writes made visible to the async proxy (TMA)
__device__ __forceinline__ void fence_async_shared() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}


// Epilogue store of one 32-column chunk of this warp's 32 rows. Lane l holds
// row l's 32 bf16 values (w, 16 words). They go through the warp's 2 KB
// staging block so that the global stores are row-contiguous: each store
// instruction writes 8 rows x 64 bytes (4 lanes per row, 16 bytes each), i.e.
// whole 32-byte sectors, instead of 32 rows x 16 bytes. In the staging block,
// rows 2p and 2p+1 share a 128-byte line and row r's 16-byte piece k sits in
// slot (r & 1) * 4 + (k ^ (p & 3)) of its line, so that neither the row-wise
// writes nor the piece-wise reads have bank conflicts.
__device__ __forceinline__ uint32_t stage_slot(int r, int k) {
    const int pr = r >> 1;
    return (uint32_t)((pr * 8 + (r & 1) * 4 + (k ^ (pr & 3))) * 16);
}

template <int D>
__device__ __forceinline__ void fwd_store_chunk(uint32_t stage, const uint32_t (&w)[16], int lane,
                                                uint16_t* o_rows, int c, int valid_rows,
                                                const uint16_t* o_end) {
    __syncwarp();   // the previous chunk's reads of the staging block are done
#pragma unroll
    for (int k = 0; k < 4; ++k)
        st_shared_v4(stage + stage_slot(lane, k), w[4 * k], w[4 * k + 1], w[4 * k + 2],
                     w[4 * k + 3]);
    __syncwarp();
    // all four pieces read from the staging block first, then the four stores
    uint4 val[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) val[i] = ld_shared_v4(stage + stage_slot(i * 8 + (lane >> 2), lane & 3));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = i * 8 + (lane >> 2), k = lane & 3;
        uint16_t* dst = o_rows + (size_t)r * D + c + 8 * k;
        if (r < valid_rows && dcheck(dst + 8 <= o_end)) *reinterpret_cast<uint4*>(dst) = val[i];
    }
}

template <int D, bool CAUSAL, bool FP8>
__device__ void fwd_softmax(const FwdParams& p, uint32_t tbase,
                            const FwdBars<FwdTraits<D, FP8>::kSlots>& b, int warp, int lane,
                            volatile int* abort_flag, const CUtensorMap* tmo) {
    using T = FwdTraits<D, FP8>;
    const int t = warp >> 2;                 // which Q tile
    const int quarter = warp & 3;            // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;       // row within the tile = TMEM lane
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t tO = tbase + lane_off + (t ? T::kColO1 : T::kColO0);
    const uint32_t bar_plo = b.p_lo(t), bar_phi = b.p_hi(t);
    const uint32_t bar_of = b.o_final(t), bar_ofree = b.o_free(t);
    uint32_t s_cnt = 0, o_use = 0;
    uint32_t p_cnt = 0;       // P_t tiles handed over so far (= P_t V products issued or due)
    uint32_t s_base = 0;      // score products issued in earlier units (three buffers)

    for (uint32_t k = 0;; ++k) {
        int u;
        const bool ok = fwd_next_unit(p, b, k, false, abort_flag, &u);
        __syncwarp();
        if (lane == 0 && ok && p.dynamic_units) mbar_arrive(b.unit_empty(k & 1));
        if (!__all_sync(0xffffffffu, ok)) return;
        if (u < 0) break;
        const FwdUnit x = fwd_unit<CAUSAL>(u, p);
        // scores in log2 units; e4m3 inputs fold their Q and K factors in here
        const float c2 = FP8 ? p.scale_log2 * p.q_descale[x.bh] * p.k_descale[x.bh]
                             : p.scale_log2;
        const int n = x.n[t];
        // sequence lengths are at most 2^30, so row indices and limits fit in int
        const int qrow = x.qb * 256 + t * 128 + r;
        const bool row_valid = qrow < p.Nq;
        int kv_lim = p.Nkv;         // keys [0, kv_lim) are visible to this row
        if (CAUSAL) kv_lim = min(kv_lim, qrow + (p.Nkv - p.Nq) + 1);
        float m_ref = -INFINITY;    // reference max, log2 units (scaled)
        float l = 0.f;              // running sum of 2^(s*c2 - m_ref)

        for (int j = 0; j < n; ++j) {
            // the TMEM columns holding S_t(j), and then P_t(j)
            const uint32_t tS =
                tbase + lane_off +
                (T::kSBufs == 3 ? ((s_base + fwd_s_pos(x, t, j)) % 3) * 128
                                : (t ? T::kColS1 : T::kColS0));
            // P_t(j): over S_t(j)'s first columns, or in its own columns (kSplit)
            const uint32_t tP = T::kSplit ? tbase + lane_off + (t ? T::kColP1 : T::kColP0) : tS;
            if (!warp_wait(b.template s_bar<T::kSBufs>(t, s_cnt),
                           FwdBars<T::kSlots>::template s_parity<T::kSBufs>(s_cnt), abort_flag))
                return;
            ++s_cnt;
            tc_fence_after_sync();
            uint32_t sr[128];
            tmem_ld128(tS, sr);
            tmem_wait_ld128(sr);
            if (T::kSplit)   // S_t(j) is in registers: its issuer may compute S_t(j+1) over it
                softmax_arrive<T::kWarpArrive>(b.s_full_b(t), lane);
            {
                // columns c >= lim of this tile are masked (-inf) for this row
                const int lim = max(-1, min(128, kv_lim - j * 128));
                if (lim < 128) {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
                }
            }
            float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
            for (int c = 0; c < 128; c += 8) {
                mx0 = fmax3(mx0, __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
                mx1 = fmax3(mx1, __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
                mx2 = fmax3(mx2, __uint_as_float(sr[c + 4]), __uint_as_float(sr[c + 5]));
                mx3 = fmax3(mx3, __uint_as_float(sr[c + 6]), __uint_as_float(sr[c + 7]));
            }
            const float mxs = fmax3(mx0, mx1, fmaxf(mx2, mx3)) * c2;
            const bool need = mxs > m_ref + T::kLazy;
            const bool any_need = __any_sync(0xffffffffu, need);
            const float m_new = need ? mxs : m_ref;
            const float alpha = need ? fast_exp2(m_ref - m_new) : 1.0f;
            m_ref = m_new;
            const float base = (m_ref == -INFINITY) ? 0.f : m_ref - T::kShift;
            const f32x2_t c2x2 = f2_pack(c2, c2);
            const f32x2_t nbx2 = f2_pack(-base, -base);
            f32x2_t lsum_a = f2_pack(0.f, 0.f), lsum_b = f2_pack(0.f, 0.f);
            // bf16 with EATTN_P_STORE_ONCE: both halves' P words, stored together
            [[maybe_unused]] uint32_t pk_all[(EATTN_P_STORE_ONCE && !FP8) ? 64 : 1];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t pk[FP8 ? 16 : 32];     // bf16 pairs or e4m3 quads
                float e_prev0 = 0.f, e_prev1 = 0.f;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int c = 64 * h + 2 * i;
                    const f32x2_t xv = f2_fma(
                        f2_pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), c2x2, nbx2);
                    float e0, e1;
                    if (kPolyEvery<D, FP8> > 0 &&
                               (i % (kPolyEvery<D, FP8> > 0 ? kPolyEvery<D, FP8> : 1)) == kPolyEvery<D, FP8> - 1) {
                        exp2_poly_pair(xv, e0, e1);
                    } else {
                        float x0, x1;
                        f2_unpack(xv, x0, x1);
                        e0 = fast_exp2(x0);
                        e1 = fast_exp2(x1);
                    }
                    if constexpr (!FP8) {
                        pk[i] = pack_bf16x2(e0, e1);
                    } else if (i & 1) {
                        pk[i / 2] = pack_e4m3x4(e_prev0, e_prev1, e0, e1);
                    } else {
                        e_prev0 = e0;
                        e_prev1 = e1;
                    }
                    if (i & 1)
                        lsum_b = f2_add(lsum_b, f2_pack(e0, e1));
                    else
                        lsum_a = f2_add(lsum_a, f2_pack(e0, e1));
                }
                // One issuer per tile: P_t(j) overwrites P_t(j-1), so P_t(j-1) V must be
                // complete (it is issued as soon as P_t(j-1) is handed over, a whole
                // softmax earlier, so this wait rarely waits); the rescale below
                // needs the same product complete.
                if (T::kSplit && h == 0 && j > 0 &&
                    !warp_wait(b.pv_done(t), (p_cnt - 1) & 1, abort_flag))
                    return;
                if (h == 0 && any_need && j > 0) {
                    // Rescale O_t by alpha (1 for rows whose max did not move)
                    // before any of P_t(j) V is released. O_t must hold P_t(j-1) V:
                    // with two score buffers the commit that signalled S_t(j)
                    // covers it; with three, S_t(j) was issued before it, so wait
                    // for its own completion (P_t(j) is not released yet, so that
                    // barrier cannot be a phase further on).
                    if (T::kSBufs == 3 && !T::kSplit &&
                        !warp_wait(b.pv_done(t), (p_cnt - 1) & 1, abort_flag))
                        return;
                    tc_fence_after_sync();
#pragma unroll
                    for (int c = 0; c < D; c += 32) {
                        uint32_t orr[32];
                        tmem_ld32(tO + c, orr);
                        tmem_wait_ld(orr);
#pragma unroll
                        for (int q = 0; q < 32; ++q)
                            orr[q] = __float_as_uint(__uint_as_float(orr[q]) * alpha);
                        tmem_st32(tO + c, orr);
                    }
                }
                if constexpr (FP8) {
                    tmem_st16(tP + 16 * h, pk);
                } else if constexpr (EATTN_P_STORE_ONCE) {
#pragma unroll
                    for (int q = 0; q < 32; ++q) pk_all[32 * h + q] = pk[q];
                    if (h == 1) tmem_st64(tP, pk_all);
                } else {
                    tmem_st32(tP + 32 * h, pk);
                }
                if (EATTN_SPLIT_P || h == 1) {
                    tmem_wait_st();
                    // three score buffers: P_t tiles alternate between p_hi and p_lo
                    softmax_arrive<T::kWarpArrive>(T::kSBufs == 3 ? ((p_cnt & 1) ? bar_plo : bar_phi)
                                                  : (h == 0 ? bar_plo : bar_phi),
                                   lane);
                }
            }
            ++p_cnt;
            float la0, la1, lb0, lb1;
            f2_unpack(lsum_a, la0, la1);
            f2_unpack(lsum_b, lb0, lb1);
            l = l * alpha + ((la0 + la1) + (lb0 + lb1));
        }

        s_base += x.n[0] + x.n[1];
        uint16_t* orow = p.o + ((size_t)x.bh * p.Nq + (size_t)(row_valid ? qrow : 0)) * D;
        // A row that sees no key at all (causal with Nq > Nkv) is O = 0, LSE = -inf by
        // definition; its polynomial exponentials of -inf scores are tiny, not zero.
        if (kv_lim <= 0) l = 0.f;
        if (n > 0) {
            if (!warp_wait(bar_of, o_use & 1, abort_flag)) return;
            tc_fence_after_sync();
            const float inv = l > 0.f ? (FP8 ? p.v_descale[x.bh] : 1.0f) / l : 0.f;
            // this warp's 32 rows: the first one and how many of them exist
            const int row0 = x.qb * 256 + t * 128 + quarter * 32;
            const int valid_rows = min(32, p.Nq - row0);
            uint16_t* o_rows = p.o + ((size_t)x.bh * p.Nq + (size_t)max(row0, 0)) * D;
            // the staging blocks sit right below the barriers
            const uint32_t stage = b.base - T::kStageBytes + warp * T::kStageWarpBytes;
            if constexpr (T::kTmaStoreO) {
                // per 64 columns: rows into the block (row = lane, 16-byte piece
                // q at position q ^ (lane % 8): the 128-byte swizzle of the O map),
                // then one TMA store of the 32 x 64 box by lane 0
#pragma unroll 1
                for (int cb = 0; cb < D; cb += 64) {
                    if (lane == 0) bulk_wait_read_all();   // the block's last store has read it
                    __syncwarp();
#pragma unroll
                    for (int ch = 0; ch < 64; ch += 32) {
                        uint32_t orr[32];
                        tmem_ld32(tO + cb + ch, orr);
                        tmem_wait_ld(orr);
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) {
                            const int q = (ch >> 3) + k4;
                            st_shared_v4(stage + lane * 128 + ((q ^ (lane & 7)) << 4),
                                         pack_bf16x2(__uint_as_float(orr[8 * k4]) * inv,
                                                     __uint_as_float(orr[8 * k4 + 1]) * inv),
                                         pack_bf16x2(__uint_as_float(orr[8 * k4 + 2]) * inv,
                                                     __uint_as_float(orr[8 * k4 + 3]) * inv),
                                         pack_bf16x2(__uint_as_float(orr[8 * k4 + 4]) * inv,
                                                     __uint_as_float(orr[8 * k4 + 5]) * inv),
                                         pack_bf16x2(__uint_as_float(orr[8 * k4 + 6]) * inv,
                                                     __uint_as_float(orr[8 * k4 + 7]) * inv));
                        }
                    }
                    fence_async_shared();
                    __syncwarp();
                    if (lane == 0 && valid_rows > 0 &&
                        dcheck(x.bh < p.BH && row0 >= 0 && row0 < p.Nq && cb + 64 <= D)) {
                        tma_store_3d(tmo, stage, cb, row0, x.bh);
                        bulk_commit_group();
                    }
                }
            } else {
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    uint32_t orr[32];
                    tmem_ld32(tO + c, orr);
                    tmem_wait_ld(orr);
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        w[i] = pack_bf16x2(__uint_as_float(orr[2 * i]) * inv,
                                           __uint_as_float(orr[2 * i + 1]) * inv);
                    if (EATTN_STAGE_O) {
                        fwd_store_chunk<D>(stage, w, lane, o_rows, c, valid_rows,
                                           p.o + (size_t)p.BH * p.Nq * D);
                    } else if (row_valid && dcheck(x.bh < p.BH)) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4)
                            dst[k4] =
                                make_uint4(w[4 * k4], w[4 * k4 + 1], w[4 * k4 + 2], w[4 * k4 + 3]);
                    }
                }
            }
            softmax_arrive<T::kWarpArrive>(bar_ofree, lane);
            ++o_use;
        } else if (row_valid && dcheck(x.bh < p.BH)) {
            uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
            for (int k = 0; k < D / 8; ++k) dst[k] = make_uint4(0, 0, 0, 0);
        }
        if (row_valid && dcheck(x.bh < p.BH))
            p.lse[(size_t)x.bh * p.Nq + qrow] =
                l > 0.f ? (m_ref - T::kShift + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
}

// ---------------------------------------------------------------- kernel --
template <int D, bool CAUSAL, bool FP8 = false>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_o, const FwdParams p) {
    using T = FwdTraits<D, FP8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sQ = smem_addr(smem);
    const uint32_t sKV = sQ + T::kQBufs * T::kTileBytes;
    // epilogue staging blocks, then the barriers (fwd_softmax finds its block
    // kStageBytes below the barrier base)
    uint8_t* bar_ptr = smem + (T::kQBufs + T::kSlots) * T::kTileBytes + T::kStageBytes;
    const uint32_t bar0 = smem_addr(bar_ptr);
    FwdBars<T::kSlots> b;
    b.base = bar0;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_ptr + 8 * FwdBars<T::kSlots>::kCount);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    b.unit_ring_ptr = reinterpret_cast<uint8_t*>(tmem_holder + 2);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < T::kSlots; ++i) {
            mbar_init(b.kv_full(i), 1);
            mbar_init(b.kv_empty(i), T::kSplit ? 2 : 1);   // one arrival per issuing thread
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(b.q_full(t), 1);
            mbar_init(b.q_empty(t), 1);
            mbar_init(b.s_full(t), 1);
            mbar_init(b.p_lo(t), T::kArrivals);
            mbar_init(b.p_hi(t), T::kArrivals);
            mbar_init(b.o_final(t), 1);
            mbar_init(b.o_free(t), T::kArrivals);
        }
        mbar_init(b.drain(), T::kSplit ? 2 : 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(b.unit_full(i), 1);
            mbar_init(b.unit_empty(i), T::kUnitReaders);
            mbar_init(b.s_full_b(i), T::kSplit ? T::kArrivals : 1);   // kSplit: "S_t free"
            mbar_init(b.pv_done(i), 1);
            mbar_init(b.q_full(2 + i), 1);
            mbar_init(b.q_empty(2 + i), 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 8 && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        if (T::kTmaStoreO) tma_prefetch_desc(&tm_o);
    }
    if (warp == 9) {
        tmem_alloc(smem_addr(tmem_holder), T::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tbase = *tmem_holder;

    if (warp < 8) {
        regs_increase<T::kSoftmaxRegs>();
        fwd_softmax<D, CAUSAL, FP8>(p, tbase, b, warp, lane, abort_flag, &tm_o);
        // every exit of the softmax role: its O stores must be complete (their
        // staging blocks are read and the writes done) before the CTA ends
        if (T::kTmaStoreO && lane == 0) bulk_wait_all();
    } else {
        regs_decrease<T::kOtherRegs>();
        const bool issuer_thread = EATTN_WARP_ISSUE ? true : lane == 0;
        if (warp == 8 && issuer_thread)
            fwd_producer<D, CAUSAL, FP8>(p, &tm_q, &tm_k, &tm_v, sQ, sKV, b, lane == 0, abort_flag);
        else if constexpr (T::kSplit) {
            if ((warp == 9 || warp == 10) && issuer_thread)   // warp 9: tile 0, warp 10: tile 1
                fwd_mma_split<D, CAUSAL, FP8>(p, tbase, sQ, sKV, b, lane == 0, abort_flag, warp - 9);
        } else if (warp == 9 && issuer_thread) {
            if constexpr (T::kSBufs == 3)
                fwd_mma_ahead<D, CAUSAL, FP8>(p, tbase, sQ, sKV, b, lane == 0, abort_flag);
            else
                fwd_mma<D, CAUSAL, FP8>(p, tbase, sQ, sKV, b, lane == 0, abort_flag);
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 9) {
        __syncwarp();
        tmem_dealloc(tbase, T::kTmemCols);
    }
    // Every role of this CTA is done, so its producer has made its last fetch.
    // The CTA that finishes last returns the queue to zero for the next launch.
    if (threadIdx.x == 0 && p.dynamic_units) {
        int* q = &g_fwd_queues[2 * p.queue_slot];
        __threadfence();
        if (atomicAdd(q + 1, 1) == (int)gridDim.x - 1) {
            atomicExch(q, 0);
            atomicExch(q + 1, 0);
        }
    }
}

}  // namespace eattn
