// bwd_sm100.cuh -- exact attention backward pass for B200, sm_100a.
//
// What it computes: the gradients of L = sum(dO * O) with respect to Q, K and
// V for O = softmax(scale * Q K^T [+ causal mask]) V, recomputing the score
// and probability tiles from Q, K and the forward pass's LSE instead of
// reading a stored P ("Describe Flash Attention at a high level"
// (mantramindai), "The two ideas", item 3: recompute in backward; "How
// FlashAttention Speeds Up the Attention Layer" (hassanahmed.net), the
// backward-pass paragraph). With P = exp(scale * S - LSE):
//   dV = P^T dO;  dP = dO V^T;  D_i = sum_c dO_ic O_ic;  dS = P o (dP - D);
//   dQ = scale * dS K;  dK = scale * dS^T Q.
//
// Three kernels, four in the deterministic form:
//   0. (deterministic form) attn_bwd_kv_bound: the largest |K| element and the
//      largest V row norm, for the dQ accumulator's fixed-point scale (below);
//   1. attn_bwd_preprocess: D = rowsum(dO o O) and LSE * log2(e) into padded
//      per-head rows (so a 64-row block of either is one aligned 256-byte
//      copy), zeroing of the dQ accumulator and (deterministic form) the
//      largest dO row norm;
//   2. attn_bwd_sm100: one CTA per (batch*head, 128-key block j), looping over
//      the 64-row query blocks that can see block j, computed transposed:
//      S^T = K_j Q_i^T and dP^T = V_j dO_i^T (M = the 128 keys, N = 64
//      queries), so that one thread owns one key row of P^T and dS^T and both
//      can stay in tensor memory as the A operand of dV += P^T dO_i and
//      dK += dS^T Q_i. dS^T also goes to shared memory as the B operand of
//      dQ_i^T = K_j^T dS^T (M = head dim), whose rows two reduction warpgroups
//      add into the dQ accumulator. Two tensor-memory stages let the tensor
//      core work on one query block while the P/dS warps work on the next.
//   3. attn_bwd_postprocess: dQ = bf16(scale * accumulator).
// The dQ accumulator is fp32, added to with fp32 atomics, so the last bits of
// dQ depend on the order in which the CTAs add. The deterministic form
// (attn_bwd_deterministic) makes it fixed point instead: int64 multiples of
// 2^-F, added with integer atomics; integer addition is exact and
// associative, so dQ is the same bits whatever the order. F is set per launch
// from a bound on every partial sum of dQ_ic / scale, from the inputs alone:
//   |sum_j dS_ij K_jc| <= max|K| * sum_j P_ij |dP_ij - D_i|
//                      <= max|K| * (max_j |dO_i . V_j| + |dO_i . O_i|)
//                      <= 2 max|K| max_i ||dO_i|| max_j ||V_j||
// (Cauchy-Schwarz, sum_j P_ij <= 1, and O_i a convex combination of the V_j);
// with a factor 2 for the bf16 rounding of P, dS and O, the bound B gives
// F = 61 - ceil(log2 2B), so every partial sum times 2^F stays below 2^61
// and the rounding of a contribution to the grid (2^-F / 2 <= B 2^-62) is far
// below bf16's resolution of dQ.
// Every mbarrier wait is bounded, as in the forward kernel.
#pragma once

#include <cstdint>

#include "ptx_sm100.cuh"
#include "tmem_wide.cuh"

namespace eattn {

struct BwdParams {
    const uint16_t* o;     // bf16 [BH, Nq, D]   (preprocess)
    const uint16_t* dout;  // bf16 [BH, Nq, D]   (preprocess)
    const float* lse;      // fp32 [BH, Nq]      (preprocess)
    float* delta;          // fp32 [BH, NqPad]: D_i, 0 past Nq
    float* lse2;           // fp32 [BH, NqPad]: LSE_i * log2(e); +inf past Nq or with no key
    void* dq_acc;          // [BH, Nq, D]: fp32, or int64 multiples of 2^-F (deterministic)
    int deterministic;     // 1: the fixed-point dQ accumulator
    unsigned* bound;       // [3]: max|K|, max ||dO_i||, max ||V_j|| (fp32 bits; zeroed first)
    const uint16_t* k;     // bf16 [BH, Nkv, D]  (kv_bound)
    const uint16_t* v;     // bf16 [BH, Nkv, D]  (kv_bound)
    uint16_t* dq;          // bf16 [BH, Nq, D]
    uint16_t* dk;          // bf16 [BH, Nkv, D]
    uint16_t* dv;          // bf16 [BH, Nkv, D]
    int BH, Nq, Nkv;
    int NqPad;             // Nq rounded up to a multiple of 64
    float scale;           // softmax scale
    float scale_log2;      // scale * log2(e)
};

// ------------------------------------------------------------- dQ bound --
// Largest of v over the warp, folded into *dst (v >= 0, so the fp32 bits of
// non-negative values order like the values).
__device__ __forceinline__ void bwd_max_into(unsigned* dst, float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    if ((threadIdx.x & 31) == 0) atomicMax(dst, __float_as_uint(v));
}

// F of the dQ accumulator's grid 2^-F (see the file header), from the three
// maxima: with 2B = m 2^e, m in [1, 2) (e the unbiased exponent), 2B < 2^(e+1).
__device__ __forceinline__ int bwd_dq_exponent(const unsigned* bound) {
    const float b = 2.f * __uint_as_float(bound[0]) * __uint_as_float(bound[1]) *
                    __uint_as_float(bound[2]);
    const int e = (int)((__float_as_uint(2.f * b) >> 23) & 0xFFu) - 127;
    return min(120, max(-60, 60 - e));
}
// 2^f as an fp32 bit pattern, f in [-126, 127]
__device__ __forceinline__ float bwd_pow2(int f) { return __uint_as_float((uint32_t)(f + 127) << 23); }

__device__ __forceinline__ float bwd_bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bwd_bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// One thread per 8 elements of a K and a V row; D/8 threads per row; rows of
// [BH, Nkv].
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_kv_bound_kernel(const BwdParams p) {
    constexpr int LPR = D / 8;
    const long long row = (long long)blockIdx.x * (256 / LPR) + threadIdx.x / LPR;
    const int cc = threadIdx.x % LPR;
    float kmax = 0.f, vsq = 0.f;
    if (row < (long long)p.BH * p.Nkv) {
        const uint4 a = *reinterpret_cast<const uint4*>(p.k + row * D + cc * 8);
        const uint4 g = *reinterpret_cast<const uint4*>(p.v + row * D + cc * 8);
        const uint32_t av[4] = {a.x, a.y, a.z, a.w}, gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            kmax = fmaxf(kmax, fmaxf(fabsf(bwd_bf16_lo(av[k])), fabsf(bwd_bf16_hi(av[k]))));
            vsq = fmaf(bwd_bf16_lo(gv[k]), bwd_bf16_lo(gv[k]), vsq);
            vsq = fmaf(bwd_bf16_hi(gv[k]), bwd_bf16_hi(gv[k]), vsq);
        }
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) vsq += __shfl_xor_sync(0xffffffffu, vsq, off);
    bwd_max_into(&p.bound[0], kmax);
    bwd_max_into(&p.bound[2], sqrtf(vsq));
}

// ------------------------------------------------------------ preprocess --
// One thread per 8 elements of a row; D/8 threads per row; rows of [BH, NqPad].
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_preprocess_kernel(const BwdParams p) {
    constexpr int LPR = D / 8;
    constexpr float kLog2e = 1.4426950408889634f;
    const long long row = (long long)blockIdx.x * (256 / LPR) + threadIdx.x / LPR;
    const int cc = threadIdx.x % LPR;
    const bool in_range = row < (long long)p.BH * p.NqPad;
    const long long bh = in_range ? row / p.NqPad : 0;
    const int i = in_range ? (int)(row % p.NqPad) : 0;
    const bool real = in_range && i < p.Nq && dcheck(bh < p.BH);
    const long long grow = bh * p.Nq + i;
    float acc = 0.f, gsq = 0.f;
    if (real) {
        const uint4 a = *reinterpret_cast<const uint4*>(p.o + grow * D + cc * 8);
        const uint4 g = *reinterpret_cast<const uint4*>(p.dout + grow * D + cc * 8);
        const uint32_t av[4] = {a.x, a.y, a.z, a.w}, gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            acc = fmaf(bwd_bf16_lo(av[k]), bwd_bf16_lo(gv[k]), acc);
            acc = fmaf(bwd_bf16_hi(av[k]), bwd_bf16_hi(gv[k]), acc);
            gsq = fmaf(bwd_bf16_lo(gv[k]), bwd_bf16_lo(gv[k]), gsq);
            gsq = fmaf(bwd_bf16_hi(gv[k]), bwd_bf16_hi(gv[k]), gsq);
        }
        // 8 elements of 4 or 8 bytes
        uint4* z = reinterpret_cast<uint4*>(static_cast<char*>(p.dq_acc) +
                                            (grow * D + cc * 8) * (p.deterministic ? 8 : 4));
        for (int k = 0; k < (p.deterministic ? 4 : 2); ++k) z[k] = make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) {
        acc += __shfl_xor_sync(0xffffffffu, acc, off);
        gsq += __shfl_xor_sync(0xffffffffu, gsq, off);
    }
    if (p.deterministic) bwd_max_into(&p.bound[1], sqrtf(gsq));
    if (in_range && cc == 0) {
        p.delta[row] = real ? acc : 0.f;
        // a row with no visible key (LSE = -inf) or past Nq gets P = 2^(s - inf) = 0
        const float l = real ? p.lse[grow] : -INFINITY;
        p.lse2[row] = (l == -INFINITY) ? INFINITY : l * kLog2e;
    }
}

// ----------------------------------------------------------- postprocess --
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_postprocess_kernel(const BwdParams p) {
    const long long i = ((long long)blockIdx.x * 256 + threadIdx.x) * 8;
    if (i >= (long long)p.BH * p.Nq * D) return;
    float f[8];
    if (p.deterministic) {
        // scale * 2^-F: a power of two times scale, exact in fp32 for F in [-60, 120]
        const float s = p.scale * bwd_pow2(-bwd_dq_exponent(p.bound));
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const longlong2 a = reinterpret_cast<const longlong2*>(p.dq_acc)[i / 2 + k];
            f[2 * k] = __ll2float_rn(a.x) * s;
            f[2 * k + 1] = __ll2float_rn(a.y) * s;
        }
    } else {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const float4 a = reinterpret_cast<const float4*>(p.dq_acc)[i / 4 + k];
            f[4 * k] = a.x * p.scale;
            f[4 * k + 1] = a.y * p.scale;
            f[4 * k + 2] = a.z * p.scale;
            f[4 * k + 3] = a.w * p.scale;
        }
    }
    *reinterpret_cast<uint4*>(p.dq + i) =
        make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                   pack_bf16x2(f[6], f[7]));
}

// ------------------------------------------------------------ main kernel --
template <int D>
struct BwdTraits {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int kQRows = 64;                   // query rows per step
    static constexpr int kKPanel = 128 * 128;           // 128 key rows x 128 bytes
    static constexpr int kKTile = (D / 64) * kKPanel;   // K_j or V_j
    static constexpr int kQPanel = 64 * 128;            // 64 query rows x 128 bytes
    static constexpr int kQTile = (D / 64) * kQPanel;   // Q_i or dO_i
    static constexpr int kStages = 3;                   // Q_i, dO_i, LSE/D ring depth
    static constexpr int kLDBytes = 2 * kQRows * 4;     // LSE*log2e and D of 64 rows
    static constexpr int kDSBytes = 128 * kQRows * 2;   // dS^T: 128 keys x 64 queries bf16
    // warps 0-7 P/dS, 8-15 dQ reduction (8-11 query columns 0-31 of a step,
    // 12-15 columns 32-63), 16 TMA, 17 MMA, 18-19 idle
    static constexpr int kThreads = 640;
    static constexpr int kComputeThreads = 256;
    static constexpr int kReduceThreads = 256;
    // Registers: the launch gives every thread kLaunchRegs (the build checks
    // that ptxas gave the kernel exactly that many); setmaxnreg then moves them
    // to the P/dS warpgroups. The split must fit the launch's total, and per
    // SM scheduler (warps w, w+4, w+8, w+12, w+16) the 16384-register file.
    static constexpr int kLaunchRegs = 96;
    static constexpr int kPdsRegs = 120, kRedRegs = 80, kOtherRegs = 72;
    static_assert(256 * kPdsRegs + 256 * kRedRegs + 128 * kOtherRegs <= kThreads * kLaunchRegs,
                  "register split exceeds the launch allocation");
    static_assert((2 * kPdsRegs + 2 * kRedRegs + kOtherRegs) * 32 <= 16384,
                  "register split exceeds a scheduler's register file");
    static constexpr int kNumBars = 16;
    static constexpr int kSmemBytes = 1024 + 2 * kKTile + kStages * (2 * kQTile + kLDBytes) +
                                      2 * kDSBytes + kNumBars * 8 + 16;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static constexpr uint32_t kTmemCols = 512;
    // TMEM: dV [0, D), dK [D, 2D), then two stages of 128 columns each:
    //   [0, 64)   S^T (fp32), later dQ^T (fp32, M = head dim)
    //   [64, 128) dP^T (fp32); P^T and dS^T (bf16 pairs) overwrite it, query
    //             block k of 16 at columns 16k (P^T) and 16k + 8 (dS^T)
    static constexpr uint32_t kColDV = 0, kColDK = D;
    __host__ __device__ static constexpr uint32_t col_stage(int b) { return 2 * D + 128 * b; }
};

// mbarriers (arrival count): kv_full(1), qd_full[3](1), qd_empty[3](1), s_full[2](1),
// p_ready[2](256), dq_full[2](1), dq_free[2](128), fin(1)
struct BwdBars {
    uint32_t base;
    __device__ __forceinline__ uint32_t kv_full() const { return base; }
    __device__ __forceinline__ uint32_t qd_full(int st) const { return base + 8 * (1 + st); }
    __device__ __forceinline__ uint32_t qd_empty(int st) const { return base + 8 * (4 + st); }
    __device__ __forceinline__ uint32_t s_full(int b) const { return base + 8 * (7 + b); }
    __device__ __forceinline__ uint32_t p_ready(int b) const { return base + 8 * (9 + b); }
    __device__ __forceinline__ uint32_t dq_full(int b) const { return base + 8 * (11 + b); }
    __device__ __forceinline__ uint32_t dq_free(int b) const { return base + 8 * (13 + b); }
    __device__ __forceinline__ uint32_t fin() const { return base + 8 * 15; }
};

// First 64-row query block that sees key block j (bottom-right causal alignment).
template <bool CAUSAL>
__device__ __forceinline__ int bwd_first_qblock(int j, const BwdParams& p) {
    if (!CAUSAL) return 0;
    const long long first_row = (long long)j * 128 - ((long long)p.Nkv - p.Nq);
    return first_row <= 0 ? 0 : (int)(first_row / 64);
}

__device__ __forceinline__ void red_add_f32(float* addr, float v) {
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(v) : "memory");
}
// Adds v, rounded to the accumulator's grid (v * 2^F to the nearest integer),
// to a fixed-point dQ element.
__device__ __forceinline__ void red_add_fixed(long long* addr, float v, float two_f) {
    const long long x = __float2ll_rn(v * two_f);
    asm volatile("red.global.add.u64 [%0], %1;" ::"l"(addr), "l"(x) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(640, 1)
    attn_bwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
    using T = BwdTraits<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sK = smem_addr(smem);
    const uint32_t sV = sK + T::kKTile;
    const uint32_t sQ0 = sV + T::kKTile;                    // Q stage st at sQ0 + st * kQTile
    const uint32_t sDO0 = sQ0 + T::kStages * T::kQTile;
    const uint32_t sDS0 = sDO0 + T::kStages * T::kQTile;    // dS^T buffer x at sDS0 + x * kDSBytes
    const uint32_t sLD0 = sDS0 + 2 * T::kDSBytes;           // LSE/D stage st at sLD0 + st * kLDBytes
    uint8_t* ld_ptr = smem + (sLD0 - sK);
    uint8_t* bar_ptr = ld_ptr + T::kStages * T::kLDBytes;
    BwdBars b;
    b.base = smem_addr(bar_ptr);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_ptr + 8 * T::kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // Launch order (x fastest, then y) -> (key block, head): heads in groups of
    // kHeadGroup, and within a group the key blocks in order, each for every head
    // of the group. Under the causal mask the early key blocks are the heavy ones,
    // so the CTAs left to run at the end are light, while the CTAs resident at
    // one time still share a few heads' Q and dO in L2.
    constexpr int kHeadGroup = 4;
    const int nkb = gridDim.x;
    const int lin = blockIdx.y * nkb + blockIdx.x;
    const int grp = lin / (kHeadGroup * nkb);
    const int heads_in_grp = min(kHeadGroup, p.BH - grp * kHeadGroup);
    const int rem = lin - grp * kHeadGroup * nkb;
    const int j = rem / heads_in_grp;                       // key block
    const int bh = grp * kHeadGroup + rem % heads_in_grp;
    const int i0 = bwd_first_qblock<CAUSAL>(j, p);
    const int nqb = (p.Nq + T::kQRows - 1) / T::kQRows;
    const int nsteps = nqb > i0 ? nqb - i0 : 0;

    if (threadIdx.x == 0) {
        mbar_init(b.kv_full(), 1);
        for (int st = 0; st < T::kStages; ++st) {
            mbar_init(b.qd_full(st), 1);
            mbar_init(b.qd_empty(st), 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(b.s_full(x), 1);
            mbar_init(b.p_ready(x), T::kComputeThreads);
            mbar_init(b.dq_full(x), 1);
            mbar_init(b.dq_free(x), T::kReduceThreads);
        }
        mbar_init(b.fin(), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 17) {
        tmem_alloc(smem_addr(tmem_holder), T::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tbase = *tmem_holder;

    if (warp >= 16) regs_decrease<T::kOtherRegs>();
    else if (warp >= 8) regs_decrease<T::kRedRegs>();
    else regs_increase<T::kPdsRegs>();

    if (warp == 16) {
        // ------------------------------------------------ TMA producer --
        if (lane == 0 && nsteps > 0) {
            int issued = 0;
            mbar_arrive_expect_tx(b.kv_full(), 2 * T::kKTile);
            for (int pn = 0; pn < D / 64; ++pn) {
                tma_load_3d(sK + pn * T::kKPanel, &tm_k, b.kv_full(), pn * 64, j * 128, bh);
                tma_load_3d(sV + pn * T::kKPanel, &tm_v, b.kv_full(), pn * 64, j * 128, bh);
            }
            for (int s = 0; s < nsteps; ++s) {
                const int st = s % T::kStages;
                if (s >= T::kStages &&
                    !mbar_wait(b.qd_empty(st), ((s / T::kStages) - 1) & 1, abort_flag,
                               &g_attn_status))
                    break;
                const int row0 = (i0 + s) * T::kQRows;
                const uint32_t bar = b.qd_full(st);
                mbar_arrive_expect_tx(bar, 2 * T::kQTile + T::kLDBytes);
                for (int pn = 0; pn < D / 64; ++pn) {
                    tma_load_3d(sQ0 + st * T::kQTile + pn * T::kQPanel, &tm_q, bar, pn * 64, row0,
                                bh);
                    tma_load_3d(sDO0 + st * T::kQTile + pn * T::kQPanel, &tm_do, bar, pn * 64,
                                row0, bh);
                }
                const size_t prow = (size_t)bh * p.NqPad + row0;   // 64-row aligned
                bulk_load(sLD0 + st * T::kLDBytes, p.lse2 + prow, T::kQRows * 4, bar);
                bulk_load(sLD0 + st * T::kLDBytes + T::kQRows * 4, p.delta + prow, T::kQRows * 4,
                          bar);
                ++issued;
            }
            // copies still in flight must land before the CTA can exit
            volatile int no_abort = 0;
            mbar_wait(b.kv_full(), 0, &no_abort, &g_attn_status);
            for (int st = 0; st < T::kStages; ++st) {
                const int cnt = (issued - st + T::kStages - 1) / T::kStages;   // loads into st
                if (cnt > 0) mbar_wait(b.qd_full(st), (cnt - 1) & 1, &no_abort, &g_attn_status);
            }
        }
    } else if (warp == 17) {
        // -------------------------------------------------- MMA issuer --
        if (lane == 0 && nsteps > 0) {
            constexpr uint32_t id_s = idesc_bf16_f32(128, T::kQRows, false);   // A, B K-major
            constexpr uint32_t id_kv = idesc_bf16_f32(128, D, true);           // B MN-major
            // dQ^T = K^T dS^T: A (K^T) and B (dS^T) both MN-major; M = 128 covers the
            // head dim (at d = 64 lanes 64-127 hold unused products)
            constexpr uint32_t id_q = idesc_bf16_f32(128, T::kQRows, true) | (1u << 15);
            const uint64_t aK = sdesc_sw128(sK, 16, 1024), aV = sdesc_sw128(sV, 16, 1024);
            const uint64_t aKt = sdesc_sw128(sK, T::kKPanel, 1024);
            bool ok = mbar_wait(b.kv_full(), 0, abort_flag, &g_attn_status);
            // S^T = K_j Q_i^T and dP^T = V_j dO_i^T for step s into tensor stage s & 1
            auto issue_s = [&](int s) -> bool {
                const int st = s % T::kStages, x = s & 1;
                if (!mbar_wait(b.qd_full(st), (s / T::kStages) & 1, abort_flag, &g_attn_status))
                    return false;
                if (s >= 2 &&
                    !mbar_wait(b.dq_free(x), ((s - 2) >> 1) & 1, abort_flag, &g_attn_status))
                    return false;
                tc_fence_after_sync();
                const uint64_t bQ = sdesc_sw128(sQ0 + st * T::kQTile, 16, 1024);
                const uint64_t bDO = sdesc_sw128(sDO0 + st * T::kQTile, 16, 1024);
                const uint32_t cs = tbase + T::col_stage(x);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t oa = ((kk / 4) * T::kKPanel + (kk % 4) * 32) >> 4;
                    const uint64_t ob = ((kk / 4) * T::kQPanel + (kk % 4) * 32) >> 4;
                    mma_bf16_ss(cs, aK + oa, bQ + ob, id_s, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t oa = ((kk / 4) * T::kKPanel + (kk % 4) * 32) >> 4;
                    const uint64_t ob = ((kk / 4) * T::kQPanel + (kk % 4) * 32) >> 4;
                    mma_bf16_ss(cs + 64, aV + oa, bDO + ob, id_s, kk > 0);
                }
                mma_commit(b.s_full(x));
                return true;
            };
            if (ok) ok = issue_s(0);
            if (ok && nsteps > 1) ok = issue_s(1);
            for (int s = 0; ok && s < nsteps; ++s) {
                const int st = s % T::kStages, x = s & 1;
                if (!mbar_wait(b.p_ready(x), (s >> 1) & 1, abort_flag, &g_attn_status)) break;
                tc_fence_after_sync();
                const uint32_t cs = tbase + T::col_stage(x);
                // dQ_i^T = K_j^T dS^T into the stage's first 64 columns (S^T was read);
                // K = 128 keys, 16 per MMA: 16 rows of K_j and of dS^T = 2048 bytes
                const uint64_t bDS = sdesc_sw128(sDS0 + x * T::kDSBytes, T::kDSBytes, 1024);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t off = (kk * 2048) >> 4;
                    mma_bf16_ss(cs, aKt + off, bDS + off, id_q, kk > 0);
                }
                mma_commit(b.dq_full(x));
                // dV += P^T dO_i and dK += dS^T Q_i, A from tensor memory (K = 64 queries)
                const uint64_t bDOt = sdesc_sw128(sDO0 + st * T::kQTile, T::kQPanel, 1024);
                const uint64_t bQt = sdesc_sw128(sQ0 + st * T::kQTile, T::kQPanel, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ts(tbase + T::kColDV, cs + 64 + 16 * kk, bDOt + ((kk * 2048) >> 4),
                                id_kv, (s > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ts(tbase + T::kColDK, cs + 64 + 16 * kk + 8,
                                bQt + ((kk * 2048) >> 4), id_kv, (s > 0 || kk > 0) ? 1u : 0u);
                mma_commit(b.qd_empty(st));
                if (s + 2 < nsteps) ok = issue_s(s + 2);
            }
            mma_commit(b.fin());
            // the CTA must not release tensor memory while products are in flight
            volatile int no_abort = 0;
            mbar_wait(b.fin(), 0, &no_abort, &g_attn_status);
        }
    } else if (warp >= 8 && warp < 16) {
        // ---------------- dQ reduction (warps 8-15, lane = head-dim index, 32 query columns) --
        const int quarter = warp & 3;
        const int cols = 32 * ((warp - 8) >> 2);   // this warp's first query column
        const int c = quarter * 32 + lane;
        const uint32_t lane_off = uint32_t(quarter * 32) << 16;
        const size_t head_off = (size_t)bh * p.Nq * D + (c < D ? c : 0);
        float* dq_head = static_cast<float*>(p.dq_acc) + head_off;
        long long* dq_head64 = static_cast<long long*>(p.dq_acc) + head_off;
        const float two_f = p.deterministic ? bwd_pow2(bwd_dq_exponent(p.bound)) : 0.f;
        for (int s = 0; s < nsteps; ++s) {
            const int x = s & 1;
            bool ok = mbar_wait(b.dq_full(x), (s >> 1) & 1, abort_flag, &g_attn_status);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after_sync();
            uint32_t v[32];
            tmem_ld32(tbase + lane_off + T::col_stage(x) + cols, v);
            tmem_wait_ld(v);
            tc_fence_before_sync();
            mbar_arrive(b.dq_free(x));
            const int row0 = (i0 + s) * T::kQRows + cols;
            if (quarter * 32 < D) {
                float* dq_rows = dq_head + (size_t)row0 * D;
                long long* dq_rows64 = dq_head64 + (size_t)row0 * D;
                const int nr = p.Nq - row0;   // rows of this block inside the head
                if (nr >= 32 && dcheck(row0 + 32 <= p.Nq && bh < p.BH)) {
                    if (p.deterministic) {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            red_add_fixed(dq_rows64 + e * D, __uint_as_float(v[e]), two_f);
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) red_add_f32(dq_rows + e * D, __uint_as_float(v[e]));
                    }
                } else if (nr < 32) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (e < nr) {
                            if (p.deterministic)
                                red_add_fixed(dq_rows64 + e * D, __uint_as_float(v[e]), two_f);
                            else
                                red_add_f32(dq_rows + e * D, __uint_as_float(v[e]));
                        }
                }
            }
        }
    } else if (warp < 8) {
        // --------------------- P^T and dS^T (warps 0-7: key row, 32-query half) --
        const int quarter = warp & 3;
        const int half = warp >> 2;
        const int r = quarter * 32 + lane;             // key row in the block = TMEM lane
        const uint32_t lane_off = uint32_t(quarter * 32) << 16;
        const int kg = j * 128 + r;
        const bool key_ok = kg < p.Nkv;
        const float c2 = p.scale_log2;
        uint8_t* ds_row0 = smem + (sDS0 - sK) + r * 128;
        bool ok = true;
        for (int s = 0; s < nsteps; ++s) {
            const int st = s % T::kStages, x = s & 1;
            const int row0 = (i0 + s) * T::kQRows;
            // query column q of this step is visible to the key iff q >= lo
            const int lo = CAUSAL ? kg - (p.Nkv - p.Nq) - row0 : -T::kQRows;
            if (!mbar_wait(b.qd_full(st), (s / T::kStages) & 1, abort_flag, &g_attn_status))
                ok = false;
            if (ok && !mbar_wait(b.s_full(x), (s >> 1) & 1, abort_flag, &g_attn_status))
                ok = false;
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after_sync();
            const uint32_t cs = tbase + lane_off + T::col_stage(x);
            const float* lse2 = reinterpret_cast<const float*>(ld_ptr + st * T::kLDBytes);
            const float* dl = lse2 + T::kQRows;
            uint8_t* ds_row = ds_row0 + x * T::kDSBytes;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                const int q0 = half * 32 + ch * 16;    // first query column of the chunk
                uint32_t sv[16], dp[16];
                tmem_ld16(cs + q0, sv);
                tmem_ld16(cs + 64 + q0, dp);
                tmem_wait_ld16(sv);
                tmem_wait_ld16(dp);
                uint32_t pw[8], dw[8];
#pragma unroll
                for (int e = 0; e < 16; e += 2) {
                    const int q = q0 + e;
                    const float p0 = (key_ok && q >= lo)
                                         ? fast_exp2(fmaf(__uint_as_float(sv[e]), c2, -lse2[q]))
                                         : 0.f;
                    const float p1 = (key_ok && q + 1 >= lo)
                                         ? fast_exp2(fmaf(__uint_as_float(sv[e + 1]), c2, -lse2[q + 1]))
                                         : 0.f;
                    pw[e / 2] = pack_bf16x2(p0, p1);
                    dw[e / 2] = pack_bf16x2(p0 * (__uint_as_float(dp[e]) - dl[q]),
                                            p1 * (__uint_as_float(dp[e + 1]) - dl[q + 1]));
                }
                // P^T and dS^T of these 16 queries over this chunk's own dP^T columns
                tmem_st8(cs + 64 + q0, pw);
                tmem_st8(cs + 64 + q0 + 8, dw);
                // dS^T row r of shared memory: 64 queries = one 128-byte swizzled row;
                // this chunk's two 16-byte pieces are chunks q0/8 and q0/8 + 1
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int chunk = (q0 / 8 + h2) ^ (r & 7);
                    *reinterpret_cast<uint4*>(ds_row + chunk * 16) =
                        make_uint4(dw[4 * h2], dw[4 * h2 + 1], dw[4 * h2 + 2], dw[4 * h2 + 3]);
                }
            }
            tmem_wait_st();
            fence_proxy_async_smem();     // generic-proxy writes -> tensor core reads
            tc_fence_before_sync();
            mbar_arrive(b.p_ready(x));
        }
        // dK and dV of this key block: TMEM lane = key row; each half writes D/2 columns
        constexpr int kHalfD = D / 2;
        uint16_t* dk_row = p.dk + ((size_t)bh * p.Nkv + (key_ok ? kg : 0)) * D + half * kHalfD;
        uint16_t* dv_row = p.dv + ((size_t)bh * p.Nkv + (key_ok ? kg : 0)) * D + half * kHalfD;
        if (nsteps == 0) {
            if (key_ok)
                for (int cc = 0; cc < kHalfD; cc += 8) {
                    *reinterpret_cast<uint4*>(dk_row + cc) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(dv_row + cc) = make_uint4(0, 0, 0, 0);
                }
        } else if (ok) {
            if (!mbar_wait(b.fin(), 0, abort_flag, &g_attn_status)) ok = false;
            if (__all_sync(0xffffffffu, ok)) {
                tc_fence_after_sync();
#pragma unroll
                for (int cc = 0; cc < kHalfD; cc += 16) {
                    uint32_t gk[16], gv[16];
                    tmem_ld16(tbase + lane_off + T::kColDK + half * kHalfD + cc, gk);
                    tmem_ld16(tbase + lane_off + T::kColDV + half * kHalfD + cc, gv);
                    tmem_wait_ld16(gk);
                    tmem_wait_ld16(gv);
                    uint32_t wk[8], wv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        wk[e] = pack_bf16x2(__uint_as_float(gk[2 * e]) * p.scale,
                                            __uint_as_float(gk[2 * e + 1]) * p.scale);
                        wv[e] = pack_bf16x2(__uint_as_float(gv[2 * e]), __uint_as_float(gv[2 * e + 1]));
                    }
                    if (key_ok) {
                        uint4* pk = reinterpret_cast<uint4*>(dk_row + cc);
                        uint4* pv = reinterpret_cast<uint4*>(dv_row + cc);
                        pk[0] = make_uint4(wk[0], wk[1], wk[2], wk[3]);
                        pk[1] = make_uint4(wk[4], wk[5], wk[6], wk[7]);
                        pv[0] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                        pv[1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
                    }
                }
            }
        }
    }

    __syncwarp();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 17) {
        tmem_dealloc(tbase, T::kTmemCols);
    }
}

}  // namespace eattn
