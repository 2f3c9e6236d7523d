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
// Three kernels:
//   1. attn_bwd_preprocess: D = rowsum(dO o O) (fp32) and zeroes the fp32 dQ
//      accumulator;
//   2. attn_bwd_sm100: one CTA per (batch*head, 128-key block j), looping over
//      the 128-row query blocks that can see block j. Tensor memory holds the
//      dV and dK accumulators of the block and the S = Q_i K_j^T and
//      dP = dO_i V_j^T tiles. Warps 0-7 (one thread per query row and column
//      half) turn S and dP into P and dS and write both, as bf16, to shared
//      memory in the 128-byte-swizzled [query][key] layout; that layout is at
//      once the MN-major A operand of P^T and dS^T and the K-major A operand of
//      dS. The MMA warp (9) then issues dV += P^T dO_i, dK += dS^T Q_i and the
//      dQ partial dS K_j (into the S columns), which warps 0-7 add into the
//      fp32 dQ accumulator with vector reductions. Warp 8 is the TMA producer;
//      Q is double-buffered so the next block's Q loads during this one.
//   3. attn_bwd_postprocess: dQ = bf16(scale * accumulator).
// Every mbarrier wait is bounded, as in the forward kernel.
#pragma once

#include <cstdint>

#include "ptx_sm100.cuh"
#include "tmem_wide.cuh"

namespace eattn {

struct BwdParams {
    const uint16_t* o;     // bf16 [BH, Nq, D]   (preprocess)
    const uint16_t* dout;  // bf16 [BH, Nq, D]   (preprocess)
    const float* lse;      // fp32 [BH, Nq]
    float* delta;          // fp32 [BH, Nq]
    float* dq_acc;         // fp32 [BH, Nq, D]
    uint16_t* dq;          // bf16 [BH, Nq, D]
    uint16_t* dk;          // bf16 [BH, Nkv, D]
    uint16_t* dv;          // bf16 [BH, Nkv, D]
    int BH, Nq, Nkv;
    float scale;           // softmax scale
    float scale_log2;      // scale * log2(e)
};

// ------------------------------------------------------------ preprocess --
// One thread per 8 elements of a row; D/8 threads per row.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_preprocess_kernel(const BwdParams p) {
    constexpr int LPR = D / 8;
    const long long row = (long long)blockIdx.x * (256 / LPR) + threadIdx.x / LPR;
    const int cc = threadIdx.x % LPR;
    const bool valid = row < (long long)p.BH * p.Nq;
    float acc = 0.f;
    if (valid) {
        const uint4 a = *reinterpret_cast<const uint4*>(p.o + row * D + cc * 8);
        const uint4 g = *reinterpret_cast<const uint4*>(p.dout + row * D + cc * 8);
        const uint32_t av[4] = {a.x, a.y, a.z, a.w}, gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc = fmaf(__uint_as_float(av[i] << 16), __uint_as_float(gv[i] << 16), acc);
            acc = fmaf(__uint_as_float(av[i] & 0xFFFF0000u), __uint_as_float(gv[i] & 0xFFFF0000u),
                       acc);
        }
        float4* z = reinterpret_cast<float4*>(p.dq_acc + row * D + cc * 8);
        z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (valid && cc == 0) p.delta[row] = acc;
}

// ----------------------------------------------------------- postprocess --
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_postprocess_kernel(const BwdParams p) {
    const long long i = ((long long)blockIdx.x * 256 + threadIdx.x) * 8;
    if (i >= (long long)p.BH * p.Nq * D) return;
    const float4 a = *reinterpret_cast<const float4*>(p.dq_acc + i);
    const float4 b = *reinterpret_cast<const float4*>(p.dq_acc + i + 4);
    const float s = p.scale;
    *reinterpret_cast<uint4*>(p.dq + i) =
        make_uint4(pack_bf16x2(a.x * s, a.y * s), pack_bf16x2(a.z * s, a.w * s),
                   pack_bf16x2(b.x * s, b.y * s), pack_bf16x2(b.z * s, b.w * s));
}

// ------------------------------------------------------------ main kernel --
template <int D>
struct BwdTraits {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int kPanelBytes = 128 * 64 * 2;         // 128 rows x 64 bf16
    static constexpr int kTileBytes = (D / 64) * kPanelBytes; // Q, K, V or dO tile
    static constexpr int kPBytes = 2 * kPanelBytes;           // P or dS: 128 x 128 bf16
    static constexpr int kQStages = 2;                        // Q is double-buffered
    static constexpr int kThreads = 320;  // warps 0-7 P/dS/dQ, 8 producer, 9 MMA issuer
    static constexpr int kComputeThreads = 256;
    static constexpr int kNumBars = 12;
    static constexpr int kSmemBytes =
        1024 + (3 + kQStages) * kTileBytes + 2 * kPBytes + kNumBars * 8 + 16;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColDV = 0, kColDK = D, kColS = 2 * D, kColDP = 2 * D + 128;
};

// mbarriers (count): kv_full(1), q_full[2](1), q_empty[2](1), do_full(1), do_empty(1),
// s_full(1), p_ready(256), dq_full(1), dq_free(256), fin(1)
struct BwdBars {
    uint32_t base;
    __device__ __forceinline__ uint32_t kv_full() const { return base; }
    __device__ __forceinline__ uint32_t q_full(int b) const { return base + 8 + 8 * b; }
    __device__ __forceinline__ uint32_t q_empty(int b) const { return base + 24 + 8 * b; }
    __device__ __forceinline__ uint32_t do_full() const { return base + 40; }
    __device__ __forceinline__ uint32_t do_empty() const { return base + 48; }
    __device__ __forceinline__ uint32_t s_full() const { return base + 56; }
    __device__ __forceinline__ uint32_t p_ready() const { return base + 64; }
    __device__ __forceinline__ uint32_t dq_full() const { return base + 72; }
    __device__ __forceinline__ uint32_t dq_free() const { return base + 80; }
    __device__ __forceinline__ uint32_t fin() const { return base + 88; }
};

// First query block that sees key block j (bottom-right causal alignment).
template <bool CAUSAL>
__device__ __forceinline__ int bwd_first_qblock(int j, const BwdParams& p) {
    if (!CAUSAL) return 0;
    const long long first_row = (long long)j * 128 - ((long long)p.Nkv - p.Nq);
    return first_row <= 0 ? 0 : (int)(first_row / 128);
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
                 "f"(c), "f"(d)
                 : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Per step s (query block i0 + s) the MMA warp issues
//   S = Q K^T, dP = dO V^T                       -> s_full
//   [P, dS written to shared memory]             <- p_ready
//   dV += P^T dO    -> do_empty (dO free)
//   dK += dS^T Q    -> q_empty  (Q buffer free)
//   dQ_part = dS K  (into the S columns)         -> dq_full
// and waits for dq_free (the partial read out) before the next S.
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(320, 1)
    attn_bwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_do, const BwdParams p) {
    using T = BwdTraits<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sK = smem_addr(smem);
    const uint32_t sV = sK + T::kTileBytes;
    const uint32_t sDO = sV + T::kTileBytes;
    const uint32_t sQ0 = sDO + T::kTileBytes;               // Q stage b at sQ0 + b * tile
    const uint32_t sP = sQ0 + T::kQStages * T::kTileBytes;
    const uint32_t sDS = sP + T::kPBytes;
    uint8_t* bar_ptr = smem + (3 + T::kQStages) * T::kTileBytes + 2 * T::kPBytes;
    BwdBars b;
    b.base = smem_addr(bar_ptr);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_ptr + 8 * T::kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int j = blockIdx.x;          // key block
    const int bh = blockIdx.y;
    const int i0 = bwd_first_qblock<CAUSAL>(j, p);
    const int nqb = (p.Nq + 127) / 128;
    const int nsteps = nqb > i0 ? nqb - i0 : 0;

    if (threadIdx.x == 0) {
        mbar_init(b.kv_full(), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(b.q_full(s), 1);
            mbar_init(b.q_empty(s), 1);
        }
        mbar_init(b.do_full(), 1);
        mbar_init(b.do_empty(), 1);
        mbar_init(b.s_full(), 1);
        mbar_init(b.p_ready(), T::kComputeThreads);
        mbar_init(b.dq_full(), 1);
        mbar_init(b.dq_free(), T::kComputeThreads);
        mbar_init(b.fin(), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(smem_addr(tmem_holder), T::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tbase = *tmem_holder;

    if (warp == 8) {
        // ------------------------------------------------ TMA producer --
        if (lane == 0 && nsteps > 0) {
            int nq = 0, nd = 0;
            mbar_arrive_expect_tx(b.kv_full(), 2 * T::kTileBytes);
            for (int pn = 0; pn < D / 64; ++pn) {
                tma_load_3d(sK + pn * T::kPanelBytes, &tm_k, b.kv_full(), pn * 64, j * 128, bh);
                tma_load_3d(sV + pn * T::kPanelBytes, &tm_v, b.kv_full(), pn * 64, j * 128, bh);
            }
            for (int s = 0; s < nsteps; ++s) {
                const int i = i0 + s;
                const int qb = s & 1;
                if (s >= 2 &&
                    !mbar_wait(b.q_empty(qb), ((s - 2) >> 1) & 1, abort_flag, &g_attn_status))
                    break;
                const uint32_t sQ = sQ0 + qb * T::kTileBytes;
                mbar_arrive_expect_tx(b.q_full(qb), T::kTileBytes);
                for (int pn = 0; pn < D / 64; ++pn)
                    tma_load_3d(sQ + pn * T::kPanelBytes, &tm_q, b.q_full(qb), pn * 64, i * 128, bh);
                ++nq;
                if (s >= 1 && !mbar_wait(b.do_empty(), (s - 1) & 1, abort_flag, &g_attn_status))
                    break;
                mbar_arrive_expect_tx(b.do_full(), T::kTileBytes);
                for (int pn = 0; pn < D / 64; ++pn)
                    tma_load_3d(sDO + pn * T::kPanelBytes, &tm_do, b.do_full(), pn * 64, i * 128,
                                bh);
                ++nd;
            }
            // copies still in flight must land before the CTA can exit
            volatile int no_abort = 0;
            mbar_wait(b.kv_full(), 0, &no_abort, &g_attn_status);
            for (int qb = 0; qb < 2; ++qb) {
                const int cnt = (nq - qb + 1) / 2;   // loads issued into stage qb
                if (cnt > 0) mbar_wait(b.q_full(qb), (cnt - 1) & 1, &no_abort, &g_attn_status);
            }
            if (nd > 0) mbar_wait(b.do_full(), (nd - 1) & 1, &no_abort, &g_attn_status);
        }
    } else if (warp == 9) {
        // -------------------------------------------------- MMA issuer --
        if (lane == 0 && nsteps > 0) {
            constexpr uint32_t id_s = idesc_bf16_f32(128, 128, false);   // A, B K-major
            // A MN-major (bit 15), B MN-major (bit 16)
            constexpr uint32_t id_kv = idesc_bf16_f32(128, D, true) | (1u << 15);
            constexpr uint32_t id_q = idesc_bf16_f32(128, D, true);      // A K-major, B MN-major
            const uint64_t dKk = sdesc_sw128(sK, 16, 1024);
            const uint64_t dDOk = sdesc_sw128(sDO, 16, 1024), dVk = sdesc_sw128(sV, 16, 1024);
            const uint64_t dPmn = sdesc_sw128(sP, T::kPanelBytes, 1024);
            const uint64_t dDSmn = sdesc_sw128(sDS, T::kPanelBytes, 1024);
            const uint64_t dDSk = sdesc_sw128(sDS, 16, 1024);
            const uint64_t dDOmn = sdesc_sw128(sDO, T::kPanelBytes, 1024);
            const uint64_t dKmn = sdesc_sw128(sK, T::kPanelBytes, 1024);
            bool ok = mbar_wait(b.kv_full(), 0, abort_flag, &g_attn_status);
            for (int s = 0; ok && s < nsteps; ++s) {
                const int qb = s & 1;
                const uint32_t sQ = sQ0 + qb * T::kTileBytes;
                const uint64_t dQk = sdesc_sw128(sQ, 16, 1024);
                const uint64_t dQmn = sdesc_sw128(sQ, T::kPanelBytes, 1024);
                if (!mbar_wait(b.q_full(qb), (s >> 1) & 1, abort_flag, &g_attn_status)) break;
                if (!mbar_wait(b.do_full(), s & 1, abort_flag, &g_attn_status)) break;
                if (s > 0 && !mbar_wait(b.dq_free(), (s - 1) & 1, abort_flag, &g_attn_status))
                    break;
                tc_fence_after_sync();
                // S = Q_i K_j^T and dP = dO_i V_j^T (K = head dim)
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = ((kk / 4) * T::kPanelBytes + (kk % 4) * 32) >> 4;
                    mma_bf16_ss(tbase + T::kColS, dQk + off, dKk + off, id_s, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = ((kk / 4) * T::kPanelBytes + (kk % 4) * 32) >> 4;
                    mma_bf16_ss(tbase + T::kColDP, dDOk + off, dVk + off, id_s, kk > 0);
                }
                mma_commit(b.s_full());
                if (!mbar_wait(b.p_ready(), s & 1, abort_flag, &g_attn_status)) break;
                tc_fence_after_sync();
                // dV += P^T dO_i (K = 128 query rows, 16 per MMA); then dO is free
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t off = (kk * 2048) >> 4;
                    mma_bf16_ss(tbase + T::kColDV, dPmn + off, dDOmn + off, id_kv,
                                (s > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(b.do_empty());
                // dK += dS^T Q_i; then this Q buffer is free
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t off = (kk * 2048) >> 4;
                    mma_bf16_ss(tbase + T::kColDK, dDSmn + off, dQmn + off, id_kv,
                                (s > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(b.q_empty(qb));
                // dQ_i partial = dS K_j into the S columns (K = 128 keys)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t offa = ((kk / 4) * T::kPanelBytes + (kk % 4) * 32) >> 4;
                    const uint64_t offb = (kk * 2048) >> 4;
                    mma_bf16_ss(tbase + T::kColS, dDSk + offa, dKmn + offb, id_q, kk > 0);
                }
                mma_commit(b.dq_full());
            }
            mma_commit(b.fin());
            // the CTA must not release tensor memory while products are in flight
            volatile int no_abort = 0;
            mbar_wait(b.fin(), 0, &no_abort, &g_attn_status);
        }
    } else {
        // ------------------------- P, dS and dQ (warps 0-7, two column halves) --
        const int quarter = warp & 3;
        const int half = warp >> 2;                    // 0: keys/columns low half, 1: high half
        const int r = quarter * 32 + lane;             // query row in the tile / key row
        const uint32_t lane_off = uint32_t(quarter * 32) << 16;
        const float c2 = p.scale_log2;
        constexpr float kLog2e = 1.4426950408889634f;
        constexpr int kHalfD = D / 2;
        uint8_t* p_row = smem + (sP - sK) + half * T::kPanelBytes + r * 128;
        uint8_t* ds_row = smem + (sDS - sK) + half * T::kPanelBytes + r * 128;
        bool ok = true;
        for (int s = 0; s < nsteps; ++s) {
            const int i = i0 + s;
            const int qrow = i * 128 + r;
            const bool row_valid = qrow < p.Nq;
            float lse2 = 0.f, dl = 0.f;
            if (row_valid) {
                lse2 = p.lse[(size_t)bh * p.Nq + qrow] * kLog2e;
                dl = p.delta[(size_t)bh * p.Nq + qrow];
            }
            // keys [0, lim) of this block are visible to the row
            int lim = row_valid ? min(128, p.Nkv - j * 128) : 0;
            if (CAUSAL && row_valid) lim = min(lim, qrow + (p.Nkv - p.Nq) + 1 - j * 128);
            if (lse2 == -INFINITY) lim = 0;            // the row sees no key at all
            lim -= half * 64;                          // relative to this half's first key
            if (!mbar_wait(b.s_full(), s & 1, abort_flag, &g_attn_status)) ok = false;
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after_sync();
#pragma unroll
            for (int c = 0; c < 64; c += 32) {
                uint32_t sv[32], dp[32];
                tmem_ld32(tbase + lane_off + T::kColS + half * 64 + c, sv);
                tmem_ld32(tbase + lane_off + T::kColDP + half * 64 + c, dp);
                tmem_wait_ld(sv);
                tmem_wait_ld(dp);
                uint32_t pw[16], dw[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int k0 = c + e;
                    const float p0 = k0 < lim ? fast_exp2(fmaf(__uint_as_float(sv[e]), c2, -lse2)) : 0.f;
                    const float p1 =
                        k0 + 1 < lim ? fast_exp2(fmaf(__uint_as_float(sv[e + 1]), c2, -lse2)) : 0.f;
                    const float d0 = p0 * (__uint_as_float(dp[e]) - dl);
                    const float d1 = p1 * (__uint_as_float(dp[e + 1]) - dl);
                    pw[e / 2] = pack_bf16x2(p0, p1);
                    dw[e / 2] = pack_bf16x2(d0, d1);
                }
                // 128-byte-swizzled [query][key] layout: this half's panel, 16-byte
                // chunk (key % 64) / 8 stored at chunk position chunk ^ (row % 8)
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int chunk = (c / 8 + q4) ^ (r & 7);
                    *reinterpret_cast<uint4*>(p_row + chunk * 16) =
                        make_uint4(pw[4 * q4], pw[4 * q4 + 1], pw[4 * q4 + 2], pw[4 * q4 + 3]);
                    *reinterpret_cast<uint4*>(ds_row + chunk * 16) =
                        make_uint4(dw[4 * q4], dw[4 * q4 + 1], dw[4 * q4 + 2], dw[4 * q4 + 3]);
                }
            }
            fence_proxy_async_smem();     // generic-proxy writes -> tensor core reads
            tc_fence_before_sync();
            mbar_arrive(b.p_ready());
            if (!mbar_wait(b.dq_full(), s & 1, abort_flag, &g_attn_status)) ok = false;
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after_sync();
            // This warp's dQ slice (32 rows x D/2 columns) leaves tensor memory
            // first, so the MMA warp can start the next block's S at once; it is
            // then added to the fp32 accumulator. To make each reduction
            // instruction cover 4 rows x 128 contiguous bytes, the rows pass
            // through this warp's own 4 KB slices of the P and dS buffers (every
            // product of the step has completed, so both are free).
            uint32_t g[kHalfD / 32][32];
#pragma unroll
            for (int cc = 0; cc < kHalfD / 32; ++cc)
                tmem_ld32(tbase + lane_off + T::kColS + half * kHalfD + cc * 32, g[cc]);
#pragma unroll
            for (int cc = 0; cc < kHalfD / 32; ++cc) tmem_wait_ld(g[cc]);
            tc_fence_before_sync();
            mbar_arrive(b.dq_free());
            const int qrow0 = i * 128 + quarter * 32;
            float* dq_blk = p.dq_acc + ((size_t)bh * p.Nq + qrow0) * D + half * kHalfD;
#pragma unroll
            for (int cc = 0; cc < kHalfD / 32; ++cc) {
                uint8_t* stage = (cc == 0 ? p_row : ds_row) - lane * 128;   // the warp's 32 rows
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    *reinterpret_cast<uint4*>(stage + lane * 128 + ((k ^ (lane & 7)) * 16)) =
                        make_uint4(g[cc][4 * k], g[cc][4 * k + 1], g[cc][4 * k + 2], g[cc][4 * k + 3]);
                __syncwarp();
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const int row = 4 * it + (lane >> 3);
                    const int ch = lane & 7;
                    const float4 v = *reinterpret_cast<const float4*>(
                        stage + row * 128 + ((ch ^ (row & 7)) * 16));
                    if (qrow0 + row < p.Nq)
                        red_add_v4(dq_blk + (size_t)row * D + cc * 32 + ch * 4, v.x, v.y, v.z, v.w);
                }
                __syncwarp();
            }
        }
        // dK and dV of this key block: TMEM lane = key row; each half writes D/2 columns
        const int krow = j * 128 + r;
        const bool key_valid = krow < p.Nkv;
        uint16_t* dk_row = p.dk + ((size_t)bh * p.Nkv + (key_valid ? krow : 0)) * D + half * kHalfD;
        uint16_t* dv_row = p.dv + ((size_t)bh * p.Nkv + (key_valid ? krow : 0)) * D + half * kHalfD;
        if (nsteps == 0) {
            if (key_valid)
                for (int c = 0; c < kHalfD; c += 8) {
                    *reinterpret_cast<uint4*>(dk_row + c) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(dv_row + c) = make_uint4(0, 0, 0, 0);
                }
        } else if (ok) {
            if (!mbar_wait(b.fin(), 0, abort_flag, &g_attn_status)) ok = false;
            if (__all_sync(0xffffffffu, ok)) {
                tc_fence_after_sync();
#pragma unroll
                for (int c = 0; c < kHalfD; c += 32) {
                    uint32_t gk[32], gv[32];
                    tmem_ld32(tbase + lane_off + T::kColDK + half * kHalfD + c, gk);
                    tmem_ld32(tbase + lane_off + T::kColDV + half * kHalfD + c, gv);
                    tmem_wait_ld(gk);
                    tmem_wait_ld(gv);
                    uint32_t wk[16], wv[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        wk[e] = pack_bf16x2(__uint_as_float(gk[2 * e]) * p.scale,
                                            __uint_as_float(gk[2 * e + 1]) * p.scale);
                        wv[e] = pack_bf16x2(__uint_as_float(gv[2 * e]), __uint_as_float(gv[2 * e + 1]));
                    }
                    if (key_valid) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            reinterpret_cast<uint4*>(dk_row + c)[q4] =
                                make_uint4(wk[4 * q4], wk[4 * q4 + 1], wk[4 * q4 + 2], wk[4 * q4 + 3]);
                            reinterpret_cast<uint4*>(dv_row + c)[q4] =
                                make_uint4(wv[4 * q4], wv[4 * q4 + 1], wv[4 * q4 + 2], wv[4 * q4 + 3]);
                        }
                    }
                }
            }
        }
    }

    __syncwarp();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 9) {
        tmem_dealloc(tbase, T::kTmemCols);
    }
}

}  // namespace eattn
