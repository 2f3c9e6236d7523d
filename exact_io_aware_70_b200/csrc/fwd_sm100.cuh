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
//     rows) = two 128-row Q tiles; units are handed out heaviest-first so the
//     causal triangle balances across the 148 SMs.
//   * Warp 8 (one elected lane) is the TMA producer: Q tiles once per unit,
//     then K_j and V_j tiles into a ring of shared-memory slots, 128-byte
//     swizzled, completion counted on mbarriers.
//   * Warp 9 (one elected lane) issues every tcgen05.mma: S_t = Q_t K_j^T into
//     tensor memory (fp32, 128x128), and O_t += P_t V_j with P_t read straight
//     from tensor memory (bf16, aliased over S_t's first 64 columns).
//   * Warps 0-3 and 4-7 are the softmax groups of Q tile 0 and Q tile 1, one
//     thread per query row (= TMEM lane). While one group exponentiates its
//     tile, the tensor core works on the other tile's products (ping-pong).
//     Each group also rescales its O tile in tensor memory when its running max
//     grows by more than 2^8 (lazy rescaling: exact, since every p and l uses
//     the same stale reference max), and runs the epilogue (O / l -> bf16,
//     LSE = ln 2 * (m + log2 l)).
//   * Exponentials are base 2 with log2(e) folded into the scale.
//   * Tensor memory columns: S0 [0,128), S1 [128,256), O0 [256,256+d),
//     O1 [256+d, 256+2d).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx_sm100.cuh"
#include "tmem_wide.cuh"

namespace eattn {


struct FwdParams {
    uint16_t* o;        // bf16 [BH, Nq, D]
    float* lse;         // fp32 [BH, Nq]
    int BH;             // batch * heads
    int Nq, Nkv;
    int num_qb;         // ceil(Nq / 256)
    int num_units;      // BH * num_qb
    float scale_log2;   // scale * log2(e)
};

template <int D>
struct FwdTraits {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int kRows = 128;                     // rows of a Q, K or V tile
    static constexpr int kPanelBytes = 128 * 64 * 2;      // 128 rows x 64 bf16 (one swizzle panel)
    static constexpr int kPanels = D / 64;
    static constexpr int kTileBytes = kPanels * kPanelBytes;
    static constexpr int kSlots = (D == 128) ? 4 : 8;     // K/V ring depth (tiles)
    static constexpr int kThreads = 320;                  // 10 warps
    static constexpr int kNumBars = 2 * kSlots + 13;
    static constexpr int kSmemBytes = 1024 + (2 + kSlots) * kTileBytes + kNumBars * 8 + 16;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS0 = 0, kColS1 = 128;
    static constexpr uint32_t kColO0 = 256, kColO1 = 256 + D;
};

struct FwdUnit {
    int bh, qb;
    int n[2];   // K/V tiles visible to Q tile 0 / Q tile 1 (0: tile has no work)
    int nmax;
};

template <bool CAUSAL>
__device__ __forceinline__ FwdUnit fwd_unit(int u, const FwdParams& p) {
    FwdUnit x;
    x.qb = p.num_qb - 1 - u / p.BH;   // heaviest (latest) query blocks first
    x.bh = u % p.BH;
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

struct FwdBars {
    uint32_t kv_full, kv_empty;   // base addresses of the slot arrays (8 bytes apart)
    uint32_t q_full, q_empty, s_full, p_ready, o_final, o_free;  // 2 each
    uint32_t drain;
};

// Bounded wait executed by a whole warp; the outcome is made warp-uniform.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    bool ok = mbar_wait(bar, parity, abort_flag, &g_attn_status);
    return __all_sync(0xffffffffu, ok);
}

// ----------------------------------------------------------- TMA producer --
template <int D, bool CAUSAL>
__device__ void fwd_producer(const FwdParams& p, const CUtensorMap* tq, const CUtensorMap* tk,
                             const CUtensorMap* tv, uint32_t sQ, uint32_t sKV, const FwdBars& b,
                             volatile int* abort_flag) {
    using T = FwdTraits<D>;
    uint32_t kv_iter = 0;
    uint32_t q_issued[2] = {0, 0};
    for (int u = blockIdx.x; u < p.num_units; u += gridDim.x) {
        const FwdUnit x = fwd_unit<CAUSAL>(u, p);
        for (int t = 0; t < 2; ++t) {
            if (q_issued[t] > 0 &&
                !mbar_wait(b.q_empty + 8 * t, (q_issued[t] - 1) & 1, abort_flag, &g_attn_status))
                goto fail;
            mbar_arrive_expect_tx(b.q_full + 8 * t, T::kTileBytes);
            for (int pn = 0; pn < T::kPanels; ++pn)
                tma_load_3d(sQ + t * T::kTileBytes + pn * T::kPanelBytes, tq, b.q_full + 8 * t,
                            pn * 64, x.qb * 256 + t * 128, x.bh);
            ++q_issued[t];
        }
        for (int j = 0; j < x.nmax; ++j) {
            for (int which = 0; which < 2; ++which) {   // K_j, then V_j
                const uint32_t slot = kv_iter % T::kSlots;
                const uint32_t round = kv_iter / T::kSlots;
                if (round > 0 &&
                    !mbar_wait(b.kv_empty + 8 * slot, (round - 1) & 1, abort_flag, &g_attn_status))
                    goto fail;
                mbar_arrive_expect_tx(b.kv_full + 8 * slot, T::kTileBytes);
                for (int pn = 0; pn < T::kPanels; ++pn)
                    tma_load_3d(sKV + slot * T::kTileBytes + pn * T::kPanelBytes,
                                which ? tv : tk, b.kv_full + 8 * slot, pn * 64, j * 128, x.bh);
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
        mbar_wait(b.kv_full + 8 * (i % T::kSlots), (i / T::kSlots) & 1, &no_abort,
                  &g_attn_status);
    for (int t = 0; t < 2; ++t)
        if (q_issued[t] > 0)
            mbar_wait(b.q_full + 8 * t, (q_issued[t] - 1) & 1, &no_abort, &g_attn_status);
}
}

// ------------------------------------------------------------ MMA issuer --
template <int D>
__device__ __forceinline__ void fwd_issue_s(uint32_t tmem_s, uint32_t sQt, uint32_t sK) {
    using T = FwdTraits<D>;
    constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk / 4) * T::kPanelBytes + (kk % 4) * 32;
        mma_bf16_ss(tmem_s, sdesc_sw128(sQt + off, 16, 1024), sdesc_sw128(sK + off, 16, 1024),
                    idesc, kk > 0 ? 1u : 0u);
    }
}

template <int D>
__device__ __forceinline__ void fwd_issue_pv(uint32_t tmem_o, uint32_t tmem_p, uint32_t sV,
                                             bool accumulate) {
    using T = FwdTraits<D>;
    constexpr uint32_t idesc = idesc_bf16_f32(128, D, true);
#pragma unroll
    for (int kk = 0; kk < 128 / 16; ++kk) {
        // P: 16 keys = 8 TMEM columns of bf16 pairs. V: 16 keys = 2 swizzle
        // atoms of 8 rows (2048 bytes); the two 64-column panels are kPanelBytes apart.
        mma_bf16_ts(tmem_o, tmem_p + kk * 8, sdesc_sw128(sV + kk * 2048, T::kPanelBytes, 1024),
                    idesc, (accumulate || kk > 0) ? 1u : 0u);
    }
}

template <int D, bool CAUSAL>
__device__ void fwd_mma(const FwdParams& p, uint32_t tbase, uint32_t sQ, uint32_t sKV,
                        const FwdBars& b, volatile int* abort_flag) {
    using T = FwdTraits<D>;
    const uint32_t colS[2] = {T::kColS0, T::kColS1};
    const uint32_t colO[2] = {T::kColO0, T::kColO1};
    uint32_t kv_iter = 0, q_use = 0;
    uint32_t o_use[2] = {0, 0}, p_phase[2] = {0, 0};
    for (int u = blockIdx.x; u < p.num_units; u += gridDim.x) {
        const FwdUnit x = fwd_unit<CAUSAL>(u, p);
        if (!mbar_wait(b.q_full, q_use & 1, abort_flag, &g_attn_status)) goto done;
        if (!mbar_wait(b.q_full + 8, q_use & 1, abort_flag, &g_attn_status)) goto done;
        tc_fence_after_sync();
        if (x.nmax > 0) {
            uint32_t kslot = kv_iter % T::kSlots;
            if (!mbar_wait(b.kv_full + 8 * kslot, (kv_iter / T::kSlots) & 1, abort_flag,
                           &g_attn_status))
                goto done;
            tc_fence_after_sync();
            for (int t = 0; t < 2; ++t)
                if (x.n[t] > 0) {
                    fwd_issue_s<D>(tbase + colS[t], sQ + t * T::kTileBytes,
                                   sKV + kslot * T::kTileBytes);
                    mma_commit(b.s_full + 8 * t);
                }
            mma_commit(b.kv_empty + 8 * kslot);
            ++kv_iter;
            for (int j = 0; j < x.nmax; ++j) {
                const uint32_t vslot = kv_iter % T::kSlots;
                if (!mbar_wait(b.kv_full + 8 * vslot, (kv_iter / T::kSlots) & 1, abort_flag,
                               &g_attn_status))
                    goto done;
                tc_fence_after_sync();
                ++kv_iter;
                const bool has_next = j + 1 < x.nmax;
                kslot = kv_iter % T::kSlots;
                const uint32_t kpar = (kv_iter / T::kSlots) & 1;
                for (int t = 0; t < 2; ++t) {
                    if (j < x.n[t]) {
                        if (!mbar_wait(b.p_ready + 8 * t, p_phase[t], abort_flag, &g_attn_status))
                            goto done;
                        p_phase[t] ^= 1;
                        if (j == 0 && o_use[t] > 0 &&
                            !mbar_wait(b.o_free + 8 * t, (o_use[t] - 1) & 1, abort_flag,
                                       &g_attn_status))
                            goto done;
                        tc_fence_after_sync();
                        fwd_issue_pv<D>(tbase + colO[t], tbase + colS[t],
                                        sKV + vslot * T::kTileBytes, j > 0);
                        if (j == x.n[t] - 1) mma_commit(b.o_final + 8 * t);
                    }
                    if (t == 0 && has_next) {
                        if (!mbar_wait(b.kv_full + 8 * kslot, kpar, abort_flag, &g_attn_status))
                            goto done;
                        tc_fence_after_sync();
                    }
                    if (t == 1) mma_commit(b.kv_empty + 8 * vslot);
                    if (j + 1 < x.n[t]) {
                        fwd_issue_s<D>(tbase + colS[t], sQ + t * T::kTileBytes,
                                       sKV + kslot * T::kTileBytes);
                        mma_commit(b.s_full + 8 * t);
                    }
                }
                if (has_next) {
                    mma_commit(b.kv_empty + 8 * kslot);
                    ++kv_iter;
                }
            }
        }
        mma_commit(b.q_empty);
        mma_commit(b.q_empty + 8);
        ++q_use;
        for (int t = 0; t < 2; ++t)
            if (x.n[t] > 0) ++o_use[t];
    }
done: {
    // Every MMA issued so far must finish before tensor memory is released.
    volatile int no_abort = 0;
    mma_commit(b.drain);
    mbar_wait(b.drain, 0, &no_abort, &g_attn_status);
}
}

// --------------------------------------------------------------- softmax --
template <int D, bool CAUSAL>
__device__ void fwd_softmax(const FwdParams& p, uint32_t tbase, const FwdBars& b, int warp,
                            int lane, volatile int* abort_flag) {
    using T = FwdTraits<D>;
    const int t = warp >> 2;                 // which Q tile
    const int quarter = warp & 3;            // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;       // row within the tile = TMEM lane
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t tS = tbase + lane_off + (t ? T::kColS1 : T::kColS0);
    const uint32_t tO = tbase + lane_off + (t ? T::kColO1 : T::kColO0);
    const uint32_t bar_s = b.s_full + 8 * t, bar_p = b.p_ready + 8 * t;
    const uint32_t bar_of = b.o_final + 8 * t, bar_ofree = b.o_free + 8 * t;
    const float c2 = p.scale_log2;
    uint32_t s_phase = 0, o_use = 0;

    for (int u = blockIdx.x; u < p.num_units; u += gridDim.x) {
        const FwdUnit x = fwd_unit<CAUSAL>(u, p);
        const int n = x.n[t];
        const long long qrow = (long long)x.qb * 256 + t * 128 + r;
        const bool row_valid = qrow < p.Nq;
        long long kv_lim = p.Nkv;   // keys [0, kv_lim) are visible to this row
        if (CAUSAL) kv_lim = min(kv_lim, qrow + ((long long)p.Nkv - p.Nq) + 1);
        float m_ref = -INFINITY;    // reference max, log2 units (scaled)
        float l = 0.f;              // running sum of 2^(s*c2 - m_ref)

        for (int j = 0; j < n; ++j) {
            if (!warp_wait(bar_s, s_phase, abort_flag)) return;
            s_phase ^= 1;
            tc_fence_after_sync();
            uint32_t sr[128];
            tmem_ld128(tS, sr);
            tmem_wait_ld128(sr);
            const long long lim = kv_lim - (long long)j * 128;
            if (lim < 128) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
            }
            float mx0 = __uint_as_float(sr[0]), mx1 = __uint_as_float(sr[1]);
            float mx2 = __uint_as_float(sr[2]), mx3 = __uint_as_float(sr[3]);
#pragma unroll
            for (int c = 4; c < 128; c += 4) {
                mx0 = fmaxf(mx0, __uint_as_float(sr[c]));
                mx1 = fmaxf(mx1, __uint_as_float(sr[c + 1]));
                mx2 = fmaxf(mx2, __uint_as_float(sr[c + 2]));
                mx3 = fmaxf(mx3, __uint_as_float(sr[c + 3]));
            }
            const float mxs = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * c2;
            const bool need = mxs > m_ref + 8.0f;
            const bool any_need = __any_sync(0xffffffffu, need);
            const float m_new = need ? mxs : m_ref;
            const float alpha = need ? fast_exp2(m_ref - m_new) : 1.0f;
            m_ref = m_new;
            const float base = (m_ref == -INFINITY) ? 0.f : m_ref;
            uint32_t pk[64];
            float l0 = 0.f, l1 = 0.f;
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                const float e0 = fast_exp2(fmaf(__uint_as_float(sr[2 * i]), c2, -base));
                const float e1 = fast_exp2(fmaf(__uint_as_float(sr[2 * i + 1]), c2, -base));
                l0 += e0;
                l1 += e1;
                pk[i] = pack_bf16x2(e0, e1);
            }
            l = l * alpha + (l0 + l1);
            tmem_st64(tS, pk);
            if (any_need && j > 0) {
                // Rescale O_t by alpha (1 for rows whose max did not move).
                // O_t is stable here: the commit that signalled S_t(j) also
                // covers the earlier P_t(j-1) V product, and P_t(j) V is not
                // issued before this group arrives on p_ready.
#pragma unroll
                for (int c = 0; c < D; c += 32) {
                    uint32_t orr[32];
                    tmem_ld32(tO + c, orr);
                    tmem_wait_ld(orr);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
                    tmem_st32(tO + c, orr);
                }
            }
            tmem_wait_st();
            tc_fence_before_sync();
            mbar_arrive(bar_p);
        }

        uint16_t* orow = p.o + ((size_t)x.bh * p.Nq + (size_t)(row_valid ? qrow : 0)) * D;
        if (n > 0) {
            if (!warp_wait(bar_of, o_use & 1, abort_flag)) return;
            tc_fence_after_sync();
            const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
            for (int c = 0; c < D; c += 32) {
                uint32_t orr[32];
                tmem_ld32(tO + c, orr);
                tmem_wait_ld(orr);
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = pack_bf16x2(__uint_as_float(orr[2 * i]) * inv,
                                       __uint_as_float(orr[2 * i + 1]) * inv);
                if (row_valid) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        dst[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
                }
            }
            tc_fence_before_sync();
            mbar_arrive(bar_ofree);
            ++o_use;
        } else if (row_valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
            for (int k = 0; k < D / 8; ++k) dst[k] = make_uint4(0, 0, 0, 0);
        }
        if (row_valid)
            p.lse[(size_t)x.bh * p.Nq + qrow] =
                l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
}

// ---------------------------------------------------------------- kernel --
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(320, 1)
    attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using T = FwdTraits<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sQ = smem_addr(smem);
    const uint32_t sKV = sQ + 2 * T::kTileBytes;
    uint8_t* bar_ptr = smem + (2 + T::kSlots) * T::kTileBytes;
    const uint32_t bar0 = smem_addr(bar_ptr);
    FwdBars b;
    b.kv_full = bar0;
    b.kv_empty = bar0 + 8 * T::kSlots;
    b.q_full = bar0 + 16 * T::kSlots;
    b.q_empty = b.q_full + 16;
    b.s_full = b.q_empty + 16;
    b.p_ready = b.s_full + 16;
    b.o_final = b.p_ready + 16;
    b.o_free = b.o_final + 16;
    b.drain = b.o_free + 16;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bar_ptr + 8 * T::kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < T::kSlots; ++i) {
            mbar_init(b.kv_full + 8 * i, 1);
            mbar_init(b.kv_empty + 8 * i, 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(b.q_full + 8 * t, 1);
            mbar_init(b.q_empty + 8 * t, 1);
            mbar_init(b.s_full + 8 * t, 1);
            mbar_init(b.p_ready + 8 * t, 128);
            mbar_init(b.o_final + 8 * t, 1);
            mbar_init(b.o_free + 8 * t, 128);
        }
        mbar_init(b.drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 8 && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
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
        fwd_softmax<D, CAUSAL>(p, tbase, b, warp, lane, abort_flag);
    } else if (warp == 8) {
        if (lane == 0) fwd_producer<D, CAUSAL>(p, &tm_q, &tm_k, &tm_v, sQ, sKV, b, abort_flag);
    } else {
        if (lane == 0) fwd_mma<D, CAUSAL>(p, tbase, sQ, sKV, b, abort_flag);
    }

    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 9) {
        __syncwarp();
        tmem_dealloc(tbase, T::kTmemCols);
    }
}

}  // namespace eattn
