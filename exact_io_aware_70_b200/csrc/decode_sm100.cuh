// decode_sm100.cuh -- split-KV decode for one query row per (batch, head).
//
// The decode method of "Describe Flash Attention at a high level"
// (mantramindai), "Follow-up questions to expect", last question: with a single
// query row there is no parallelism across query tiles, so the KV sequence is
// split across thread blocks, each block computes the attention of the row
// over its chunk of keys, and the partial results are merged with the same
// max-and-sum trick the online softmax uses.
//
// With one query row the work is about one multiply-add per byte of K and V,
// so it is bound by HBM bandwidth, not by the tensor cores: the partial kernel
// streams K and V once with 16-byte non-caching loads, many in flight per
// thread, and does the dot products and the P.V accumulation on the fp32 CUDA
// cores. Within a chunk it walks sub-blocks of kSub keys with the online
// softmax (running max, running sum, rescaled accumulator).
#pragma once

#include <cstdint>

#include "ptx_sm100.cuh"

namespace eattn {

struct DecodeParams {
    const uint16_t* q;   // bf16 [BH, D]
    const uint16_t* k;   // bf16 [BH, Nkv, D]; paged: [num_pages, H, page_size, D]
    const uint16_t* v;   // same layout as k
    float* o_part;       // fp32 [BH, S, D]
    float* lse_part;     // fp32 [BH, S]
    int Nkv;             // keys per row (contiguous layout)
    int S;               // number of chunks
    int L;               // keys per chunk = ceil(Nkv / S) (contiguous layout)
    float scale_log2;    // scale * log2(e)
    // paged layout only
    const int* block_table;   // [B, max_pages]: physical page of each logical page
    const int* seq_lens;      // [B]
    int H, page_shift, max_pages, num_pages;
};

// Bit of the device status word: a block-table entry or sequence length was
// out of range (the keys concerned were skipped, nothing out of range was read).
constexpr unsigned kDevErrBadIndex = 2u;

// 1: K/V loads of the decode kernel are marked evict-first in L2 (each byte is
//    read exactly once). Measured: no gain for a prefill that follows, and
//    0.4% less decode bandwidth, so off by default.
#ifndef EATTN_DECODE_EVICT_FIRST
#define EATTN_DECODE_EVICT_FIRST 0
#endif

// 16-byte streaming load: not kept in L1, 256-byte L2 prefetch, L2 policy `pol`.
__device__ __forceinline__ uint4 ld_stream_16B(const void* p, uint64_t pol) {
    uint4 r;
#if EATTN_DECODE_EVICT_FIRST
    asm volatile(
        "ld.global.nc.L1::no_allocate.L2::cache_hint.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p), "l"(pol));
#else
    (void)pol;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
#endif
    return r;
}

// bf16 pair packed in a 32-bit word -> two fp32 (exact)
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float dot8(const uint4& kv, const float (&q)[8]) {
    float a = bf16_lo(kv.x) * q[0];
    a = fmaf(bf16_hi(kv.x), q[1], a);
    a = fmaf(bf16_lo(kv.y), q[2], a);
    a = fmaf(bf16_hi(kv.y), q[3], a);
    a = fmaf(bf16_lo(kv.z), q[4], a);
    a = fmaf(bf16_hi(kv.z), q[5], a);
    a = fmaf(bf16_lo(kv.w), q[6], a);
    a = fmaf(bf16_hi(kv.w), q[7], a);
    return a;
}

__device__ __forceinline__ void axpy8(float p, const uint4& kv, float (&acc)[8]) {
    acc[0] = fmaf(p, bf16_lo(kv.x), acc[0]);
    acc[1] = fmaf(p, bf16_hi(kv.x), acc[1]);
    acc[2] = fmaf(p, bf16_lo(kv.y), acc[2]);
    acc[3] = fmaf(p, bf16_hi(kv.y), acc[3]);
    acc[4] = fmaf(p, bf16_lo(kv.z), acc[4]);
    acc[5] = fmaf(p, bf16_hi(kv.z), acc[5]);
    acc[6] = fmaf(p, bf16_lo(kv.w), acc[6]);
    acc[7] = fmaf(p, bf16_hi(kv.w), acc[7]);
}

// 16-byte K (then V) rows each thread has in flight per pass, and the
// minimum resident CTAs per SM the contiguous kernel is compiled for. Three
// CTAs per SM (76 registers, no spills) measured 1.152 ms against 1.230 ms
// with two (89 registers) on decode_32k: 7.45 against 6.98 TB/s of K/V; four
// (64 registers) 1.156 ms; 16 rows in flight per thread (two CTAs) 1.285 ms.
#ifndef EATTN_DECODE_BATCH
#define EATTN_DECODE_BATCH 8
#endif
#ifndef EATTN_DECODE_MIN_CTAS
#define EATTN_DECODE_MIN_CTAS 3
#endif

template <int D>
struct DecodeTraits {
    static constexpr int kThreads = 256;
    static constexpr int kLanesPerRow = D / 8;                     // 16-byte pieces per row
    static constexpr int kRowsPerPass = kThreads / kLanesPerRow;   // rows covered by one load of all threads
    static constexpr int kBatch = EATTN_DECODE_BATCH;              // rows in flight per thread
    static_assert(kBatch % 8 == 0, "the score pass reduces rows in groups of 8");
    static constexpr int kSub = kRowsPerPass * kBatch * 4;         // keys per sub-block
};

// Sum 8 per-lane partial values over the kLanes lanes of a row group so that
// each lane ends with one complete sum: a transpose-reduce (each exchange step
// halves the number of values a lane carries). On return, lane l of the group
// holds the sum for value index ((l >> 1) & 7) when kLanes == 16, or (l & 7)
// when kLanes == 8.
template <int kLanes>
__device__ __forceinline__ float group_transpose_reduce8(float (&v)[8], int lane) {
    // step: 8 values -> 4
    {
        constexpr int off = kLanes / 2;
        const bool hi = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float send = hi ? v[i] : v[i + 4];
            const float keep = hi ? v[i + 4] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    // 4 -> 2
    {
        constexpr int off = kLanes / 4;
        const bool hi = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float send = hi ? v[i] : v[i + 2];
            const float keep = hi ? v[i + 2] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    // 2 -> 1
    {
        constexpr int off = kLanes / 8;
        const bool hi = (lane & off) != 0;
        const float send = hi ? v[0] : v[1];
        const float keep = hi ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
    if (kLanes == 16) v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
    return v[0];
}

template <int D>
__device__ __forceinline__ int reduce_owner_index(int glane) {
    // which of the 8 values a lane of its row group ends up holding
    return DecodeTraits<D>::kLanesPerRow == 16
               ? ((glane >> 3) & 1) * 4 + ((glane >> 2) & 1) * 2 + ((glane >> 1) & 1)
               : ((glane >> 2) & 1) * 4 + ((glane >> 1) & 1) * 2 + (glane & 1);
}

// PAGED: token j of sequence b is in physical page block_table[b][j >> page_shift],
// slot j & (page_size - 1), of a cache laid out [num_pages][H][page_size][D].
// The paged instantiation is held to 64 registers (4 CTAs per SM): measured
// 6.63 TB/s against 4.83 TB/s at its unconstrained 80 registers (3 CTAs).
template <int D, bool PAGED>
__global__ void __launch_bounds__(256, PAGED ? 4 : EATTN_DECODE_MIN_CTAS)
    attn_decode_partials_kernel(const DecodeParams p) {
    using T = DecodeTraits<D>;
    constexpr int LPR = T::kLanesPerRow, RPP = T::kRowsPerPass, NB = T::kBatch;
    constexpr int SUB = T::kSub;
    __shared__ float s_score[SUB];
    __shared__ float s_red[32];
    // paged layout: physical page of each logical page touched by the current
    // sub-block (-1: out of range, skipped); page_size >= 16 bounds the count
    __shared__ int s_page[PAGED ? SUB / 16 + 2 : 1];
    __shared__ float s_acc[RPP][D + 4];

    const int c = blockIdx.x;            // chunk
    const int bh = blockIdx.y;
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int cc = tid % LPR;            // which 16-byte piece of a row
    const int rs = tid / LPR;            // row slot within a pass
    const int glane = tid % LPR;         // lane within the row group

    int nkv = p.Nkv, L = p.L;
    int b = 0, h = 0;
    if (PAGED) {
        b = bh / p.H;
        h = bh - b * p.H;
        const int len = p.seq_lens[b];
        const int cap = p.max_pages << p.page_shift;
        nkv = min(max(len, 0), cap);
        if ((len < 0 || len > cap) && tid == 0 && c == 0) atomicOr(&g_attn_status, kDevErrBadIndex);
        L = (nkv + p.S - 1) / p.S;
    }
    const long long j0 = (long long)c * L;
    const long long j1 = min(j0 + (long long)L, (long long)nkv);
    const int n = j1 > j0 ? (int)(j1 - j0) : 0;
    float* o_out = p.o_part + ((size_t)bh * p.S + c) * D;
    if (!dcheck(c < p.S && (!PAGED || b < (int)gridDim.y / p.H))) return;

    if (n == 0) {   // empty chunk: weight zero in the merge
        for (int x = tid; x < D; x += blockDim.x) o_out[x] = 0.f;
        if (tid == 0) p.lse_part[(size_t)bh * p.S + c] = -INFINITY;
        return;
    }

    // this thread's 8 query elements, pre-scaled so scores come out in log2 units
    float qv[8];
    {
        const uint4 qq = *reinterpret_cast<const uint4*>(p.q + (size_t)bh * D + cc * 8);
        const float s = p.scale_log2;
        qv[0] = bf16_lo(qq.x) * s; qv[1] = bf16_hi(qq.x) * s;
        qv[2] = bf16_lo(qq.y) * s; qv[3] = bf16_hi(qq.y) * s;
        qv[4] = bf16_lo(qq.z) * s; qv[5] = bf16_hi(qq.z) * s;
        qv[6] = bf16_lo(qq.w) * s; qv[7] = bf16_hi(qq.w) * s;
    }
    const uint16_t* kbase = p.k + ((size_t)bh * p.Nkv + j0) * D + cc * 8;
    const uint16_t* vbase = p.v + ((size_t)bh * p.Nkv + j0) * D + cc * 8;
    // paged layout: the sub-block's pages are staged in s_page; the element
    // offset of key j0 + i within the cache is then one shared-memory read away
    const int* table = PAGED ? p.block_table + (size_t)b * p.max_pages : nullptr;
    const uint16_t* kpaged = p.k + cc * 8;
    const uint16_t* vpaged = p.v + cc * 8;
    const int pmask = (1 << p.page_shift) - 1;
    auto page_of = [&](int i, int lp0) -> int {   // i: key index within the chunk
        return s_page[(((int)j0 + i) >> p.page_shift) - lp0];
    };
    auto paged_offset = [&](int i, int page) -> long long {
        const int j = (int)j0 + i;
        return ((((long long)page * p.H + h) << p.page_shift) + (j & pmask)) * D;
    };
    const uint64_t pol = l2_policy_evict_first();   // used only with EATTN_DECODE_EVICT_FIRST
    float m_run = -INFINITY, l_run = 0.f;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;

    for (int sb = 0; sb < n; sb += SUB) {
        const int nsub = min(SUB, n - sb);
        int lp0 = 0;
        if (PAGED) {
            lp0 = ((int)j0 + sb) >> p.page_shift;
            const int lp1 = ((int)j0 + sb + nsub - 1) >> p.page_shift;
            for (int x = tid; x <= lp1 - lp0; x += blockDim.x) {
                const int page = __ldg(table + lp0 + x);
                const bool ok = page >= 0 && page < p.num_pages;
                if (!ok) atomicOr(&g_attn_status, kDevErrBadIndex);
                s_page[x] = ok ? page : -1;
            }
            __syncthreads();
        }
        // ---- scores for this sub-block: s_i = (scale*log2e) q . k_i
        for (int base = 0; base < SUB; base += RPP * NB) {
            uint4 kr[NB];
#pragma unroll
            for (int r = 0; r < NB; ++r) {
                const int i = base + rs + RPP * r;
                if (PAGED) {
                    const int page = i < nsub ? page_of(sb + i, lp0) : -1;
                    kr[r] = page >= 0 ? ld_stream_16B(kpaged + paged_offset(sb + i, page), pol)
                                      : make_uint4(0, 0, 0, 0);
                } else {
                    kr[r] = (i < nsub && dcheck(j0 + sb + i < p.Nkv))
                                ? ld_stream_16B(kbase + (size_t)(sb + i) * D, pol)
                                : make_uint4(0, 0, 0, 0);
                }
            }
            // the transpose-reduce sums 8 rows at a time
#pragma unroll
            for (int g = 0; g < NB / 8; ++g) {
                float part[8];
#pragma unroll
                for (int r = 0; r < 8; ++r) part[r] = dot8(kr[8 * g + r], qv);
                const float sum = group_transpose_reduce8<LPR>(part, glane);
                const int owner = 8 * g + reduce_owner_index<D>(glane);
                const bool writer = (LPR == 16) ? ((glane & 1) == 0) : true;
                if (writer) {
                    const int i = base + rs + RPP * owner;
                    bool skipped = i >= nsub;
                    if (PAGED && !skipped) skipped = page_of(sb + i, lp0) < 0;
                    s_score[i] = skipped ? -INFINITY : sum;
                }
            }
        }
        __syncthreads();
        // ---- sub-block max
        float mx = -INFINITY;
        for (int i = tid; i < SUB; i += blockDim.x) mx = fmaxf(mx, s_score[i]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) s_red[warp] = mx;
        __syncthreads();
        mx = s_red[0];
#pragma unroll
        for (int w = 1; w < 8; ++w) mx = fmaxf(mx, s_red[w]);
        // m_new is finite unless every key so far was skipped (bad block-table
        // entries); then nothing is accumulated and alpha stays 1.
        const float m_new = fmaxf(m_run, mx);
        const bool none = m_new == -INFINITY;
        const float alpha = none ? 1.0f : fast_exp2(m_run - m_new);   // 0 on the first sub-block
        const float base = none ? 0.0f : m_new;
        // ---- probabilities (unnormalised) and their sum
        float ls = 0.f;
        for (int i = tid; i < SUB; i += blockDim.x) {
            const float e = fast_exp2(s_score[i] - base);
            s_score[i] = e;
            ls += e;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
        __syncthreads();                 // all reads of s_red (max) done
        if (lane == 0) s_red[warp] = ls;
        __syncthreads();
        float lsum = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) lsum += s_red[w];
        l_run = l_run * alpha + lsum;
        m_run = m_new;
        // ---- accumulate P.V for this thread's 8 columns
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] *= alpha;
        for (int base = 0; base < SUB; base += RPP * NB) {
            uint4 vr[NB];
#pragma unroll
            for (int r = 0; r < NB; ++r) {
                const int i = base + rs + RPP * r;
                if (PAGED) {
                    const int page = i < nsub ? page_of(sb + i, lp0) : -1;
                    vr[r] = page >= 0 ? ld_stream_16B(vpaged + paged_offset(sb + i, page), pol)
                                      : make_uint4(0, 0, 0, 0);
                } else {
                    vr[r] = (i < nsub && dcheck(j0 + sb + i < p.Nkv))
                                ? ld_stream_16B(vbase + (size_t)(sb + i) * D, pol)
                                : make_uint4(0, 0, 0, 0);
                }
            }
#pragma unroll
            for (int r = 0; r < NB; ++r) axpy8(s_score[base + rs + RPP * r], vr[r], acc);
        }
        __syncthreads();                 // s_score and s_red are reused next sub-block
    }
    // ---- combine the RPP row slots, normalise, write the partial
#pragma unroll
    for (int i = 0; i < 8; ++i) s_acc[rs][cc * 8 + i] = acc[i];
    __syncthreads();
    const float inv = l_run > 0.f ? 1.0f / l_run : 0.f;   // l_run = 0: every key skipped
    for (int x = tid; x < D; x += blockDim.x) {
        float s = 0.f;
#pragma unroll 4
        for (int r = 0; r < RPP; ++r) s += s_acc[r][x];
        o_out[x] = s * inv;
    }
    if (tid == 0)
        p.lse_part[(size_t)bh * p.S + c] =
            l_run > 0.f ? (m_run + log2f(l_run)) * 0.69314718055994531f : -INFINITY;
}

// ------------------------------------------------------------------ merge --
// One block of kMergeThreads per (batch, head):
//   M = max_c lse_c;  w_c = exp(lse_c - M);  LSE = M + ln sum_c w_c;
//   O = sum_c w_c O_c / sum_c w_c.
// The chunks may come from R groups (the KV shards of R GPUs, gathered one
// after another): chunk s of group r of row bh is at ((r * BH + bh) * S + s),
// which for R = 1 is the plain [BH, S] layout of attn_decode_partials.
// Each thread owns 4 output columns of one chunk slot: D / 4 threads read one
// partial row as one coalesced run of 16-byte loads, and the block covers
// kMergeThreads / (D / 4) chunks per pass; the slots' sums are then added in
// a fixed order through shared memory, so the result is deterministic.
// VEC: o_part is 16-byte aligned (one 16-byte load per thread and chunk);
// otherwise four 4-byte loads.
constexpr int kMergeThreads = 256;

template <bool VEC>
__device__ __forceinline__ float4 load_f32x4(const float* p) {
    if constexpr (VEC) return *reinterpret_cast<const float4*>(p);
    return make_float4(p[0], p[1], p[2], p[3]);
}

template <int D, bool VEC>
__global__ void __launch_bounds__(kMergeThreads)
    attn_lse_merge_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                          uint16_t* __restrict__ o, float* __restrict__ lse, int S, int R,
                          int BH) {
    constexpr int kColThreads = D / 4;                       // threads per partial row
    constexpr int kSlots = kMergeThreads / kColThreads;      // chunks per pass
    __shared__ float s_red[kMergeThreads / 32];
    __shared__ float4 s_acc[kSlots][kColThreads];
    __shared__ float s_w[kSlots];
    const int bh = blockIdx.x;
    const int tid = threadIdx.x;
    const int C = S * R;
    // chunk c (0 <= c < C) of this row: group c / S, chunk c % S within it
    auto row_of = [&](int c) -> size_t {
        const int r = c / S;
        const size_t row = ((size_t)r * BH + bh) * S + (c - r * S);
        return dcheck(row < (size_t)R * BH * S) ? row : 0;
    };
    // ---- M = max_c lse_c
    float M = -INFINITY;
    for (int c = tid; c < C; c += kMergeThreads) M = fmaxf(M, lse_part[row_of(c)]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    if ((tid & 31) == 0) s_red[tid >> 5] = M;
    __syncthreads();
    M = s_red[0];
#pragma unroll
    for (int w = 1; w < kMergeThreads / 32; ++w) M = fmaxf(M, s_red[w]);
    // ---- weighted sums, one chunk slot per group of kColThreads threads
    const int slot = tid / kColThreads, col = tid % kColThreads;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float W = 0.f;
    if (M != -INFINITY) {
        constexpr float kLog2e = 1.4426950408889634f;
        for (int c = slot; c < C; c += kSlots) {
            const size_t row = row_of(c);
            const float w = fast_exp2((lse_part[row] - M) * kLog2e);
            const float4 x = load_f32x4<VEC>(o_part + row * D + 4 * col);
            W += w;
            acc.x = fmaf(w, x.x, acc.x);
            acc.y = fmaf(w, x.y, acc.y);
            acc.z = fmaf(w, x.z, acc.z);
            acc.w = fmaf(w, x.w, acc.w);
        }
    }
    s_acc[slot][col] = acc;
    if (col == 0) s_w[slot] = W;
    __syncthreads();
    // ---- add the slots in order; threads 0 .. kColThreads-1 write the row
    if (tid < kColThreads) {
        float4 t = s_acc[0][tid];
        float Wt = s_w[0];
#pragma unroll
        for (int k = 1; k < kSlots; ++k) {
            const float4 u = s_acc[k][tid];
            t.x += u.x; t.y += u.y; t.z += u.z; t.w += u.w;
            Wt += s_w[k];
        }
        const bool any = Wt > 0.f;
        const uint32_t lo = pack_bf16x2(any ? t.x / Wt : 0.f, any ? t.y / Wt : 0.f);
        const uint32_t hi = pack_bf16x2(any ? t.z / Wt : 0.f, any ? t.w / Wt : 0.f);
        uint16_t* dst = o + (size_t)bh * D + 4 * tid;
        if ((reinterpret_cast<uintptr_t>(dst) & 7) == 0) {
            *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
        } else {   // o is only required to be 2-byte aligned
            dst[0] = (uint16_t)(lo & 0xFFFFu);
            dst[1] = (uint16_t)(lo >> 16);
            dst[2] = (uint16_t)(hi & 0xFFFFu);
            dst[3] = (uint16_t)(hi >> 16);
        }
        if (tid == 0) lse[bh] = Wt > 0.f ? M + logf(Wt) : -INFINITY;
    }
}

}  // namespace eattn
