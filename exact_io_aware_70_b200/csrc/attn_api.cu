// attn_api.cu -- the C ABI declared in include/exact_attn.h.
//
// Argument checking, TMA tensor-map encoding and kernel launches. This is the
// only translation unit of the library that includes the kernels (they live
// in the .cuh files below) and defines the device status word, so that word
// has a single definition. The library's other translation unit,
// attn_noalloc.cu, holds the allocation-free decode's scratch array and calls
// only the extern "C" entry points defined here.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "exact_attn.h"

namespace eattn {
// Device status word: kernels OR error bits into it; attn_status() reads and clears it.
__device__ unsigned g_attn_status = 0;
}  // namespace eattn

#include "bwd_sm100.cuh"
#include "decode_sm100.cuh"
#include "fwd_sm100.cuh"

using namespace eattn;

namespace eattn {
// Waits on an mbarrier that nothing ever arrives on, through the same bounded
// wait every pipeline kernel uses, so the give-up path can be exercised
// without faulting or hanging the GPU.
__global__ void attn_wait_selftest_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_addr(&bar), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_limit(smem_addr(&bar), 0, &abort_flag, &g_attn_status, limit_ns);
}
}  // namespace eattn

namespace {

constexpr int kAbiVersion = 1;
constexpr float kLog2e = 1.4426950408889634f;
constexpr long long kMaxSeq = 1ll << 30;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Tensor map over a bf16 tensor viewed as [BH][N][D]; box = box_rows rows x 64
// columns, 128-byte swizzle, out-of-range rows read as zero.
bool encode_bf16_map(CUtensorMap* map, const void* base, int BH, int N, int D,
                     int box_rows = 128) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)N * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Tensor map over an 8-bit tensor viewed as [BH][N][D] with D = 128 or 64: box =
// 128 rows x D bytes, 128-byte swizzle (64-byte swizzle for D = 64), rows past
// N read as zero.
bool encode_u8_map(CUtensorMap* map, const void* base, int BH, int N, int D) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D, (cuuint64_t)N * D};
    cuuint32_t box[3] = {(cuuint32_t)D, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     D == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

struct DeviceInfo {
    int sms = 0;
    bool fwd_attr_set[8] = {false, false, false, false, false, false, false, false};
    bool bwd_attr_set[4] = {false, false, false, false};
};
DeviceInfo g_dev[64];
std::mutex g_dev_mu;

int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev;
}

// Unit-queue entry of the next forward launch (round robin): two launches
// share an entry only if kFwdQueueSlots further launches are started while
// the first is still running.
std::atomic<unsigned> g_fwd_queue_rr{0};

// Heads per group of the forward's unit order: as many heads as keep their
// K and V within EATTN_FWD_GROUP_BYTES, so the CTAs in flight find them in
// L2. Measured at 16K (8 MB of K/V per head): 16, 32, 48, 64, 96 and 128 MB
// groups ran 3.63, 3.55-3.59, 3.58, 3.50-3.54, 3.67 and 3.58 ms.
#ifndef EATTN_FWD_GROUP_BYTES
#define EATTN_FWD_GROUP_BYTES (64ll << 20)
#endif
int fwd_group_heads(int BH, int Nkv, int d, int elem_bytes) {
    const long long per_head = 2ll * Nkv * d * elem_bytes;
    long long g = EATTN_FWD_GROUP_BYTES / (per_head > 0 ? per_head : 1);
    if (g < 1) g = 1;
    return g < BH ? (int)g : BH;
}
// Units are dealt dynamically, in head groups, only when the K and V of all
// heads exceed this (the launch's K/V then cannot stay in the 126 MB L2 while
// every head is in flight); below it a static deal of the heaviest-first
// order is used. 0 forces the dynamic queue, a huge value the static deal.
// 1: the static deal also walks the units in head groups (measured slower)
#ifndef EATTN_FWD_STATIC_GROUPS
#define EATTN_FWD_STATIC_GROUPS 0
#endif
#ifndef EATTN_FWD_QUEUE_MIN_BYTES
#define EATTN_FWD_QUEUE_MIN_BYTES (192ll << 20)
#endif

template <int D, bool CAUSAL, bool FP8 = false>
attn_status_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& to, FwdParams p, cudaStream_t stream) {
    using T = FwdTraits<D, FP8>;
    const int dev = current_device();
    if (dev < 0 || dev >= 64) return ATTN_ERR_CUDA;
    auto kern = attn_fwd_sm100_kernel<D, CAUSAL, FP8>;
    int sms;
    {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        DeviceInfo& di = g_dev[dev];
        if (di.sms == 0 &&
            cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return ATTN_ERR_CUDA;
        const int slot = (FP8 ? 4 : 0) + (D == 128 ? 2 : 0) + (CAUSAL ? 1 : 0);
        if (!di.fwd_attr_set[slot]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     T::kSmemBytes) != cudaSuccess)
                return ATTN_ERR_CUDA;
            di.fwd_attr_set[slot] = true;
        }
        sms = di.sms;
    }
    const int grid = p.num_units < sms ? p.num_units : sms;
    p.dynamic_units =
        2ll * p.BH * p.Nkv * D * T::kElemBytes > EATTN_FWD_QUEUE_MIN_BYTES ? 1 : 0;
    // EXACT_ATTN_FWD_SCHEDULE=dynamic|static overrides the choice (for tests
    // and measurements; the result is the same either way)
    if (const char* sched = std::getenv("EXACT_ATTN_FWD_SCHEDULE")) {
        if (std::strcmp(sched, "dynamic") == 0) p.dynamic_units = 1;
        if (std::strcmp(sched, "static") == 0) p.dynamic_units = 0;
    }
    p.group_heads = (p.dynamic_units || EATTN_FWD_STATIC_GROUPS)
                        ? fwd_group_heads(p.BH, p.Nkv, D, T::kElemBytes)
                        : p.BH;
    p.queue_slot = (int)(g_fwd_queue_rr.fetch_add(1, std::memory_order_relaxed) % kFwdQueueSlots);
    kern<<<grid, T::kThreads, T::kSmemBytes, stream>>>(tq, tk, tv, to, p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <int D, bool CAUSAL>
attn_status_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& tdo, const BwdParams& p, cudaStream_t stream) {
    using T = BwdTraits<D>;
    const int dev = current_device();
    if (dev < 0 || dev >= 64) return ATTN_ERR_CUDA;
    auto kern = attn_bwd_sm100_kernel<D, CAUSAL>;
    {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        DeviceInfo& di = g_dev[dev];
        const int slot = (D == 128 ? 2 : 0) + (CAUSAL ? 1 : 0);
        if (!di.bwd_attr_set[slot]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     T::kSmemBytes) != cudaSuccess)
                return ATTN_ERR_CUDA;
            di.bwd_attr_set[slot] = true;
        }
    }
    const long long prows = (long long)p.BH * p.NqPad;
    constexpr int kRowsPerBlock = 256 / (D / 8);
    if (p.deterministic) {
        if (cudaMemsetAsync(p.bound, 0, 3 * sizeof(unsigned), stream) != cudaSuccess)
            return ATTN_ERR_CUDA;
        const long long kvrows = (long long)p.BH * p.Nkv;
        attn_bwd_kv_bound_kernel<D>
            <<<(unsigned)((kvrows + kRowsPerBlock - 1) / kRowsPerBlock), 256, 0, stream>>>(p);
    }
    attn_bwd_preprocess_kernel<D>
        <<<(unsigned)((prows + kRowsPerBlock - 1) / kRowsPerBlock), 256, 0, stream>>>(p);
    const long long rows = (long long)p.BH * p.Nq;
    // key blocks along x so that the CTAs resident at one time share a few
    // heads' Q and dO tiles in L2
    dim3 grid((p.Nkv + 127) / 128, p.BH);
    kern<<<grid, T::kThreads, T::kSmemBytes, stream>>>(tq, tk, tv, tdo, p);
    attn_bwd_postprocess_kernel<D>
        <<<(unsigned)((rows * D / 8 + 255) / 256), 256, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t check_sizes(int B, int H, long long N1, long long N2) {
    if (B < 1 || H < 1 || N1 < 1 || N2 < 1) return ATTN_ERR_INVALID_ARG;
    if (N1 > kMaxSeq || N2 > kMaxSeq) return ATTN_ERR_INVALID_ARG;
    if ((long long)B * H > (1ll << 24)) return ATTN_ERR_INVALID_ARG;
    return ATTN_OK;
}

}  // namespace

extern "C" {

int attn_abi_version(void) { return kAbiVersion; }

const char* attn_strerror(attn_status_t s) {
    switch (s) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_INVALID_ARG: return "invalid argument (null pointer or bad size)";
        case ATTN_ERR_UNSUPPORTED: return "unsupported configuration (head dim must be 64 or 128)";
        case ATTN_ERR_ALIGNMENT: return "misaligned pointer (bf16 tensors need 16 bytes, fp32 4)";
        case ATTN_ERR_CUDA: return "CUDA error while launching or running a kernel";
        case ATTN_ERR_TIMEOUT: return "a kernel pipeline wait timed out; outputs are invalid";
        case ATTN_ERR_SCRATCH_LIMIT:
            return "partials exceed the library's fixed 32 MiB decode scratch array";
        case ATTN_ERR_BAD_INDEX:
            return "a block-table entry or sequence length was out of range; those keys were skipped";
        case ATTN_ERR_INDEX_CHECK:
            return "debug build: a kernel computed an index outside its tensor; the access was skipped";
    }
    return "unknown status";
}

attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int H, int Nq, int Nkv, int d, int causal, float scale, void* stream) {
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    attn_status_t s = check_sizes(B, H, Nq, Nkv);
    if (s != ATTN_OK) return s;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(lse, 4))
        return ATTN_ERR_ALIGNMENT;

    const int BH = B * H;
    CUtensorMap tq, tk, tv, to;
    // O: stored by the softmax warps as boxes of 32 rows x 64 columns
    if (!encode_bf16_map(&tq, q, BH, Nq, d) || !encode_bf16_map(&tk, k, BH, Nkv, d) ||
        !encode_bf16_map(&tv, v, BH, Nkv, d) || !encode_bf16_map(&to, o, BH, Nq, d, 32))
        return ATTN_ERR_CUDA;
    FwdParams p;
    p.o = static_cast<uint16_t*>(o);
    p.lse = lse;
    p.q_descale = p.k_descale = p.v_descale = nullptr;
    p.BH = BH;
    p.Nq = Nq;
    p.Nkv = Nkv;
    p.num_qb = (Nq + 255) / 256;
    const long long units = (long long)BH * p.num_qb;
    if (units > (1ll << 30)) return ATTN_ERR_INVALID_ARG;
    p.num_units = (int)units;
    p.scale_log2 = scale * kLog2e;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d == 128)
        return causal ? launch_fwd<128, true>(tq, tk, tv, to, p, st)
                      : launch_fwd<128, false>(tq, tk, tv, to, p, st);
    return causal ? launch_fwd<64, true>(tq, tk, tv, to, p, st)
                  : launch_fwd<64, false>(tq, tk, tv, to, p, st);
}

attn_status_t attn_fwd_fp8(const void* q, const void* k, const void* v, const float* q_descale,
                           const float* k_descale, const float* v_descale, void* o, float* lse,
                           int B, int H, int Nq, int Nkv, int d, int causal, float scale,
                           void* stream) {
    if (!q || !k || !v || !q_descale || !k_descale || !v_descale || !o || !lse)
        return ATTN_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    attn_status_t s = check_sizes(B, H, Nq, Nkv);
    if (s != ATTN_OK) return s;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(lse, 4) || !aligned(q_descale, 4) || !aligned(k_descale, 4) ||
        !aligned(v_descale, 4))
        return ATTN_ERR_ALIGNMENT;
    const int BH = B * H;
    CUtensorMap tq, tk, tv, to;
    if (!encode_u8_map(&tq, q, BH, Nq, d) || !encode_u8_map(&tk, k, BH, Nkv, d) ||
        !encode_u8_map(&tv, v, BH, Nkv, d) || !encode_bf16_map(&to, o, BH, Nq, d, 32))
        return ATTN_ERR_CUDA;
    FwdParams p;
    p.o = static_cast<uint16_t*>(o);
    p.lse = lse;
    p.q_descale = q_descale;
    p.k_descale = k_descale;
    p.v_descale = v_descale;
    p.BH = BH;
    p.Nq = Nq;
    p.Nkv = Nkv;
    p.num_qb = (Nq + 255) / 256;
    const long long units = (long long)BH * p.num_qb;
    if (units > (1ll << 30)) return ATTN_ERR_INVALID_ARG;
    p.num_units = (int)units;
    p.scale_log2 = scale * kLog2e;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d == 128)
        return causal ? launch_fwd<128, true, true>(tq, tk, tv, to, p, st)
                      : launch_fwd<128, false, true>(tq, tk, tv, to, p, st);
    return causal ? launch_fwd<64, true, true>(tq, tk, tv, to, p, st)
                  : launch_fwd<64, false, true>(tq, tk, tv, to, p, st);
}

attn_status_t attn_decode_partials(const void* q, const void* k, const void* v, float* o_part,
                                   float* lse_part, int B, int H, int Nkv, int d, float scale,
                                   int num_splits, void* stream) {
    if (!q || !k || !v || !o_part || !lse_part) return ATTN_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    attn_status_t s = check_sizes(B, H, Nkv, 1);
    if (s != ATTN_OK) return s;
    if (num_splits < 1 || num_splits > 65535) return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o_part, 4) ||
        !aligned(lse_part, 4))
        return ATTN_ERR_ALIGNMENT;
    DecodeParams p;
    p.q = static_cast<const uint16_t*>(q);
    p.k = static_cast<const uint16_t*>(k);
    p.v = static_cast<const uint16_t*>(v);
    p.o_part = o_part;
    p.lse_part = lse_part;
    p.Nkv = Nkv;
    p.S = num_splits;
    p.L = (int)(((long long)Nkv + num_splits - 1) / num_splits);
    p.scale_log2 = scale * kLog2e;
    dim3 grid(num_splits, B * H);
    if (B * H > 65535) return ATTN_ERR_INVALID_ARG;   // grid.y limit
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    p.block_table = nullptr;
    p.seq_lens = nullptr;
    p.H = H;
    p.page_shift = p.max_pages = p.num_pages = 0;
    if (d == 128)
        attn_decode_partials_kernel<128, false><<<grid, DecodeTraits<128>::kThreads, 0, st>>>(p);
    else
        attn_decode_partials_kernel<64, false><<<grid, DecodeTraits<64>::kThreads, 0, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t attn_decode_paged_partials(const void* q, const void* k_cache, const void* v_cache,
                                         const int* block_table, const int* seq_lens,
                                         float* o_part, float* lse_part, int B, int H, int d,
                                         int page_size, int max_pages_per_seq, int num_pages,
                                         float scale, int num_splits, void* stream) {
    if (!q || !k_cache || !v_cache || !block_table || !seq_lens || !o_part || !lse_part)
        return ATTN_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    attn_status_t s = check_sizes(B, H, 1, 1);
    if (s != ATTN_OK) return s;
    if (num_splits < 1 || num_splits > 65535 || B * H > 65535) return ATTN_ERR_INVALID_ARG;
    if (page_size < 16 || page_size > 1024 || (page_size & (page_size - 1)) != 0)
        return ATTN_ERR_INVALID_ARG;
    if (max_pages_per_seq < 1 || num_pages < 1) return ATTN_ERR_INVALID_ARG;
    if ((long long)max_pages_per_seq * page_size > kMaxSeq) return ATTN_ERR_INVALID_ARG;
    if ((long long)num_pages * H * page_size * d > (1ll << 46)) return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_table, 4) || !aligned(seq_lens, 4) || !aligned(o_part, 4) ||
        !aligned(lse_part, 4))
        return ATTN_ERR_ALIGNMENT;
    DecodeParams p;
    p.q = static_cast<const uint16_t*>(q);
    p.k = static_cast<const uint16_t*>(k_cache);
    p.v = static_cast<const uint16_t*>(v_cache);
    p.o_part = o_part;
    p.lse_part = lse_part;
    p.Nkv = 0;
    p.L = 0;
    p.S = num_splits;
    p.scale_log2 = scale * kLog2e;
    p.block_table = block_table;
    p.seq_lens = seq_lens;
    p.H = H;
    p.page_shift = 0;
    while ((1 << p.page_shift) < page_size) ++p.page_shift;
    p.max_pages = max_pages_per_seq;
    p.num_pages = num_pages;
    dim3 grid(num_splits, B * H);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d == 128)
        attn_decode_partials_kernel<128, true><<<grid, DecodeTraits<128>::kThreads, 0, st>>>(p);
    else
        attn_decode_partials_kernel<64, true><<<grid, DecodeTraits<64>::kThreads, 0, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t attn_decode_paged(const void* q, const void* k_cache, const void* v_cache,
                                const int* block_table, const int* seq_lens, void* o, float* lse,
                                int B, int H, int d, int page_size, int max_pages_per_seq,
                                int num_pages, float scale, int num_splits, void* workspace,
                                size_t workspace_bytes, void* stream) {
    if (!workspace || !o || !lse) return ATTN_ERR_INVALID_ARG;
    const size_t need = attn_decode_workspace_bytes(B, H, d, num_splits);
    if (need == 0) {
        if (d != 64 && d != 128 && B >= 1 && H >= 1 && num_splits >= 1)
            return ATTN_ERR_UNSUPPORTED;
        return ATTN_ERR_INVALID_ARG;
    }
    if (workspace_bytes < need) return ATTN_ERR_INVALID_ARG;
    if (!aligned(workspace, 256) || !aligned(o, 2) || !aligned(lse, 4)) return ATTN_ERR_ALIGNMENT;
    float* o_part = static_cast<float*>(workspace);
    const size_t o_bytes = ((size_t)B * H * num_splits * d * 4 + 255) / 256 * 256;
    float* lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + o_bytes);
    attn_status_t s = attn_decode_paged_partials(q, k_cache, v_cache, block_table, seq_lens,
                                                 o_part, lse_part, B, H, d, page_size,
                                                 max_pages_per_seq, num_pages, scale, num_splits,
                                                 stream);
    if (s != ATTN_OK) return s;
    return attn_lse_merge(o_part, lse_part, o, lse, B, H, num_splits, d, stream);
}

}  // extern "C"

namespace {
attn_status_t launch_merge(const float* o_part, const float* lse_part, void* o, float* lse,
                           int B, int H, int S, int R, int d, void* stream) {
    if (!o_part || !lse_part || !o || !lse) return ATTN_ERR_INVALID_ARG;
    attn_status_t s = check_sizes(B, H, 1, 1);
    if (s != ATTN_OK) return s;
    if (S < 1 || S > 65535 || R < 1 || R > 65535) return ATTN_ERR_INVALID_ARG;
    if ((long long)S * R > (1ll << 24)) return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (!aligned(o_part, 4) || !aligned(lse_part, 4) || !aligned(o, 2) || !aligned(lse, 4))
        return ATTN_ERR_ALIGNMENT;
    const int BH = B * H;
    if ((long long)BH * S * R * d >= (1ll << 46)) return ATTN_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint16_t* ob = static_cast<uint16_t*>(o);
    const bool vec = aligned(o_part, 16);
    if (d == 128) {
        if (vec)
            attn_lse_merge_kernel<128, true><<<BH, kMergeThreads, 0, st>>>(o_part, lse_part, ob,
                                                                          lse, S, R, BH);
        else
            attn_lse_merge_kernel<128, false><<<BH, kMergeThreads, 0, st>>>(o_part, lse_part, ob,
                                                                           lse, S, R, BH);
    } else {
        if (vec)
            attn_lse_merge_kernel<64, true><<<BH, kMergeThreads, 0, st>>>(o_part, lse_part, ob,
                                                                         lse, S, R, BH);
        else
            attn_lse_merge_kernel<64, false><<<BH, kMergeThreads, 0, st>>>(o_part, lse_part, ob,
                                                                          lse, S, R, BH);
    }
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}
}  // namespace

extern "C" {

attn_status_t attn_lse_merge(const float* o_part, const float* lse_part, void* o, float* lse,
                             int B, int H, int S, int d, void* stream) {
    return launch_merge(o_part, lse_part, o, lse, B, H, S, 1, d, stream);
}

attn_status_t attn_lse_merge_gathered(const float* o_part, const float* lse_part, void* o,
                                      float* lse, int R, int B, int H, int S, int d,
                                      void* stream) {
    return launch_merge(o_part, lse_part, o, lse, B, H, S, R, d, stream);
}

size_t attn_decode_workspace_bytes(int B, int H, int d, int num_splits) {
    if (B < 1 || H < 1 || num_splits < 1 || (d != 64 && d != 128)) return 0;
    const size_t bhs = (size_t)B * H * num_splits;
    const size_t o_bytes = (bhs * d * 4 + 255) / 256 * 256;
    const size_t l_bytes = (bhs * 4 + 255) / 256 * 256;
    return o_bytes + l_bytes;
}

attn_status_t attn_decode_splitkv(const void* q, const void* k, const void* v, void* o,
                                  float* lse, int B, int H, int Nkv, int d, float scale,
                                  int num_splits, void* workspace, size_t workspace_bytes,
                                  void* stream) {
    if (!workspace) return ATTN_ERR_INVALID_ARG;
    const size_t need = attn_decode_workspace_bytes(B, H, d, num_splits);
    if (need == 0) {
        if (d != 64 && d != 128 && B >= 1 && H >= 1 && num_splits >= 1)
            return ATTN_ERR_UNSUPPORTED;
        return ATTN_ERR_INVALID_ARG;
    }
    if (workspace_bytes < need) return ATTN_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return ATTN_ERR_ALIGNMENT;
    if (!o || !lse) return ATTN_ERR_INVALID_ARG;
    if (!aligned(o, 2) || !aligned(lse, 4)) return ATTN_ERR_ALIGNMENT;
    float* o_part = static_cast<float*>(workspace);
    const size_t o_bytes = ((size_t)B * H * num_splits * d * 4 + 255) / 256 * 256;
    float* lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + o_bytes);
    attn_status_t s = attn_decode_partials(q, k, v, o_part, lse_part, B, H, Nkv, d, scale,
                                           num_splits, stream);
    if (s != ATTN_OK) return s;
    return attn_lse_merge(o_part, lse_part, o, lse, B, H, num_splits, d, stream);
}

size_t attn_bwd_workspace_bytes(int B, int H, int Nq, int d) {
    if (B < 1 || H < 1 || Nq < 1 || (d != 64 && d != 128)) return 0;
    const size_t prow = (size_t)B * H * (((size_t)Nq + 63) / 64 * 64);
    return 2 * ((prow * 4 + 255) / 256 * 256) + 256 + (size_t)B * H * Nq * d * 8;
}

}  // extern "C"

namespace {
attn_status_t bwd_entry(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                        int H, int Nq, int Nkv, int d, int causal, float scale, void* workspace,
                        size_t workspace_bytes, void* stream, bool deterministic) {
    if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace)
        return ATTN_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    attn_status_t s = check_sizes(B, H, Nq, Nkv);
    if (s != ATTN_OK) return s;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    const int BH = B * H;
    if (BH > 65535) return ATTN_ERR_INVALID_ARG;   // grid.y limit
    if ((long long)BH * Nq * d / 2048 >= (1ll << 31)) return ATTN_ERR_INVALID_ARG;
    if (workspace_bytes < attn_bwd_workspace_bytes(B, H, Nq, d)) return ATTN_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
        !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
        !aligned(lse, 4) || !aligned(workspace, 256))
        return ATTN_ERR_ALIGNMENT;
    CUtensorMap tq, tk, tv, tdo;
    if (!encode_bf16_map(&tq, q, BH, Nq, d, 64) || !encode_bf16_map(&tk, k, BH, Nkv, d) ||
        !encode_bf16_map(&tv, v, BH, Nkv, d) || !encode_bf16_map(&tdo, dout, BH, Nq, d, 64))
        return ATTN_ERR_CUDA;
    const int NqPad = (Nq + 63) / 64 * 64;
    const size_t pbytes = ((size_t)BH * NqPad * 4 + 255) / 256 * 256;
    BwdParams p;
    p.o = static_cast<const uint16_t*>(o);
    p.dout = static_cast<const uint16_t*>(dout);
    p.lse = lse;
    p.delta = static_cast<float*>(workspace);
    p.lse2 = reinterpret_cast<float*>(static_cast<char*>(workspace) + pbytes);
    p.bound = reinterpret_cast<unsigned*>(static_cast<char*>(workspace) + 2 * pbytes);
    p.dq_acc = static_cast<char*>(workspace) + 2 * pbytes + 256;
    p.deterministic = deterministic ? 1 : 0;
    p.k = static_cast<const uint16_t*>(k);
    p.v = static_cast<const uint16_t*>(v);
    p.NqPad = NqPad;
    p.dq = static_cast<uint16_t*>(dq);
    p.dk = static_cast<uint16_t*>(dk);
    p.dv = static_cast<uint16_t*>(dv);
    p.BH = BH;
    p.Nq = Nq;
    p.Nkv = Nkv;
    p.scale = scale;
    p.scale_log2 = scale * kLog2e;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (d == 128)
        return causal ? launch_bwd<128, true>(tq, tk, tv, tdo, p, st)
                      : launch_bwd<128, false>(tq, tk, tv, tdo, p, st);
    return causal ? launch_bwd<64, true>(tq, tk, tv, tdo, p, st)
                  : launch_bwd<64, false>(tq, tk, tv, tdo, p, st);
}
}  // namespace

extern "C" {

attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o,
                       const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                       int H, int Nq, int Nkv, int d, int causal, float scale, void* workspace,
                       size_t workspace_bytes, void* stream) {
    return bwd_entry(q, k, v, o, dout, lse, dq, dk, dv, B, H, Nq, Nkv, d, causal, scale,
                     workspace, workspace_bytes, stream, false);
}

attn_status_t attn_bwd_deterministic(const void* q, const void* k, const void* v, const void* o,
                                     const void* dout, const float* lse, void* dq, void* dk,
                                     void* dv, int B, int H, int Nq, int Nkv, int d, int causal,
                                     float scale, void* workspace, size_t workspace_bytes,
                                     void* stream) {
    return bwd_entry(q, k, v, o, dout, lse, dq, dk, dv, B, H, Nq, Nkv, d, causal, scale,
                     workspace, workspace_bytes, stream, true);
}

attn_status_t attn_selftest_wait_timeout(unsigned limit_us, void* stream) {
    if (limit_us < 1 || limit_us > 1000000) return ATTN_ERR_INVALID_ARG;
    attn_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        (unsigned long long)limit_us * 1000ull);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t attn_status(void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return ATTN_ERR_CUDA;
    unsigned word = 0;
    if (cudaMemcpyFromSymbol(&word, g_attn_status, sizeof(word)) != cudaSuccess)
        return ATTN_ERR_CUDA;
    if (word != 0) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(g_attn_status, &zero, sizeof(zero)) != cudaSuccess)
            return ATTN_ERR_CUDA;
    }
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    if (word & kDevErrTimeout) return ATTN_ERR_TIMEOUT;
    if (word & kDevErrIndexCheck) return ATTN_ERR_INDEX_CHECK;
    if (word & kDevErrBadIndex) return ATTN_ERR_BAD_INDEX;
    return ATTN_OK;
}

}  // extern "C"
