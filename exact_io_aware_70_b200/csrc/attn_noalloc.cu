// attn_noalloc.cu -- split-KV decode that needs no device allocation at all.
//
// attn_decode_splitkv() asks its caller for a workspace that holds the
// per-chunk partials. Some callers have no way to provide one: code running
// where cudaMalloc is not allowed or not wanted (inside a custom allocator's
// own callbacks, in a plugin whose host framework owns every device
// allocation, on a hot path that must never touch the allocator), or code
// that simply has no device buffer of the right size at hand.
// attn_decode_splitkv_noalloc() serves them: its partials live in a fixed
// array that belongs to this library's module, so the caller passes only the
// inputs and outputs.
//
// Properties a user must know:
//   * The array is kDecodeScratchBytes (32 MiB) on every GPU that loads this
//     library, held until the process exits. Calls whose partials would not
//     fit are refused with ATTN_ERR_SCRATCH_LIMIT.
//   * The array is shared by every call on a device and keeps the last call's
//     contents. Nothing in it needs to start at zero: the partial kernel writes
//     every entry the merge kernel reads. Calls that overlap on the GPU (for
//     example on two streams at once) race on the array and give wrong
//     results; serialise them.
//   * The first call on each device looks up the array's device address with
//     cudaGetSymbolAddress (host code cannot use the symbol itself: on the host
//     it is only a stand-in, not a device address). Make that first call before
//     any stream capture begins.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "exact_attn.h"

namespace {

constexpr size_t kDecodeScratchBytes = size_t(32) << 20;   // 32 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kDecodeScratchBytes];

void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of this device's scratch array (set up once per device, with
// that device current). Returns nullptr if the lookup failed.
void* scratch_for_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = ptr;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" attn_status_t attn_decode_splitkv_noalloc(const void* q, const void* k, const void* v,
                                                     void* o, float* lse, int B, int H, int Nkv,
                                                     int d, float scale, int num_splits,
                                                     void* stream) {
    // Same arguments as attn_decode_splitkv, minus the workspace.
    if (B < 1 || H < 1 || num_splits < 1) return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    const size_t need = attn_decode_workspace_bytes(B, H, d, num_splits);
    if (need == 0) return ATTN_ERR_INVALID_ARG;
    if (need > kDecodeScratchBytes) return ATTN_ERR_SCRATCH_LIMIT;
    void* scratch = scratch_for_current_device();
    if (scratch == nullptr) return ATTN_ERR_CUDA;
    // Partials layout as in attn_decode_splitkv: O_c first, then lse_c, each
    // rounded up to 256 bytes.
    const size_t o_bytes = ((size_t)B * H * num_splits * d * 4 + 255) / 256 * 256;
    float* o_part = static_cast<float*>(scratch);
    float* lse_part = reinterpret_cast<float*>(static_cast<unsigned char*>(scratch) + o_bytes);
    attn_status_t s = attn_decode_partials(q, k, v, o_part, lse_part, B, H, Nkv, d, scale,
                                           num_splits, stream);
    if (s != ATTN_OK) return s;
    return attn_lse_merge(o_part, lse_part, o, lse, B, H, num_splits, d, stream);
}
