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
// This translation unit holds only that array and the entry point; it calls
// the library's other extern "C" entry points and includes no kernel.
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
//   * The first call in each CUDA context looks up the array's device address
//     with cudaGetSymbolAddress (host code cannot use the symbol itself: on the
//     host it is only a stand-in, not a device address). Make that first call
//     before any stream capture begins. The address is cached per device
//     together with the context's unique id, so a context that was torn down
//     and created again (cudaDeviceReset, for instance) gets a fresh lookup
//     instead of a stale address.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "exact_attn.h"

namespace {

constexpr size_t kDecodeScratchBytes = size_t(32) << 20;   // 32 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kDecodeScratchBytes];

struct ScratchSlot {
    unsigned long long ctx_id = 0;   // id of the context the address belongs to
    void* ptr = nullptr;
};
ScratchSlot g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

template <class Fn>
Fn driver_fn(const char* name) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion(name, &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(p);
}

// Unique id of the calling thread's current context (0 if none is current).
bool current_ctx_id(unsigned long long* id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
        get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    });
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS) return false;
    if (ctx == nullptr) {
        *id = 0;
        return true;
    }
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array in the current context, with the
// device current. Returns nullptr if the lookup failed.
void* scratch_for_current_context() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    unsigned long long id = 0;
    if (!current_ctx_id(&id)) return nullptr;
    ScratchSlot& s = g_scratch[dev];
    if (id != 0 && s.ptr != nullptr && s.ctx_id == id) return s.ptr;
    // First use in this context (or no context yet: the lookup below makes the
    // runtime create the device's primary context and make it current).
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess) return nullptr;
    if (!current_ctx_id(&id) || id == 0) return nullptr;
    s.ctx_id = id;
    s.ptr = ptr;
    return ptr;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" attn_status_t attn_decode_splitkv_noalloc(const void* q, const void* k, const void* v,
                                                     void* o, float* lse, int B, int H, int Nkv,
                                                     int d, float scale, int num_splits,
                                                     void* stream) {
    // Same arguments and checks as attn_decode_splitkv, minus the workspace.
    // Every argument is checked here, before anything is enqueued, so that no
    // partial kernel is launched into the shared array for a call that the
    // merge step would then refuse.
    if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || Nkv < 1 || Nkv > (1 << 30)) return ATTN_ERR_INVALID_ARG;
    if ((long long)B * H > 65535) return ATTN_ERR_INVALID_ARG;   // grid.y of both kernels
    if (num_splits < 1 || num_splits > 65535) return ATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 2) ||
        !aligned(lse, 4))
        return ATTN_ERR_ALIGNMENT;
    const size_t need = attn_decode_workspace_bytes(B, H, d, num_splits);
    if (need == 0) return ATTN_ERR_INVALID_ARG;
    if (need > kDecodeScratchBytes) return ATTN_ERR_SCRATCH_LIMIT;
    void* scratch = scratch_for_current_context();
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
