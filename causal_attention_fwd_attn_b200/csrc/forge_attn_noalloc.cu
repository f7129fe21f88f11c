// forge_attn_noalloc.cu -- the backward for callers that cannot allocate device
// memory.
//
// forge_attn_bwd needs a workspace (the row statistics and the fp32 dQ accumulator) that
// the caller allocates.  Some callers cannot: code that runs after a fixed memory
// budget has been handed out at start-up (a serving process or an embedded runtime
// that forbids allocation once running), code whose allocator is not reachable
// from the call site (a plugin handed only raw device pointers), or code that must
// not hit the allocator's synchronisation on a latency-critical path.  This file
// gives them the same backward with its scratch in a fixed, file-scope device
// array instead.
//
// The array is allocated when the library's device code is loaded onto a GPU and
// is held on every GPU that loads the library until the process exits.  All calls
// on a device share it and it keeps the last call's contents; the D pre-pass
// rewrites the row statistics and clears the dQ accumulator at the start of every
// call, so nothing
// leaks from one call into the next.  Two calls whose kernels overlap on the GPU
// (different streams, no ordering between them) race on the array.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "forge_attn.h"
#include "forge_internal.h"

namespace forge {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[FORGE_ATTN_NOALLOC_SCRATCH_BYTES];

// Device addresses of the array, one per CUDA context it was looked up in.  The
// array's address belongs to the copy of the library's device code loaded into a
// context; a new context on the same device (after cudaDeviceReset, or a
// caller-created context) has its own copy, so entries are keyed by the context's
// process-unique ID rather than by the device ordinal.
struct ScratchEntry {
    unsigned long long ctx_id;
    void* addr;
};
constexpr int kMaxContexts = 64;
std::mutex g_scratch_mutex;
ScratchEntry g_scratch_addr[kMaxContexts] = {};
int g_scratch_next = 0;

using GetCurrentFn = CUresult (*)(CUcontext*);
using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// ID of the calling thread's current context (0 when none is current or the driver
// cannot say).
unsigned long long current_context_id() {
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the scratch array in the current context.  The host-side name
// g_noalloc_scratch is only a stand-in for the symbol; the address a kernel can use
// comes from cudaGetSymbolAddress, looked up once per context with that context
// current (the first call in a context also loads the library's device code there).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    unsigned long long id = current_context_id();
    if (id != 0)
        for (const ScratchEntry& s : g_scratch_addr)
            if (s.ctx_id == id && s.addr) {
                *out = s.addr;
                return cudaSuccess;
            }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    if (id == 0) id = current_context_id();  // the lookup made the primary context current
    if (id != 0) {
        g_scratch_addr[g_scratch_next] = {id, p};
        g_scratch_next = (g_scratch_next + 1) % kMaxContexts;
    }
    *out = p;
    return cudaSuccess;
}

size_t round_up_256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace
}  // namespace forge

using namespace forge;

extern "C" int forge_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                      const void* dO, const float* lse, void* dq, void* dk,
                                      void* dv, int B, int H, int T, int d, float scale,
                                      int causal, void* stream) {
    if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv)
        return FORGE_ATTN_ERR_INVALID_ARG;
    // every argument is checked here, before the first of the three launches
    if (B < 1 || H < 1 || T < 1 || d < 1) return FORGE_ATTN_ERR_INVALID_ARG;
    const size_t need = forge_attn_bwd_workspace_size(B, H, T, d);
    if (need == 0) return FORGE_ATTN_ERR_UNSUPPORTED;
    if (!std::isfinite(scale)) return FORGE_ATTN_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return FORGE_ATTN_ERR_INVALID_ARG;
    for (const void* p : {q, k, v, o, dO, (const void*)dq, (const void*)dk, (const void*)dv})
        if (reinterpret_cast<uintptr_t>(p) & 15u) return FORGE_ATTN_ERR_MISALIGNED;
    if (reinterpret_cast<uintptr_t>(lse) & 3u) return FORGE_ATTN_ERR_MISALIGNED;
    // the fixed array plays the part of the workspace: sizes that need more are refused
    if (need > (size_t)FORGE_ATTN_NOALLOC_SCRATCH_BYTES) return FORGE_ATTN_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return FORGE_ATTN_ERR_CUDA;
    // same layout as the workspace of forge_attn_bwd: padded row statistics, then the
    // fp32 dQ accumulator
    const size_t t_pad = (size_t)((T + 127) / 128) * 128;
    float* rowstats = static_cast<float*>(scratch);
    float* acc = reinterpret_cast<float*>(static_cast<char*>(scratch) +
                                          round_up_256(2 * (size_t)B * H * t_pad * sizeof(float)));
    int s = forge_attn_bwd_preprocess(o, dO, lse, rowstats, acc, B, H, T, d, 0, stream);
    if (s != FORGE_ATTN_OK) return s;
    s = forge_attn_bwd_dkdv(q, k, v, dO, rowstats, acc, dk, dv, B, H, T, d, scale, causal, 0,
                            stream);
    if (s != FORGE_ATTN_OK) return s;
    return forge_attn_bwd_dq_convert(acc, dq, B, H, T, d, stream);
}
