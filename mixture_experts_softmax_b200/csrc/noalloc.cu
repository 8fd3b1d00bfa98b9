// noalloc.cu -- routing (router + dispatch) for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: code that runs inside an arena whose device
// memory is fixed up front (an inference server's pre-sized pool, an embedded runtime
// with a hard budget), or code driven from a framework that owns the allocator and does
// not hand out raw device memory.  moe_route_noalloc gives them the layer's routing
// without any allocation: the caller passes the inputs and the outputs, and the
// dispatch step's own working arrays live in one file-scope device array that every
// GPU loading this library holds until the process exits.
#include <cudaTypedefs.h>

#include <mutex>

#include "../../include/moe.h"
#include "kernels.cuh"

namespace {

constexpr int kE = moe::kExperts;
constexpr int kRouteBn = 16;   // padding granularity of dispatch's row map (the smallest tile width)
// dispatch's working arrays, in 4-byte words:
//   counts [E] | padded offsets [E+1] | row -> route map [2T + E*(bn-1)] | route -> row map [2T]
constexpr int kOffCounts = 0;
constexpr int kOffPoff = 64;
constexpr int kOffRperm = 128;
constexpr int kOffSlot = kOffRperm + ((2 * MOE_NOALLOC_MAX_TOKENS + kE * (kRouteBn - 1) + 63) / 64) * 64;
constexpr int kScratchWords = kOffSlot + 2 * MOE_NOALLOC_MAX_TOKENS;

}  // namespace

// the scratch itself: 256-byte aligned, kScratchWords * 4 bytes (about 1 MB)
static __device__ __align__(256) int g_route_scratch[kScratchWords];

namespace {

std::mutex g_mu;
// device address of g_route_scratch per CUDA device, with the context it was looked up in:
// the module (and so the array) is loaded again in a new context, for instance after
// cudaDeviceReset, so an address is reused only while the same context is current
int *g_scratch_dev[64];
CUcontext g_scratch_ctx[64];

CUcontext current_context()
{
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    }
    CUcontext c = nullptr;
    return fn(&c) == CUDA_SUCCESS ? c : nullptr;
}

// Device address of the scratch on the current device.  Looked up once per device (and
// context) with that device current: in host code the array's name is only a host-side
// stand-in.
int scratch_on_current_device(int **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return MOE_ENODEV;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    const CUcontext ctx = current_context();
    if (!g_scratch_dev[dev] || !ctx || ctx != g_scratch_ctx[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return MOE_ECUDA;
        }
        g_scratch_dev[dev] = static_cast<int *>(p);
        g_scratch_ctx[dev] = current_context();   // the lookup made the device's context current
    }
    *out = g_scratch_dev[dev];
    return MOE_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" MOE_API int moe_route_noalloc(int T, int d, const void *x, const float *router_w, const float *bias,
                                         int32_t *idx, float *gate, int32_t *offsets, int32_t *perm, void *stream)
{
    if (T < 0 || T > MOE_NOALLOC_MAX_TOKENS) return MOE_EINVAL;   // beyond the static scratch
    if (T == 0) return MOE_OK;
    if (d <= 0 || d % 8 != 0) return MOE_EINVAL;
    const void *ptrs[] = {x, router_w, idx, gate, offsets, perm};
    for (const void *p : ptrs)
        if (!p || !aligned16(p)) return MOE_EINVAL;
    if (bias && !aligned16(bias)) return MOE_EINVAL;
    int *scratch = nullptr;
    int rc = scratch_on_current_device(&scratch);
    if (rc != MOE_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    moe::RouteArgs ra{T, d, static_cast<const __nv_bfloat16 *>(x), router_w, bias, idx, gate};
    if (moe::launch_router(ra, s) != cudaSuccess) return MOE_ECUDA;
    // dispatch only writes the scratch (its row maps and padded offsets, which the full
    // layer's GEMMs would read); no word is read before this launch writes it, so nothing
    // needs clearing between calls
    moe::DispatchArgs da{T, kE, kRouteBn, idx, scratch + kOffCounts, offsets, scratch + kOffPoff,
                         perm, scratch + kOffRperm, scratch + kOffSlot};
    if (moe::launch_dispatch(da, s) != cudaSuccess) return MOE_ECUDA;
    return MOE_OK;
}
