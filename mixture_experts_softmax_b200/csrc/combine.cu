// combine.cu -- sum the gate-weighted expert outputs back in token order
// ("Grok-1 Admin & Architecture Guide", section 3, "Mixture of Experts", step 4),
// and the residual-block variant with the post-MoE RMSNorm and residual add
// ("Transformer stack and language model head": h += h_dense).
//
// The down-projection epilogue has already written gate * s1 * (partial sum) of
// every route into its own slot [split, t, j, :].  Here each output element is the
// sum of its 2 * splits slots in a fixed order (split ascending, slot 0 before
// slot 1), so the result does not depend on scheduling.
#include "kernels.cuh"
#include "ptx.cuh"

namespace moe {

namespace {

__device__ __forceinline__ float4 ld4(const float *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }

__device__ __forceinline__ void add4(float4 &a, const float4 &b)
{
    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
}

// fixed-order sum of one token's slots for 4 consecutive features.  The split loop runs to
// the compile-time maximum MAXS with the unused splits predicated off, so that all the loads
// of a chunk are in flight together instead of one L2 round trip per split.
template <int MAXS>
__device__ __forceinline__ float4 slot_sum(const CombineArgs &a, int t, int c)
{
    const size_t plane = static_cast<size_t>(a.T) * 2 * a.d;
    const float *p = a.slots + (static_cast<size_t>(t) * 2) * a.d + c;
    float4 v0[MAXS], v1[MAXS];
#pragma unroll
    for (int s = 0; s < MAXS; ++s) {
        if (s < a.splits) {
            v0[s] = ld4(p + s * plane);
            v1[s] = ld4(p + s * plane + a.d);
        }
    }
    float4 y0 = v0[0], y1 = v1[0];
#pragma unroll
    for (int s = 1; s < MAXS; ++s) {
        if (s < a.splits) {
            add4(y0, v0[s]);
            add4(y1, v1[s]);
        }
    }
    add4(y0, y1);
    return y0;
}

template <int MAXS>
__global__ void __launch_bounds__(256) combine_kernel(CombineArgs a)
{
    griddep_wait();   // launched to overlap the down-projection's end: its slots first
    const int per_row = a.d >> 2;
    const size_t n = static_cast<size_t>(a.T) * per_row;
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const int t = static_cast<int>(i / per_row), c = static_cast<int>(i % per_row) * 4;
        // a padding token (expert -1) has no slots: its output row is 0
        const float4 y = __ldg(a.idx + 2 * t) < 0 ? make_float4(0.f, 0.f, 0.f, 0.f) : slot_sum<MAXS>(a, t, c);
        __nv_bfloat162 lo = __floats2bfloat162_rn(y.x, y.y), hi = __floats2bfloat162_rn(y.z, y.w);
        uint2 v;
        v.x = *reinterpret_cast<uint32_t *>(&lo);
        v.y = *reinterpret_cast<uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(a.out + static_cast<size_t>(t) * a.d + c) = v;
    }
}

// one block per token: y = sum of slots; h <- bf16( h + y * rsqrt(mean(y^2) + eps) * g_post )
template <int MAXS>
__global__ void __launch_bounds__(256) combine_postnorm_kernel(CombineArgs a)
{
    __shared__ float red[8];
    griddep_wait();   // launched to overlap the down-projection's end: its slots first
    const int t = blockIdx.x;
    if (__ldg(a.idx + 2 * t) < 0) return;   // a padding token: the residual row passes through unchanged
    float ss = 0.f;
    for (int c = threadIdx.x * 4; c < a.d; c += blockDim.x * 4) {
        const float4 y = slot_sum<MAXS>(a, t, c);
        ss = fmaf(y.x, y.x, fmaf(y.y, y.y, fmaf(y.z, y.z, fmaf(y.w, y.w, ss))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += red[w];
    const float r = rsqrtf(tot / static_cast<float>(a.d) + a.eps);
    __nv_bfloat16 *hr = a.h_io + static_cast<size_t>(t) * a.d;
    for (int c = threadIdx.x * 4; c < a.d; c += blockDim.x * 4) {
        const float4 y = slot_sum<MAXS>(a, t, c);
        const float yv[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float hv = __bfloat162float(hr[c + q]);
            hr[c + q] = __float2bfloat16_rn(hv + yv[q] * r * __bfloat162float(a.g_post[c + q]));
        }
    }
}

}  // namespace

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t s)
{
    if (a.T <= 0) return cudaSuccess;
    // programmatic stream serialization: the blocks may be scheduled while the down-projection
    // ends; each waits for it before reading the slots
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    // one split (large batches): the plain loop; several: all split loads in flight together
    if (a.h_io) {
        cfg.gridDim = dim3(a.T);
        return a.splits == 1 ? cudaLaunchKernelEx(&cfg, combine_postnorm_kernel<1>, a)
                             : cudaLaunchKernelEx(&cfg, combine_postnorm_kernel<kMaxSplits>, a);
    }
    const size_t n = static_cast<size_t>(a.T) * (a.d >> 2);
    const size_t want = (n + 255) / 256;
    cfg.gridDim = dim3(static_cast<unsigned>(want < 148 * 16 ? want : 148 * 16));
    return a.splits == 1 ? cudaLaunchKernelEx(&cfg, combine_kernel<1>, a)
                         : cudaLaunchKernelEx(&cfg, combine_kernel<kMaxSplits>, a);
}

}  // namespace moe
