// router.cu -- routing logits, softmax and top-2 ("Grok-1 Admin & Architecture Guide",
// section 3, "Mixture of Experts (MoELayer + Router)", steps 1-2), with the pre-MoE
// RMSNorm of the residual block ("Transformer stack and language model head") folded in:
// the routed row is then the normalised one, which the kernel also stores for the gather.
#include "kernels.cuh"
#include "ptx.cuh"
#include "route_common.cuh"

namespace moe {

namespace {

constexpr int kRouterWarps = 16;      // large-T variant: warps per block
constexpr int kTokensPerWarp = 4;     // large-T variant: tokens sharing each router-weight load
constexpr size_t kRouterSmemMax = 224 * 1024;   // large-T variant: the staged router weight (d <= 7168)
constexpr int kSmallT = 256;          // up to this many tokens: one block per token

// Few tokens: one block per token (route_token, shared with the fused small-batch routing).
__global__ void __launch_bounds__(kRouteTokenThreads) router_small_kernel(RouteArgs a) { route_token(a, blockIdx.x); }

// Many tokens: each warp takes 4 tokens, so every router-weight load feeds 4 tokens; lane
// partial sums are reduced with a butterfly (fixed order; every lane ends with the same sum).
// The block first stages the whole router weight ([d, 8] fp32, 32 bytes per input row) in
// shared memory, then walks groups of 16 warps x 4 tokens.  Lane l reads the 8 rows of its
// 8-element chunk c as 16 float4 units; unit u of chunk c sits at unit slot u ^ (c & 7), so
// the 32 lanes of a warp (consecutive chunks) spread over the 8 bank groups instead of all
// landing on one.
// With a.g_pre set (the residual block), the routed rows are u = bf16(x * rsqrt(mean(x^2) +
// eps) * g_pre): a first pass takes each token's sum of squares (lane partials over the
// lane's chunks in order, then the butterfly), the second forms each 8-element chunk of u in
// fp32, rounds it to bf16, stores it to a.u (for the gather) and routes on it.
__global__ void __launch_bounds__(kRouterWarps * 32, 1) router_kernel(RouteArgs a)
{
    extern __shared__ float4 wsm[];   // [d / 8 chunks][16 units], swizzled
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int chunks = a.d >> 3;
    const float4 *w4 = reinterpret_cast<const float4 *>(a.w);
    for (int i = threadIdx.x; i < chunks * 16; i += blockDim.x) {
        const int c = i >> 4, u = i & 15;
        wsm[c * 16 + (u ^ (c & 7))] = __ldg(w4 + i);
    }
    __syncthreads();
    constexpr int kGroup = kRouterWarps * kTokensPerWarp;
    for (int g0 = blockIdx.x * kGroup; g0 < a.T; g0 += gridDim.x * kGroup) {
        const int t0 = g0 + warp * kTokensPerWarp;
        if (t0 >= a.T) continue;   // warp-uniform; no block barrier follows
        float acc[kTokensPerWarp][kExperts];
#pragma unroll
        for (int j = 0; j < kTokensPerWarp; ++j)
#pragma unroll
            for (int e = 0; e < kExperts; ++e) acc[j][e] = 0.f;
        float rn[kTokensPerWarp];   // RMSNorm factor of each token (residual block only)
        if (a.g_pre) {
            float ss[kTokensPerWarp];
#pragma unroll
            for (int j = 0; j < kTokensPerWarp; ++j) ss[j] = 0.f;
            for (int c = lane; c < chunks; c += 32) {
#pragma unroll
                for (int j = 0; j < kTokensPerWarp; ++j) {
                    const int t = min(t0 + j, a.T - 1);
                    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(a.x + static_cast<size_t>(t) * a.d) + c);
                    const uint32_t hv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float lo = __uint_as_float(hv[q] << 16), hi = __uint_as_float(hv[q] & 0xffff0000u);
                        ss[j] = fmaf(lo, lo, ss[j]);
                        ss[j] = fmaf(hi, hi, ss[j]);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < kTokensPerWarp; ++j) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) ss[j] += __shfl_xor_sync(0xffffffffu, ss[j], o);
                rn[j] = rsqrtf(ss[j] / static_cast<float>(a.d) + a.eps);
            }
        }
        for (int c = lane; c < chunks; c += 32) {
            uint4 xv[kTokensPerWarp];
#pragma unroll
            for (int j = 0; j < kTokensPerWarp; ++j) {
                const int t = min(t0 + j, a.T - 1);
                xv[j] = __ldg(reinterpret_cast<const uint4 *>(a.x + static_cast<size_t>(t) * a.d) + c);
            }
            if (a.g_pre) {
                const uint4 g = __ldg(reinterpret_cast<const uint4 *>(a.g_pre) + c);
                const uint32_t gv[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
                for (int j = 0; j < kTokensPerWarp; ++j) {
                    const uint32_t hv[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
                    uint32_t uv[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float lo = __uint_as_float(hv[q] << 16) * rn[j] * __uint_as_float(gv[q] << 16);
                        const float hi =
                            __uint_as_float(hv[q] & 0xffff0000u) * rn[j] * __uint_as_float(gv[q] & 0xffff0000u);
                        const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
                        uv[q] = *reinterpret_cast<const uint32_t *>(&p);
                    }
                    xv[j] = make_uint4(uv[0], uv[1], uv[2], uv[3]);
                    if (t0 + j < a.T)
                        reinterpret_cast<uint4 *>(a.u + static_cast<size_t>(t0 + j) * a.d)[c] = xv[j];
                }
            }
            const uint32_t *wv = reinterpret_cast<const uint32_t *>(xv);
            const float4 *wc = wsm + c * 16;
            const int sw = c & 7;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                // rows 8c + 2q (units 4q, 4q+1) and 8c + 2q + 1 (units 4q+2, 4q+3)
                const float4 a0 = wc[(4 * q) ^ sw], a1 = wc[(4 * q + 1) ^ sw];
                const float4 b0 = wc[(4 * q + 2) ^ sw], b1 = wc[(4 * q + 3) ^ sw];
#pragma unroll
                for (int j = 0; j < kTokensPerWarp; ++j) {
                    const uint32_t pv = wv[j * 4 + q];
                    const float x0 = __uint_as_float(pv << 16);
                    const float x1 = __uint_as_float(pv & 0xffff0000u);
                    float *ac = acc[j];
                    ac[0] = fmaf(x0, a0.x, ac[0]); ac[1] = fmaf(x0, a0.y, ac[1]);
                    ac[2] = fmaf(x0, a0.z, ac[2]); ac[3] = fmaf(x0, a0.w, ac[3]);
                    ac[4] = fmaf(x0, a1.x, ac[4]); ac[5] = fmaf(x0, a1.y, ac[5]);
                    ac[6] = fmaf(x0, a1.z, ac[6]); ac[7] = fmaf(x0, a1.w, ac[7]);
                    ac[0] = fmaf(x1, b0.x, ac[0]); ac[1] = fmaf(x1, b0.y, ac[1]);
                    ac[2] = fmaf(x1, b0.z, ac[2]); ac[3] = fmaf(x1, b0.w, ac[3]);
                    ac[4] = fmaf(x1, b1.x, ac[4]); ac[5] = fmaf(x1, b1.y, ac[5]);
                    ac[6] = fmaf(x1, b1.z, ac[6]); ac[7] = fmaf(x1, b1.w, ac[7]);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kTokensPerWarp; ++j)
#pragma unroll
            for (int e = 0; e < kExperts; ++e) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc[j][e] += __shfl_xor_sync(0xffffffffu, acc[j][e], o);
            }
        if (lane < kTokensPerWarp && t0 + lane < a.T) {
            float mine[kExperts];
#pragma unroll
            for (int e = 0; e < kExperts; ++e) {
                float v = acc[0][e];
#pragma unroll
                for (int j = 1; j < kTokensPerWarp; ++j)
                    if (lane == j) v = acc[j][e];
                mine[e] = v;
            }
            if (is_padding(a, t0 + lane))
                write_padding_route(t0 + lane, a.idx, a.gate);
            else
                select_top2(mine, a.bias, t0 + lane, a.idx, a.gate);
        }
    }
}

}  // namespace

cudaError_t launch_router(const RouteArgs &a, cudaStream_t s)
{
    if (a.T <= 0) return cudaSuccess;
    const size_t smem = static_cast<size_t>(a.d) * kExperts * sizeof(float);   // the staged router weight
    if (a.T <= kSmallT || smem > kRouterSmemMax) {
        router_small_kernel<<<a.T, kRouteTokenThreads, 0, s>>>(a);
        return cudaGetLastError();
    }
    static int sms = 0;   // persistent blocks, one per SM (the staged weight fills its shared memory)
    if (sms == 0) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRouterSmemMax);
        if (e != cudaSuccess) {
            sms = 0;
            return e;
        }
    }
    const int per_block = kRouterWarps * kTokensPerWarp;
    const int groups = (a.T + per_block - 1) / per_block;
    router_kernel<<<groups < sms ? groups : sms, kRouterWarps * 32, smem, s>>>(a);
    return cudaGetLastError();
}


}  // namespace moe
