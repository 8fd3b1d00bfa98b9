// router.cu -- routing logits, softmax and top-2 ("Grok-1 Admin & Architecture Guide",
// section 3, "Mixture of Experts (MoELayer + Router)", steps 1-2), and the pre-MoE
// RMSNorm of the residual block ("Transformer stack and language model head").
#include "kernels.cuh"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kRouterWarps = 8;   // tokens per block (one warp per token)

// One warp per token.  Lane l reads 8 consecutive bf16 of x (16 B) per step and the
// matching 8 rows of the fp32 router weight (8 x E floats), keeping E fp32 partial
// sums; a butterfly reduction then gives every lane the E logits.  The selection
// is taken on the fp32 logits (strictly larger wins, equal logits keep the lower
// expert index); the gates are the fp32 softmax probabilities of the two picks.
__global__ void __launch_bounds__(kRouterWarps * 32) router_kernel(RouteArgs a)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kRouterWarps + warp;
    if (t >= a.T) return;
    const uint4 *xr = reinterpret_cast<const uint4 *>(a.x + static_cast<size_t>(t) * a.d);
    const float4 *w4 = reinterpret_cast<const float4 *>(a.w);
    float acc[kExperts];
#pragma unroll
    for (int e = 0; e < kExperts; ++e) acc[e] = 0.f;
    const int chunks = a.d >> 3;
    for (int c = lane; c < chunks; c += 32) {
        uint4 v = __ldg(xr + c);
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float x0 = __uint_as_float(wv[q] << 16);
            const float x1 = __uint_as_float(wv[q] & 0xffff0000u);
            const int row = c * 8 + 2 * q;
            // rows `row` and `row+1`, E = 8 floats each = 2 float4 per row
            const float4 a0 = __ldg(w4 + row * 2), a1 = __ldg(w4 + row * 2 + 1);
            const float4 b0 = __ldg(w4 + row * 2 + 2), b1 = __ldg(w4 + row * 2 + 3);
            acc[0] = fmaf(x0, a0.x, acc[0]); acc[1] = fmaf(x0, a0.y, acc[1]);
            acc[2] = fmaf(x0, a0.z, acc[2]); acc[3] = fmaf(x0, a0.w, acc[3]);
            acc[4] = fmaf(x0, a1.x, acc[4]); acc[5] = fmaf(x0, a1.y, acc[5]);
            acc[6] = fmaf(x0, a1.z, acc[6]); acc[7] = fmaf(x0, a1.w, acc[7]);
            acc[0] = fmaf(x1, b0.x, acc[0]); acc[1] = fmaf(x1, b0.y, acc[1]);
            acc[2] = fmaf(x1, b0.z, acc[2]); acc[3] = fmaf(x1, b0.w, acc[3]);
            acc[4] = fmaf(x1, b1.x, acc[4]); acc[5] = fmaf(x1, b1.y, acc[5]);
            acc[6] = fmaf(x1, b1.z, acc[6]); acc[7] = fmaf(x1, b1.w, acc[7]);
        }
    }
#pragma unroll
    for (int e = 0; e < kExperts; ++e) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    }
    if (lane != 0) return;
    if (a.bias) {
#pragma unroll
        for (int e = 0; e < kExperts; ++e) acc[e] += __ldg(a.bias + e);
    }
    int e0 = 0;
#pragma unroll
    for (int e = 1; e < kExperts; ++e)
        if (acc[e] > acc[e0]) e0 = e;
    int e1 = (e0 == 0) ? 1 : 0;
#pragma unroll
    for (int e = 0; e < kExperts; ++e)
        if (e != e0 && acc[e] > acc[e1]) e1 = e;
    const float m = acc[e0];
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < kExperts; ++e) s += expf(acc[e] - m);
    const float inv = 1.f / s;
    a.idx[2 * t] = e0;
    a.idx[2 * t + 1] = e1;
    a.gate[2 * t] = inv;                        // exp(0) / s
    a.gate[2 * t + 1] = expf(acc[e1] - m) * inv;
}

// u = bf16( h * rsqrt(mean(h^2) + eps) * g ), one block per token, fp32 math.
__global__ void __launch_bounds__(256) prenorm_kernel(NormArgs a)
{
    __shared__ float red[8];
    const int t = blockIdx.x;
    const __nv_bfloat16 *hr = a.h + static_cast<size_t>(t) * a.d;
    float ss = 0.f;
    for (int i = threadIdx.x; i < a.d; i += blockDim.x) {
        const float v = __bfloat162float(hr[i]);
        ss = fmaf(v, v, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += red[w];
    const float r = rsqrtf(tot / static_cast<float>(a.d) + a.eps);
    __nv_bfloat16 *ur = a.u + static_cast<size_t>(t) * a.d;
    for (int i = threadIdx.x; i < a.d; i += blockDim.x)
        ur[i] = __float2bfloat16_rn(__bfloat162float(hr[i]) * r * __bfloat162float(a.g[i]));
}

}  // namespace

cudaError_t launch_router(const RouteArgs &a, cudaStream_t s)
{
    if (a.T <= 0) return cudaSuccess;
    const int blocks = (a.T + kRouterWarps - 1) / kRouterWarps;
    router_kernel<<<blocks, kRouterWarps * 32, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_prenorm(const NormArgs &a, cudaStream_t s)
{
    if (a.T <= 0) return cudaSuccess;
    prenorm_kernel<<<a.T, 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
