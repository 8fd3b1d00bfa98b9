// route_common.cuh -- per-token routing arithmetic shared by the router kernels: the
// fp32 logits of "Grok-1 Admin & Architecture Guide", section 3, "Mixture of Experts
// (MoELayer + Router)", step 1, and the softmax / top-2 choice of step 2.
#pragma once

#include "kernels.cuh"

namespace moe {

// x (8 bf16 packed in a uint4) times 8 rows of the [d, 8] fp32 router weight starting at `row`
__device__ __forceinline__ void dot8(const uint4 &v, const float4 *w4, int row, float (&acc)[kExperts])
{
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float x0 = __uint_as_float(wv[q] << 16);
        const float x1 = __uint_as_float(wv[q] & 0xffff0000u);
        const int r = row + 2 * q;
        const float4 a0 = __ldg(w4 + r * 2), a1 = __ldg(w4 + r * 2 + 1);
        const float4 b0 = __ldg(w4 + r * 2 + 2), b1 = __ldg(w4 + r * 2 + 3);
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

// logits (+ bias) -> top-2 on the fp32 logits (strictly larger wins, equal logits keep
// the lower expert index) and the fp32 softmax probabilities of the two picks
__device__ __forceinline__ void select_top2(float (&acc)[kExperts], const float *bias, int t, int *idx, float *gate)
{
    if (bias) {
#pragma unroll
        for (int e = 0; e < kExperts; ++e) acc[e] += __ldg(bias + e);
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
    idx[2 * t] = e0;
    idx[2 * t + 1] = e1;
    gate[2 * t] = inv;                        // exp(0) / s
    gate[2 * t + 1] = expf(acc[e1] - m) * inv;
}


constexpr int kRouteTokenThreads = 256;

// a padding token (padding mask 0) is routed nowhere: experts -1, gates 0
__device__ __forceinline__ bool is_padding(const RouteArgs &a, int t) { return a.mask && !__ldg(a.mask + t); }

__device__ __forceinline__ void write_padding_route(int t, int *idx, float *gate)
{
    idx[2 * t] = -1;
    idx[2 * t + 1] = -1;
    gate[2 * t] = 0.f;
    gate[2 * t + 1] = 0.f;
}

// The logits of token t by one block of kRouteTokenThreads threads splitting d: every
// thread issues all its loads at once (one memory latency), then a fixed-order reduction
// (lane tree, then the warp partials in warp order) gives the logits; thread 0 writes the
// token's top-2 experts and gates.  With a.g_pre set, the routed row is the RMS-normalised
// u = bf16(x * rsqrt(mean(x^2) + eps) * g) of the residual block, which is also written to
// a.u: the sum of squares is reduced first (same fixed order), then every 8-element chunk
// of u is formed in fp32, rounded to bf16, stored and used.
__device__ __forceinline__ void route_token(const RouteArgs &a, int t)
{
    if (is_padding(a, t)) {   // uniform over the block
        if (threadIdx.x == 0) write_padding_route(t, a.idx, a.gate);
        return;
    }
    constexpr int kWarps = kRouteTokenThreads / 32;
    __shared__ float part[kWarps][kExperts];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint4 *xr = reinterpret_cast<const uint4 *>(a.x + static_cast<size_t>(t) * a.d);
    const float4 *w4 = reinterpret_cast<const float4 *>(a.w);
    const int chunks = a.d >> 3;
    float acc[kExperts];
#pragma unroll
    for (int e = 0; e < kExperts; ++e) acc[e] = 0.f;
    if (a.g_pre) {
        float ss = 0.f;
        for (int c = threadIdx.x; c < chunks; c += kRouteTokenThreads) {
            const uint4 v = __ldg(xr + c);
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float lo = __uint_as_float(wv[q] << 16), hi = __uint_as_float(wv[q] & 0xffff0000u);
                ss = fmaf(lo, lo, ss);
                ss = fmaf(hi, hi, ss);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) part[warp][0] = ss;
        __syncthreads();
        float tot = 0.f;
        for (int w = 0; w < kWarps; ++w) tot += part[w][0];
        __syncthreads();   // part is reused for the logits below
        const float r = rsqrtf(tot / static_cast<float>(a.d) + a.eps);
        const uint4 *gr = reinterpret_cast<const uint4 *>(a.g_pre);
        uint4 *ur = reinterpret_cast<uint4 *>(a.u + static_cast<size_t>(t) * a.d);
        for (int c = threadIdx.x; c < chunks; c += kRouteTokenThreads) {
            const uint4 v = __ldg(xr + c), g = __ldg(gr + c);
            const uint32_t hv[4] = {v.x, v.y, v.z, v.w}, gv[4] = {g.x, g.y, g.z, g.w};
            uint32_t uv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float lo = __uint_as_float(hv[q] << 16) * r * __uint_as_float(gv[q] << 16);
                const float hi = __uint_as_float(hv[q] & 0xffff0000u) * r * __uint_as_float(gv[q] & 0xffff0000u);
                const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
                uv[q] = *reinterpret_cast<const uint32_t *>(&p);
            }
            const uint4 u = make_uint4(uv[0], uv[1], uv[2], uv[3]);
            ur[c] = u;
            dot8(u, w4, c * 8, acc);
        }
    } else {
#pragma unroll 4
        for (int c = threadIdx.x; c < chunks; c += kRouteTokenThreads) dot8(__ldg(xr + c), w4, c * 8, acc);
    }
#pragma unroll
    for (int e = 0; e < kExperts; ++e) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    }
    if (lane == 0) {
#pragma unroll
        for (int e = 0; e < kExperts; ++e) part[warp][e] = acc[e];
    }
    __syncthreads();
    if (threadIdx.x == 0) {
#pragma unroll
        for (int e = 0; e < kExperts; ++e) {
            float v = 0.f;
            for (int w = 0; w < kWarps; ++w) v += part[w][e];
            acc[e] = v;
        }
        select_top2(acc, a.bias, t, a.idx, a.gate);
    }
}

// The logits of token t over the chunks [c0, c1) of its row (8 elements per chunk), one
// chunk per thread and pass: every thread's loads are issued together, the dot products
// take the chunk's rows in order, and the block reduces in a fixed order (lane tree, then
// the warps in order) into thread 0's `acc`.  With a.g_pre set the routed row is the
// RMS-normalised u of the residual block: the sum of squares is taken over the whole row
// (the same fixed order in every block that calls this for token t, so all of them get the
// same scale), and the slice's chunks of u are formed, rounded to bf16, stored to a.u and
// used.  Without a.g_pre and with a.u set, the slice's chunks of x are copied to a.u (in place
// when a.u is a.x: each chunk is read and written by one thread).  With a.u_scaled the chunks
// go to a.u at kActScale times their value; the routing itself uses the values.
__device__ __forceinline__ void route_slice(const RouteArgs &a, int t, int c0, int c1, float (&acc)[kExperts])
{
    constexpr int kWarps = kRouteTokenThreads / 32;
    __shared__ float part[kWarps][kExperts];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint4 *xr = reinterpret_cast<const uint4 *>(a.x + static_cast<size_t>(t) * a.d);
    const float4 *w4 = reinterpret_cast<const float4 *>(a.w);
    uint4 *ur = a.u ? reinterpret_cast<uint4 *>(a.u + static_cast<size_t>(t) * a.d) : nullptr;
#pragma unroll
    for (int e = 0; e < kExperts; ++e) acc[e] = 0.f;
    float r = 0.f;
    if (a.g_pre) {
        const int chunks = a.d >> 3;
        float ss = 0.f;
        for (int c = threadIdx.x; c < chunks; c += kRouteTokenThreads) {
            const uint4 v = __ldg(xr + c);
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float lo = __uint_as_float(wv[q] << 16), hi = __uint_as_float(wv[q] & 0xffff0000u);
                ss = fmaf(lo, lo, ss);
                ss = fmaf(hi, hi, ss);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) part[warp][0] = ss;
        __syncthreads();
        float tot = 0.f;
        for (int w = 0; w < kWarps; ++w) tot += part[w][0];
        __syncthreads();   // part is reused for the logits below
        r = rsqrtf(tot / static_cast<float>(a.d) + a.eps);
    }
    for (int c = c0 + threadIdx.x; c < c1; c += kRouteTokenThreads) {
        uint4 v = __ldg(xr + c);
        if (a.g_pre) {
            const uint4 g = __ldg(reinterpret_cast<const uint4 *>(a.g_pre) + c);
            const uint32_t hv[4] = {v.x, v.y, v.z, v.w}, gv[4] = {g.x, g.y, g.z, g.w};
            uint32_t uv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float lo = __uint_as_float(hv[q] << 16) * r * __uint_as_float(gv[q] << 16);
                const float hi = __uint_as_float(hv[q] & 0xffff0000u) * r * __uint_as_float(gv[q] & 0xffff0000u);
                const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
                uv[q] = *reinterpret_cast<const uint32_t *>(&p);
            }
            v = make_uint4(uv[0], uv[1], uv[2], uv[3]);
        }
        if (ur) ur[c] = a.u_scaled ? scale_bf16x8(v, kActScale) : v;
        dot8(v, w4, c * 8, acc);
    }
#pragma unroll
    for (int e = 0; e < kExperts; ++e) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    }
    if (lane == 0) {
#pragma unroll
        for (int e = 0; e < kExperts; ++e) part[warp][e] = acc[e];
    }
    __syncthreads();
    if (threadIdx.x == 0) {
#pragma unroll
        for (int e = 0; e < kExperts; ++e) {
            float v = 0.f;
            for (int w = 0; w < kWarps; ++w) v += part[w][e];
            acc[e] = v;
        }
    }
}

}  // namespace moe
