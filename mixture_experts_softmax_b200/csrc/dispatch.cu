// dispatch.cu -- group the routes by expert (histogram, prefix sum, stable permute)
// and gather the token rows into the grouped, padded order the grouped GEMMs read.
//
// The method's own MoE selects expert outputs with one-hot masks over a dense
// all-experts product ("Grok-1 Admin & Architecture Guide", section 3, "Mixture of
// Experts", step 4); grouping the routes by expert computes the same sums for the
// chosen experts only.
#include "kernels.cuh"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kDispatchThreads = 1024;
constexpr int kMaxE = 32;

// Single block.  Pass 1 counts routes per expert; thread 0 forms the exclusive
// prefix sums (plain and padded to multiples of bn rows).  Pass 2 walks the tokens
// in chunks of 1024 in ascending order; within a chunk the rank of a route among
// the routes to the same expert is (routes in earlier chunks) + (routes in earlier
// warps, by a per-expert warp scan) + (earlier lanes, by ballot/popc).  Every
// value is a count, so the result is exact and independent of scheduling.
__global__ void __launch_bounds__(kDispatchThreads) dispatch_kernel(DispatchArgs a)
{
    __shared__ int s_cnt[kMaxE], s_off[kMaxE + 1], s_poff[kMaxE + 1], s_run[kMaxE];
    __shared__ int s_warp[kDispatchThreads / 32][kMaxE];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = a.E;
    if (tid < kMaxE) { s_cnt[tid] = 0; s_run[tid] = 0; }
    __syncthreads();
    for (int t = tid; t < a.T; t += kDispatchThreads) {
        atomicAdd(&s_cnt[a.idx[2 * t]], 1);
        atomicAdd(&s_cnt[a.idx[2 * t + 1]], 1);
    }
    __syncthreads();
    if (tid == 0) {
        s_off[0] = 0;
        s_poff[0] = 0;
        for (int e = 0; e < E; ++e) {
            s_off[e + 1] = s_off[e] + s_cnt[e];
            s_poff[e + 1] = s_poff[e] + (s_cnt[e] + a.bn - 1) / a.bn * a.bn;
        }
    }
    __syncthreads();
    if (tid < E) a.counts[tid] = s_cnt[tid];
    if (tid <= E) { a.offsets[tid] = s_off[tid]; a.poff[tid] = s_poff[tid]; }

    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int c0 = 0; c0 < a.T; c0 += kDispatchThreads) {
        const int t = c0 + tid;
        const bool valid = t < a.T;
        const int e0 = valid ? a.idx[2 * t] : -1;
        const int e1 = valid ? a.idx[2 * t + 1] : -1;
        for (int e = 0; e < E; ++e) {
            const uint32_t m = __ballot_sync(0xffffffffu, e0 == e || e1 == e);
            if (lane == 0) s_warp[warp][e] = __popc(m);
        }
        __syncthreads();
        if (tid < E) {   // exclusive scan over the warps of this chunk, continuing s_run
            int run = s_run[tid];
            for (int w = 0; w < kDispatchThreads / 32; ++w) {
                const int cnt = s_warp[w][tid];
                s_warp[w][tid] = run;
                run += cnt;
            }
            s_run[tid] = run;
        }
        __syncthreads();
        int rank0 = 0, rank1 = 0;
        for (int e = 0; e < E; ++e) {
            const uint32_t m = __ballot_sync(0xffffffffu, e0 == e || e1 == e);
            const int pre = s_warp[warp][e] + __popc(m & lt_mask);
            if (e0 == e) rank0 = pre;
            if (e1 == e) rank1 = pre;
        }
        if (valid) {
            const int r0 = 2 * t, r1 = 2 * t + 1;
            a.perm[s_off[e0] + rank0] = r0;
            a.perm[s_off[e1] + rank1] = r1;
            const int p0 = s_poff[e0] + rank0, p1 = s_poff[e1] + rank1;
            a.rperm[p0] = r0;
            a.rperm[p1] = r1;
            a.slot_of_route[r0] = p0;
            a.slot_of_route[r1] = p1;
        }
        __syncthreads();   // s_warp is rewritten by the next chunk
    }
    // padding rows of every expert segment carry route id -1
    for (int e = 0; e < E; ++e)
        for (int r = s_poff[e] + s_cnt[e] + tid; r < s_poff[e + 1]; r += kDispatchThreads) a.rperm[r] = -1;
}

// Xp[r, :] = x[token of route rperm[r], :], zero rows for padding.  16-byte copies.
__global__ void __launch_bounds__(256) gather_kernel(GatherArgs a)
{
    const int rows = min(*a.poff_end, a.max_rows);
    const int chunks = a.d >> 3;
    for (int r = blockIdx.x; r < rows; r += gridDim.x) {
        const int route = a.rperm[r];
        uint4 *dst = reinterpret_cast<uint4 *>(a.xp + static_cast<size_t>(r) * a.d);
        if (route >= 0) {
            const uint4 *src = reinterpret_cast<const uint4 *>(a.x + static_cast<size_t>(route >> 1) * a.d);
            for (int c = threadIdx.x; c < chunks; c += blockDim.x) dst[c] = __ldg(src + c);
        } else {
            for (int c = threadIdx.x; c < chunks; c += blockDim.x) dst[c] = make_uint4(0, 0, 0, 0);
        }
    }
}

}  // namespace

cudaError_t launch_dispatch(const DispatchArgs &a, cudaStream_t s)
{
    dispatch_kernel<<<1, kDispatchThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_gather(const GatherArgs &a, cudaStream_t s)
{
    if (a.max_rows <= 0) return cudaSuccess;
    const int grid = a.max_rows < 148 * 8 ? a.max_rows : 148 * 8;
    gather_kernel<<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
