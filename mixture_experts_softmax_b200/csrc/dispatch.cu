// dispatch.cu -- group the routes by expert (histogram, prefix sum, stable permute)
// and gather the token rows into the grouped, padded order the grouped GEMMs read.
//
// The method's own MoE selects expert outputs with one-hot masks over a dense
// all-experts product ("Grok-1 Admin & Architecture Guide", section 3, "Mixture of
// Experts", step 4); grouping the routes by expert computes the same sums for the
// chosen experts only.
#include "kernels.cuh"
#include "ptx.cuh"
#include "route_common.cuh"

namespace moe {

namespace {

constexpr int kDispatchThreads = 1024;
constexpr int kMaxE = 32;
constexpr int kFusedMaxT = 32;      // batches routed by route_small_kernel

// The dispatch of one block of NT threads.  Pass 1 counts routes per expert; thread 0
// forms the exclusive prefix sums (plain and padded to multiples of bn rows).  Pass 2
// walks the tokens in chunks of NT in ascending order; within a chunk the rank of a
// route among the routes to the same expert is (routes in earlier chunks) + (routes in
// earlier warps, by a per-expert warp scan) + (earlier lanes, by ballot/popc).  Every
// value is a count, so the result is exact and independent of scheduling.  The expert
// indices are read through L2 (.cg): in the fused routing they were written by other
// blocks of the same launch.
template <int NT>
__device__ __forceinline__ void dispatch_block(const DispatchArgs &a)
{
    __shared__ int s_cnt[kMaxE], s_off[kMaxE + 1], s_poff[kMaxE + 1], s_run[kMaxE];
    __shared__ int s_warp[NT / 32][kMaxE];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = a.E;
    if (tid < kMaxE) { s_cnt[tid] = 0; s_run[tid] = 0; }
    __syncthreads();
    for (int t = tid; t < a.T; t += NT) {   // expert -1: a padding token's route, not dispatched
        const int e0 = __ldcg(a.idx + 2 * t), e1 = __ldcg(a.idx + 2 * t + 1);
        if (e0 >= 0) atomicAdd(&s_cnt[e0], 1);
        if (e1 >= 0) atomicAdd(&s_cnt[e1], 1);
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
    for (int c0 = 0; c0 < a.T; c0 += NT) {
        const int t = c0 + tid;
        const bool valid = t < a.T;
        const int e0 = valid ? __ldcg(a.idx + 2 * t) : -1;
        const int e1 = valid ? __ldcg(a.idx + 2 * t + 1) : -1;
        for (int e = 0; e < E; ++e) {
            const uint32_t m = __ballot_sync(0xffffffffu, e0 == e || e1 == e);
            if (lane == 0) s_warp[warp][e] = __popc(m);
        }
        __syncthreads();
        if (tid < E) {   // exclusive scan over the warps of this chunk, continuing s_run
            int run = s_run[tid];
            for (int w = 0; w < NT / 32; ++w) {
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
            if (e0 >= 0) {
                a.perm[s_off[e0] + rank0] = r0;
                a.rperm[s_poff[e0] + rank0] = r0;
                a.slot_of_route[r0] = s_poff[e0] + rank0;
            } else {
                a.slot_of_route[r0] = -1;
            }
            if (e1 >= 0) {
                a.perm[s_off[e1] + rank1] = r1;
                a.rperm[s_poff[e1] + rank1] = r1;
                a.slot_of_route[r1] = s_poff[e1] + rank1;
            } else {
                a.slot_of_route[r1] = -1;
            }
        }
        __syncthreads();   // s_warp is rewritten by the next chunk
    }
    // padding rows of every expert segment carry route id -1
    for (int e = 0; e < E; ++e)
        for (int r = s_poff[e] + s_cnt[e] + tid; r < s_poff[e + 1]; r += NT) a.rperm[r] = -1;
}

__global__ void __launch_bounds__(kDispatchThreads) dispatch_kernel(DispatchArgs a)
{
    dispatch_block<kDispatchThreads>(a);
}

// Xp[slot_of_route[2t + j], :] = x[t, :] for the T tokens and their two routes; 16-byte
// copies, each token row read once.  Padding rows are left as they are: every MMA output
// column depends on its own B row only, and both GEMM epilogues skip rows whose route id
// is -1.  The calling block takes groups of kGatherTokens tokens (group0, group0 + step,
// ...), its threads the row's chunks, with the group's loads in flight together.
constexpr int kGatherTokens = 8;

__device__ __forceinline__ void gather_rows(const GatherArgs &g, int T, const int *slot_of_route, int group0,
                                            int group_step)
{
    const int chunks = g.d >> 3;
    for (int t0 = group0 * kGatherTokens; t0 < T; t0 += group_step * kGatherTokens) {
        const int n = min(kGatherTokens, T - t0);
        for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
            uint4 v[kGatherTokens];
#pragma unroll
            for (int u = 0; u < kGatherTokens; ++u)
                if (u < n) v[u] = __ldg(reinterpret_cast<const uint4 *>(g.x + static_cast<size_t>(t0 + u) * g.d) + c);
#pragma unroll
            for (int u = 0; u < kGatherTokens; ++u) {
                if (u < n) {   // slot -1: a padding token's route
                    const int r = 2 * (t0 + u);
                    const int p0 = slot_of_route[r], p1 = slot_of_route[r + 1];
                    if (p0 >= 0) reinterpret_cast<uint4 *>(g.xp + static_cast<size_t>(p0) * g.d)[c] = v[u];
                    if (p1 >= 0) reinterpret_cast<uint4 *>(g.xp + static_cast<size_t>(p1) * g.d)[c] = v[u];
                }
            }
        }
    }
}

__global__ void __launch_bounds__(256) gather_kernel(GatherArgs g, int T, const int *slot_of_route)
{
    gather_rows(g, T, slot_of_route, blockIdx.x, gridDim.x);
}

// Small batches in one launch: block t computes token t's logits and top-2 (route_token);
// every block then takes a ticket, and the block holding the last one, which sees every
// block's expert choice, runs the dispatch and gathers the 2T rows.  The ticket counter
// is a workspace word that the last block sets back to 0 for the next launch.
__global__ void __launch_bounds__(kRouteTokenThreads) route_small_kernel(RouteArgs ra, DispatchArgs da, GatherArgs ga,
                                                                          unsigned int *ticket)
{
    __shared__ bool s_last;
    route_token(ra, blockIdx.x);
    __threadfence();   // this block's idx / gate before its ticket
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(ticket, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();   // every other block's idx / gate is visible after their tickets
    if (threadIdx.x == 0) *ticket = 0u;
    dispatch_block<kRouteTokenThreads>(da);
    __syncthreads();   // slot_of_route of this block's dispatch, read back below
    gather_rows(ga, da.T, da.slot_of_route, 0, 1);
}

}  // namespace

int route_small_max_tokens() { return kFusedMaxT; }

cudaError_t launch_route_small(const RouteArgs &ra, const DispatchArgs &da, const GatherArgs &ga, unsigned int *ticket,
                               cudaStream_t s)
{
    if (ra.T <= 0 || ra.T > kFusedMaxT) return cudaErrorInvalidValue;
    route_small_kernel<<<ra.T, kRouteTokenThreads, 0, s>>>(ra, da, ga, ticket);
    return cudaGetLastError();
}

cudaError_t launch_dispatch(const DispatchArgs &a, cudaStream_t s)
{
    dispatch_kernel<<<1, kDispatchThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_gather(const GatherArgs &a, int T, const int *slot_of_route, cudaStream_t s)
{
    if (T <= 0) return cudaSuccess;
    const int groups = (T + kGatherTokens - 1) / kGatherTokens;
    gather_kernel<<<groups < 148 * 4 ? groups : 148 * 4, 256, 0, s>>>(a, T, slot_of_route);
    return cudaGetLastError();
}

}  // namespace moe
