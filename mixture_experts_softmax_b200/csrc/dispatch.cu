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

// Xp[slot_of_route[2t + j], :] = x[t, :] (times kActScale when g.scaled) for the T tokens and
// their two routes; 16-byte copies, each token row read once.  Padding rows are left as they are: every MMA output
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
                    const uint4 o = g.scaled ? scale_bf16x8(v[u], kActScale) : v[u];
                    if (p0 >= 0) reinterpret_cast<uint4 *>(g.xp + static_cast<size_t>(p0) * g.d)[c] = o;
                    if (p1 >= 0) reinterpret_cast<uint4 *>(g.xp + static_cast<size_t>(p1) * g.d)[c] = o;
                }
            }
        }
    }
}

__global__ void __launch_bounds__(256) gather_kernel(GatherArgs g, int T, const int *slot_of_route)
{
    gather_rows(g, T, slot_of_route, blockIdx.x, gridDim.x);
}

// The dispatch of T <= kFusedMaxT tokens by one block whose expert indices are already in
// shared memory (s_idx[2t + j], -1 for a padding token's routes).  A route's rank within its
// expert is the number of routes with a smaller id and the same expert: the two routes of a
// token go to different experts, so this is the token-ordered stable grouping that
// dispatch_block forms.  s_slot receives slot_of_route.
__device__ __forceinline__ void dispatch_small(const DispatchArgs &a, const int *s_idx, int *s_slot)
{
    __shared__ int s_cnt[kMaxE], s_off[kMaxE + 1], s_poff[kMaxE + 1];
    const int tid = threadIdx.x, R = 2 * a.T, E = a.E;
    if (tid < E) {
        int n = 0;
        for (int r = 0; r < R; ++r) n += s_idx[r] == tid;
        s_cnt[tid] = n;
        a.counts[tid] = n;
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
    if (tid <= E) { a.offsets[tid] = s_off[tid]; a.poff[tid] = s_poff[tid]; }
    if (tid < R) {
        const int e = s_idx[tid];
        int slot = -1;
        if (e >= 0) {
            int rank = 0;
            for (int r = 0; r < tid; ++r) rank += s_idx[r] == e;
            a.perm[s_off[e] + rank] = tid;
            a.rperm[s_poff[e] + rank] = tid;
            slot = s_poff[e] + rank;
        }
        a.slot_of_route[tid] = slot;
        s_slot[tid] = slot;
    }
    for (int e = 0; e < E; ++e)   // padding rows of every expert segment carry route id -1
        for (int r = s_poff[e] + s_cnt[e] + tid; r < s_poff[e + 1]; r += blockDim.x) a.rperm[r] = -1;
    __syncthreads();
}

// Small batches in one launch.  Block b takes slice b % S of token b / S's row (S row
// slices per token, S * T blocks) and writes the slice's partial logits to part[b][E]
// (route_slice).  Every block then takes a ticket; the block holding the last one sums
// each token's S partials in slice order, picks the top-2 and gates, dispatches from
// shared memory and, when ga.xp is set, gathers the 2T rows.  The ticket counter is a
// workspace word that the last block sets back to 0 for the next launch.
__global__ void __launch_bounds__(kRouteTokenThreads) route_small_kernel(RouteArgs ra, DispatchArgs da, GatherArgs ga,
                                                                          float *part, int S, unsigned int *ticket)
{
    __shared__ bool s_last;
    __shared__ float s_logit[kFusedMaxT][kExperts];
    __shared__ int s_idx[2 * kFusedMaxT], s_slot[2 * kFusedMaxT];
    // the up-projection, launched next with programmatic serialization, may set up on free SMs
    // (it waits for this grid before it reads anything)
    if (threadIdx.x == 0) griddep_launch_dependents();
    const int t = blockIdx.x / S, sl = blockIdx.x - t * S;
    if (!is_padding(ra, t)) {   // uniform over the block
        const int per = (ra.d >> 3) / S;
        float acc[kExperts];
        route_slice(ra, t, sl * per, sl == S - 1 ? (ra.d >> 3) : (sl + 1) * per, acc);
        if (threadIdx.x == 0) {
#pragma unroll
            for (int e = 0; e < kExperts; ++e) part[blockIdx.x * kExperts + e] = acc[e];
        }
    }
    __threadfence();   // this block's partials (and u) before its ticket
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(ticket, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();   // every other block's partials are visible after their tickets
    const int T = ra.T;
    if (threadIdx.x == 0) *ticket = 0u;
    if (threadIdx.x < T * kExperts) {   // fixed order: slices 0 .. S-1
        const int tt = threadIdx.x / kExperts, e = threadIdx.x % kExperts;
        float v = 0.f;
        for (int q = 0; q < S; ++q) v += __ldcg(part + (tt * S + q) * kExperts + e);
        s_logit[tt][e] = v;
    }
    __syncthreads();
    if (threadIdx.x < T) {
        const int tt = threadIdx.x;
        if (is_padding(ra, tt)) {
            s_idx[2 * tt] = -1;
            s_idx[2 * tt + 1] = -1;
            write_padding_route(tt, ra.idx, ra.gate);
        } else {
            float acc[kExperts], g[2];
#pragma unroll
            for (int e = 0; e < kExperts; ++e) acc[e] = s_logit[tt][e];
            select_top2(acc, ra.bias, 0, s_idx + 2 * tt, g);
            ra.idx[2 * tt] = s_idx[2 * tt];
            ra.idx[2 * tt + 1] = s_idx[2 * tt + 1];
            ra.gate[2 * tt] = g[0];
            ra.gate[2 * tt + 1] = g[1];
        }
    }
    __syncthreads();
    dispatch_small(da, s_idx, s_slot);
    if (ga.xp) gather_rows(ga, T, s_slot, 0, 1);
}

}  // namespace

int route_small_max_tokens() { return kFusedMaxT; }

int route_small_slices(int T, int d, int num_sms)
{
    const int chunks = d >> 3;
    int S = 1;   // row slices per token: the most that keep one wave and a warp's worth of chunks each
    while (T * 2 * S <= num_sms && chunks % (2 * S) == 0 && chunks / (2 * S) >= 32) S *= 2;
    return S;
}

cudaError_t launch_route_small(const RouteArgs &ra, const DispatchArgs &da, const GatherArgs &ga, float *part, int S,
                               unsigned int *ticket, cudaStream_t s)
{
    if (ra.T <= 0 || ra.T > kFusedMaxT || S <= 0 || (ra.d >> 3) < S || da.E > kMaxE) return cudaErrorInvalidValue;
    route_small_kernel<<<ra.T * S, kRouteTokenThreads, 0, s>>>(ra, da, ga, part, S, ticket);
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
