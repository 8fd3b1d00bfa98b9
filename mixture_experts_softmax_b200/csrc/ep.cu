// ep.cu -- the device steps of the expert-parallel layer: the pages' own layout spreads the
// experts over the devices of the `model` mesh axis ("Grok-1 Admin & Architecture Guide",
// section 6 "Sharding & Parallelism Deep Dive").  Here rank r of W holds E/W consecutive
// experts; each rank routes its own tokens, sends every routed row to the rank holding its
// expert, runs the grouped GEMMs of its experts on the rows it received, sends the results
// back, and combines them in token order (step 4 of "Mixture of Experts (MoELayer + Router)").
//
// The kernels here are the glue around the layer's own router, dispatch and GEMMs:
//   ep_layout    -- the grouped, padded row order of the received rows (one block);
//   ep_gather    -- received rows into that order (the GEMMs' B operand);
//   ep_split_sum -- fixed-order sum of the down-projection's K-split partials per row;
//   ep_combine   -- gate-weighted sum of each token's two returned rows, slot 0 first.
#include "kernels.cuh"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kLayoutThreads = 1024;
constexpr int kMaxSrcExperts = kEpMaxRuns;

// Received rows are ordered by source rank, and within a source by local expert (a source
// sends its rows grouped by expert, and a rank's experts are consecutive).  Local expert k's
// grouped segment (padded to bn rows) takes its rows source after source, each source's rows
// in the order they arrived: row i of source s, j-th of that source's rows for expert k, goes
// to poff[k] + (rows of k from sources before s) + j.
__global__ void __launch_bounds__(kLayoutThreads) ep_layout_kernel(EpLayoutArgs a)
{
    __shared__ int s_cnt[kMaxSrcExperts];
    __shared__ int s_src0[kMaxSrcExperts];   // first received row of each (source, expert) run
    __shared__ int s_dst0[kMaxSrcExperts];   // its first grouped row
    __shared__ int s_tot[65], s_poff[65], s_rows;
    const int El = a.E_local, NS = a.n_src, tid = threadIdx.x;
    for (int i = tid; i < NS * El; i += kLayoutThreads) s_cnt[i] = a.recv_counts[i];
    __syncthreads();
    if (tid == 0) {
        int off = 0, poff = 0;
        for (int k = 0; k < El; ++k) {
            int n = 0;
            for (int s = 0; s < NS; ++s) n += s_cnt[s * El + k];
            s_tot[k] = n;
            a.counts[k] = n;
            a.offsets[k] = off;
            a.poff[k] = poff;
            s_poff[k] = poff;
            off += n;
            poff += (n + a.bn - 1) / a.bn * a.bn;
        }
        a.offsets[El] = off;
        a.poff[El] = poff;
        s_poff[El] = poff;
        s_rows = min(off, a.R);   // R is the counts' sum (the host forms both)
        int src0 = 0;
        for (int s = 0; s < NS; ++s)
            for (int k = 0; k < El; ++k) {
                s_src0[s * El + k] = src0;
                src0 += s_cnt[s * El + k];
            }
        for (int k = 0; k < El; ++k) {
            int dst = s_poff[k];
            for (int s = 0; s < NS; ++s) {
                s_dst0[s * El + k] = dst;
                dst += s_cnt[s * El + k];
            }
        }
    }
    __syncthreads();
    const int runs = NS * El;
    for (int i = tid; i < s_rows; i += kLayoutThreads) {
        int run = 0;   // the (source, expert) run holding received row i; runs are in row order
        while (run + 1 < runs && s_src0[run + 1] <= i) ++run;
        const int pos = s_dst0[run] + (i - s_src0[run]);
        a.rperm[pos] = i;
        a.slot[i] = pos;
        a.ones[i] = 1.f;
    }
    for (int k = 0; k < El; ++k)   // padding rows of every expert segment carry route id -1
        for (int r = s_poff[k] + s_tot[k] + tid; r < s_poff[k + 1]; r += kLayoutThreads) a.rperm[r] = -1;
}

// xp[slot[i]] = rows[i] (times kActScale when `scaled`) for the R received rows, 16-byte copies
__global__ void __launch_bounds__(256) ep_gather_kernel(int R, int d, const __nv_bfloat16 *rows, const int *slot,
                                                       __nv_bfloat16 *xp, int scaled)
{
    const int per_row = d >> 3;
    const size_t n = static_cast<size_t>(R) * per_row;
    for (size_t q = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; q < n;
         q += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const int i = static_cast<int>(q / per_row), c = static_cast<int>(q % per_row);
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(rows + static_cast<size_t>(i) * d) + c);
        reinterpret_cast<uint4 *>(xp + static_cast<size_t>(__ldg(slot + i)) * d)[c] =
            scaled ? scale_bf16x8(v, kActScale) : v;
    }
}

// y[i] = sum over s = 0 .. splits-1 of part[s][i] (planes `plane` floats apart), in that order
__global__ void __launch_bounds__(256) ep_split_sum_kernel(int R, int d, int splits, size_t plane, const float *part,
                                                          float *y)
{
    const int per_row = d >> 2;
    const size_t n = static_cast<size_t>(R) * per_row;
    for (size_t q = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; q < n;
         q += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const size_t o = q * 4;
        float4 acc = __ldg(reinterpret_cast<const float4 *>(part + o));
        for (int s = 1; s < splits; ++s) {
            const float4 v = __ldg(reinterpret_cast<const float4 *>(part + s * plane + o));
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        *reinterpret_cast<float4 *>(y + o) = acc;
    }
}

// out[t] = bf16( gate[t,0] * y[slot(2t)] + gate[t,1] * y[slot(2t+1)] ), 0 for a padding token
__global__ void __launch_bounds__(256) ep_combine_kernel(EpCombineArgs a)
{
    const int per_row = a.d >> 2;
    const size_t n = static_cast<size_t>(a.T) * per_row;
    for (size_t q = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; q < n;
         q += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const int t = static_cast<int>(q / per_row), c = static_cast<int>(q % per_row) * 4;
        float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
        if (__ldg(a.idx + 2 * t) >= 0) {
            const float g0 = __ldg(a.gate + 2 * t), g1 = __ldg(a.gate + 2 * t + 1);
            const int p0 = __ldg(a.slot_of_route + 2 * t), p1 = __ldg(a.slot_of_route + 2 * t + 1);
            const float4 y0 = __ldg(reinterpret_cast<const float4 *>(a.y + static_cast<size_t>(p0) * a.d + c));
            const float4 y1 = __ldg(reinterpret_cast<const float4 *>(a.y + static_cast<size_t>(p1) * a.d + c));
            r.x = g0 * y0.x + g1 * y1.x;
            r.y = g0 * y0.y + g1 * y1.y;
            r.z = g0 * y0.z + g1 * y1.z;
            r.w = g0 * y0.w + g1 * y1.w;
        }
        __nv_bfloat162 lo = __floats2bfloat162_rn(r.x, r.y), hi = __floats2bfloat162_rn(r.z, r.w);
        uint2 v;
        v.x = *reinterpret_cast<uint32_t *>(&lo);
        v.y = *reinterpret_cast<uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(a.out + static_cast<size_t>(t) * a.d + c) = v;
    }
}

int grid_for(size_t n)
{
    const size_t want = (n + 255) / 256;
    return static_cast<int>(want < 148 * 16 ? (want ? want : 1) : 148 * 16);
}

}  // namespace

cudaError_t launch_ep_layout(const EpLayoutArgs &a, cudaStream_t s)
{
    if (a.n_src <= 0 || a.E_local <= 0 || a.n_src * a.E_local > kMaxSrcExperts)
        return cudaErrorInvalidValue;
    ep_layout_kernel<<<1, kLayoutThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_ep_gather(int R, int d, const __nv_bfloat16 *rows, const int *slot, __nv_bfloat16 *xp, int scaled,
                             cudaStream_t s)
{
    if (R <= 0) return cudaSuccess;
    ep_gather_kernel<<<grid_for(static_cast<size_t>(R) * (d >> 3)), 256, 0, s>>>(R, d, rows, slot, xp, scaled);
    return cudaGetLastError();
}

cudaError_t launch_ep_split_sum(int R, int d, int splits, size_t plane, const float *part, float *y, cudaStream_t s)
{
    if (R <= 0) return cudaSuccess;
    ep_split_sum_kernel<<<grid_for(static_cast<size_t>(R) * (d >> 2)), 256, 0, s>>>(R, d, splits, plane, part, y);
    return cudaGetLastError();
}

cudaError_t launch_ep_combine(const EpCombineArgs &a, cudaStream_t s)
{
    if (a.T <= 0) return cudaSuccess;
    ep_combine_kernel<<<grid_for(static_cast<size_t>(a.T) * (a.d >> 2)), 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
