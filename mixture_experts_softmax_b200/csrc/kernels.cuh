// kernels.cuh -- launch interface between the C ABI (moe_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr int kExperts = 8;       // E supported by the router kernel
constexpr int kScaleBlock = 128;   // reduction rows sharing a scale in the per-block scale format
constexpr int kTopK = 2;          // picks per token
constexpr int kBM = 128;          // output features per GEMM tile (TMEM lanes)
constexpr int kBK = 64;           // reduction elements per pipeline stage (128 B of bf16)
constexpr int kMaxSplits = 8;     // K-splits of the down-projection

// The packed weight layout and its operand scaling (the TMEM-operand GEMMs).  Packed weights
// hold each int8 value w as a sign bit and a 7-bit magnitude (so w = -128 has no packed form),
// four consecutive reduction elements to a 32-bit word with the signs crossed over within each
// 16-bit half (gemm_common.cuh, pk_lo).  A converter turns a value into the bf16 with its sign,
// a zero exponent field and |w| as its mantissa: the value w * 2^-133, exactly (bf16 numbers
// with a zero exponent field are the multiples of 2^-133 below 2^-126).  Products with such an operand are
// 2^133 times too small, so the other operand, the routed rows and H, is kept at kActScale times
// its value, which holds the fp32 accumulator above its own subnormal range for activations down
// to about 1e-20; the epilogues multiply the scales by kAccScaleChannel.  Every step is an exact
// power-of-two scaling, as long as the routed rows and H stay below 2^64 in magnitude (beyond
// that their scaled copies overflow) and the scales below 2^59.  With per-block scales the converters form bf16(w * s) as
// normal numbers instead, and the epilogues multiply by kActUnscale.
constexpr float kActScale = 0x1p64f;
constexpr float kActUnscale = 0x1p-64f;
constexpr float kAccScaleChannel = 0x1p69f;   // 2^133 / kActScale

// two bf16 values (a 32-bit pair) or eight (16 bytes) times f, through fp32: exact for a
// power of two f while the results stay finite (bf16 subnormals are fp32 subnormals, kept
// without flushing)
__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t w, float f)
{
    const __nv_bfloat162 r = __floats2bfloat162_rn(__uint_as_float(w << 16) * f, __uint_as_float(w & 0xffff0000u) * f);
    return *reinterpret_cast<const uint32_t *>(&r);
}
__device__ __forceinline__ uint4 scale_bf16x8(uint4 v, float f)
{
    return make_uint4(scale_bf16x2(v.x, f), scale_bf16x2(v.y, f), scale_bf16x2(v.z, f), scale_bf16x2(v.w, f));
}

// device error word values (the first error wins)
constexpr int kErrTimeoutBase = 0x1000;   // + wait site

struct RouteArgs {
    int T, d;
    const __nv_bfloat16 *x;     // [T, d]
    const float *w;             // [d, E]
    const float *bias;          // [E] or nullptr
    int *idx;                   // [T, 2]
    float *gate;                // [T, 2]
    // optional pre-MoE RMSNorm of the residual block: route on u = bf16(x * rsqrt(mean x^2 + eps) * g),
    // written to u for the gather (every routing kernel)
    const __nv_bfloat16 *g_pre; // [d] or nullptr
    float eps;
    __nv_bfloat16 *u;           // [T, d]
    const uint8_t *mask;        // [T] padding mask (0 = padding: experts -1, gates 0) or nullptr
    int u_scaled;               // 1: u is written at kActScale times its value (the small-batch
                                //    routing launch, when u is the packed up-projection's operand)
};

struct DispatchArgs {
    int T, E, bn;
    const int *idx;             // [T, 2]
    int *counts;                // [E]
    int *offsets;               // [E+1]   unpadded grouped offsets
    int *poff;                  // [E+1]   offsets with each expert's segment padded to bn rows
    int *perm;                  // [2T]    grouped row -> route id (2t + slot)
    int *rperm;                 // [rows]  padded row -> route id, -1 for padding
    int *slot_of_route;         // [2T]    route id -> padded row
};

struct GatherArgs {
    int d;
    const __nv_bfloat16 *x;     // [T, d]
    __nv_bfloat16 *xp;          // [rows, d]; only the rows of real routes are written
    int scaled;                 // 1: rows written at kActScale times their value (packed layout)
};

// one grouped GEMM of the layer:  for every expert e and padded row r of e
//   UP   (two A matrices):  H[r, f]  = bf16( gelu(s0[e,f] * A0) * (s1[e,f] * A1) )
//   DOWN (one A matrix):    slot[s, t, j, f] = gate[t, j] * s0[e, f] * A0_partial(s)
// where A_i[f, r] = sum_k W_i[e, k, f] * B[r, k] over this split's k range.
struct GemmArgs {
    int T;                      // tokens
    int E;
    int M;                      // output features (F for UP, d for DOWN)
    int K;                      // reduction length (d for UP, F for DOWN)
    int ksteps;                 // k-steps of kBK per split
    int splits;                 // K-splits (DOWN); 1 for UP
    const int *poff;            // [E+1] expert segments, padded to tile width
    const int *offsets;         // [E+1] the same without padding: real rows of expert e are the first
                                //       offsets[e+1] - offsets[e] rows of its segment
    const int *rperm;           // [rows]
    const float *gate;          // [T, 2]
    const __nv_bfloat16 *s0;    // [E, M]
    const __nv_bfloat16 *s1;    // [E, M] (UP only)
    __nv_bfloat16 *h;           // UP output   [rows, M]
    float *slots;               // DOWN output [splits, T, 2, M]
    int *err;                   // device error word
    long long timeout_ns;
    // scale format: 0 = one scale per output channel, s0/s1 [E, M] (applied in the epilogue);
    // kScaleBlock = per block of kScaleBlock reduction rows, s0/s1 [E, K / kScaleBlock, M]
    // (applied while dequantising, TMEM-operand kernels only)
    int kblock;
    // last-wave pieces (TMEM-operand kernels): partial accumulators and per-tile tickets
    float *part;                // [gridDim.x, 128, accumulator columns] fp32, or nullptr: no pieces
    unsigned int *tickets;      // [gridDim.x], zero, left zero by every launch that completes
    // TMEM-operand up-projection with tiles of at most 32 rows: 1 = the B map covers the routed
    // rows [T, K] with one-row boxes and each tile row is loaded from row rperm >> 1 of it
    // (no gathered copy); 0 = the B map covers the gathered rows [rows, K]
    int gather;
    // TMEM-operand kernels (packed layout): the factor taking an accumulator to its value
    // (kAccScaleChannel, or kActUnscale with per-block scales); H is written at kActScale
    float accf;
};

struct CombineArgs {
    int T, d, splits;
    const float *slots;         // [splits, T, 2, d]
    const int *idx;             // [T, 2] experts; -1: a padding token (no slots written), output 0
    __nv_bfloat16 *out;         // [T, d]
    // residual block variant
    __nv_bfloat16 *h_io;        // [T, d] residual stream (nullptr: plain combine)
    const __nv_bfloat16 *g_post;
    float eps;
};


// expert-parallel steps (ep.cu)
constexpr int kEpMaxRuns = 64;   // n_src * E_local: (source rank, local expert) pairs
struct EpLayoutArgs {
    int n_src, E_local, bn, R;  // R = the sum of recv_counts
    int recv_counts[kEpMaxRuns]; // [n_src, E_local] rows received from each source for each local expert
    int *counts;                // [E_local]
    int *offsets;               // [E_local + 1] unpadded grouped offsets
    int *poff;                  // [E_local + 1] offsets with each expert's segment padded to bn rows
    int *rperm;                 // [rows] padded grouped row -> received row, -1 for padding
    int *slot;                  // [R] received row -> padded grouped row
    float *ones;                // [R] set to 1: the GEMMs' gate (the source applies the real gates)
};

struct EpCombineArgs {
    int T, d;
    const int *idx;             // [T, 2] experts (-1: padding token)
    const float *gate;          // [T, 2]
    const int *slot_of_route;   // [2T] route -> its row in the sent (and returned) order
    const float *y;             // [rows sent, d] expert outputs returned by their ranks
    __nv_bfloat16 *out;         // [T, d]
};

cudaError_t launch_ep_layout(const EpLayoutArgs &a, cudaStream_t s);
// xp[slot[i]] = rows[i], i < R
cudaError_t launch_ep_gather(int R, int d, const __nv_bfloat16 *rows, const int *slot, __nv_bfloat16 *xp, int scaled,
                             cudaStream_t s);
// y[i] = sum_s part[s * plane + i * d ...], s ascending
cudaError_t launch_ep_split_sum(int R, int d, int splits, size_t plane, const float *part, float *y, cudaStream_t s);
cudaError_t launch_ep_combine(const EpCombineArgs &a, cudaStream_t s);

cudaError_t launch_router(const RouteArgs &a, cudaStream_t s);
cudaError_t launch_dispatch(const DispatchArgs &a, cudaStream_t s);
// Xp[slot_of_route[r]] = x[r / 2] for the 2T routes
cudaError_t launch_gather(const GatherArgs &a, int T, const int *slot_of_route, cudaStream_t s);
// router + dispatch (+ gather when ga.xp is set) in one launch of T * S blocks for
// T <= route_small_max_tokens(), S = route_small_slices(T, d, SMs) row slices per token;
// `part` is fp32 scratch of T * S * 8 words, `ticket` a zero-initialised device word owned by
// the caller (left at 0 after the launch)
int route_small_max_tokens();
int route_small_slices(int T, int d, int num_sms);
cudaError_t launch_route_small(const RouteArgs &ra, const DispatchArgs &da, const GatherArgs &ga, float *part, int S,
                               unsigned int *ticket, cudaStream_t s);
cudaError_t launch_gemm_up(int bn, const CUtensorMap &wl, const CUtensorMap &wv, const CUtensorMap &xp,
                           const GemmArgs &a, int grid, cudaStream_t s);
cudaError_t launch_gemm_down(int bn, const CUtensorMap &w1, const CUtensorMap &h, const GemmArgs &a,
                             int grid, cudaStream_t s);
// the same GEMMs for K-major ([E, out, in]) weights, dequantised into TMEM
cudaError_t launch_gemm_up_ts(int bn, const CUtensorMap &wl, const CUtensorMap &wv, const CUtensorMap &xp,
                              const GemmArgs &a, int grid, cudaStream_t s);
cudaError_t launch_gemm_down_ts(int bn, const CUtensorMap &w1, const CUtensorMap &h, const GemmArgs &a,
                                int grid, cudaStream_t s);
// The GEMMs of a plan with tile width bn on CTA pairs (M = 256 per MMA across two SMs), for
// bn = 32 (tiles of 32 routes) and bn = 128 (up-projection tiles of 128 routes, down-projection
// tiles of two 128-row segments).  gemm_pair_tn: routes per pair tile, 0 if bn has no pair
// kernel; each CTA holds tn / 2 route rows, so the activation map (xp for the up-projection, or
// the routed-rows map with a.gather; H for the down-projection) has boxes of tn / 2 rows.
// gemm_pair_ready: the device can run a full wave of that kernel's pairs.  a.M a multiple of 256.
int gemm_pair_tn(bool up, int bn);
bool gemm_pair_ready(bool up, int bn, int num_sms);
cudaError_t launch_gemm_up_pair(int bn, const CUtensorMap &wl, const CUtensorMap &wv, const CUtensorMap &xp,
                                const GemmArgs &a, int num_sms, cudaStream_t s);
cudaError_t launch_gemm_down_pair(int bn, const CUtensorMap &w1, const CUtensorMap &h, const GemmArgs &a, int num_sms,
                                  cudaStream_t s);
// reduction elements per pipeline stage of the TMEM-operand GEMM (up- or down-projection, tile width bn)
int gemm_ts_kstage(bool up, int bn);
// out[e, m, k] = in[e, k, m] for E int8 [K, M] matrices (K, M multiples of 64)
cudaError_t launch_pack_i8(const int8_t *in, int8_t *out, int E, int K, int M, int *range_flag, cudaStream_t s);
cudaError_t launch_scale_rows(const __nv_bfloat16 *in, __nv_bfloat16 *out, size_t n, float f, cudaStream_t s);
cudaError_t launch_combine(const CombineArgs &a, cudaStream_t s);

// dynamic shared memory each GEMM variant needs (for cudaFuncSetAttribute)
size_t gemm_smem_bytes(bool up, int bn);

}  // namespace moe
