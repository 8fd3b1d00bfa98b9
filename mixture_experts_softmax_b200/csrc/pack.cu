// pack.cu -- one-time weight layout change for the TMEM-operand GEMMs: every expert's
// int8 matrix stored [in, out] (x @ W orientation) becomes [out, in], so that the
// reduction elements of one output feature are contiguous.  Values are copied, not
// changed; scales are untouched (they stay per output channel).
#include "kernels.cuh"

namespace moe {

namespace {

// 64 x 64-byte tiles through shared memory: out[e, m, k] = in[e, k, m]
__global__ void __launch_bounds__(256) transpose_i8_kernel(const int8_t *in, int8_t *out, int K, int M)
{
    __shared__ uint32_t tile[64][17];   // [k][m / 4], padded
    const int e = blockIdx.z, k0 = blockIdx.y * 64, m0 = blockIdx.x * 64;
    const int r = threadIdx.x >> 2, c = threadIdx.x & 3;
    const uint4 v = *reinterpret_cast<const uint4 *>(in + (static_cast<size_t>(e) * K + k0 + r) * M + m0 + c * 16);
    tile[r][c * 4 + 0] = v.x;
    tile[r][c * 4 + 1] = v.y;
    tile[r][c * 4 + 2] = v.z;
    tile[r][c * 4 + 3] = v.w;
    __syncthreads();
    const int mm = threadIdx.x >> 2, ks = (threadIdx.x & 3) * 16;
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t acc = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const uint32_t byte = (tile[ks + q * 4 + b][mm >> 2] >> (8 * (mm & 3))) & 0xffu;
            acc |= byte << (8 * b);
        }
        w[q] = acc;
    }
    *reinterpret_cast<uint4 *>(out + (static_cast<size_t>(e) * M + m0 + mm) * K + k0 + ks) =
        make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace

cudaError_t launch_transpose_i8(const int8_t *in, int8_t *out, int E, int K, int M, cudaStream_t s)
{
    dim3 grid(M / 64, K / 64, E);
    transpose_i8_kernel<<<grid, 256, 0, s>>>(in, out, K, M);
    return cudaGetLastError();
}

}  // namespace moe
