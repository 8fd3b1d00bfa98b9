// pack.cu -- one-time weight layout change for the TMEM-operand GEMMs: every expert's
// int8 matrix stored [in, out] (x @ W orientation) becomes [out, in], so that the
// reduction elements of one output feature are contiguous, and every four consecutive
// values w[k..k+3] become one 32-bit word of sign bits and 7-bit magnitudes with the signs
// crossed over within each 16-bit half (the layout gemm_common.cuh's pk_lo / pk_hi read:
// bytes sign(w[k+2]) | |w[k]|, sign(w[k]) | |w[k+2]|, sign(w[k+3]) | |w[k+1]|,
// sign(w[k+1]) | |w[k+3]|), which the GEMMs' converters turn into bf16 operands in three
// instructions per four values (kActScale in kernels.cuh).  -128 has no such form: it is
// reported through `range_flag`.  Scales are untouched (they stay per output channel).
#include "kernels.cuh"

namespace moe {

namespace {

// four two's-complement bytes w[k..k+3] (byte i of `w4` = w[k+i]) -> the packed word
__device__ __forceinline__ uint32_t pack_word(uint32_t w4)
{
    uint32_t mag[4], sgn[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t b = (w4 >> (8 * i)) & 0xFFu;
        sgn[i] = b >> 7;
        mag[i] = (sgn[i] ? 0x100u - b : b) & 0x7Fu;   // -128 gives 0: flagged by the caller
    }
    return (mag[0] | sgn[2] << 7) | (mag[2] | sgn[0] << 7) << 8 | (mag[1] | sgn[3] << 7) << 16 |
           (mag[3] | sgn[1] << 7) << 24;
}

// 64 x 64-byte tiles through shared memory: out[e, m, k] = in[e, k, m], four k at a time packed
__global__ void __launch_bounds__(256) pack_i8_kernel(const int8_t *in, int8_t *out, int K, int M, int *range_flag)
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
    bool minus128 = false;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t acc = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const uint32_t byte = (tile[ks + q * 4 + b][mm >> 2] >> (8 * (mm & 3))) & 0xffu;
            minus128 |= byte == 0x80u;
            acc |= byte << (8 * b);
        }
        w[q] = pack_word(acc);
    }
    *reinterpret_cast<uint4 *>(out + (static_cast<size_t>(e) * M + m0 + mm) * K + k0 + ks) =
        make_uint4(w[0], w[1], w[2], w[3]);
    if (minus128) *range_flag = 1;
}

// out = in * f for n bf16 values (n a multiple of 8), in fp32: exact for a power of two f
// while the results stay finite
__global__ void __launch_bounds__(256) scale_rows_kernel(const uint4 *in, uint4 *out, size_t n8, float f)
{
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n8;
         i += static_cast<size_t>(gridDim.x) * blockDim.x)
        out[i] = scale_bf16x8(in[i], f);
}

}  // namespace

cudaError_t launch_pack_i8(const int8_t *in, int8_t *out, int E, int K, int M, int *range_flag, cudaStream_t s)
{
    dim3 grid(M / 64, K / 64, E);
    pack_i8_kernel<<<grid, 256, 0, s>>>(in, out, K, M, range_flag);
    return cudaGetLastError();
}

cudaError_t launch_scale_rows(const __nv_bfloat16 *in, __nv_bfloat16 *out, size_t n, float f, cudaStream_t s)
{
    const size_t n8 = n / 8;
    if (n8 == 0) return cudaSuccess;
    const unsigned int blocks = static_cast<unsigned int>(n8 / 256 + 1 < 4096 ? n8 / 256 + 1 : 4096);
    scale_rows_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const uint4 *>(in), reinterpret_cast<uint4 *>(out), n8,
                                             f);
    return cudaGetLastError();
}

}  // namespace moe
