// pack.cu -- one-time weight layout change for the TMEM-operand GEMMs.  Every expert's
// int8 matrix stored [in, out] (x @ W orientation) is rewritten as contiguous 16 KB
// tiles, one per (block of 128 output features, block of 128 reduction elements), in
// the order the GEMM streams them; inside a tile each output feature owns a 128-byte
// row of its reduction elements, with the 16-byte chunks rotated by the 128-byte
// swizzle (chunk j of row r stored at chunk j ^ (r % 8)) so that the converter warps
// read it without shared-memory bank conflicts.  Values are copied, not changed;
// scales are untouched.
#include "kernels.cuh"

namespace moe {

namespace {

__global__ void __launch_bounds__(256) pack_tiles_kernel(const int8_t *in, int8_t *out, int K, int M)
{
    __shared__ uint32_t tile[128][33];   // [k][m / 4], padded
    const int e = blockIdx.z, kt = blockIdx.y, mt = blockIdx.x;
    const int k0 = kt * 128, m0 = mt * 128;
    for (int idx = threadIdx.x; idx < 1024; idx += blockDim.x) {
        const int row = idx >> 3, c = idx & 7;
        const uint4 v = *reinterpret_cast<const uint4 *>(in + (static_cast<size_t>(e) * K + k0 + row) * M + m0 + c * 16);
        tile[row][c * 4 + 0] = v.x;
        tile[row][c * 4 + 1] = v.y;
        tile[row][c * 4 + 2] = v.z;
        tile[row][c * 4 + 3] = v.w;
    }
    __syncthreads();
    int8_t *base = out + ((static_cast<size_t>(e) * (M / 128) + mt) * (K / 128) + kt) * 16384;
    for (int idx = threadIdx.x; idx < 1024; idx += blockDim.x) {
        const int r = idx >> 3, j = idx & 7;
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t acc = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const uint32_t byte = (tile[j * 16 + q * 4 + b][r >> 2] >> (8 * (r & 3))) & 0xffu;
                acc |= byte << (8 * b);
            }
            w[q] = acc;
        }
        *reinterpret_cast<uint4 *>(base + r * 128 + ((j ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

}  // namespace

cudaError_t launch_pack_tiles(const int8_t *in, int8_t *out, int E, int K, int M, cudaStream_t s)
{
    dim3 grid(M / 128, K / 128, E);
    pack_tiles_kernel<<<grid, 256, 0, s>>>(in, out, K, M);
    return cudaGetLastError();
}

}  // namespace moe
