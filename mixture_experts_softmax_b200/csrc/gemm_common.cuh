// gemm_common.cuh -- pieces shared by the two grouped-GEMM kernels (weights from the
// reference [E, in, out] layout through shared memory, and pre-packed K-major weights
// through TMEM): descriptors, the int8 -> bf16 conversion, GELU, bounded waits and the
// device-side tile list.
#pragma once

#include "kernels.cuh"
#include "ptx.cuh"

namespace moe {

constexpr int cmin(int a, int b) { return a < b ? a : b; }
constexpr int pow2_at_least(int v)
{
    int p = 32;
    while (p < v) p <<= 1;
    return p;
}

#ifdef MOE_PIPE_STATS
// cycles spent in each wait site, summed over the CTA (instrumented builds only; one
// array per translation unit)
static __device__ unsigned long long g_pipe_stats[64];
#endif

// UMMA shared-memory descriptor, 128-byte swizzle, sm_100 version bits.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo)
{
    return static_cast<uint64_t>((addr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(lbo >> 4) << 16) |
           (static_cast<uint64_t>(sbo >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// The same descriptor as its two 32-bit halves: the low word holds the address field and the
// leading byte offset, the high word the stride, the version and the swizzle mode.  For a
// 16-byte-aligned shared-memory address below 256 KB, moving the operand by off bytes (a multiple
// of 16) adds off >> 4 to the low word and nothing else, so an MMA loop forms each descriptor
// with one 32-bit add.
__device__ __forceinline__ uint32_t desc_sw128_lo(uint32_t addr, uint32_t lbo)
{
    return ((addr & 0x3FFFFu) >> 4) | ((lbo >> 4) << 16);
}
__host__ __device__ constexpr uint32_t desc_sw128_hi(uint32_t sbo) { return (sbo >> 4) | (1u << 14) | (2u << 29); }
__device__ __forceinline__ uint64_t desc_join(uint32_t lo, uint32_t hi)
{
    return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Two signed bytes (chosen by `sel`) -> two exact bf16 values (the [E, in, out] layout's
// weights, two's complement).  With the byte b in
// the low 7 mantissa bits under exponent 2^7, hi = 128 + (b & 127); lo is 128, or
// 256 when b's sign bit is set (it lands on the exponent's lowest bit); hi - lo = b
// exactly (an integer of at most 8 significant bits).
__device__ __forceinline__ uint32_t i8x2_to_bf16x2(uint32_t w, uint32_t sel)
{
    const uint32_t p = __byte_perm(w, 0x43434343u, sel);
    const uint32_t hi = p & 0xFF7FFF7Fu;
    const uint32_t lo = p & 0xFF80FF80u;
    __nv_bfloat162 r = __hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&hi),
                               *reinterpret_cast<const __nv_bfloat162 *>(&lo));
    return *reinterpret_cast<uint32_t *>(&r);
}

// The packed form.  A packed 32-bit word holds the weights of four consecutive reduction
// elements k .. k+3, each as a sign bit and a 7-bit magnitude, with the signs crossed over within
// each 16-bit half: byte 0 = sign(w[k+2]) << 7 | |w[k]|,   byte 1 = sign(w[k]) << 7 | |w[k+2]|,
//                   byte 2 = sign(w[k+3]) << 7 | |w[k+1]|, byte 3 = sign(w[k+1]) << 7 | |w[k+3]|.
// Masked with 0x807F807F the word is the bf16 pair (w[k], w[k+1]) with zero exponent fields:
// the values w * 2^-133, exactly (bf16 numbers with a zero exponent field are the multiples of
// 2^-133 below 2^-126).  With the bytes of each half swapped first (prmt 0x2301), the same mask
// gives (w[k+2], w[k+3]).  Three integer instructions per two pairs.
//   pk_lo / pk_hi:        the pairs (w[k], w[k+1]) / (w[k+2], w[k+3]) as w * 2^-133;
//   pk_exact:             a masked-ready word's pair as the normal bf16 values w themselves, formed as
//                         (+-(128 + m)) - (+-128): both terms have exponent 2^7 and the sign of w, and
//                         their difference is exact.
__device__ __forceinline__ uint32_t pk_swap(uint32_t q)
{
    uint32_t p;
    asm("prmt.b32 %0, %1, %1, 0x2301;" : "=r"(p) : "r"(q));
    return p;
}
__device__ __forceinline__ uint32_t pk_lo(uint32_t q) { return q & 0x807F807Fu; }
__device__ __forceinline__ uint32_t pk_hi(uint32_t q) { return pk_swap(q) & 0x807F807Fu; }
__device__ __forceinline__ uint32_t pk_exact(uint32_t q)
{
    const uint32_t hi = (q & 0x807F807Fu) | 0x43004300u;
    const uint32_t lo = (q & 0x80008000u) | 0x43004300u;
    __nv_bfloat162 r = __hsub2(*reinterpret_cast<const __nv_bfloat162 *>(&hi),
                               *reinterpret_cast<const __nv_bfloat162 *>(&lo));
    return *reinterpret_cast<uint32_t *>(&r);
}

// One 16-byte chunk of packed weights (16 values) -> 8 bf16 pairs for one 8-column TMEM store,
// in the form convert_group describes.
template <bool KBLOCK>
__device__ __forceinline__ void convert_chunk(const uint4 &v, uint32_t (&words)[8], __nv_bfloat162 sc2)
{
    const uint32_t q[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if constexpr (KBLOCK) {
            words[2 * j] = pk_exact(q[j]);
            words[2 * j + 1] = pk_exact(pk_swap(q[j]));
        } else {
            words[2 * j] = pk_lo(q[j]);
            words[2 * j + 1] = pk_hi(q[j]);
        }
    }
    if constexpr (KBLOCK) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            __nv_bfloat162 wq = *reinterpret_cast<const __nv_bfloat162 *>(&words[k]);
            wq = __hmul2(wq, sc2);
            words[k] = *reinterpret_cast<const uint32_t *>(&wq);
        }
    }
}

// Four 16-byte chunks of packed weights (64 values) -> 32 bf16 pairs for one 32-column TMEM
// store: the subnormal form (per-channel scales, applied in the epilogue), or the exact
// values times the block scale sc2 (per-block scales).
template <bool KBLOCK>
__device__ __forceinline__ void convert_group(const uint4 *v, uint32_t (&words)[32], __nv_bfloat162 sc2)
{
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const uint32_t q[4] = {v[h].x, v[h].y, v[h].z, v[h].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if constexpr (KBLOCK) {
                words[8 * h + 2 * j] = pk_exact(q[j]);
                words[8 * h + 2 * j + 1] = pk_exact(pk_swap(q[j]));
            } else {
                words[8 * h + 2 * j] = pk_lo(q[j]);
                words[8 * h + 2 * j + 1] = pk_hi(q[j]);
            }
        }
    }
    if constexpr (KBLOCK) {
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            __nv_bfloat162 wq = *reinterpret_cast<const __nv_bfloat162 *>(&words[k]);
            wq = __hmul2(wq, sc2);
            words[k] = *reinterpret_cast<const uint32_t *>(&wq);
        }
    }
}

__device__ __forceinline__ float gelu_tanh(float a)
{
    // 0.5 a (1 + tanh(sqrt(2/pi) (a + 0.044715 a^3)))
    const float k0 = 0.7978845608028654f, k1 = 0.044715f * 0.7978845608028654f;
    const float u = a * fmaf(k1, a * a, k0);
    const float h = 0.5f * a;
    return fmaf(h, tanh_approx(u), h);
}

struct Waiter {
    volatile uint32_t *abort;
    int *err;
    long long timeout_ns;
    int stat_base;   // instrumented builds: first stats slot of this kernel

    // wait for the phase of `bar` with parity `par`; false if the CTA aborted or the limit ran out
    __device__ __forceinline__ bool wait(uint32_t bar, uint32_t par, int site) const
    {
        if (mbar_try_wait(bar, par)) return true;
        const uint64_t t0 = global_timer_ns();
        while (true) {
            if (mbar_try_wait(bar, par)) return true;
            if (*abort) return false;
            if (static_cast<long long>(global_timer_ns() - t0) > timeout_ns) {
                *abort = 1u;
                atomicCAS(err, 0, kErrTimeoutBase + site);
                return false;
            }
        }
    }
};

// Instrumented builds (-DMOE_PIPE_STATS): cycle counters kept per thread in registers and
// added to g_pipe_stats once per warp at the end of the kernel.
#ifdef MOE_PIPE_STATS
#define PS_VAR(v) long long v = 0
#define PS_NOW(t) const long long t = clock64()
#define PS_ADD(v, t0) (v) += clock64() - (t0)
#define PS_FLUSH(slot, v) atomicAdd(&g_pipe_stats[slot], static_cast<unsigned long long>(v))
#else
#define PS_VAR(v)
#define PS_NOW(t)
#define PS_ADD(v, t0)
#define PS_FLUSH(slot, v)
#endif

// wait used only while draining after an abort: fixed 1 s limit, ignores the abort flag
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t par)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, par))
        if (global_timer_ns() - t0 > 1000000000ull) return;
}

// tile index -> expert e, output tile m, route tile n, reduction split s: splits vary
// fastest, then route tiles, then output tiles, expert after expert.  A route tile covers
// `pair` consecutive BN-row segments of its expert (the expert's last tile may cover fewer).
template <int BN>
__device__ __forceinline__ void decode_tile(int tile, const int *prefix, const int *poff, int m_tiles,
                                            int splits, int &e, int &m, int &n, int &s, int pair = 1)
{
    e = 0;
    while (tile >= prefix[e + 1]) ++e;
    int local = tile - prefix[e];
    s = local % splits;
    local /= splits;
    const int nt = ((poff[e + 1] - poff[e]) / BN + pair - 1) / pair;   // tiles of `pair` BN-row segments
    n = local % nt;
    m = local / nt;
}


// The persistent CTAs' work list.  Tiles fill whole waves of gridDim.x CTAs; the r tiles of
// a last, partial wave are each cut along the reduction into P = gridDim.x / r pieces
// (stream-K for the last wave only), so every CTA runs the same number of whole tiles and
// at most one piece.  A piece leaves its fp32 accumulator in a workspace; the piece that
// finishes last (a ticket per tile) adds the P partial sums in piece order and applies the
// tile's epilogue.  P < 2 means no pieces; so do fewer tiles than CTAs (test-sized problems).
struct WorkList {
    int whole;    // items [0, whole): whole tiles 0 .. whole-1
    int P;        // pieces per split tile
    int items;    // whole + (tiles - whole) * P
};

__device__ __forceinline__ WorkList make_work_list(int tiles, int grid, int ksteps)
{
    WorkList q;
    const int r = tiles % grid;
    int P = r ? grid / r : 0;
    if (P > ksteps) P = ksteps;
    if (P < 2 || tiles < grid) P = 0;   // pieces only behind at least one full wave of whole tiles
    q.P = P;
    q.whole = P ? tiles - r : tiles;
    q.items = q.whole + (P ? r * P : 0);
    return q;
}

struct WorkItem {
    int tile;     // tile index (decode_tile)
    int k0, k1;   // stages [k0, k1) of the tile's split
    int piece;    // -1: the whole tile; else the piece's slot in the partial-sum workspace
};

__device__ __forceinline__ WorkItem work_item(const WorkList &q, int i, int ksteps)
{
    if (i < q.whole) return {i, 0, ksteps, -1};
    const int j = i - q.whole, t = j / q.P, p = j - t * q.P;
    return {q.whole + t, p * ksteps / q.P, (p + 1) * ksteps / q.P, j};
}

}  // namespace moe
