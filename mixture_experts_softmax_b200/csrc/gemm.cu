// gemm.cu -- grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// Computes the expert MLP of "Grok-1 Admin & Architecture Guide", section 3,
// "Mixture of Experts (MoELayer + Router)" step 3, linear_1(gelu(linear(x)) * linear_v(x)),
// with the 8-bit weights of section 3 "Quantized weights" (int8 value * scale).
//
// Orientation: the weights are the MMA's A operand (M = 128 output features per
// tile), the grouped token rows are B (N = BN rows per tile), K is the reduction:
//     D[f, r] = sum_k W[e, k, f] * X[r, k]            (fp32 in TMEM)
// Each weight tile is read from HBM once per N-tile, so a decode step with a few
// rows per expert streams every touched weight byte exactly once, and per-output-
// channel scales are one value per TMEM lane in the epilogue.
//
// Per pipeline stage (kBK = 64 reduction elements):
//   - a TMA producer thread copies the int8 weight tile(s) [64 k x 128 f] into a
//     staging ring (128-byte swizzle);
//   - 16 converter warps turn each int8 tile into bf16 in the canonical
//     MN-major 128-byte-swizzled UMMA layout (int8 -> bf16 is exact);
//   - a second TMA producer thread copies the bf16 activation tile [BN r x 64 k]
//     (K-major, 128-byte swizzle) straight into the operand ring;
//   - one thread issues tcgen05.mma (kind::f16, bf16 x bf16 -> fp32) and commits
//     stage release and accumulator-ready events to mbarriers;
//   - 4 epilogue warps read the double-buffered accumulators out of TMEM and apply
//       UP:   H[r, f] = bf16( gelu(sl[f] * D_l) * (sv[f] * D_v) )
//       DOWN: slot[split, t, j, f] = gate[t, j] * s1[f] * D      (scatter to token order)
//     The DOWN result of every route lands in its own slot, so the combine that
//     sums the slots is deterministic.
// The CTA is persistent: tiles are taken in a fixed order from a tile list derived
// on the device from the padded expert offsets.  Every wait on an mbarrier is
// bounded in time; on expiry the kernel records an error, stops, drains its own
// in-flight copies and MMAs and frees TMEM.
#include "gemm_common.cuh"

namespace moe {

namespace {

constexpr int kThreads = 768;                  // 24 warps
constexpr int kWarpTmaA = 0, kWarpMma = 1, kWarpTmaB = 2;
constexpr int kWarpEpi0 = 4;                   // warps 4..7: epilogue (TMEM lanes 0..127)
constexpr int kWarpConv0 = 8;                  // warps 8..23: int8 -> bf16 converters
constexpr int kConvThreads = (kThreads / 32 - kWarpConv0) * 32;
static_assert(kConvThreads == kBM * kBK / 16, "one 16-byte unit per converter thread and matrix");
constexpr int kSmemBudget = 216 * 1024;

template <bool UP, int BN>
struct Cfg {
    static constexpr int NA = UP ? 2 : 1;                 // weight matrices per stage
    static constexpr int STG = NA * kBM * kBK;            // int8 staging bytes per stage
    static constexpr int ABYTES = NA * kBM * kBK * 2;     // bf16 A bytes per stage
    static constexpr int BBYTES = BN * kBK * 2;           // bf16 B bytes per stage
    static constexpr int S2 = UP ? 3 : 4;                 // operand ring depth
    static constexpr int S1 = cmin(12, (kSmemBudget - S2 * (ABYTES + BBYTES)) / STG);   // staging ring
    static constexpr int ACC = NA * BN;                   // TMEM columns of one accumulator buffer
    static constexpr int TMEM_COLS = pow2_at_least(2 * ACC);
    static constexpr int OFF_STG = 0;
    static constexpr int OFF_A = OFF_STG + S1 * STG;
    static constexpr int OFF_B = OFF_A + S2 * ABYTES;
    static constexpr int OFF_BAR = OFF_B + S2 * BBYTES;
    // barriers: stg_full[S1] stg_empty[S1] a_full[S2] b_full[S2] op_empty[S2] acc_full[2] acc_empty[2] drain
    static constexpr int NBAR = 2 * S1 + 3 * S2 + 5;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int MISC_BYTES = 16 + 2 * 4 * 40;    // tmem addr, abort flag, prefix[40], poff[40]
    static constexpr int SMEM = OFF_MISC + MISC_BYTES + 1024;   // + alignment slack
    static_assert(S1 >= 2, "staging ring too shallow");
    static_assert(SMEM <= 227 * 1024, "shared memory over the per-CTA limit");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128 is 16..256 in steps of 16");
    static_assert(TMEM_COLS <= 512, "TMEM has 512 columns");
};

// kind::f16 instruction descriptor: D fp32, A and B bf16, A MN-major, B K-major, M = 128.
template <int BN>
__device__ __forceinline__ constexpr uint32_t idesc_bf16()
{
    return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (static_cast<uint32_t>(BN >> 3) << 17) |
           (static_cast<uint32_t>(kBM >> 4) << 24);
}

template <bool UP, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                const __grid_constant__ CUtensorMap tmB, const GemmArgs a)
{
    using C = Cfg<UP, BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * i; };
    auto stg_full = [&](int s) { return bar(s); };
    auto stg_empty = [&](int s) { return bar(C::S1 + s); };
    auto a_full = [&](int s) { return bar(2 * C::S1 + s); };
    auto b_full = [&](int s) { return bar(2 * C::S1 + C::S2 + s); };
    auto op_empty = [&](int s) { return bar(2 * C::S1 + 2 * C::S2 + s); };
    auto acc_full = [&](int b) { return bar(2 * C::S1 + 3 * C::S2 + b); };
    auto acc_empty = [&](int b) { return bar(2 * C::S1 + 3 * C::S2 + 2 + b); };
    const uint32_t drain_bar = bar(2 * C::S1 + 3 * C::S2 + 4);

    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile uint32_t *abort_flag = misc + 1;
    int *prefix = reinterpret_cast<int *>(misc + 4);
    int *poff = prefix + 40;
    const int m_tiles = a.M / kBM;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::S1; ++s) {
            mbar_init(stg_full(s), 1);
            mbar_init(stg_empty(s), kConvThreads / 32);
        }
        for (int s = 0; s < C::S2; ++s) {
            mbar_init(a_full(s), kConvThreads / 32);
            mbar_init(b_full(s), 1);
            mbar_init(op_empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(acc_full(b), 1);
            mbar_init(acc_empty(b), 4);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0u;
        prefix[0] = 0;
        for (int e = 0; e <= a.E; ++e) poff[e] = a.poff[e];
        for (int e = 0; e < a.E; ++e)
            prefix[e + 1] = prefix[e] + m_tiles * ((poff[e + 1] - poff[e]) / BN) * a.splits;
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(smem_u32(misc), C::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == kWarpTmaA && lane == 0) {
        prefetch_tmap(&tmA0);
        if (UP) prefetch_tmap(&tmA1);
        prefetch_tmap(&tmB);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc[0];
    const int total = prefix[a.E];
#ifdef MOE_PIPE_STATS
    if (threadIdx.x == 0) atomicAdd(&g_pipe_stats[UP ? 28 : 29], static_cast<unsigned long long>(clock64()));
#endif
    const Waiter w{abort_flag, a.err, a.timeout_ns, UP ? 0 : 10};

    if (warp == kWarpTmaA) {
        // ---- int8 weight tiles -> staging ring ------------------------------------
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            uint32_t st = 0, ph = 0, issued = 0, par = 0;
            for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
                int e, m, n, s;
                decode_tile<BN>(tile, prefix, poff, m_tiles, a.splits, e, m, n, s);
                const int kb = s * a.ksteps;
                for (int ks = 0; ks < a.ksteps; ++ks) {
                    if (!w.wait(stg_empty(st), ph ^ 1u, 1)) goto a_done;
                    mbar_arrive_expect_tx(stg_full(st), C::STG);
                    const int y = e * a.K + (kb + ks) * kBK;
                    const uint32_t dst = sbase + C::OFF_STG + st * C::STG;
                    tma_load_2d(dst, &tmA0, stg_full(st), m * kBM, y, pol);
                    if (UP) tma_load_2d(dst + kBM * kBK, &tmA1, stg_full(st), m * kBM, y, pol);
                    issued |= 1u << st;
                    par = (par & ~(1u << st)) | (ph << st);
                    if (++st == C::S1) { st = 0; ph ^= 1u; }
                }
            }
        a_done:
            for (int s = 0; s < C::S1; ++s)   // every copy issued has landed before the CTA may exit
                if (issued & (1u << s)) wait_drain(stg_full(s), (par >> s) & 1u);
        }
        __syncwarp();
    } else if (warp == kWarpTmaB) {
        // ---- bf16 activation tiles -> operand ring ---------------------------------
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_last();
            uint32_t st = 0, ph = 0, issued = 0, par = 0;
            for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
                int e, m, n, s;
                decode_tile<BN>(tile, prefix, poff, m_tiles, a.splits, e, m, n, s);
                const int kb = s * a.ksteps;
                const int row = poff[e] + n * BN;
                for (int ks = 0; ks < a.ksteps; ++ks) {
                    if (!w.wait(op_empty(st), ph ^ 1u, 2)) goto b_done;
                    mbar_arrive_expect_tx(b_full(st), C::BBYTES);
                    tma_load_2d(sbase + C::OFF_B + st * C::BBYTES, &tmB, b_full(st), (kb + ks) * kBK, row, pol);
                    issued |= 1u << st;
                    par = (par & ~(1u << st)) | (ph << st);
                    if (++st == C::S2) { st = 0; ph ^= 1u; }
                }
            }
        b_done:
            for (int s = 0; s < C::S2; ++s)
                if (issued & (1u << s)) wait_drain(b_full(s), (par >> s) & 1u);
        }
        __syncwarp();
    } else if (warp == kWarpMma) {
        // ---- tensor-core issue -----------------------------------------------------
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16<BN>();
            uint32_t st = 0, ph = 0;
            int it = 0;
            for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
                const int b = it & 1;
                const uint32_t aph = (it >> 1) & 1;
                if (!w.wait(acc_empty(b), aph ^ 1u, 3)) break;
                tc_fence_after();
                const uint32_t dcol = tmem_base + b * C::ACC;
                bool ok = true;
                for (int ks = 0; ks < a.ksteps; ++ks) {
                    if (!w.wait(a_full(st), ph, 4) || !w.wait(b_full(st), ph, 5)) { ok = false; break; }
                    tc_fence_after();
                    // descriptor low words once per stage; each MMA adds its offset in 16-byte units
                    const uint32_t alo = desc_sw128_lo(sbase + C::OFF_A + st * C::ABYTES, 1024);
                    const uint32_t blo = desc_sw128_lo(sbase + C::OFF_B + st * C::BBYTES, 16);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t bdesc = desc_join(blo + ((kk * 32) >> 4), desc_sw128_hi(1024));
#pragma unroll
                        for (int mat = 0; mat < C::NA; ++mat) {
                            const uint64_t adesc =
                                desc_join(alo + ((mat * kBM * kBK * 2 + kk * 4096) >> 4), desc_sw128_hi(2048));
                            umma_bf16(dcol + mat * BN, adesc, bdesc, idesc, (ks | kk) != 0);
                        }
                    }
                    umma_commit(op_empty(st));
                    if (++st == C::S2) { st = 0; ph ^= 1u; }
                }
                if (!ok) break;
                umma_commit(acc_full(b));
            }
            umma_commit(drain_bar);          // all MMAs issued above have completed after this
            wait_drain(drain_bar, 0);
        }
        __syncwarp();
    } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + 4) {
        // ---- epilogue: TMEM -> registers -> global ---------------------------------
        const int ew = warp - kWarpEpi0;
        int it = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
            int e, m, n, s;
            decode_tile<BN>(tile, prefix, poff, m_tiles, a.splits, e, m, n, s);
            const int b = it & 1;
            const uint32_t aph = (it >> 1) & 1;
            const bool ok = __all_sync(0xffffffffu, w.wait(acc_full(b), aph, 6));
            if (!ok) break;
            tc_fence_after();
            const int f = m * kBM + ew * 32 + lane;
            const uint32_t tl = tmem_base + (static_cast<uint32_t>(ew * 32) << 16) + b * C::ACC;
            const int row0 = poff[e] + n * BN;
            if constexpr (UP) {
                const float sa = __bfloat162float(a.s0[static_cast<size_t>(e) * a.M + f]);
                const float sb = __bfloat162float(a.s1[static_cast<size_t>(e) * a.M + f]);
#pragma unroll 1
                for (int c = 0; c < BN; c += 16) {
                    float va[16], vb[16];
                    __syncwarp();   // tcgen05.ld is warp-collective (.sync.aligned): converge first
                    tmem_ld16(tl + c, va);
                    tmem_ld16(tl + BN + c, vb);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int r = row0 + c + i;
                        if (__ldg(a.rperm + r) >= 0)
                            a.h[static_cast<size_t>(r) * a.M + f] =
                                __float2bfloat16_rn(gelu_tanh(sa * va[i]) * (sb * vb[i]));
                    }
                }
            } else {
                const float sc = __bfloat162float(a.s0[static_cast<size_t>(e) * a.M + f]);
#pragma unroll 1
                for (int c = 0; c < BN; c += 16) {
                    float v[16];
                    __syncwarp();   // tcgen05.ld is warp-collective (.sync.aligned): converge first
                    tmem_ld16(tl + c, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int route = __ldg(a.rperm + row0 + c + i);
                        if (route >= 0) {
                            const float g = __ldg(a.gate + route);
                            const size_t o = ((static_cast<size_t>(s) * a.T + (route >> 1)) * 2 + (route & 1)) *
                                                 static_cast<size_t>(a.M) + f;
                            a.slots[o] = g * (sc * v[i]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty(b));
        }
    } else if (warp >= kWarpConv0) {
        // ---- int8 staging -> bf16 UMMA operand (MN-major, 128-byte swizzle) --------
        // Thread ct owns one 16-byte unit of every [64 k x 128 f] int8 tile: reduction
        // row k = (ct & 7) | (ct >> 6) << 3 and 16-feature chunk mc = (ct >> 3) & 7.
        // 8 consecutive lanes take 8 rows of one chunk, so both the swizzled reads and
        // the swizzled writes are free of bank conflicts.
        const int ct = threadIdx.x - kWarpConv0 * 32;
        const int k = (ct & 7) | ((ct >> 6) << 3);
        const int mc = (ct >> 3) & 7;
        const int kr = k & 7;
        const uint32_t src_off = k * 128 + ((mc ^ kr) << 4);
        const uint32_t atom = ((((k >> 3) * 2 + (mc >> 2)) << 10) + kr * 128);
        const uint32_t dst_lo = atom + ((((mc & 3) * 2) ^ kr) << 4);
        const uint32_t dst_hi = atom + (((((mc & 3) * 2) ^ kr) ^ 1) << 4);
        uint32_t st = 0, ph = 0, st2 = 0, ph2 = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            bool ok = true;
            for (int ks = 0; ks < a.ksteps; ++ks) {
                ok = __all_sync(0xffffffffu, w.wait(stg_full(st), ph, 7) && w.wait(op_empty(st2), ph2 ^ 1u, 8));
                if (!ok) break;
                const uint32_t src0 = sbase + C::OFF_STG + st * C::STG + src_off;
                const uint32_t dst0 = sbase + C::OFF_A + st2 * C::ABYTES;
                uint4 v[C::NA];
#pragma unroll
                for (int mat = 0; mat < C::NA; ++mat) v[mat] = lds128(src0 + mat * kBM * kBK);
#pragma unroll
                for (int mat = 0; mat < C::NA; ++mat) {
                    uint4 lo, hi;
                    lo.x = i8x2_to_bf16x2(v[mat].x, 0x4140);
                    lo.y = i8x2_to_bf16x2(v[mat].x, 0x4342);
                    lo.z = i8x2_to_bf16x2(v[mat].y, 0x4140);
                    lo.w = i8x2_to_bf16x2(v[mat].y, 0x4342);
                    hi.x = i8x2_to_bf16x2(v[mat].z, 0x4140);
                    hi.y = i8x2_to_bf16x2(v[mat].z, 0x4342);
                    hi.z = i8x2_to_bf16x2(v[mat].w, 0x4140);
                    hi.w = i8x2_to_bf16x2(v[mat].w, 0x4342);
                    const uint32_t d = dst0 + mat * kBM * kBK * 2;
                    sts128(d + dst_lo, lo);
                    sts128(d + dst_hi, hi);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(stg_empty(st));
                    mbar_arrive(a_full(st2));
                }
                if (++st == C::S1) { st = 0; ph ^= 1u; }
                if (++st2 == C::S2) { st2 = 0; ph2 ^= 1u; }
            }
            if (!ok) break;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
#ifdef MOE_PIPE_STATS
    if (threadIdx.x == 0) atomicAdd(&g_pipe_stats[UP ? 30 : 31], static_cast<unsigned long long>(clock64()));
#endif
}

template <bool UP, int BN>
cudaError_t launch_one(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &b, const GemmArgs &args,
                       int grid, cudaStream_t s)
{
    using C = Cfg<UP, BN>;
    static bool configured = false;   // attribute set once per process (per device is not needed: same value)
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemm_kernel<UP, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    gemm_kernel<UP, BN><<<grid, kThreads, C::SMEM, s>>>(a0, a1, b, args);
    return cudaGetLastError();
}

}  // namespace

size_t gemm_smem_bytes(bool up, int bn)
{
    switch (bn) {
    case 16: return up ? Cfg<true, 16>::SMEM : Cfg<false, 16>::SMEM;
    case 32: return up ? Cfg<true, 32>::SMEM : Cfg<false, 32>::SMEM;
    case 64: return up ? Cfg<true, 64>::SMEM : Cfg<false, 64>::SMEM;
    case 128: return up ? Cfg<true, 128>::SMEM : Cfg<false, 128>::SMEM;
    default: return 0;
    }
}

cudaError_t launch_gemm_up(int bn, const CUtensorMap &wl, const CUtensorMap &wv, const CUtensorMap &xp,
                           const GemmArgs &a, int grid, cudaStream_t s)
{
    switch (bn) {
    case 16: return launch_one<true, 16>(wl, wv, xp, a, grid, s);
    case 32: return launch_one<true, 32>(wl, wv, xp, a, grid, s);
    case 64: return launch_one<true, 64>(wl, wv, xp, a, grid, s);
    case 128: return launch_one<true, 128>(wl, wv, xp, a, grid, s);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_gemm_down(int bn, const CUtensorMap &w1, const CUtensorMap &h, const GemmArgs &a, int grid,
                             cudaStream_t s)
{
    switch (bn) {
    case 16: return launch_one<false, 16>(w1, w1, h, a, grid, s);
    case 32: return launch_one<false, 32>(w1, w1, h, a, grid, s);
    case 64: return launch_one<false, 64>(w1, w1, h, a, grid, s);
    case 128: return launch_one<false, 128>(w1, w1, h, a, grid, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe

#ifdef MOE_PIPE_STATS
// instrumented builds only: copy (and optionally clear) the per-site wait-cycle sums
extern "C" __attribute__((visibility("default"))) int moe_debug_pipe_stats(unsigned long long *out, int reset)
{
    if (cudaMemcpyFromSymbol(out, moe::g_pipe_stats, sizeof(unsigned long long) * 64) != cudaSuccess) return -4;
    if (reset) {
        unsigned long long z[64] = {};
        if (cudaMemcpyToSymbol(moe::g_pipe_stats, z, sizeof z) != cudaSuccess) return -4;
    }
    return 0;
}
#endif


