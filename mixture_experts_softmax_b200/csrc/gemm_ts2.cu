// gemm_ts2.cu -- the grouped expert GEMMs of the packed layout on CTA pairs: one tcgen05 MMA of
// M = 256 output features spans the two SMs of a two-CTA cluster.  It computes the expert MLP of
// "Grok-1 Admin & Architecture Guide", section 3, "Mixture of Experts (MoELayer + Router)" step 3,
// linear_1(gelu(linear(x)) * linear_v(x)), with the 8-bit weights of section 3 "Quantized
// weights", and the gate-weighted scatter of step 4.
//
// Why pairs.  In the one-CTA kernel (gemm_ts.cu) a prefill stage of 128 reduction elements moves
// 160 KB through one SM's shared memory against 1024 MMA cycles (the int8 weight boxes in and
// out again to the converters, the activation tile in, and read by every MMA), above the
// ~128 B/clk shared memory delivers.  On a pair the activation tile is split: each CTA loads
// and serves half of the routes' rows, and every MMA reads both halves, so a CTA moves 112 KB
// (up-projection) or 96 KB (down-projection) per stage.  For small batches, where one thread
// issuing MMAs of few columns is the limit, each MMA of a pair covers twice the features.
//
// Tiles (TN routes, segments padded to SEG rows by the dispatch):
//   up-projection    TN = 128 (large batches) or 32 (small): both matrices, two issuers;
//   down-projection  TN = 256 (two 128-row segments of an expert; one matrix, one issuer), or
//                    TN = 32 with two consecutive 128-element k-boxes per stage, each with an
//                    issuer and accumulator of its own, summed by the epilogue in box order;
//                    both with optional K-splits.
// CTA c of the pair converts the int8 weights of features 256 m + 128 c .. + 127 into its own
// TMEM (its half of the MMA's A operand) and loads route rows row0 + c TN/2 .. + TN/2 - 1 into
// its shared memory (its half of B).  The even CTA issues the MMAs; each CTA's accumulators hold
// its 128 features x TN routes, and each CTA's epilogue writes its features: H for the
// up-projection (gelu(s_lin A0) * (s_v A1)), gate * s_1 * A into the route's slot for the
// down-projection.  A 256-route tile over an expert's odd last segment still runs N = 256 (the
// odd CTA's rows belong to no route of this tile); its epilogue stops at the tile's own rows.
// Small up-projections can load their activation rows straight from the routed rows (four-row
// TMA gathers from a one-row-box map): rows past the tile's real count repeat its first token.
//
// Last wave: when the tiles fill at least one wave of pairs, the r tiles of a last, partial wave
// are cut along the reduction into P = pairs / r pieces.  Each CTA of a piece stores its fp32
// accumulators in the workspace and takes a ticket for its half of the tile; the CTA holding the
// last ticket adds the P partial sums in piece order and applies the epilogue.
//
// Cross-CTA signals (all other barriers are local):
//   a_full    -- both CTAs' converter warps arrive on the even CTA's barrier;
//   b_full    -- the even CTA expects both halves' bytes; each CTA's TMA loads count their bytes
//                on the even CTA's barrier (.cta_group::2 form, no multicast);
//   op_empty, acc_full -- the MMA completion is committed to the barrier in both CTAs;
//   acc_empty -- both CTAs' epilogue warps arrive on the even CTA's barrier.
// A cluster barrier after set-up and before teardown keeps each CTA's shared memory and TMEM
// alive while the pair's MMAs can read them.  Every wait is bounded (2 s default): a CTA that
// gives up drains what it issued (1 s limit) and still reaches the teardown barrier.
#include "gemm_common.cuh"

namespace moe {

namespace {

constexpr int kThreads = 640;                  // 20 warps, the roles of the one-CTA kernel
constexpr int kWarpTmaA = 0, kWarpMma = 1, kWarpTmaB = 2, kWarpMma2 = 3;
constexpr int kWarpEpi0 = 4;
constexpr int kEpiWarps = 8;
constexpr int kWarpConv0 = 12;
constexpr int kConvWarps = 8;
constexpr int kBKT = 128;                      // reduction elements per weight box
constexpr int kPM = 2 * kBM;                   // features per pair tile (MMA M)
constexpr int kSmemBudget = 208 * 1024;

template <bool UP, int TN_>
struct Cfg2 {
    static constexpr int TN = TN_;                          // routes per tile (MMA N)
    static constexpr bool K2 = !UP && TN <= 64;             // two consecutive k-boxes per stage
    static constexpr int NB = UP || K2 ? 2 : 1;             // weight boxes per stage
    static constexpr int NACC = NB;                         // issuers / accumulators, one per box
    static constexpr int KSTAGE = K2 ? 2 * kBKT : kBKT;     // reduction elements per stage
    static constexpr int SEG = (!UP && TN == 256) ? 128 : TN;   // rows of a dispatch segment
    static constexpr int SEGS = TN / SEG;                   // segments per tile
    static constexpr int HALF = TN / 2;                     // route rows each CTA holds
    static constexpr int KP = kConvWarps / 4 / NB;          // converter warps per (quadrant, box)
    static constexpr int CH = (kBKT / 16) / KP;             // 16-byte chunks per converter thread and stage
    static constexpr int STG = NB * kBM * kBKT;             // int8 staging bytes per stage
    static constexpr int BBYTES = HALF * KSTAGE * 2;        // this CTA's bf16 activation bytes per stage
    static constexpr int ACC = NACC * TN;                   // accumulator columns
    static constexpr int A_COLS = NB * kBKT / 2;            // TMEM columns of one A stage
    static constexpr int S2 = cmin(4, (512 - ACC) / A_COLS);   // A (TMEM) + B (smem) ring
    static constexpr int S1 = cmin(12, (kSmemBudget - S2 * BBYTES) / STG);   // int8 staging ring
    static constexpr int A_BASE = ACC;
    static constexpr int TMEM_COLS = 512;
    static constexpr int OFF_STG = 0;
    static constexpr int OFF_B = OFF_STG + S1 * STG;
    static constexpr int OFF_BAR = OFF_B + S2 * BBYTES;
    // barriers: stg_full[S1] stg_empty[S1] a_full[S2] b_full[S2] op_empty[S2] acc_full acc_empty drain[2]
    static constexpr int NBAR = 2 * S1 + 3 * S2 + 2 + 2;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int MISC_BYTES = 16 + 3 * 4 * 40;
    static constexpr int SMEM = OFF_MISC + MISC_BYTES + 1024;
    static_assert(S1 >= 2 && S2 >= 2, "rings too shallow");
    static_assert(ACC + S2 * A_COLS <= TMEM_COLS, "TMEM has 512 columns");
    static_assert(SMEM <= 227 * 1024, "shared memory over the per-CTA limit");
    static_assert(KP >= 1 && CH * KP == kBKT / 16, "converter warps must split the 8 chunks of a row");
    static_assert(TN % 32 == 0 && TN <= 256, "pair MMA N is 32..256 in steps of 32");
    static_assert(HALF % 16 == 0 && (TN / 2) % 16 == 0, "epilogue chunks of 16 columns");
};

// kind::f16 instruction descriptor: D fp32, A and B bf16, both K-major, M = 256 (the pair)
template <int TN>
__device__ __forceinline__ constexpr uint32_t idesc_pair()
{
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(TN >> 3) << 17) |
           (static_cast<uint32_t>(kPM >> 4) << 24);
}

// bounded wait at cluster scope (arrivals of the peer CTA)
struct WaiterC {
    volatile uint32_t *abort;
    int *err;
    long long timeout_ns;

    __device__ __forceinline__ bool wait(uint32_t bar, uint32_t par, int site) const
    {
        if (mbar_try_wait_cluster(bar, par)) return true;
        const uint64_t t0 = global_timer_ns();
        while (true) {
            if (mbar_try_wait_cluster(bar, par)) return true;
            if (*abort) return false;
            if (static_cast<long long>(global_timer_ns() - t0) > timeout_ns) {
                *abort = 1u;
                atomicCAS(err, 0, kErrTimeoutBase + site);
                return false;
            }
        }
    }
};

__device__ __forceinline__ void wait_drain_cluster(uint32_t bar, uint32_t par)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait_cluster(bar, par))
        if (global_timer_ns() - t0 > 1000000000ull) return;
}

// four rows of a one-row-box tensor map (tma_gather4), completion counted on either CTA of the pair
__device__ __forceinline__ void tma_gather4_pair(uint32_t dst, const CUtensorMap *map, uint32_t bar_cluster,
                                                 int32_t x, int32_t r0, int32_t r1, int32_t r2, int32_t r3,
                                                 uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4, %5, %6, %7}], [%2], %8;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3),
        "l"(policy)
        : "memory");
}

// The tile epilogue on columns c .. c+15 of this CTA's accumulator row (TMEM lane = feature f).
// The packed operands are scaled (kActScale): sc0 and sc1 are the scales times the factor
// taking a sum to its value.
//   up-projection:   H[r, f] = bf16( gelu(sc0 * x0) * (sc1 * x1) ) for the tile's real rows,
//                    stored at kActScale times it;
//   down-projection: slot[s, t, j, f] = gate[t, j] * sc0 * (x0 + x1)   (k-box sums in box order)
template <bool UP, int NACC>
__device__ __forceinline__ void pair_epilogue_chunk(const GemmArgs &a, int row0, int nreal, int c, int f, int s,
                                                    float sc0, float sc1, const float (&x0)[16],
                                                    const float (&x1)[16])
{
    if constexpr (UP) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if (c + i < nreal)
                a.h[static_cast<size_t>(row0 + c + i) * a.M + f] =
                    __float2bfloat16_rn(gelu_tanh(sc0 * x0[i]) * (sc1 * x1[i]) * kActScale);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int route = __ldg(a.rperm + row0 + c + i);
            if (route >= 0) {
                const float v = NACC == 2 ? x0[i] + x1[i] : x0[i];
                const float g = __ldg(a.gate + route);
                const size_t o =
                    ((static_cast<size_t>(s) * a.T + (route >> 1)) * 2 + (route & 1)) * static_cast<size_t>(a.M) + f;
                a.slots[o] = g * (sc0 * v);
            }
        }
    }
}

// The CTA holding a split tile's last ticket: add the P pieces' partial sums of this thread's row
// (p0 = piece 0's row, pieces `pstride` floats apart) in piece order, then the tile epilogue.
template <bool UP, int TN, int NACC>
__device__ __noinline__ void pair_finish_pieces(const GemmArgs a, const float *p0, size_t pstride, int P, int c0,
                                                int c1, int row0, int nreal, int f, int s, float sc0, float sc1)
{
    for (int c = c0; c < c1; c += 16) {
        float x0[16], x1[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x0[i] = x1[i] = 0.f;
        for (int p = 0; p < P; ++p) {
            const float4 *r0 = reinterpret_cast<const float4 *>(p0 + p * pstride + c);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 u = __ldcg(r0 + i);
                x0[4 * i] += u.x; x0[4 * i + 1] += u.y; x0[4 * i + 2] += u.z; x0[4 * i + 3] += u.w;
            }
            if constexpr (NACC == 2) {
                const float4 *r1 = reinterpret_cast<const float4 *>(p0 + p * pstride + TN + c);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 u = __ldcg(r1 + i);
                    x1[4 * i] += u.x; x1[4 * i + 1] += u.y; x1[4 * i + 2] += u.z; x1[4 * i + 3] += u.w;
                }
            }
        }
        pair_epilogue_chunk<UP, NACC>(a, row0, nreal, c, f, s, sc0, sc1, x0, x1);
    }
}

// One converter thread's share of a stage in the per-block scale format: CH 16-byte chunks of
// its feature row (chunks j0 .. j0+CH-1, 128-byte swizzle: chunk j at (j ^ sw) * 16) loaded from
// the staging ring at src, each value turned into bf16(w * scale), stored to TMEM at taddr.
template <int CH>
__device__ __noinline__ void pair_convert_stage_kblock(uint32_t src, int j0, int sw, uint32_t taddr,
                                                       __nv_bfloat162 sc2)
{
    uint4 v[CH];
#pragma unroll
    for (int c = 0; c < CH; ++c) v[c] = lds128(src + (((j0 + c) ^ sw) << 4));
    __syncwarp();   // tcgen05.st is warp-collective (.sync.aligned): converge first
#pragma unroll
    for (int c = 0; c < CH; ++c) {
        uint32_t words[8];
        convert_chunk<true>(v[c], words, sc2);
        tmem_st8(taddr + c * 8, words);
    }
}

template <bool UP, int TN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                     const __grid_constant__ CUtensorMap tmB, const GemmArgs a)
{
    using C = Cfg2<UP, TN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t cta = cluster_ctarank();          // 0: issues the MMAs, 1: its peer
    const uint32_t pair = cluster_id_x(), npairs = num_clusters_x();

    auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * i; };
    auto stg_full = [&](int s) { return bar(s); };
    auto stg_empty = [&](int s) { return bar(C::S1 + s); };
    auto a_full = [&](int s) { return bar(2 * C::S1 + s); };
    auto b_full = [&](int s) { return bar(2 * C::S1 + C::S2 + s); };
    auto op_empty = [&](int s) { return bar(2 * C::S1 + 2 * C::S2 + s); };
    const uint32_t acc_full = bar(2 * C::S1 + 3 * C::S2);
    const uint32_t acc_empty = bar(2 * C::S1 + 3 * C::S2 + 1);
    const uint32_t drain_bar = bar(2 * C::S1 + 3 * C::S2 + 2);
    // the even CTA's copy of a barrier, as a shared::cluster address
    auto lead = [&](uint32_t b) { return mapa_shared(b, 0); };

    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile uint32_t *abort_flag = misc + 1;
    int *prefix = reinterpret_cast<int *>(misc + 4);
    int *poff = prefix + 40;
    int *roff = prefix + 80;
    const int m_tiles = a.M / kPM;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::S1; ++s) {
            mbar_init(stg_full(s), 1);
            mbar_init(stg_empty(s), kConvWarps);
        }
        for (int s = 0; s < C::S2; ++s) {
            mbar_init(a_full(s), 2 * kConvWarps);   // both CTAs' converters (used in the even CTA)
            mbar_init(b_full(s), 1);                // the even CTA's expect; both CTAs' bytes
            mbar_init(op_empty(s), C::NACC);        // one commit per issuer, sent to both CTAs
        }
        mbar_init(acc_full, C::NACC);
        mbar_init(acc_empty, 2 * kEpiWarps);        // both CTAs' epilogue warps (used in the even CTA)
        mbar_init(drain_bar, 1);
        mbar_init(drain_bar + 8, 1);
        *abort_flag = 0u;
        prefix[0] = 0;
        for (int e = 0; e <= a.E; ++e) poff[e] = a.poff[e];
        for (int e = 0; e <= a.E; ++e) roff[e] = a.offsets[e];
        for (int e = 0; e < a.E; ++e)
            prefix[e + 1] =
                prefix[e] + m_tiles * (((poff[e + 1] - poff[e]) / C::SEG + C::SEGS - 1) / C::SEGS) * a.splits;
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc_pair(smem_u32(misc), C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    if (warp == kWarpTmaA && lane == 0) {
        prefetch_tmap(&tmA0);
        if (UP) prefetch_tmap(&tmA1);
        prefetch_tmap(&tmB);
    }
    tc_fence_before();
    __syncthreads();
    __syncwarp();
    cluster_sync();   // both CTAs' barriers are initialised before any cross-CTA signal
    tc_fence_after();
    const uint32_t tmem_base = misc[0];
    const int total = prefix[a.E];
    const WorkList wl = a.part ? make_work_list(total, static_cast<int>(npairs), a.ksteps) : WorkList{total, 0, total};
    const WaiterC w{abort_flag, a.err, a.timeout_ns};
    const int SB = (UP ? 0 : 32) + (cta ? 16 : 0);   // first stats slot (instrumented builds)
    (void)SB;
    PS_NOW(t_start);

    if (warp == kWarpTmaA) {
        // ---- this CTA's int8 weight tiles [128 f x 128 k] -> staging ring ---------------------
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            uint32_t st = 0, ph = 0, issued = 0, par = 0;
            PS_VAR(c_wait);
            for (int item = pair; item < wl.items && !*abort_flag; item += npairs) {
                const WorkItem wi = work_item(wl, item, a.ksteps);
                int e, m, n, s;
                decode_tile<C::SEG>(wi.tile, prefix, poff, m_tiles, a.splits, e, m, n, s, C::SEGS);
                const int y = e * a.M + m * kPM + static_cast<int>(cta) * kBM;
                const int kb = s * a.ksteps;
                for (int ks = wi.k0; ks < wi.k1; ++ks) {
                    PS_NOW(t0);
                    if (!w.wait(stg_empty(st), ph ^ 1u, 1)) goto a_done;
                    PS_ADD(c_wait, t0);
                    mbar_arrive_expect_tx(stg_full(st), C::STG);
                    const uint32_t dst = sbase + C::OFF_STG + st * C::STG;
#pragma unroll
                    for (int bx = 0; bx < C::NB; ++bx)
                        tma_load_2d(dst + bx * kBM * kBKT, (UP && bx == 1) ? &tmA1 : &tmA0, stg_full(st),
                                    (kb + ks) * C::KSTAGE + (UP ? 0 : bx * kBKT), y, pol);
                    issued |= 1u << st;
                    par = (par & ~(1u << st)) | (ph << st);
                    if (++st == C::S1) { st = 0; ph ^= 1u; }
                }
            }
        a_done:
            for (int s = 0; s < C::S1; ++s)
                if (issued & (1u << s)) wait_drain(stg_full(s), (par >> s) & 1u);
            PS_FLUSH(SB + 1, c_wait);
        }
        __syncwarp();
    } else if (warp == kWarpTmaB) {
        // ---- this CTA's half of the activation tile: HALF rows x KSTAGE k (64-wide boxes) ------
        // gathered: tmB covers the routed rows [T, K] with one-row boxes; the CTA's rows are tile
        // rows c HALF .. c HALF + HALF - 1, four per lane 0 .. HALF/4 - 1 (tokens rperm >> 1; rows
        // past the tile's real count repeat its first token)
        const bool gather = UP && a.gather;
        const uint64_t pol = l2_policy_evict_last();
        uint32_t st = 0, ph = 0, issued = 0, par = 0;
        bool ok = true;
        PS_VAR(c_bwait);
        for (int item = pair; ok && item < wl.items; item += npairs) {
            if (__shfl_sync(0xffffffffu, lane == 0 ? static_cast<int>(*abort_flag) : 0, 0)) break;
            const WorkItem wi = work_item(wl, item, a.ksteps);
            int e, m, n, s;
            decode_tile<C::SEG>(wi.tile, prefix, poff, m_tiles, a.splits, e, m, n, s, C::SEGS);
            const int row0 = poff[e] + n * C::TN;
            const int row = row0 + static_cast<int>(cta) * C::HALF;
            const int kb = s * a.ksteps;
            int g[4] = {0, 0, 0, 0};
            if (gather) {
                const int nreal = min(C::TN, roff[e + 1] - roff[e] - n * C::TN);
                const int tok0 = __ldg(a.rperm + row0) >> 1;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = static_cast<int>(cta) * C::HALF + 4 * lane + i;   // row within the tile
                    g[i] = (4 * lane + i < C::HALF && r < nreal) ? (__ldg(a.rperm + row0 + r) >> 1) : tok0;
                }
            }
            for (int ks = wi.k0; ks < wi.k1; ++ks) {
                PS_NOW(t0);
                if (lane == 0) ok = w.wait(op_empty(st), ph ^ 1u, 2);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                PS_ADD(c_bwait, t0);
                if (!ok) break;
                if (lane == 0 && cta == 0) mbar_arrive_expect_tx(b_full(st), 2 * C::BBYTES);
                __syncwarp();
                const uint32_t dst = sbase + C::OFF_B + st * C::BBYTES;
                const uint32_t fb = lead(b_full(st));
                const int x = (kb + ks) * C::KSTAGE;
                if (gather) {
                    if (lane < C::HALF / 4) {
#pragma unroll
                        for (int j = 0; j < C::KSTAGE / 64; ++j)
                            tma_gather4_pair(dst + j * C::HALF * 128 + lane * 4 * 128, &tmB, fb, x + 64 * j, g[0],
                                             g[1], g[2], g[3], pol);
                    }
                } else if (lane == 0) {
#pragma unroll
                    for (int j = 0; j < C::KSTAGE / 64; ++j)
                        tma_load_2d_pair(dst + j * C::HALF * 128, &tmB, fb, x + 64 * j, row, pol);
                }
                issued |= 1u << st;
                par = (par & ~(1u << st)) | (ph << st);
                if (++st == C::S2) { st = 0; ph ^= 1u; }
            }
        }
        // every copy issued has landed before the CTA may exit: the even CTA sees both halves
        // on its b_full; the odd one sees its stage released by the MMAs that read it
        if (lane == 0)
            for (int s = 0; s < C::S2; ++s)
                if (issued & (1u << s)) {
                    if (cta == 0)
                        wait_drain_cluster(b_full(s), (par >> s) & 1u);
                    else
                        wait_drain_cluster(op_empty(s), (par >> s) & 1u);
                }
        if (lane == 0) PS_FLUSH(SB + 2, c_bwait);
        __syncwarp();
    } else if (warp == kWarpMma || (C::NACC == 2 && warp == kWarpMma2)) {
        // ---- tensor-core issue (even CTA): issuer i, box i, accumulator i ---------------------
        const int mine = warp == kWarpMma ? 0 : 1;
        if (cta == 0 && lane == 0) {
            uint32_t st = 0, ph = 0;
            int it = 0;
            bool issued_any = false;
            PS_VAR(c_acc);
            PS_VAR(c_a);
            PS_VAR(c_b);
            PS_VAR(c_issue);
            for (int item = pair; item < wl.items; item += npairs, ++it) {
                const WorkItem wi = work_item(wl, item, a.ksteps);
                PS_NOW(t0);
                if (!w.wait(acc_empty, (it & 1) ^ 1u, 3)) break;
                PS_ADD(c_acc, t0);
                tc_fence_after();
                const uint32_t dcol = tmem_base + mine * C::TN;
                bool ok = true;
                for (int ks = wi.k0; ks < wi.k1; ++ks) {
                    PS_NOW(t1);
                    if (!w.wait(a_full(st), ph, 4)) { ok = false; break; }
                    PS_ADD(c_a, t1);
                    PS_NOW(t2);
                    if (!w.wait(b_full(st), ph, 5)) { ok = false; break; }
                    PS_ADD(c_b, t2);
                    PS_NOW(t3);
                    tc_fence_after();
                    const uint32_t acol = tmem_base + C::A_BASE + st * C::A_COLS + mine * (kBKT / 2);
                    const uint32_t blo = desc_sw128_lo(sbase + C::OFF_B + st * C::BBYTES, 16);
#pragma unroll
                    for (int kk = 0; kk < kBKT / 16; ++kk) {
                        // K slice of the stage's activation tile: both matrices of the up-projection
                        // use the same slices, the k-boxes of the down-projection consecutive ones
                        const int kg = (UP ? 0 : mine * (kBKT / 16)) + kk;
                        const uint64_t bdesc = desc_join(
                            blo + (((kg >> 2) * (C::HALF * 128) + (kg & 3) * 32) >> 4), desc_sw128_hi(1024));
                        umma_bf16_ts_pair(dcol, acol + kk * 8, bdesc, idesc_pair<TN>(), ((ks - wi.k0) | kk) != 0);
                    }
                    issued_any = true;
                    umma_commit_pair_mc(op_empty(st), 0x3);
                    PS_ADD(c_issue, t3);
                    if (++st == C::S2) { st = 0; ph ^= 1u; }
                }
                if (!ok) break;
                umma_commit_pair_mc(acc_full, 0x3);
            }
            if (issued_any) {
                umma_commit_pair(drain_bar + 8 * mine);   // all MMAs this thread issued have completed after this
                wait_drain_cluster(drain_bar + 8 * mine, 0);
            }
            PS_FLUSH(SB + 3, c_acc);
            PS_FLUSH(SB + 4, c_a);
            PS_FLUSH(SB + 5, c_b);
            PS_FLUSH(SB + 6, c_issue);
        }
        __syncwarp();
    } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + kEpiWarps) {
        // ---- epilogue: this CTA's 128 features x TN routes ------------------------------------
        // warp (q, hc): TMEM lane quadrant q = warp % 4, column half hc of the tile
        const int q = warp & 3;
        const int hc = (warp - kWarpEpi0) >> 2;
        const int c0 = hc * (TN / 2);
        const uint32_t empty_lead = lead(acc_empty);
        volatile uint32_t *last_flag = misc + 2;
        auto epilogue_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory"); };
        int it = 0;
        PS_VAR(c_ewait);
        PS_VAR(c_ework);
        for (int item = pair; item < wl.items; item += npairs, ++it) {
            const WorkItem wi = work_item(wl, item, a.ksteps);
            int e, m, n, s;
            decode_tile<C::SEG>(wi.tile, prefix, poff, m_tiles, a.splits, e, m, n, s, C::SEGS);
            PS_NOW(t0);
            w.wait(acc_full, it & 1, 6);   // a wait that gives up sets the CTA's abort flag
            // one decision for all epilogue warps: a piece's epilogue meets at a named barrier,
            // so no warp may leave the loop while the others go on
            epilogue_sync();
            if (*abort_flag) break;
            PS_ADD(c_ewait, t0);
            PS_NOW(t1);
            tc_fence_after();
            const int f = m * kPM + static_cast<int>(cta) * kBM + q * 32 + lane;
            const uint32_t tl = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
            const int row0 = poff[e] + n * C::TN;
            const int nreal = roff[e + 1] - roff[e] - n * C::TN;   // real rows of this tile (may exceed TN)
            // the tile's own rows: a 256-route tile over an expert's odd last segment fills 128 columns
            const int c1 = max(c0, min(c0 + TN / 2, poff[e + 1] - row0));
            // the scales times the factor taking a sum of scaled operands to its value (exact while
            // |s| < 2^59); the per-block format applied its scales while dequantising
            const float sc0 = (a.kblock ? 1.f : __bfloat162float(a.s0[static_cast<size_t>(e) * a.M + f])) * a.accf;
            const float sc1 =
                !UP ? 0.f : (a.kblock ? 1.f : __bfloat162float(a.s1[static_cast<size_t>(e) * a.M + f])) * a.accf;
            const bool whole = wi.piece < 0;   // uniform over the pair
            if (!whole) {
                // a piece: this CTA's partial sums go to the workspace, [piece][cta][row][column]
                float *pp = a.part + ((static_cast<size_t>(wi.piece) * 2 + cta) * kBM + q * 32 + lane) * C::ACC;
#pragma unroll 1
                for (int c = c0; c < c1; c += 16) {
                    float x0[16], x1[16];
                    __syncwarp();   // tcgen05.ld is warp-collective (.sync.aligned): converge first
                    tmem_ld16(tl + c, x0);
                    if constexpr (C::NACC == 2) tmem_ld16(tl + TN + c, x1);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; i += 4) {
                        *reinterpret_cast<float4 *>(pp + c + i) = make_float4(x0[i], x0[i + 1], x0[i + 2], x0[i + 3]);
                        if constexpr (C::NACC == 2)
                            *reinterpret_cast<float4 *>(pp + TN + c + i) =
                                make_float4(x1[i], x1[i + 1], x1[i + 2], x1[i + 3]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(empty_lead);   // the accumulator is no longer needed
                __threadfence();                                   // partial sums before the ticket
                epilogue_sync();
                if (warp == kWarpEpi0 && lane == 0) {
                    unsigned int *tk = a.tickets + (wi.tile - wl.whole) * 2 + cta;
                    const bool last = atomicAdd(tk, 1u) == static_cast<unsigned int>(wl.P - 1);
                    if (last) *tk = 0u;                            // every piece of this half has arrived
                    *last_flag = last ? 1u : 0u;
                }
                epilogue_sync();
                if (*last_flag) {
                    __threadfence();   // the other pieces' sums, visible after their tickets
                    // the tile's pieces are consecutive: piece (tile - whole) * P + p, this CTA's half
                    const size_t pstride = 2 * static_cast<size_t>(kBM) * C::ACC;
                    const float *p0 = a.part + ((static_cast<size_t>(wi.tile - wl.whole) * wl.P * 2 + cta) * kBM +
                                                q * 32 + lane) * C::ACC;
                    pair_finish_pieces<UP, TN, C::NACC>(a, p0, pstride, wl.P, c0, c1, row0, nreal, f, s, sc0, sc1);
                }
            } else {
#pragma unroll 1
                for (int c = c0; c < c1; c += 16) {
                    float x0[16], x1[16];
                    __syncwarp();   // tcgen05.ld is warp-collective (.sync.aligned): converge first
                    tmem_ld16(tl + c, x0);
                    if constexpr (C::NACC == 2) tmem_ld16(tl + TN + c, x1);
                    tmem_wait_ld();
                    pair_epilogue_chunk<UP, C::NACC>(a, row0, nreal, c, f, s, sc0, sc1, x0, x1);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(empty_lead);
            }
            PS_ADD(c_ework, t1);
        }
        if (lane == 0) {
            PS_FLUSH(SB + 7, c_ewait);
            PS_FLUSH(SB + 8, c_ework);
        }
    } else if (warp >= kWarpConv0) {
        // ---- this CTA's int8 staging -> bf16 A operand in its TMEM -----------------------------
        const int cw = warp - kWarpConv0;
        const int q = warp & 3;
        const int part = cw >> 2;
        const int box = part / C::KP;
        const int j0 = (part % C::KP) * C::CH;
        const int fr = q * 32 + lane;
        const uint32_t src_row = box * kBM * kBKT + fr * 128;
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        uint32_t st = 0, ph = 0, st2 = 0, ph2 = 0;
        PS_VAR(c_cwait);
        PS_VAR(c_cwork);
        PS_VAR(c_cst);
        PS_VAR(c_ctail);
        for (int item = pair; item < wl.items; item += npairs) {
            const WorkItem wi = work_item(wl, item, a.ksteps);
            // per-block scale format: this thread's feature row in the scale rows of its box; the
            // scale row of a box is its first reduction row / kScaleBlock
            const __nv_bfloat16 *srow = nullptr;
            if (a.kblock) {
                int e, m, n, s;
                decode_tile<C::SEG>(wi.tile, prefix, poff, m_tiles, a.splits, e, m, n, s, C::SEGS);
                const int k0 = s * a.ksteps * C::KSTAGE + (UP ? 0 : box * kBKT);
                srow = ((UP && box == 1) ? a.s1 : a.s0) +
                       (static_cast<size_t>(e) * (a.K / kScaleBlock) + k0 / kScaleBlock) * a.M + m * kPM +
                       static_cast<int>(cta) * kBM + fr;
            }
            bool ok = true;
            for (int ks = wi.k0; ks < wi.k1; ++ks) {
                PS_NOW(t0);
                ok = __all_sync(0xffffffffu, w.wait(stg_full(st), ph, 7) && w.wait(op_empty(st2), ph2 ^ 1u, 8));
                if (!ok) break;
                PS_ADD(c_cwait, t0);
                PS_NOW(t1);
                tc_fence_after();
                const uint32_t src = sbase + C::OFF_STG + st * C::STG + src_row;
                const uint32_t taddr = tmem_base + lane_base + C::A_BASE + st2 * C::A_COLS + box * (kBKT / 2) + j0 * 8;
                if (a.kblock) {
                    // per-block scale format, out of line (keeps the register pressure of the loop below)
                    const __nv_bfloat16 sv = srow[static_cast<size_t>(ks) * (C::KSTAGE / kScaleBlock) * a.M];
                    pair_convert_stage_kblock<C::CH>(src, j0, fr & 7, taddr, __halves2bfloat162(sv, sv));
                } else {
                    uint4 v[C::CH];
#pragma unroll
                    for (int c = 0; c < C::CH; ++c) v[c] = lds128(src + (((j0 + c) ^ (fr & 7)) << 4));
                    __syncwarp();   // tcgen05.st is warp-collective (.sync.aligned): converge first
#pragma unroll
                    for (int c = 0; c < C::CH; ++c) {
                        uint32_t words[8];
                        convert_chunk<false>(v[c], words, __nv_bfloat162{});
                        tmem_st8(taddr + c * 8, words);
                    }
                }
                PS_ADD(c_cwork, t1);
                PS_NOW(t2);
                tmem_wait_st();
                PS_ADD(c_cst, t2);
                PS_NOW(t3);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(stg_empty(st));
                    mbar_arrive_cluster(lead(a_full(st2)));
                }
                PS_ADD(c_ctail, t3);
                if (++st == C::S1) { st = 0; ph ^= 1u; }
                if (++st2 == C::S2) { st2 = 0; ph2 ^= 1u; }
            }
            if (!ok) break;
        }
        if (lane == 0) {
            PS_FLUSH(SB + 9, c_cwait);
            PS_FLUSH(SB + 10, c_cwork);
            PS_FLUSH(SB + 11, c_cst);
            PS_FLUSH(SB + 12, c_ctail);
        }
    }

    tc_fence_before();
    __syncthreads();
    __syncwarp();
    cluster_sync();   // the pair's MMAs have completed (the even CTA drained them) before any teardown
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
#ifdef MOE_PIPE_STATS
    if (threadIdx.x == 0) PS_FLUSH(SB + 0, clock64() - t_start);
#endif
}

cudaLaunchConfig_t pair_config(int grid, size_t smem, cudaStream_t s, cudaLaunchAttribute *attr)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    attr->id = cudaLaunchAttributeClusterDimension;
    attr->val.clusterDim.x = 2;
    attr->val.clusterDim.y = 1;
    attr->val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

// CTAs of a full wave of pairs of one kernel (0 if pairs cannot be launched); the same for every
// launch in the process (one device)
template <bool UP, int TN>
int pair_grid(int num_sms)
{
    static int grid = -1;
    if (grid < 0) {
        if (cudaFuncSetAttribute(gemm_pair_kernel<UP, TN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg2<UP, TN>::SMEM) != cudaSuccess) {
            cudaGetLastError();
            grid = 0;
            return 0;
        }
        cudaLaunchAttribute attr;
        cudaLaunchConfig_t cfg = pair_config(2 * (num_sms / 2), Cfg2<UP, TN>::SMEM, nullptr, &attr);
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, gemm_pair_kernel<UP, TN>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            clusters = 0;
        }
        grid = 2 * clusters;
    }
    return grid;
}

template <bool UP, int TN>
cudaError_t launch_pair(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &b, const GemmArgs &args,
                        cudaStream_t s, int num_sms)
{
    const int grid = pair_grid<UP, TN>(num_sms);
    if (grid < 2 || grid % 2 || args.M % kPM) return cudaErrorInvalidValue;
    cudaLaunchAttribute attr;
    cudaLaunchConfig_t cfg = pair_config(grid, Cfg2<UP, TN>::SMEM, s, &attr);
    return cudaLaunchKernelEx(&cfg, gemm_pair_kernel<UP, TN>, a0, a1, b, args);
}

}  // namespace

int gemm_pair_tn(bool up, int bn) { return bn == 32 ? 32 : bn == 128 ? (up ? 128 : 256) : 0; }

// CTAs of a full wave of the pair kernel for (up, bn), 0 if there is none
int gemm_pair_grid(bool up, int bn, int num_sms)
{
    switch (gemm_pair_tn(up, bn)) {
    case 32: return up ? pair_grid<true, 32>(num_sms) : pair_grid<false, 32>(num_sms);
    case 128: return pair_grid<true, 128>(num_sms);
    case 256: return pair_grid<false, 256>(num_sms);
    default: return 0;
    }
}

bool gemm_pair_ready(bool up, int bn, int num_sms) { return gemm_pair_grid(up, bn, num_sms) >= 2; }

cudaError_t launch_gemm_up_pair(int bn, const CUtensorMap &wl, const CUtensorMap &wv, const CUtensorMap &xp,
                                const GemmArgs &a, int num_sms, cudaStream_t s)
{
    switch (bn) {
    case 32: return launch_pair<true, 32>(wl, wv, xp, a, s, num_sms);
    case 128: return launch_pair<true, 128>(wl, wv, xp, a, s, num_sms);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_gemm_down_pair(int bn, const CUtensorMap &w1, const CUtensorMap &h, const GemmArgs &a, int num_sms,
                                  cudaStream_t s)
{
    switch (bn) {
    case 32: return launch_pair<false, 32>(w1, w1, h, a, s, num_sms);
    case 128: return launch_pair<false, 256>(w1, w1, h, a, s, num_sms);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe

#ifdef MOE_PIPE_STATS
extern "C" __attribute__((visibility("default"))) int moe_debug_pipe_stats_pair(unsigned long long *out, int reset)
{
    if (cudaMemcpyFromSymbol(out, moe::g_pipe_stats, sizeof(unsigned long long) * 64) != cudaSuccess) return -4;
    if (reset) {
        unsigned long long z[64] = {};
        if (cudaMemcpyToSymbol(moe::g_pipe_stats, z, sizeof z) != cudaSuccess) return -4;
    }
    return 0;
}

extern "C" __attribute__((visibility("default"))) int moe_debug_pair_grid(int up, int bn, int num_sms)
{
    return moe::gemm_pair_grid(up != 0, bn, num_sms);
}
#endif
