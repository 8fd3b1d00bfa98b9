// gemm_ts2.cu -- the grouped expert GEMMs of large batches (128-route tiles, packed weights) on
// CTA pairs: one tcgen05 MMA of M = 256 output features spans the two SMs of a two-CTA cluster.
// It computes the expert MLP of "Grok-1 Admin & Architecture Guide", section 3, "Mixture of
// Experts (MoELayer + Router)" step 3, linear_1(gelu(linear(x)) * linear_v(x)), with the 8-bit
// weights of section 3 "Quantized weights", and the gate-weighted scatter of step 4.
//
// Why pairs.  In the one-CTA kernel (gemm_ts.cu) a stage of 128 reduction elements moves
// 160 KB through one SM's shared memory against 1024 MMA cycles (the int8 weight boxes in and
// out again to the converters, the activation tile in, and read by every MMA), above the
// ~128 B/clk shared memory delivers.  On a pair the activation tile is split: each CTA loads
// and serves half of the routes' rows, and every MMA reads both halves, so a CTA moves
// 112 KB (up-projection) or 96 KB (down-projection) per stage.
//
// Tiles.  Expert e, features [256 m, 256 m + 256), TN route rows from row0:
//   up-projection   TN = 128, both matrices (linear, linear_v), two issuers and accumulators;
//   down-projection TN = 256 (two consecutive 128-row segments of the expert), one matrix,
//                   optionally a K-split s of the reduction.
// CTA c of the pair converts the int8 weights of features 256 m + 128 c .. + 127 into its own
// TMEM (its half of the MMA's A operand) and loads route rows row0 + c TN/2 .. + TN/2 - 1 into
// its shared memory (its half of B).  The even CTA issues the MMAs; each CTA's accumulators hold
// its 128 features x TN routes, and each CTA's epilogue writes its features: H for the
// up-projection (gelu(s_lin A0) * (s_v A1)), gate * s_1 * A0 into the route's slot for the
// down-projection.  A down tile over an expert's odd last segment still runs N = 256 (the odd
// CTA's rows belong to no route of this tile); its epilogue stops at the tile's own rows.
//
// Cross-CTA signals (all other barriers are local):
//   a_full    -- both CTAs' converter warps arrive on the even CTA's barrier;
//   b_full    -- the even CTA expects both halves' bytes; each CTA's TMA load counts its bytes
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
constexpr int kBKT = 128;                      // reduction elements per stage
constexpr int kPM = 2 * kBM;                   // features per pair tile (MMA M)
constexpr int kSmemBudget = 208 * 1024;

template <bool UP>
struct Cfg2 {
    static constexpr int NB = UP ? 2 : 1;                   // weight boxes per stage (matrices)
    static constexpr int NACC = NB;                         // issuers / accumulators
    static constexpr int TN = UP ? 128 : 256;               // routes per tile (MMA N)
    static constexpr int SEGS = TN / 128;                   // 128-row segments per tile
    static constexpr int HALF = TN / 2;                     // route rows each CTA holds
    static constexpr int KP = kConvWarps / 4 / NB;          // converter warps per (quadrant, box)
    static constexpr int CH = (kBKT / 16) / KP;             // 16-byte chunks per converter thread and stage
    static constexpr int STG = NB * kBM * kBKT;             // int8 staging bytes per stage
    static constexpr int BBYTES = HALF * kBKT * 2;          // this CTA's bf16 activation bytes per stage
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

template <bool UP>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                     const __grid_constant__ CUtensorMap tmB, const GemmArgs a)
{
    using C = Cfg2<UP>;
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
            prefix[e + 1] = prefix[e] + m_tiles * (((poff[e + 1] - poff[e]) / kBM + C::SEGS - 1) / C::SEGS) * a.splits;
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
    const WaiterC w{abort_flag, a.err, a.timeout_ns};

    if (warp == kWarpTmaA) {
        // ---- this CTA's int8 weight tiles [128 f x 128 k] (one per matrix) -> staging ring ---
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            uint32_t st = 0, ph = 0, issued = 0, par = 0;
            for (int tile = pair; tile < total && !*abort_flag; tile += npairs) {
                int e, m, n, s;
                decode_tile<kBM>(tile, prefix, poff, m_tiles, a.splits, e, m, n, s, C::SEGS);
                const int y = e * a.M + m * kPM + static_cast<int>(cta) * kBM;
                const int k0 = s * a.ksteps;
                for (int ks = 0; ks < a.ksteps; ++ks) {
                    if (!w.wait(stg_empty(st), ph ^ 1u, 1)) goto a_done;
                    mbar_arrive_expect_tx(stg_full(st), C::STG);
                    const uint32_t dst = sbase + C::OFF_STG + st * C::STG;
                    tma_load_2d(dst, &tmA0, stg_full(st), (k0 + ks) * kBKT, y, pol);
                    if (UP) tma_load_2d(dst + kBM * kBKT, &tmA1, stg_full(st), (k0 + ks) * kBKT, y, pol);
                    issued |= 1u << st;
                    par = (par & ~(1u << st)) | (ph << st);
                    if (++st == C::S1) { st = 0; ph ^= 1u; }
                }
            }
        a_done:
            for (int s = 0; s < C::S1; ++s)
                if (issued & (1u << s)) wait_drain(stg_full(s), (par >> s) & 1u);
        }
        __syncwarp();
    } else if (warp == kWarpTmaB) {
        // ---- this CTA's half of the activation tile: TN/2 rows x 128 k (two 64-wide boxes) ----
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_last();
            uint32_t st = 0, ph = 0, issued = 0, par = 0;
            for (int tile = pair; tile < total && !*abort_flag; tile += npairs) {
                int e, m, n, s;
                decode_tile<kBM>(tile, prefix, poff, m_tiles, a.splits, e, m, n, s, C::SEGS);
                const int row = poff[e] + n * C::TN + static_cast<int>(cta) * C::HALF;
                const int k0 = s * a.ksteps;
                for (int ks = 0; ks < a.ksteps; ++ks) {
                    if (!w.wait(op_empty(st), ph ^ 1u, 2)) goto b_done;
                    if (cta == 0) mbar_arrive_expect_tx(b_full(st), 2 * C::BBYTES);
                    const uint32_t dst = sbase + C::OFF_B + st * C::BBYTES;
                    const uint32_t fb = lead(b_full(st));
                    tma_load_2d_pair(dst, &tmB, fb, (k0 + ks) * kBKT, row, pol);
                    tma_load_2d_pair(dst + C::HALF * 128, &tmB, fb, (k0 + ks) * kBKT + 64, row, pol);
                    issued |= 1u << st;
                    par = (par & ~(1u << st)) | (ph << st);
                    if (++st == C::S2) { st = 0; ph ^= 1u; }
                }
            }
        b_done:
            // every copy issued has landed before the CTA may exit: the even CTA sees both halves
            // on its b_full; the odd one sees its stage released by the MMAs that read it
            for (int s = 0; s < C::S2; ++s)
                if (issued & (1u << s)) {
                    if (cta == 0)
                        wait_drain_cluster(b_full(s), (par >> s) & 1u);
                    else
                        wait_drain_cluster(op_empty(s), (par >> s) & 1u);
                }
        }
        __syncwarp();
    } else if (warp == kWarpMma || (UP && warp == kWarpMma2)) {
        // ---- tensor-core issue (even CTA): issuer i, matrix i, accumulator i ------------------
        const int mine = warp == kWarpMma ? 0 : 1;
        if (cta == 0 && lane == 0) {
            uint32_t st = 0, ph = 0;
            int it = 0;
            bool issued_any = false;
            for (int tile = pair; tile < total; tile += npairs, ++it) {
                if (!w.wait(acc_empty, (it & 1) ^ 1u, 3)) break;
                tc_fence_after();
                const uint32_t dcol = tmem_base + mine * C::TN;
                bool ok = true;
                for (int ks = 0; ks < a.ksteps; ++ks) {
                    if (!w.wait(a_full(st), ph, 4)) { ok = false; break; }
                    if (!w.wait(b_full(st), ph, 5)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t acol = tmem_base + C::A_BASE + st * C::A_COLS + mine * (kBKT / 2);
                    const uint32_t bbase = sbase + C::OFF_B + st * C::BBYTES;
#pragma unroll
                    for (int kk = 0; kk < kBKT / 16; ++kk) {
                        const uint64_t bdesc =
                            desc_sw128(bbase + (kk >> 2) * (C::HALF * 128) + (kk & 3) * 32, 16, 1024);
                        umma_bf16_ts_pair(dcol, acol + kk * 8, bdesc, idesc_pair<C::TN>(), (ks | kk) != 0);
                    }
                    issued_any = true;
                    umma_commit_pair_mc(op_empty(st), 0x3);
                    if (++st == C::S2) { st = 0; ph ^= 1u; }
                }
                if (!ok) break;
                umma_commit_pair_mc(acc_full, 0x3);
            }
            if (issued_any) {
                umma_commit_pair(drain_bar + 8 * mine);   // all MMAs this thread issued have completed after this
                wait_drain_cluster(drain_bar + 8 * mine, 0);
            }
        }
        __syncwarp();
    } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + kEpiWarps) {
        // ---- epilogue: this CTA's 128 features x TN routes ------------------------------------
        const int q = warp & 3;
        const int hc = (warp - kWarpEpi0) >> 2;
        const uint32_t empty_lead = lead(acc_empty);
        int it = 0;
        for (int tile = pair; tile < total; tile += npairs, ++it) {
            int e, m, n, s;
            decode_tile<kBM>(tile, prefix, poff, m_tiles, a.splits, e, m, n, s, C::SEGS);
            const bool ok = __all_sync(0xffffffffu, w.wait(acc_full, it & 1, 6));
            if (!ok) break;
            tc_fence_after();
            const int f = m * kPM + static_cast<int>(cta) * kBM + q * 32 + lane;
            const uint32_t tl = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
            const int row0 = poff[e] + n * C::TN;
            const int c0 = hc * (C::TN / 2);
            const float sc0 = a.kblock ? 1.f : __bfloat162float(a.s0[static_cast<size_t>(e) * a.M + f]);
            if constexpr (UP) {
                const int nreal = roff[e + 1] - roff[e] - n * C::TN;   // real rows of this tile (may exceed TN)
                const float sc1 = a.kblock ? 1.f : __bfloat162float(a.s1[static_cast<size_t>(e) * a.M + f]);
#pragma unroll 1
                for (int c = c0; c < c0 + C::TN / 2; c += 16) {
                    float x0[16], x1[16];
                    __syncwarp();   // tcgen05.ld is warp-collective (.sync.aligned): converge first
                    tmem_ld16(tl + c, x0);
                    tmem_ld16(tl + C::TN + c, x1);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        if (c + i < nreal)
                            a.h[static_cast<size_t>(row0 + c + i) * a.M + f] =
                                __float2bfloat16_rn(gelu_tanh(sc0 * x0[i]) * (sc1 * x1[i]));
                    }
                }
            } else {
                // the tile's own rows: an expert's odd last segment fills only the first 128 columns
                const int c1 = max(c0, min(c0 + C::TN / 2, poff[e + 1] - row0));
#pragma unroll 1
                for (int c = c0; c < c1; c += 16) {
                    float x0[16];
                    __syncwarp();
                    tmem_ld16(tl + c, x0);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int route = __ldg(a.rperm + row0 + c + i);
                        if (route >= 0) {
                            const float g = __ldg(a.gate + route);
                            const size_t o = ((static_cast<size_t>(s) * a.T + (route >> 1)) * 2 + (route & 1)) *
                                                 static_cast<size_t>(a.M) + f;
                            a.slots[o] = g * (sc0 * x0[i]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(empty_lead);
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
        for (int tile = pair; tile < total; tile += npairs) {
            const __nv_bfloat16 *srow = nullptr;
            if (a.kblock) {
                int e, m, n, s;
                decode_tile<kBM>(tile, prefix, poff, m_tiles, a.splits, e, m, n, s, C::SEGS);
                srow = ((UP && box == 1) ? a.s1 : a.s0) +
                       (static_cast<size_t>(e) * (a.K / kScaleBlock) + s * a.ksteps) * a.M + m * kPM +
                       static_cast<int>(cta) * kBM + fr;
            }
            bool ok = true;
            for (int ks = 0; ks < a.ksteps; ++ks) {
                ok = __all_sync(0xffffffffu, w.wait(stg_full(st), ph, 7) && w.wait(op_empty(st2), ph2 ^ 1u, 8));
                if (!ok) break;
                tc_fence_after();
                const uint32_t src = sbase + C::OFF_STG + st * C::STG + src_row;
                uint4 v[C::CH];
#pragma unroll
                for (int c = 0; c < C::CH; ++c) v[c] = lds128(src + (((j0 + c) ^ (fr & 7)) << 4));
                __nv_bfloat162 sc2;
                if (a.kblock) {   // one scale row per stage (128 reduction rows)
                    const __nv_bfloat16 sv = srow[static_cast<size_t>(ks) * a.M];
                    sc2 = __halves2bfloat162(sv, sv);
                }
                const uint32_t taddr = tmem_base + lane_base + C::A_BASE + st2 * C::A_COLS + box * (kBKT / 2) + j0 * 8;
                __syncwarp();   // tcgen05.st is warp-collective (.sync.aligned): converge first
#pragma unroll
                for (int c = 0; c < C::CH; ++c) {
                    uint32_t words[8];
                    words[0] = i8x2_to_bf16x2(v[c].x, 0x4140);
                    words[1] = i8x2_to_bf16x2(v[c].x, 0x4342);
                    words[2] = i8x2_to_bf16x2(v[c].y, 0x4140);
                    words[3] = i8x2_to_bf16x2(v[c].y, 0x4342);
                    words[4] = i8x2_to_bf16x2(v[c].z, 0x4140);
                    words[5] = i8x2_to_bf16x2(v[c].z, 0x4342);
                    words[6] = i8x2_to_bf16x2(v[c].w, 0x4140);
                    words[7] = i8x2_to_bf16x2(v[c].w, 0x4342);
                    if (a.kblock) {
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            __nv_bfloat162 wq = *reinterpret_cast<const __nv_bfloat162 *>(&words[k]);
                            wq = __hmul2(wq, sc2);
                            words[k] = *reinterpret_cast<const uint32_t *>(&wq);
                        }
                    }
                    tmem_st8(taddr + c * 8, words);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(stg_empty(st));
                    mbar_arrive_cluster(lead(a_full(st2)));
                }
                if (++st == C::S1) { st = 0; ph ^= 1u; }
                if (++st2 == C::S2) { st2 = 0; ph2 ^= 1u; }
            }
            if (!ok) break;
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
template <bool UP>
int pair_grid(int num_sms)
{
    static int grid = -1;
    if (grid < 0) {
        if (cudaFuncSetAttribute(gemm_pair_kernel<UP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg2<UP>::SMEM) != cudaSuccess) {
            cudaGetLastError();
            grid = 0;
            return 0;
        }
        cudaLaunchAttribute attr;
        cudaLaunchConfig_t cfg = pair_config(2 * (num_sms / 2), Cfg2<UP>::SMEM, nullptr, &attr);
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, gemm_pair_kernel<UP>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            clusters = 0;
        }
        grid = 2 * clusters;
    }
    return grid;
}

template <bool UP>
cudaError_t launch_pair(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &b, const GemmArgs &args,
                        int grid, cudaStream_t s)
{
    if (grid < 2 || grid % 2 || args.M % kPM) return cudaErrorInvalidValue;
    cudaLaunchAttribute attr;
    cudaLaunchConfig_t cfg = pair_config(grid, Cfg2<UP>::SMEM, s, &attr);
    return cudaLaunchKernelEx(&cfg, gemm_pair_kernel<UP>, a0, a1, b, args);
}

}  // namespace

int gemm_up_pair_grid(int num_sms) { return pair_grid<true>(num_sms); }
int gemm_down_pair_grid(int num_sms) { return pair_grid<false>(num_sms); }

cudaError_t launch_gemm_up_pair(const CUtensorMap &wl, const CUtensorMap &wv, const CUtensorMap &xp,
                                const GemmArgs &a, int grid, cudaStream_t s)
{
    return launch_pair<true>(wl, wv, xp, a, grid, s);
}

cudaError_t launch_gemm_down_pair(const CUtensorMap &w1, const CUtensorMap &h, const GemmArgs &a, int grid,
                                  cudaStream_t s)
{
    return launch_pair<false>(w1, w1, h, a, grid, s);
}

}  // namespace moe
