// gemm_ts.cu -- grouped expert GEMMs for int8 weights stored K-major ([E, out, in], one
// row of reduction elements per output feature), with the dequantised bf16 weights
// kept in tensor memory (TMEM) as the MMA's A operand.
//
// Computes the expert MLP of "Grok-1 Admin & Architecture Guide", section 3,
// "Mixture of Experts (MoELayer + Router)" step 3, linear_1(gelu(linear(x)) * linear_v(x)),
// with the 8-bit weights of section 3 "Quantized weights" (int8 value * scale).
//
// Same tile orientation as the shared-memory variant (weights = A, M = 128 output
// features; grouped token rows = B, N = BN rows), but per pipeline stage of 128
// reduction elements:
//   - a TMA producer thread copies the int8 weight tile(s) [128 f x 128 k] (128-byte
//     swizzle) into a shared-memory staging ring;
//   - 16 converter warps each own 32 feature rows (one TMEM lane quadrant) and a slice
//     of the 128 reduction elements: they read their bytes from the staging tile,
//     convert int8 -> bf16 exactly and store the bf16 pairs into the A ring in TMEM
//     with tcgen05.st (one 32-bit TMEM column holds two consecutive k);
//   - a second TMA producer copies the bf16 activation tile [BN r x 128 k] into the
//     shared-memory operand ring;
//   - one thread issues tcgen05.mma with A from TMEM and B from shared memory; where a
//     stage holds two weight boxes with accumulators of their own, two threads on different
//     SM sub-partitions (warps 1 and 3) issue one box each;
//   - 4 epilogue warps apply the same fused epilogues as the shared-memory variant.
// Shared-memory traffic per weight byte is the TMA write plus one read (against
// also a bf16 write and an MMA read of 2 bytes each when the dequantised tile goes
// through shared memory), which takes shared-memory bandwidth off the critical path.
#include "gemm_common.cuh"

namespace moe {

namespace {

constexpr int kThreads = 640;                  // 20 warps
constexpr int kWarpTmaA = 0, kWarpMma = 1, kWarpTmaB = 2, kWarpMma2 = 3;
constexpr int kWarpEpi0 = 4;                   // warps 4..11: epilogue, two per TMEM lane quadrant
constexpr int kEpiWarps = 8;
constexpr int kWarpConv0 = 12;                 // warps 12..19: converters, two per TMEM lane quadrant
constexpr int kConvWarps = 8;
constexpr int kBKT = 128;                      // reduction elements per stage
constexpr int kSmemBudget = 208 * 1024;
static_assert(kWarpConv0 % 4 == 0 && kWarpEpi0 % 4 == 0, "warp w must own TMEM lane quadrant w % 4");
static_assert(kWarpConv0 + kConvWarps == kThreads / 32 && kWarpEpi0 + kEpiWarps == kWarpConv0, "warp roles");

// Weight tiles are [128 features x 128 reduction elements] int8 "boxes" of 16 KB.  A pipeline
// stage carries NB boxes: the up-projection one box of each of its two matrices (same k), the
// down-projection with narrow tiles two consecutive k-boxes of its one matrix (so every stage
// moves 32 KB), the down-projection with 128-route (wide, 256-route) tiles one box.
template <bool UP, int BN>
struct CfgTS {
    static constexpr bool K2 = !UP && BN <= 64;             // two k-boxes per stage
    // The 128-route down-projection takes route tiles of two consecutive 128-row segments of an
    // expert: one N = 256 MMA per K slice (N = 128 for an expert's odd last segment), so each
    // converted weight box serves 256 routes and a stage carries 1024 MMA cycles against
    // 160 KB of shared-memory traffic, the balance of the up-projection.
    static constexpr bool WIDE = !UP && BN == 128;
    static constexpr int PAIR = WIDE ? 2 : 1;               // BN-row segments per route tile
    static constexpr int TN = PAIR * BN;                    // MMA N (accumulator columns) of a full tile
    static constexpr int NB = UP ? 2 : (K2 ? 2 : 1);        // weight boxes per stage
    static constexpr int KSTAGE = K2 ? 2 * kBKT : kBKT;     // reduction elements per stage
    static constexpr int KP = kConvWarps / 4 / NB;          // converter warps per (quadrant, box)
    static constexpr int CH = (kBKT / 16) / KP;             // 16-byte chunks per converter thread and stage
    static constexpr int STG = NB * kBM * kBKT;             // int8 staging bytes per stage
    static constexpr int BBYTES = TN * KSTAGE * 2;          // bf16 activation bytes per stage
    // Two MMA issuers, one per box of a stage, each into an accumulator of its own: the
    // up-projection (one accumulator per matrix anyway) and the narrowest down-projections (one
    // per k-box; the epilogue sums the two).  The converter warps keep every SM sub-partition's
    // issue slots busy, and a single issuing thread, which spends several instructions per MMA,
    // then falls behind the tensor core.
    static constexpr bool DUAL = UP || (K2 && BN <= 32);
    static constexpr int NACC = DUAL ? 2 : 1;               // accumulators per tile
    static constexpr int ACC = NACC * TN;                   // TMEM columns of one accumulator buffer
    static constexpr int NDB = ACC > 128 ? 1 : 2;           // accumulator buffers in TMEM
    static constexpr int A_COLS = NB * kBKT / 2;            // TMEM columns of one A stage
    static constexpr int S2 = cmin(cmin(4, (512 - NDB * ACC) / A_COLS), (kSmemBudget - 2 * STG) / BBYTES);   // A (TMEM) + B (smem) ring
    static constexpr int S1 = cmin(12, (kSmemBudget - S2 * BBYTES) / STG);   // int8 staging ring
    static constexpr int A_BASE = NDB * ACC;                // first TMEM column of the A ring
    static constexpr int TMEM_COLS = pow2_at_least(NDB * ACC + S2 * A_COLS);
    static constexpr int OFF_STG = 0;
    static constexpr int OFF_B = OFF_STG + S1 * STG;
    static constexpr int OFF_BAR = OFF_B + S2 * BBYTES;
    // barriers: stg_full[S1] stg_empty[S1] a_full[S2] b_full[S2] op_empty[S2] acc_full[NDB] acc_empty[NDB] drain[2]
    static constexpr int NBAR = 2 * S1 + 3 * S2 + 2 * NDB + 2;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int MISC_BYTES = 16 + 3 * 4 * 40;   // tmem addr, flags, prefix[40], poff[40], roff[40]
    static constexpr int SMEM = OFF_MISC + MISC_BYTES + 1024;
    static_assert(S1 >= 2 && S2 >= 2, "rings too shallow");
    static_assert(SMEM <= 227 * 1024, "shared memory over the per-CTA limit");
    static_assert(TMEM_COLS <= 512, "TMEM has 512 columns");
    static_assert(KP >= 1 && CH * KP == kBKT / 16, "converter warps must split the 8 chunks of a row");
    static_assert(TN % 16 == 0 && BN >= 16 && TN <= 256, "UMMA N for M=128 is 16..256 in steps of 16");
};

// kind::f16 instruction descriptor: D fp32, A and B bf16, both K-major, M = 128.
template <int BN>
__device__ __forceinline__ constexpr uint32_t idesc_ts()
{
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
           (static_cast<uint32_t>(kBM >> 4) << 24);
}

// The tile epilogue on columns c .. c+15 of one accumulator row (TMEM lane = feature f),
// from the full-K sums x0 (and x1: the second matrix, or the second k-box).  The packed
// operands are scaled (kActScale): sc0 and sc1 are the scales times the factor taking a sum
// to its value.
//   up-projection:   H[r, f] = bf16( gelu(s0 * x0) * (s1 * x1) ), stored at kActScale times it
//   down-projection: slot[s, t, j, f] = gate[t, j] * s0 * (x0 + x1)   (k-box sums in this order)
// padding rows (route id -1; for the up-projection: tile rows from nreal on) are skipped.
struct EpiOut {
    const int *rperm;
    const float *gate;
    __nv_bfloat16 *h;
    float *slots;
    int M, T;
};

template <bool UP, int NACC>
__device__ __forceinline__ void epilogue_chunk(const EpiOut &a, int row0, int nreal, int c, int f, int s, float sc0,
                                               float sc1, const float (&x0)[16], const float (&x1)[16])
{
    if constexpr (UP) {
        // the tile's real rows are its first nreal rows (the rest pad the expert's segment)
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int r = row0 + c + i;
            if (c + i < nreal)
                a.h[static_cast<size_t>(r) * a.M + f] =
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

// The last piece of a split tile: add the P pieces' partial sums of this thread's row (p0 =
// piece 0's row, pieces kBM * ACC floats apart) in piece order, then the tile epilogue.  Out
// of line: it runs at most once per split tile and would otherwise raise the register
// pressure of the whole kernel.
template <bool UP, int BN, int NACC, int ACC>
__device__ __noinline__ void finish_pieces(const EpiOut a, const float *p0, int P, int c0, int c1, int row0,
                                           int nreal, int f, int s, float sc0, float sc1)
{
    const size_t pstride = static_cast<size_t>(kBM) * ACC;
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
                const float4 *r1 = reinterpret_cast<const float4 *>(p0 + p * pstride + BN + c);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 u = __ldcg(r1 + i);
                    x1[4 * i] += u.x; x1[4 * i + 1] += u.y; x1[4 * i + 2] += u.z; x1[4 * i + 3] += u.w;
                }
            }
        }
        epilogue_chunk<UP, NACC>(a, row0, nreal, c, f, s, sc0, sc1, x0, x1);
    }
}

// One converter thread's share of a stage in the per-block scale format: CH 16-byte chunks of
// its feature row (chunks j0 .. j0+CH-1, 128-byte swizzle: chunk j at (j ^ sw) * 16) loaded from
// the staging ring at src, each value turned into bf16(w * scale), stored to TMEM at taddr.
template <int CH>
__device__ __noinline__ void convert_stage_kblock(uint32_t src, int j0, int sw, uint32_t taddr, __nv_bfloat162 sc2)
{
    uint4 v[CH];
#pragma unroll
    for (int c = 0; c < CH; ++c) v[c] = lds128(src + (((j0 + c) ^ sw) << 4));
    __syncwarp();   // tcgen05.st is warp-collective (.sync.aligned): converge first
#pragma unroll
    for (int c = 0; c < CH; c += 4) {
        uint32_t words[32];
        convert_group<true>(v + c, words, sc2);
        tmem_st32(taddr + c * 8, words);
    }
}

template <bool UP, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_ts_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                   const __grid_constant__ CUtensorMap tmB, const GemmArgs a)
{
    using C = CfgTS<UP, BN>;
    // launched to overlap the previous kernel's end: the up-projection reads the routing from its
    // first instruction on, so all of it waits for that kernel (the down-projection waits later)
    if (UP) griddep_wait();
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
    auto acc_empty = [&](int b) { return bar(2 * C::S1 + 3 * C::S2 + C::NDB + b); };
    const uint32_t drain_bar = bar(2 * C::S1 + 3 * C::S2 + 2 * C::NDB);

    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile uint32_t *abort_flag = misc + 1;
    int *prefix = reinterpret_cast<int *>(misc + 4);
    int *poff = prefix + 40;
    int *roff = prefix + 80;   // unpadded offsets
    const int m_tiles = a.M / kBM;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::S1; ++s) {
            mbar_init(stg_full(s), 1);
            mbar_init(stg_empty(s), kConvWarps);
        }
        for (int s = 0; s < C::S2; ++s) {
            mbar_init(a_full(s), kConvWarps);
            mbar_init(b_full(s), 1);
            mbar_init(op_empty(s), C::NACC);   // one commit per issuer
        }
        for (int b = 0; b < C::NDB; ++b) {
            mbar_init(acc_full(b), C::NACC);
            mbar_init(acc_empty(b), kEpiWarps);
        }
        mbar_init(drain_bar, 1);
        mbar_init(drain_bar + 8, 1);
        *abort_flag = 0u;
        prefix[0] = 0;
        for (int e = 0; e <= a.E; ++e) poff[e] = a.poff[e];
        for (int e = 0; e <= a.E; ++e) roff[e] = a.offsets[e];
        for (int e = 0; e < a.E; ++e)
            prefix[e + 1] = prefix[e] + m_tiles * (((poff[e + 1] - poff[e]) / BN + C::PAIR - 1) / C::PAIR) * a.splits;
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
    // the next kernel (the down-projection after the up-projection, the combine after the
    // down-projection) may be scheduled onto SMs as this grid's CTAs leave them
    if (threadIdx.x == 0) griddep_launch_dependents();
    const uint32_t tmem_base = misc[0];
    const int total = prefix[a.E];
    const WorkList wl = a.part ? make_work_list(total, gridDim.x, a.ksteps) : WorkList{total, 0, total};
    const int SB = UP ? 0 : 32;   // first stats slot of this kernel (instrumented builds)
    PS_NOW(t_start);
    const Waiter w{abort_flag, a.err, a.timeout_ns, SB};

    if (warp == kWarpTmaA) {
        // ---- int8 weight tiles [128 f x 128 k] -> staging ring ------------------------
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            uint32_t st = 0, ph = 0, issued = 0, par = 0;
            PS_VAR(c_wait);
            for (int item = blockIdx.x; item < wl.items && !*abort_flag; item += gridDim.x) {
                const WorkItem wi = work_item(wl, item, a.ksteps);
                int e, m, n, s;
                decode_tile<BN>(wi.tile, prefix, poff, m_tiles, a.splits, e, m, n, s, C::PAIR);
                const int kb = s * a.ksteps;
                const int y = e * a.M + m * kBM;
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
            for (int s = 0; s < C::S1; ++s)   // every copy issued has landed before the CTA may exit
                if (issued & (1u << s)) wait_drain(stg_full(s), (par >> s) & 1u);
            PS_FLUSH(SB + 1, c_wait);
        }
        __syncwarp();
    } else if (UP && BN <= 32 && warp == kWarpTmaB && a.gather) {
        // ---- small batches: the activation rows straight from the routed rows -----------
        // tmB covers the routed rows [T, d] with one-row boxes.  Lane q copies tile rows
        // 4q .. 4q+3 (tokens rperm >> 1) with one four-row gather per 64-wide box, into the
        // place the tiled load gives those rows; rows from nreal on repeat row 0's token.
        // Each accumulator column depends on its own B row only, and the epilogue skips the
        // columns from nreal on.
        const uint64_t pol = l2_policy_evict_last();
        uint32_t st = 0, ph = 0, issued = 0, par = 0;
        bool ok = true;
        for (int item = blockIdx.x; ok && item < wl.items; item += gridDim.x) {
            if (__shfl_sync(0xffffffffu, lane == 0 ? static_cast<int>(*abort_flag) : 0, 0)) break;
            const WorkItem wi = work_item(wl, item, a.ksteps);
            int e, m, n, s;
            decode_tile<BN>(wi.tile, prefix, poff, m_tiles, a.splits, e, m, n, s, C::PAIR);
            const int kb = s * a.ksteps;
            const int row = poff[e] + n * BN;
            const int nreal = min(BN, roff[e + 1] - roff[e] - n * BN);
            const int ngroups = (nreal + 3) >> 2;
            const int tok = lane < nreal ? (__ldg(a.rperm + row + lane) >> 1) : -1;
            const int tok0 = __shfl_sync(0xffffffffu, tok, 0);
            int g[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int v = __shfl_sync(0xffffffffu, tok, (4 * lane + i) & 31);
                g[i] = 4 * lane + i < nreal ? v : tok0;
            }
            for (int ks = wi.k0; ks < wi.k1; ++ks) {
                if (lane == 0) ok = w.wait(op_empty(st), ph ^ 1u, 2);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (lane == 0) mbar_arrive_expect_tx(b_full(st), static_cast<uint32_t>(ngroups) * 4 * C::KSTAGE * 2);
                __syncwarp();
                const uint32_t dst = sbase + C::OFF_B + st * C::BBYTES + lane * 4 * 128;
                const int x = (kb + ks) * C::KSTAGE;
                if (lane < ngroups) {
#pragma unroll
                    for (int j = 0; j < C::KSTAGE / 64; ++j)
                        tma_gather4(dst + j * BN * 128, &tmB, b_full(st), x + 64 * j, g[0], g[1], g[2], g[3], pol);
                }
                issued |= 1u << st;
                par = (par & ~(1u << st)) | (ph << st);
                if (++st == C::S2) { st = 0; ph ^= 1u; }
            }
        }
        if (lane == 0)
            for (int s = 0; s < C::S2; ++s)
                if (issued & (1u << s)) wait_drain(b_full(s), (par >> s) & 1u);
        __syncwarp();
    } else if (warp == kWarpTmaB) {
        // ---- bf16 activation tiles [BN r x 128 k] (two 64-wide boxes) -> operand ring --
        // The down-projection is launched to overlap the up-projection's last CTAs (its weight
        // loads and conversions do not depend on them): its activations, H, are read only once
        // the up-projection has completed.
        if (!UP) griddep_wait();
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_last();
            uint32_t st = 0, ph = 0, issued = 0, par = 0;
            PS_VAR(c_bwait);
            for (int item = blockIdx.x; item < wl.items && !*abort_flag; item += gridDim.x) {
                const WorkItem wi = work_item(wl, item, a.ksteps);
                int e, m, n, s;
                decode_tile<BN>(wi.tile, prefix, poff, m_tiles, a.splits, e, m, n, s, C::PAIR);
                const int kb = s * a.ksteps;
                const int row = poff[e] + n * C::TN;
                const int nseg = min(C::PAIR, (poff[e + 1] - row) / BN);   // BN-row segments of the tile
                for (int ks = wi.k0; ks < wi.k1; ++ks) {
                    PS_NOW(t0);
                    if (!w.wait(op_empty(st), ph ^ 1u, 2)) goto b_done;
                    PS_ADD(c_bwait, t0);
                    mbar_arrive_expect_tx(b_full(st), static_cast<uint32_t>(nseg) * BN * C::KSTAGE * 2);
                    const uint32_t dst = sbase + C::OFF_B + st * C::BBYTES;
                    const int x = (kb + ks) * C::KSTAGE;
#pragma unroll
                    for (int j = 0; j < C::KSTAGE / 64; ++j)   // 64-element (128-byte) wide boxes of TN rows
                        for (int g = 0; g < nseg; ++g)
                            tma_load_2d(dst + (j * C::TN + g * BN) * 128, &tmB, b_full(st), x + 64 * j, row + g * BN,
                                        pol);
                    issued |= 1u << st;
                    par = (par & ~(1u << st)) | (ph << st);
                    if (++st == C::S2) { st = 0; ph ^= 1u; }
                }
            }
        b_done:
            for (int s = 0; s < C::S2; ++s)
                if (issued & (1u << s)) wait_drain(b_full(s), (par >> s) & 1u);
            PS_FLUSH(SB + 2, c_bwait);
        }
        __syncwarp();
    } else if (warp == kWarpMma || (C::DUAL && warp == kWarpMma2)) {
        // ---- tensor-core issue: A from TMEM, B from shared memory --------------------
        // with two issuers, issuer i takes box i of every stage into accumulator i
        const int mine = warp == kWarpMma ? 0 : 1;
        if (lane == 0) {
            uint32_t st = 0, ph = 0;
            int it = 0;
            PS_VAR(c_acc);
            PS_VAR(c_a);
            PS_VAR(c_b);
            PS_VAR(c_issue);
            for (int item = blockIdx.x; item < wl.items; item += gridDim.x, ++it) {
                const WorkItem wi = work_item(wl, item, a.ksteps);
                uint32_t idesc = idesc_ts<C::TN>();
                if constexpr (C::WIDE) {   // an expert's odd last segment: N = BN
                    int e, m, n, s;
                    decode_tile<BN>(wi.tile, prefix, poff, m_tiles, a.splits, e, m, n, s, C::PAIR);
                    if (poff[e + 1] - (poff[e] + n * C::TN) < C::TN) idesc = idesc_ts<BN>();
                }
                const int b = it % C::NDB;
                const uint32_t aph = (it / C::NDB) & 1;
                PS_NOW(t0);
                if (!w.wait(acc_empty(b), aph ^ 1u, 3)) break;
                PS_ADD(c_acc, t0);
                tc_fence_after();
                const uint32_t dcol = tmem_base + b * C::ACC;
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
                    const uint32_t acol = tmem_base + C::A_BASE + st * C::A_COLS;
                    const uint32_t blo = desc_sw128_lo(sbase + C::OFF_B + st * C::BBYTES, 16);
#pragma unroll
                    for (int bx = 0; bx < C::NB; ++bx) {
#pragma unroll
                        for (int kk = 0; kk < kBKT / 16; ++kk) {
                            // issuer / accumulator of this MMA: the box
                            if (C::DUAL && bx != mine) continue;
                            // K slice of the stage's activation tile; both matrices of the
                            // up-projection use the same slices, the k-boxes of the down-projection
                            // consecutive ones
                            const int kg = (UP ? 0 : bx * (kBKT / 16)) + kk;
                            const uint64_t bdesc = desc_join(
                                blo + (((kg >> 2) * (C::TN * 128) + (kg & 3) * 32) >> 4), desc_sw128_hi(1024));
                            // the item's first MMA into an accumulator starts it
                            const int kr = ks - wi.k0;
                            const uint32_t acc = C::DUAL ? ((kr | kk) != 0) : ((kr | bx | kk) != 0);
                            umma_bf16_ts(dcol + (C::DUAL ? bx : 0) * BN, acol + bx * (kBKT / 2) + kk * 8, bdesc,
                                         idesc, acc);
                        }
                    }
                    umma_commit(op_empty(st));
                    PS_ADD(c_issue, t3);
                    if (++st == C::S2) { st = 0; ph ^= 1u; }
                }
                if (!ok) break;
                umma_commit(acc_full(b));
            }
            umma_commit(drain_bar + 8 * mine);   // all MMAs this thread issued have completed after this
            wait_drain(drain_bar + 8 * mine, 0);
            PS_FLUSH(SB + 3, c_acc);
            PS_FLUSH(SB + 4, c_a);
            PS_FLUSH(SB + 5, c_b);
            PS_FLUSH(SB + 6, c_issue);
        }
        __syncwarp();
    } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + kEpiWarps) {
        // ---- epilogue: TMEM -> registers -> global -----------------------------------
        // warp (q, hc): TMEM lane quadrant q = warp % 4, column half hc of the tile (narrowest
        // tiles: the first four warps take all 16 columns, the others only hand the buffer back)
        const int q = warp & 3;
        const int hc = (warp - kWarpEpi0) >> 2;
        constexpr int kCols = BN >= 32 ? C::TN / 2 : BN;
        const int c0 = BN >= 32 ? hc * kCols : 0;
        const int c1_full = BN >= 32 || hc == 0 ? c0 + kCols : c0;
        volatile uint32_t *last_flag = misc + 2;
        const EpiOut eo{a.rperm, a.gate, a.h, a.slots, a.M, a.T};
        // the down-projection's slots, pieces and tickets: after the up-projection has completed
        if (!UP) griddep_wait();
        auto epilogue_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory"); };
        int it = 0;
        PS_VAR(c_ewait);
        PS_VAR(c_ework);
        for (int item = blockIdx.x; item < wl.items; item += gridDim.x, ++it) {
            const WorkItem wi = work_item(wl, item, a.ksteps);
            int e, m, n, s;
            decode_tile<BN>(wi.tile, prefix, poff, m_tiles, a.splits, e, m, n, s, C::PAIR);
            const int b = it % C::NDB;
            const uint32_t aph = (it / C::NDB) & 1;
            PS_NOW(t0);
            w.wait(acc_full(b), aph, 6);   // a wait that gives up sets the CTA's abort flag
            // one decision for all epilogue warps: a piece's epilogue meets at a named barrier,
            // so no warp may leave the loop while the others go on
            epilogue_sync();
            if (*abort_flag) break;
            PS_ADD(c_ewait, t0);
            PS_NOW(t1);
            tc_fence_after();
            const int f = m * kBM + q * 32 + lane;
            const uint32_t tl = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * C::ACC;
            const int row0 = poff[e] + n * C::TN;
            const int nreal = roff[e + 1] - roff[e] - n * C::TN;   // real rows of this tile (may exceed TN)
            // a wide tile over an expert's odd last segment has BN columns
            const int c1 = C::WIDE ? max(c0, min(c1_full, poff[e + 1] - row0)) : c1_full;
            // per-channel scales here (the per-block format applied them while dequantising), times
            // the factor taking a sum of scaled operands to its value: exact while |s| < 2^59
            const float sc0 = (a.kblock ? 1.f : __bfloat162float(a.s0[static_cast<size_t>(e) * a.M + f])) * a.accf;
            const float sc1 =
                !UP ? 0.f : (a.kblock ? 1.f : __bfloat162float(a.s1[static_cast<size_t>(e) * a.M + f])) * a.accf;
            const bool whole = wi.piece < 0;   // uniform over the CTA
            if (!whole) {
                // a piece: its partial sums go to the workspace, [piece][row][accumulator column]
                float *pp = a.part + (static_cast<size_t>(wi.piece) * kBM + q * 32 + lane) * C::ACC;
#pragma unroll 1
                for (int c = c0; c < c1; c += 16) {
                    float x0[16], x1[16];
                    __syncwarp();   // tcgen05.ld is warp-collective (.sync.aligned): converge first
                    tmem_ld16(tl + c, x0);
                    if constexpr (C::NACC == 2) tmem_ld16(tl + BN + c, x1);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; i += 4) {
                        *reinterpret_cast<float4 *>(pp + c + i) = make_float4(x0[i], x0[i + 1], x0[i + 2], x0[i + 3]);
                        if constexpr (C::NACC == 2)
                            *reinterpret_cast<float4 *>(pp + BN + c + i) =
                                make_float4(x1[i], x1[i + 1], x1[i + 2], x1[i + 3]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty(b));   // the accumulator is no longer needed
                __threadfence();                             // partial sums before the ticket
                epilogue_sync();
                if (warp == kWarpEpi0 && lane == 0) {
                    unsigned int *tk = a.tickets + (wi.tile - wl.whole);
                    const bool last = atomicAdd(tk, 1u) == static_cast<unsigned int>(wl.P - 1);
                    if (last) *tk = 0u;                      // every piece of the tile has arrived
                    *last_flag = last ? 1u : 0u;
                }
                epilogue_sync();
                if (*last_flag) __threadfence();   // the other pieces' sums, visible after their tickets
            }
            if (whole && UP && kCols == 64) {
                // the 128-route up-projection: this warp's 64 columns of H, packed as bf16 pairs in
                // registers, so that the accumulator goes back to the MMA issuers before the stores
                // (8-column loads keep the peak at 16 accumulator registers beside the 32 packed)
                uint32_t hp[32];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    float x0[8], x1[8];
                    __syncwarp();   // tcgen05.ld is warp-collective (.sync.aligned): converge first
                    tmem_ld8(tl + c0 + 8 * k, x0);
                    tmem_ld8(tl + BN + c0 + 8 * k, x1);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float h0 = gelu_tanh(sc0 * x0[2 * i]) * (sc1 * x1[2 * i]);
                        const float h1 = gelu_tanh(sc0 * x0[2 * i + 1]) * (sc1 * x1[2 * i + 1]);
                        const __nv_bfloat162 v = __floats2bfloat162_rn(h0 * kActScale, h1 * kActScale);
                        hp[4 * k + i] = *reinterpret_cast<const uint32_t *>(&v);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty(b));
                // the tile's real rows are its first nreal rows (the rest pad the expert's segment)
                __nv_bfloat16 *hrow = a.h + static_cast<size_t>(row0 + c0) * a.M + f;
                const int lim = nreal - c0;   // this warp's real columns
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    if (2 * j < lim) *hrow = __ushort_as_bfloat16(hp[j] & 0xFFFFu);
                    hrow += a.M;
                    if (2 * j + 1 < lim) *hrow = __ushort_as_bfloat16(hp[j] >> 16);
                    hrow += a.M;
                }
            } else if (whole) {
#pragma unroll 1
                for (int c = c0; c < c1; c += 16) {
                    float x0[16], x1[16];
                    __syncwarp();   // tcgen05.ld is warp-collective (.sync.aligned): converge first
                    tmem_ld16(tl + c, x0);
                    if constexpr (C::NACC == 2) tmem_ld16(tl + BN + c, x1);
                    tmem_wait_ld();
                    epilogue_chunk<UP, C::NACC>(eo, row0, nreal, c, f, s, sc0, sc1, x0, x1);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty(b));
            } else if (*last_flag) {
                // the tile's pieces are consecutive in the workspace
                const float *p0 =
                    a.part + (static_cast<size_t>(wi.tile - wl.whole) * wl.P * kBM + q * 32 + lane) * C::ACC;
                finish_pieces<UP, BN, C::NACC, C::ACC>(eo, p0, wl.P, c0, c1, row0, nreal, f, s, sc0, sc1);
            }
            PS_ADD(c_ework, t1);
        }
        if (lane == 0) {
            PS_FLUSH(SB + 7, c_ewait);
            PS_FLUSH(SB + 8, c_ework);
        }
    } else if (warp >= kWarpConv0) {
        // ---- int8 staging -> bf16 A operand in TMEM ------------------------------------
        // Converter warp cw owns TMEM lane quadrant q = warp % 4 (feature rows 32q..32q+31
        // of the tile), weight box `box` of the stage and chunks [j0, j0 + CH) of the 8
        // 16-byte chunks of each 128-byte feature row.  Lanes of one 8-lane phase read 8
        // different rows, whose 128-byte swizzle puts the same logical chunk in 8
        // different bank groups.
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
        for (int item = blockIdx.x; item < wl.items; item += gridDim.x) {
            const WorkItem wi = work_item(wl, item, a.ksteps);
            // per-block scale format: this thread's feature row in the scale rows of its box;
            // the scale row of a stage is its first reduction row / kScaleBlock
            const __nv_bfloat16 *srow = nullptr;
            if (a.kblock) {
                int e, m, n, s;
                decode_tile<BN>(wi.tile, prefix, poff, m_tiles, a.splits, e, m, n, s, C::PAIR);
                const int k0 = s * a.ksteps * C::KSTAGE + (UP ? 0 : box * kBKT);
                srow = ((UP && box == 1) ? a.s1 : a.s0) +
                       (static_cast<size_t>(e) * (a.K / kScaleBlock) + k0 / kScaleBlock) * a.M + m * kBM + fr;
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
                static_assert(C::CH % 4 == 0, "chunks go to TMEM in fours");
                if (a.kblock) {
                    // this row's block scale (per-block format); out of line, so that this rarer
                    // form does not add to the register pressure of the loop below
                    const __nv_bfloat16 sv = srow[static_cast<size_t>(ks) * (C::KSTAGE / kScaleBlock) * a.M];
                    convert_stage_kblock<C::CH>(src, j0, fr & 7, taddr, __halves2bfloat162(sv, sv));
                } else {
                    uint4 v[C::CH];
#pragma unroll
                    for (int c = 0; c < C::CH; ++c) v[c] = lds128(src + (((j0 + c) ^ (fr & 7)) << 4));
                    __syncwarp();   // tcgen05.st is warp-collective (.sync.aligned): converge first
                    // each group of four 16-byte chunks (64 reduction elements = 32 TMEM columns) is
                    // stored with one 32-column store as soon as it is converted, so the TMEM writes
                    // spread over the conversion work in few, wide instructions
#pragma unroll
                    for (int c = 0; c < C::CH; c += 4) {
                        uint32_t words[32];
                        convert_group<false>(v + c, words, __nv_bfloat162{});
                        tmem_st32(taddr + c * 8, words);
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
                    mbar_arrive(a_full(st2));
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
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
#ifdef MOE_PIPE_STATS
    if (threadIdx.x == 0) PS_FLUSH(SB + 0, clock64() - t_start);
#endif
}

template <bool UP, int BN>
cudaError_t launch_one_ts(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &b, const GemmArgs &args,
                          int grid, cudaStream_t s)
{
    using C = CfgTS<UP, BN>;
    static bool configured = false;   // the attribute is the same for every launch in the process
    if (!configured) {
        cudaError_t e =
            cudaFuncSetAttribute(gemm_ts_kernel<UP, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    // programmatic stream serialization: the CTAs may start while the previous kernel ends (the
    // kernel waits for it where it must); the down-projection's weight streaming overlaps the
    // up-projection's last CTAs
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemm_ts_kernel<UP, BN>, a0, a1, b, args);
}

}  // namespace

int gemm_ts_kstage(bool up, int bn) { return (!up && bn <= 64) ? 2 * kBKT : kBKT; }

cudaError_t launch_gemm_up_ts(int bn, const CUtensorMap &wl, const CUtensorMap &wv, const CUtensorMap &xp,
                              const GemmArgs &a, int grid, cudaStream_t s)
{
    switch (bn) {
    case 16: return launch_one_ts<true, 16>(wl, wv, xp, a, grid, s);
    case 32: return launch_one_ts<true, 32>(wl, wv, xp, a, grid, s);
    case 64: return launch_one_ts<true, 64>(wl, wv, xp, a, grid, s);
    case 128: return launch_one_ts<true, 128>(wl, wv, xp, a, grid, s);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_gemm_down_ts(int bn, const CUtensorMap &w1, const CUtensorMap &h, const GemmArgs &a, int grid,
                                cudaStream_t s)
{
    switch (bn) {
    case 16: return launch_one_ts<false, 16>(w1, w1, h, a, grid, s);
    case 32: return launch_one_ts<false, 32>(w1, w1, h, a, grid, s);
    case 64: return launch_one_ts<false, 64>(w1, w1, h, a, grid, s);
    case 128: return launch_one_ts<false, 128>(w1, w1, h, a, grid, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe

#ifdef MOE_PIPE_STATS
extern "C" __attribute__((visibility("default"))) int moe_debug_pipe_stats_ts(unsigned long long *out, int reset)
{
    if (cudaMemcpyFromSymbol(out, moe::g_pipe_stats, sizeof(unsigned long long) * 64) != cudaSuccess) return -4;
    if (reset) {
        unsigned long long z[64] = {};
        if (cudaMemcpyToSymbol(moe::g_pipe_stats, z, sizeof z) != cudaSuccess) return -4;
    }
    return 0;
}
#endif
