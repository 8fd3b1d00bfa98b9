// moe_api.cu -- the C ABI declared in include/moe.h: handle, argument checks,
// workspace, TMA descriptors and the launch sequence of one MoE layer.
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/moe.h"
#include "kernels.cuh"

using namespace moe;

namespace {

enum KernelId { K_ROUTER = 0, K_DISPATCH, K_GATHER, K_UP, K_DOWN, K_COMBINE, K_PRENORM, K_ROUTE_SMALL };

struct DevBuf {
    void *ptr = nullptr;
    size_t bytes = 0;
};

struct WeightMap {
    const void *ptr = nullptr;
    int kind = -1;     // 0: linear / linear_v   1: linear_1
    int layout = -1;   // MOE_LAYOUT_IN_OUT or MOE_LAYOUT_PACKED
    int experts = 0;   // experts in the tensor
    CUtensorMap map;
};

struct PendingEvent {
    int id;
    cudaEvent_t a, b;
};

}  // namespace

struct moe_ctx {
    int d, F, E, k;
    int device = -1;
    int num_sms = 0;
    cudaStream_t last_stream = nullptr;
    bool used = false;

    // workspace
    DevBuf b_route;    // idx [2T] int, gate [2T] float, counts/offsets/poff, perm [2T], slot_of_route [2T]
    DevBuf b_rperm;    // [rows]
    DevBuf b_xp;       // bf16 [rows, d]
    DevBuf b_h;        // bf16 [rows, F]
    DevBuf b_slots;    // fp32 [splits, T, 2, d]
    DevBuf b_stage;    // bf16 [T, d] x2: host-API input/output staging, block pre-norm output
    // kCtlWords zeroed words: [0] the device error word, [32] the routing ticket, [64 ..) the
    // GEMMs' last-wave tickets (one per SM)
    int *err = nullptr;
    DevBuf b_part;     // fp32 [num_sms, 128, 256]: the GEMMs' last-wave partial sums
    // host-buffer forwards with host overlap on (moe_set_host_overlap): two staging slots, each
    // x [T, d] then out [T, d] bf16, used by alternate calls.  A call copies its input in on
    // copy_in and its result out on copy_out, so both copies overlap the neighbouring calls'
    // layers on the caller's stream.
    bool host_overlap = false;
    DevBuf b_host[2];
    int host_slot = 0;
    cudaStream_t copy_in = nullptr, copy_out = nullptr;
    cudaEvent_t ev_in[2] = {nullptr, nullptr};     // slot k's input has landed
    cudaEvent_t ev_layer[2] = {nullptr, nullptr};  // slot k's layer has written its result
    cudaEvent_t ev_done[2] = {nullptr, nullptr};   // slot k's last call has copied its output out
    bool slot_used[2] = {false, false};
    const char *slot_out[2] = {nullptr, nullptr};  // the host output range of slot k's last call
    size_t slot_out_bytes[2] = {0, 0};
    int rows_cap = 0;       // rows the xp / h buffers hold
    int route_cap = 0;      // T the route buffer holds
    int map_gen = 0;        // bumps when b_xp / b_h move
    int last_T = -1;
    int last_block_T = -1;  // T of the last forward if it was moe_block_forward (u is staged), else -1
    bool stage_scaled = false;   // that staged u is at kActScale (packed small-batch path)
    int ep_T = -1;          // T of the last moe_ep_dispatch (its routing waits for moe_ep_combine), else -1
    DevBuf b_ep;            // expert-parallel layout of received rows: counts, offsets, poff, rperm, slot, ones

    // TMA descriptors
    std::vector<WeightMap> wmaps;
    CUtensorMap xp_map[4], h_map[4];
    CUtensorMap stage_map;              // b_stage as bf16 [rows, d], one-row boxes (small-batch B rows)
    const void *stage_map_ptr = nullptr;
    size_t stage_map_bytes = 0;
    int xp_map_gen[4] = {-1, -1, -1, -1}, h_map_gen[4] = {-1, -1, -1, -1};

    const float *bias = nullptr;
    const uint8_t *mask = nullptr;   // padding mask of the next forwards (device, >= T bytes)
    int kblock = 0;                  // scale format: 0 per output channel, kScaleBlock per block
    long long timeout_ns = 2000000000LL;
    int layout = MOE_LAYOUT_IN_OUT;
    // GEMMs on CTA pairs (packed layout): 0 never, 1 the down-projection of 128-route plans,
    // 2 both GEMMs of 128-route plans, 3 also both GEMMs of 32-route plans
    int cta_pairs = 1;

    // profiling
    bool prof = false;
    std::vector<PendingEvent> pending;
    std::vector<cudaEvent_t> event_pool;
};

namespace {

constexpr int kCtlWords = 1024;     // words of the handle's zeroed control block
constexpr int kCtlRouteTicket = 32;
constexpr int kCtlPackRange = 48;   // moe_pack_weight: set when a weight is -128
constexpr int kCtlTickets = 64;     // first GEMM ticket

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// the packed layout's power-of-two steps must undo each other exactly: weights enter the tensor
// cores at 2^-133 times their value, activations at kActScale times theirs
static_assert(static_cast<double>(kAccScaleChannel) * static_cast<double>(kActScale) == 0x1p133,
              "per-channel epilogue factor must be 2^133 / kActScale");
static_assert(static_cast<double>(kActUnscale) * static_cast<double>(kActScale) == 1.0,
              "kActUnscale must be the inverse of kActScale");

// the GEMM epilogues' factor from an accumulator to its value: the packed layout's operands are
// scaled (kActScale); the shared-memory kernels of the [E, in, out] layout ignore it
float acc_factor(const moe_ctx *h)
{
    if (h->layout != MOE_LAYOUT_PACKED) return 1.f;
    return h->kblock ? kActUnscale : kAccScaleChannel;
}

// the up- (up = true) or down-projection of plans of tile width bn on CTA pairs on this handle
bool pairs_for(const moe_ctx *h, int bn, bool up)
{
    if (h->layout != MOE_LAYOUT_PACKED || h->d % 256 || h->F % 256) return false;
    if (bn == 128) return h->cta_pairs >= (up ? 2 : 1);
    if (bn == 32) return h->cta_pairs >= 3;
    return false;
}

// routes per GEMM tile (the dispatch pads each expert's segment to it) for batches of about
// `rows_per_expert` routes per expert; CTA pairs at small batches need 32-route tiles
int plan_bn_rows(const moe_ctx *h, int rows_per_expert)
{
    if (rows_per_expert <= 16 && !pairs_for(h, 32, true)) return 16;
    if (rows_per_expert <= 32) return 32;
    if (rows_per_expert <= 64) return 64;
    return 128;
}

int plan_bn(const moe_ctx *h, int T)
{
    // by T: T <= 16 -> 16 (32 with small-batch pairs), <= 32 -> 32, <= 64 -> 64, else 128
    return plan_bn_rows(h, T);
}

int bn_slot(int bn) { return bn == 16 ? 0 : bn == 32 ? 1 : bn == 64 ? 2 : 3; }

// reduction elements per pipeline stage of the up- / down-projection kernel of the handle's layout
int kstage_of(const moe_ctx *h, bool up, int bn)
{
    return h->layout == MOE_LAYOUT_PACKED ? gemm_ts_kstage(up, bn) : kBK;
}

// K-splits of the down-projection: double while the tiles of `experts` experts with about
// `per_expert` rows each fill fewer than 16 waves and the stages still divide evenly
int splits_for(const moe_ctx *h, int experts, int per_expert, int bn)
{
    const long nt = per_expert <= bn ? 1 : (per_expert + bn - 1) / bn;
    const long tiles = static_cast<long>(experts) * (h->d / kBM) * nt;
    const int ksteps = h->F / kstage_of(h, false, bn);
    const int sms = h->num_sms > 0 ? h->num_sms : 148;
    int s = 1;
    while (s < kMaxSplits && tiles * s < 16L * sms && ksteps % (2 * s) == 0) s *= 2;
    return s;
}

int plan_splits(const moe_ctx *h, int T, int bn)
{
    const int per_expert = (2 * T + h->E - 1) / h->E;
    const long nt = per_expert <= bn ? 1 : (per_expert + bn - 1) / bn;
    const long tiles = static_cast<long>(h->E) * (h->d / kBM) * nt;
    const int ksteps = h->F / kstage_of(h, false, bn);
    const int sms = h->num_sms > 0 ? h->num_sms : 148;
    int s = 1;
    while (s < kMaxSplits && tiles * s < 16L * sms && ksteps % (2 * s) == 0) s *= 2;
    return s;
}

int rows_for(const moe_ctx *h, int T, int bn) { return ((2 * T + h->E * (bn - 1)) + 127) / 128 * 128; }

// route buffer layout (ints/floats), all offsets in 4-byte words
struct RouteLayout {
    size_t idx, gate, counts, offsets, poff, perm, slot, words;
};

RouteLayout route_layout(int T, int E)
{
    auto up = [](size_t v) { return (v + 63) / 64 * 64; };
    RouteLayout L;
    size_t o = 0;
    L.idx = o; o += up(2 * static_cast<size_t>(T));
    L.gate = o; o += up(2 * static_cast<size_t>(T));
    L.counts = o; o += up(E);
    L.offsets = o; o += up(E + 1);
    L.poff = o; o += up(E + 1);
    L.perm = o; o += up(2 * static_cast<size_t>(T));
    L.slot = o; o += up(2 * static_cast<size_t>(T));
    L.words = o;
    return L;
}

int sync_last(moe_ctx *h)
{
    if (h->copy_in && cudaStreamSynchronize(h->copy_in) != cudaSuccess) return MOE_ECUDA;
    if (h->copy_out && cudaStreamSynchronize(h->copy_out) != cudaSuccess) return MOE_ECUDA;
    if (!h->used) return MOE_OK;
    return cudaStreamSynchronize(h->last_stream) == cudaSuccess ? MOE_OK : MOE_ECUDA;
}

// grow a buffer to at least `bytes` (contents are not kept)
int ensure(moe_ctx *h, DevBuf &b, size_t bytes, bool *moved = nullptr)
{
    if (b.bytes >= bytes) return MOE_OK;
    if (b.ptr) {
        if (sync_last(h) != MOE_OK) return MOE_ECUDA;
        cudaFree(b.ptr);
        b.ptr = nullptr;
        b.bytes = 0;
    }
    size_t want = bytes + bytes / 4;   // headroom against repeated small growth
    if (cudaMalloc(&b.ptr, want) != cudaSuccess) {
        cudaGetLastError();
        b.ptr = nullptr;
        if (cudaMalloc(&b.ptr, bytes) != cudaSuccess) {
            cudaGetLastError();
            b.ptr = nullptr;
            return MOE_ENOMEM;
        }
        want = bytes;
    }
    b.bytes = want;
    if (moved) *moved = true;
    return MOE_OK;
}

int ensure_device(moe_ctx *h)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ENODEV;
    }
    if (h->device < 0) {
        cudaDeviceProp p;
        if (cudaGetDeviceProperties(&p, dev) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ENODEV;
        }
        if (p.major != 10) return MOE_ENODEV;   // built for sm_100a only
        h->device = dev;
        h->num_sms = p.multiProcessorCount;
        if (h->num_sms + kCtlTickets > kCtlWords) return MOE_EUNSUPPORTED;
        if (cudaMalloc(reinterpret_cast<void **>(&h->err), kCtlWords * 4) != cudaSuccess) {
            cudaGetLastError();
            return MOE_ENOMEM;
        }
        if (cudaMemset(h->err, 0, kCtlWords * 4) != cudaSuccess) return MOE_ECUDA;
    } else if (dev != h->device) {
        return MOE_EINVAL;   // the handle belongs to another device
    }
    return MOE_OK;
}

// grouped-row buffers (rperm, Xp, H) for at least `rows` rows
int ensure_rows(moe_ctx *h, int rows)
{
    int rc;
    if (rows > h->rows_cap) {
        if ((rc = ensure(h, h->b_rperm, static_cast<size_t>(rows) * 4)) != MOE_OK) return rc;
        if ((rc = ensure(h, h->b_xp, static_cast<size_t>(rows) * h->d * 2)) != MOE_OK) return rc;
        if ((rc = ensure(h, h->b_h, static_cast<size_t>(rows) * h->F * 2)) != MOE_OK) return rc;
        h->rows_cap = rows;
        // the descriptors cover rows_cap rows: rebuild them all
        h->map_gen++;
    }
    return MOE_OK;
}

int ensure_workspace(moe_ctx *h, int T, int bn, int splits)
{
    int rc;
    const RouteLayout L = route_layout(T, h->E);
    if ((rc = ensure(h, h->b_route, L.words * 4)) != MOE_OK) return rc;
    if ((rc = ensure_rows(h, rows_for(h, T, bn))) != MOE_OK) return rc;
    if ((rc = ensure(h, h->b_slots, static_cast<size_t>(splits) * T * 2 * h->d * 4)) != MOE_OK) return rc;
    if ((rc = ensure(h, h->b_stage, static_cast<size_t>(T) * h->d * 2 * 2)) != MOE_OK) return rc;
    // last-wave partial sums of the TMEM GEMMs: one 128-row tile of up to 256 fp32 columns per SM
    if (h->layout == MOE_LAYOUT_PACKED &&
        (rc = ensure(h, h->b_part, static_cast<size_t>(h->num_sms) * 128 * 256 * 4)) != MOE_OK)
        return rc;
    return MOE_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        else
            cudaGetLastError();
    }
    return fn;
}

// 2-D tiled map with 128-byte swizzle: inner extent `cols` elements, `rows` rows
int encode_2d(CUtensorMap *m, CUtensorMapDataType dt, int esize, const void *ptr, uint64_t cols, uint64_t rows,
              uint32_t box_cols, uint32_t box_rows)
{
    auto fn = encode_fn();
    if (!fn) return MOE_ECUDA;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * static_cast<uint64_t>(esize)};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MOE_OK : MOE_ECUDA;
}

// int8 weight descriptor.  [E, in, out] layout: rows = E*in, box = 64 k-rows x 128 features.
// [E, out, in] (packed) layout: rows = E*out, box = 128 feature-rows x 128 k.
// The tensor map of a weight, from the handle's cache (encoded on first use).  The map is
// copied out: a pointer into the cache would dangle once a later insertion moves it.
// E_w: experts the weight tensor holds (the handle's E, or a rank's local experts)
int weight_map(moe_ctx *h, const void *ptr, int kind, CUtensorMap *out, int E_w = 0)
{
    if (E_w <= 0) E_w = h->E;
    for (auto &w : h->wmaps)
        if (w.ptr == ptr && w.kind == kind && w.layout == h->layout && w.experts == E_w) {
            *out = w.map;
            return MOE_OK;
        }
    WeightMap w;
    w.ptr = ptr;
    w.kind = kind;
    w.layout = h->layout;
    w.experts = E_w;
    const uint64_t in = kind == 0 ? h->d : h->F, outf = kind == 0 ? h->F : h->d;
    int rc;
    if (h->layout == MOE_LAYOUT_PACKED)
        rc = encode_2d(&w.map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ptr, in, static_cast<uint64_t>(E_w) * outf,
                       128, kBM);
    else
        rc = encode_2d(&w.map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ptr, outf, static_cast<uint64_t>(E_w) * in,
                       kBM, kBK);
    if (rc != MOE_OK) return rc;
    if (h->wmaps.size() >= 64) h->wmaps.erase(h->wmaps.begin());
    h->wmaps.push_back(w);
    *out = w.map;
    return MOE_OK;
}

int act_maps(moe_ctx *h, int bn, const CUtensorMap **xp, const CUtensorMap **hm)
{
    const int s = bn_slot(bn);
    int rc;
    if (h->xp_map_gen[s] != h->map_gen) {
        if ((rc = encode_2d(&h->xp_map[s], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, h->b_xp.ptr, h->d, h->rows_cap, kBK,
                            bn)) != MOE_OK)
            return rc;
        h->xp_map_gen[s] = h->map_gen;
    }
    if (h->h_map_gen[s] != h->map_gen) {
        if ((rc = encode_2d(&h->h_map[s], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, h->b_h.ptr, h->F, h->rows_cap, kBK,
                            bn)) != MOE_OK)
            return rc;
        h->h_map_gen[s] = h->map_gen;
    }
    *xp = &h->xp_map[s];
    *hm = &h->h_map[s];
    return MOE_OK;
}

// the routed rows of a small batch (b_stage as bf16 [rows, d]) with one-row boxes of kBK
// columns, for the up-projection's per-row loads
int stage_map(moe_ctx *h, const CUtensorMap **out)
{
    if (h->stage_map_ptr != h->b_stage.ptr || h->stage_map_bytes != h->b_stage.bytes) {
        const uint64_t rows = h->b_stage.bytes / (static_cast<uint64_t>(h->d) * 2);
        const int rc = encode_2d(&h->stage_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, h->b_stage.ptr, h->d, rows, kBK, 1);
        if (rc != MOE_OK) return rc;
        h->stage_map_ptr = h->b_stage.ptr;
        h->stage_map_bytes = h->b_stage.bytes;
    }
    *out = &h->stage_map;
    return MOE_OK;
}

cudaEvent_t take_event(moe_ctx *h)
{
    if (!h->event_pool.empty()) {
        cudaEvent_t e = h->event_pool.back();
        h->event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return e;
}

// run one launch, bracketed by events when profiling
template <class F>
cudaError_t timed(moe_ctx *h, int id, cudaStream_t s, F &&launch)
{
    cudaEvent_t a = nullptr, b = nullptr;
    if (h->prof) {
        a = take_event(h);
        b = take_event(h);
        if (a) cudaEventRecord(a, s);
    }
    cudaError_t e = launch();
    if (h->prof && a && b) {
        cudaEventRecord(b, s);
        h->pending.push_back({id, a, b});
    }
    return e;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb)
{
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

int check_weights(const moe_ctx *h, const float *router_w, const int8_t *w_lin, const void *s_lin, const int8_t *w_v,
                  const void *s_v, const int8_t *w_1, const void *s_1)
{
    const void *ps[] = {router_w, w_lin, s_lin, w_v, s_v, w_1, s_1};
    for (const void *p : ps)
        if (!p || !aligned16(p)) return MOE_EINVAL;
    (void)h;
    return MOE_OK;
}

cudaError_t launch_up(moe_ctx *h, int bn, const CUtensorMap &m_wl, const CUtensorMap &m_wv, const CUtensorMap &m_b,
                      const GemmArgs &up, cudaStream_t s);
cudaError_t launch_down(moe_ctx *h, int bn, const CUtensorMap &m_w1, const CUtensorMap &m_h, const GemmArgs &dn,
                        cudaStream_t s);

// the layer on x (device, bf16 [T, d]); result into `out` (plain) or added into h_io (residual block)
int run_layer(moe_ctx *h, int T, const void *x, const float *router_w, const int8_t *w_lin, const void *s_lin,
              const int8_t *w_v, const void *s_v, const int8_t *w_1, const void *s_1, void *out, void *h_io,
              const void *g_pre, const void *g_post, float eps, cudaStream_t s)
{
    int rc;
    const int bn = plan_bn(h, T);
    const int splits = plan_splits(h, T, bn);
    const RouteLayout L = route_layout(T, h->E);
    int *rw = static_cast<int *>(h->b_route.ptr);
    int *idx = rw + L.idx;
    float *gate = reinterpret_cast<float *>(rw + L.gate);
    int *poff = rw + L.poff;
    int *rperm = static_cast<int *>(h->b_rperm.ptr);

    const bool ts = h->layout == MOE_LAYOUT_PACKED;
    if (h->kblock && !ts) return MOE_EUNSUPPORTED;   // block scales: TMEM-operand kernels only
    CUtensorMap m_wl, m_wv, m_w1;
    const CUtensorMap *m_xp, *m_h;   // in the handle's fixed arrays
    if ((rc = weight_map(h, w_lin, 0, &m_wl)) != MOE_OK) return rc;
    if ((rc = weight_map(h, w_v, 0, &m_wv)) != MOE_OK) return rc;
    if ((rc = weight_map(h, w_1, 1, &m_w1)) != MOE_OK) return rc;
    if ((rc = act_maps(h, bn, &m_xp, &m_h)) != MOE_OK) return rc;

    // residual block: the routed rows are u = pre-RMSNorm(x); the routing kernels normalise
    // each row as they read it and leave u in the staging buffer for the gather
    const bool small = T <= route_small_max_tokens();
    __nv_bfloat16 *u = static_cast<__nv_bfloat16 *>(h->b_stage.ptr);
    const __nv_bfloat16 *routed = static_cast<const __nv_bfloat16 *>(x);
    RouteArgs ra{T, h->d, routed, router_w, h->bias, idx, gate};
    ra.mask = h->mask;
    if (g_pre) {
        ra.g_pre = static_cast<const __nv_bfloat16 *>(g_pre);
        ra.eps = eps;
        ra.u = u;
    }
    DispatchArgs da{T, h->E, bn, idx, rw + L.counts, rw + L.offsets, poff, rw + L.perm, rperm, rw + L.slot};
    GatherArgs ga{h->d, g_pre ? u : routed, static_cast<__nv_bfloat16 *>(h->b_xp.ptr)};
    ga.scaled = ts ? 1 : 0;   // the packed GEMMs take their B rows at kActScale
    // small batches on the TMEM-operand kernels: the routing launch leaves the routed rows in
    // the staging buffer at kActScale (in place when they were staged there) and the
    // up-projection loads its B rows from it, so nothing is gathered
    const bool gather_in_gemm = small && ts;
    const CUtensorMap *m_b = m_xp;
    if (gather_in_gemm) {
        if ((rc = stage_map(h, &m_b)) != MOE_OK) return rc;
        ra.u = u;
        ra.u_scaled = 1;
        ga.xp = nullptr;
    }
    if (small) {
        unsigned int *ticket = reinterpret_cast<unsigned int *>(h->err + kCtlRouteTicket);
        // the partial logits go to the combine's slot buffer, which is free until the down-projection
        float *part = static_cast<float *>(h->b_slots.ptr);
        const int S = route_small_slices(T, h->d, h->num_sms);
        if (timed(h, K_ROUTE_SMALL, s, [&] { return launch_route_small(ra, da, ga, part, S, ticket, s); }) !=
            cudaSuccess)
            return MOE_ECUDA;
    } else {
        if (timed(h, K_ROUTER, s, [&] { return launch_router(ra, s); }) != cudaSuccess) return MOE_ECUDA;
        if (timed(h, K_DISPATCH, s, [&] { return launch_dispatch(da, s); }) != cudaSuccess) return MOE_ECUDA;
        if (timed(h, K_GATHER, s, [&] { return launch_gather(ga, T, rw + L.slot, s); }) != cudaSuccess)
            return MOE_ECUDA;
    }

    GemmArgs up{};
    up.T = T;
    up.E = h->E;
    up.M = h->F;
    up.K = h->d;
    up.ksteps = h->d / kstage_of(h, true, bn);
    up.splits = 1;
    up.poff = poff;
    up.offsets = rw + L.offsets;
    up.rperm = rperm;
    up.gate = gate;
    up.s0 = static_cast<const __nv_bfloat16 *>(s_lin);
    up.s1 = static_cast<const __nv_bfloat16 *>(s_v);
    up.h = static_cast<__nv_bfloat16 *>(h->b_h.ptr);
    up.err = h->err;
    up.timeout_ns = h->timeout_ns;
    up.kblock = h->kblock;
    up.gather = gather_in_gemm ? 1 : 0;
    up.accf = acc_factor(h);
    if (ts) {
        up.part = static_cast<float *>(h->b_part.ptr);
        up.tickets = reinterpret_cast<unsigned int *>(h->err + kCtlTickets);
    }
    if (timed(h, K_UP, s, [&] { return launch_up(h, bn, m_wl, m_wv, ts ? *m_b : *m_xp, up, s); }) != cudaSuccess)
        return MOE_ECUDA;

    GemmArgs dn = up;
    dn.gather = 0;
    dn.M = h->d;
    dn.K = h->F;
    dn.splits = splits;
    dn.ksteps = h->F / kstage_of(h, false, bn) / splits;
    dn.s0 = static_cast<const __nv_bfloat16 *>(s_1);
    dn.s1 = nullptr;
    dn.h = nullptr;
    dn.slots = static_cast<float *>(h->b_slots.ptr);
    if (timed(h, K_DOWN, s, [&] { return launch_down(h, bn, m_w1, *m_h, dn, s); }) != cudaSuccess)
        return MOE_ECUDA;

    h->last_block_T = g_pre ? T : -1;
    h->stage_scaled = g_pre && gather_in_gemm;   // u in the staging buffer is at kActScale
    h->ep_T = -1;   // the route buffer now holds this forward's routing
    CombineArgs ca{T, h->d, splits, static_cast<const float *>(h->b_slots.ptr), idx, static_cast<__nv_bfloat16 *>(out),
                   static_cast<__nv_bfloat16 *>(h_io), static_cast<const __nv_bfloat16 *>(g_post), eps};
    if (timed(h, K_COMBINE, s, [&] { return launch_combine(ca, s); }) != cudaSuccess) return MOE_ECUDA;
    h->last_T = T;
    return MOE_OK;
}

int begin_call(moe_ctx *h, int T, cudaStream_t s)
{
    int rc;
    if ((rc = ensure_device(h)) != MOE_OK) return rc;
    if (h->used && s != h->last_stream) {
        // work of the previous stream may still use the workspace
        if (cudaStreamSynchronize(h->last_stream) != cudaSuccess) return MOE_ECUDA;
    }
    const int bn = plan_bn(h, T);
    if ((rc = ensure_workspace(h, T, bn, plan_splits(h, T, bn))) != MOE_OK) return rc;
    h->last_stream = s;
    h->used = true;
    return MOE_OK;
}

// the up-projection launch of the handle's layout and plan: CTA pairs where the plan has them and
// the device can hold a wave of them, else one CTA per tile.  m_b: the routed-rows map (one-row
// boxes) when up.gather, else the gathered rows with bn-row boxes.
cudaError_t launch_up(moe_ctx *h, int bn, const CUtensorMap &m_wl, const CUtensorMap &m_wv, const CUtensorMap &m_b,
                      const GemmArgs &up, cudaStream_t s)
{
    if (h->layout != MOE_LAYOUT_PACKED) return launch_gemm_up(bn, m_wl, m_wv, m_b, up, h->num_sms, s);
    if (pairs_for(h, bn, true) && gemm_pair_ready(true, bn, h->num_sms)) {
        if (up.gather) return launch_gemm_up_pair(bn, m_wl, m_wv, m_b, up, h->num_sms, s);
        const CUtensorMap *xph, *hh;   // maps with boxes of half a pair tile
        if (act_maps(h, gemm_pair_tn(true, bn) / 2, &xph, &hh) == MOE_OK)
            return launch_gemm_up_pair(bn, m_wl, m_wv, *xph, up, h->num_sms, s);
    }
    return launch_gemm_up_ts(bn, m_wl, m_wv, m_b, up, h->num_sms, s);
}

// the down-projection launch: CTA pairs where the plan has them (same rule as launch_up)
cudaError_t launch_down(moe_ctx *h, int bn, const CUtensorMap &m_w1, const CUtensorMap &m_h, const GemmArgs &dn,
                        cudaStream_t s)
{
    if (h->layout != MOE_LAYOUT_PACKED) return launch_gemm_down(bn, m_w1, m_h, dn, h->num_sms, s);
    if (pairs_for(h, bn, false) && gemm_pair_ready(false, bn, h->num_sms)) {
        const CUtensorMap *xph, *hh;
        if (act_maps(h, gemm_pair_tn(false, bn) / 2, &xph, &hh) == MOE_OK)
            return launch_gemm_down_pair(bn, m_w1, *hh, dn, h->num_sms, s);
    }
    return launch_gemm_down_ts(bn, m_w1, m_h, dn, h->num_sms, s);
}

// ---- expert parallelism (device steps; the exchange between ranks is the caller's) ----------

// the expert-parallel layout arrays in b_ep, in 4-byte words
struct EpLayout {
    size_t counts, offsets, poff, rperm, slot, ones, words;
};

EpLayout ep_layout(int rows, int R)
{
    auto up = [](size_t v) { return (v + 63) / 64 * 64; };
    EpLayout L;
    size_t o = 0;
    L.counts = o; o += 64;
    L.offsets = o; o += 128;
    L.poff = o; o += 128;
    L.rperm = o; o += up(rows);
    L.slot = o; o += up(R);
    L.ones = o; o += up(R);
    L.words = o;
    return L;
}

// routing + grouping by expert (no padding: grouped row i is route perm[i]) + the routed rows
// gathered into send_rows in that order
int run_ep_dispatch(moe_ctx *h, int T, const void *x, const float *router_w, void *send_rows, int32_t *send_counts,
                    cudaStream_t s)
{
    const RouteLayout L = route_layout(T, h->E);
    int *rw = static_cast<int *>(h->b_route.ptr);
    int *idx = rw + L.idx;
    float *gate = reinterpret_cast<float *>(rw + L.gate);
    RouteArgs ra{T, h->d, static_cast<const __nv_bfloat16 *>(x), router_w, h->bias, idx, gate};
    ra.mask = h->mask;
    DispatchArgs da{T, h->E, 1, idx, rw + L.counts, rw + L.offsets, rw + L.poff, rw + L.perm,
                    static_cast<int *>(h->b_rperm.ptr), rw + L.slot};
    GatherArgs ga{h->d, static_cast<const __nv_bfloat16 *>(x), static_cast<__nv_bfloat16 *>(send_rows)};
    if (T <= route_small_max_tokens()) {
        unsigned int *ticket = reinterpret_cast<unsigned int *>(h->err + kCtlRouteTicket);
        float *part = static_cast<float *>(h->b_slots.ptr);
        const int S = route_small_slices(T, h->d, h->num_sms);
        if (timed(h, K_ROUTE_SMALL, s, [&] { return launch_route_small(ra, da, ga, part, S, ticket, s); }) !=
            cudaSuccess)
            return MOE_ECUDA;
    } else {
        if (timed(h, K_ROUTER, s, [&] { return launch_router(ra, s); }) != cudaSuccess) return MOE_ECUDA;
        if (timed(h, K_DISPATCH, s, [&] { return launch_dispatch(da, s); }) != cudaSuccess) return MOE_ECUDA;
        if (timed(h, K_GATHER, s, [&] { return launch_gather(ga, T, rw + L.slot, s); }) != cudaSuccess)
            return MOE_ECUDA;
    }
    if (cudaMemcpyAsync(send_counts, rw + L.counts, static_cast<size_t>(h->E) * 4, cudaMemcpyDeviceToDevice, s) !=
        cudaSuccess)
        return MOE_ECUDA;
    h->last_T = T;
    h->last_block_T = -1;
    h->ep_T = T;
    return MOE_OK;
}

int run_ep_experts(moe_ctx *h, int n_src, int E_local, const int32_t *counts, int R, int max_rows,
                   const void *recv_rows, const int8_t *w_lin, const void *s_lin, const int8_t *w_v, const void *s_v,
                   const int8_t *w_1, const void *s_1, float *y_rows, cudaStream_t s)
{
    int rc;
    const int bn = plan_bn_rows(h, max_rows);
    const int splits = splits_for(h, E_local, max_rows, bn);
    const int Tp = (R + 1) / 2;   // the down-projection's slots [splits, Tp, 2, d] hold rows [splits, 2 Tp, d]
    const int rows = ((R + E_local * (bn - 1)) + 127) / 128 * 128;
    if ((rc = ensure_rows(h, rows)) != MOE_OK) return rc;
    if (splits > 1 && (rc = ensure(h, h->b_slots, static_cast<size_t>(splits) * Tp * 2 * h->d * 4)) != MOE_OK)
        return rc;
    if (h->layout == MOE_LAYOUT_PACKED &&
        (rc = ensure(h, h->b_part, static_cast<size_t>(h->num_sms) * 128 * 256 * 4)) != MOE_OK)
        return rc;
    const EpLayout L = ep_layout(h->rows_cap, R);
    if ((rc = ensure(h, h->b_ep, L.words * 4)) != MOE_OK) return rc;

    const bool ts = h->layout == MOE_LAYOUT_PACKED;
    if (h->kblock && !ts) return MOE_EUNSUPPORTED;
    CUtensorMap m_wl, m_wv, m_w1;
    const CUtensorMap *m_xp, *m_h;
    if ((rc = weight_map(h, w_lin, 0, &m_wl, E_local)) != MOE_OK) return rc;
    if ((rc = weight_map(h, w_v, 0, &m_wv, E_local)) != MOE_OK) return rc;
    if ((rc = weight_map(h, w_1, 1, &m_w1, E_local)) != MOE_OK) return rc;
    if ((rc = act_maps(h, bn, &m_xp, &m_h)) != MOE_OK) return rc;

    int *ew = static_cast<int *>(h->b_ep.ptr);
    float *ones = reinterpret_cast<float *>(ew + L.ones);
    EpLayoutArgs la{};
    la.n_src = n_src;
    la.E_local = E_local;
    la.bn = bn;
    la.R = R;
    for (int i = 0; i < n_src * E_local; ++i) la.recv_counts[i] = counts[i];
    la.counts = ew + L.counts;
    la.offsets = ew + L.offsets;
    la.poff = ew + L.poff;
    la.rperm = ew + L.rperm;
    la.slot = ew + L.slot;
    la.ones = ones;
    if (timed(h, K_DISPATCH, s, [&] { return launch_ep_layout(la, s); }) != cudaSuccess) return MOE_ECUDA;
    if (timed(h, K_GATHER, s, [&] {
            return launch_ep_gather(R, h->d, static_cast<const __nv_bfloat16 *>(recv_rows), la.slot,
                                    static_cast<__nv_bfloat16 *>(h->b_xp.ptr), ts ? 1 : 0, s);
        }) != cudaSuccess)
        return MOE_ECUDA;

    GemmArgs up{};
    up.T = Tp;
    up.E = E_local;
    up.M = h->F;
    up.K = h->d;
    up.ksteps = h->d / kstage_of(h, true, bn);
    up.splits = 1;
    up.poff = la.poff;
    up.offsets = la.offsets;
    up.rperm = la.rperm;
    up.gate = ones;
    up.s0 = static_cast<const __nv_bfloat16 *>(s_lin);
    up.s1 = static_cast<const __nv_bfloat16 *>(s_v);
    up.h = static_cast<__nv_bfloat16 *>(h->b_h.ptr);
    up.err = h->err;
    up.timeout_ns = h->timeout_ns;
    up.kblock = h->kblock;
    up.gather = 0;
    up.accf = acc_factor(h);
    if (ts) {
        up.part = static_cast<float *>(h->b_part.ptr);
        up.tickets = reinterpret_cast<unsigned int *>(h->err + kCtlTickets);
    }
    if (timed(h, K_UP, s, [&] { return launch_up(h, bn, m_wl, m_wv, *m_xp, up, s); }) != cudaSuccess)
        return MOE_ECUDA;
    GemmArgs dn = up;
    dn.M = h->d;
    dn.K = h->F;
    dn.splits = splits;
    dn.ksteps = h->F / kstage_of(h, false, bn) / splits;
    dn.s0 = static_cast<const __nv_bfloat16 *>(s_1);
    dn.s1 = nullptr;
    dn.h = nullptr;
    // one split: route id i lands in row i of [Tp, 2, d] = y_rows itself
    dn.slots = splits == 1 ? y_rows : static_cast<float *>(h->b_slots.ptr);
    if (timed(h, K_DOWN, s, [&] { return launch_down(h, bn, m_w1, *m_h, dn, s); }) != cudaSuccess)
        return MOE_ECUDA;
    if (splits > 1 && timed(h, K_COMBINE, s, [&] {
            return launch_ep_split_sum(R, h->d, splits, static_cast<size_t>(Tp) * 2 * h->d,
                                       static_cast<const float *>(h->b_slots.ptr), y_rows, s);
        }) != cudaSuccess)
        return MOE_ECUDA;
    return MOE_OK;
}

}  // namespace

extern "C" {

MOE_API const char *moe_strerror(int code)
{
    switch (code) {
    case MOE_OK: return "ok";
    case MOE_EINVAL: return "invalid argument";
    case MOE_EUNSUPPORTED: return "unsupported shape or option";
    case MOE_ENOMEM: return "out of device memory";
    case MOE_ECUDA: return "CUDA error";
    case MOE_ETIMEOUT: return "device-side wait timed out";
    case MOE_ENODEV: return "no sm_100 CUDA device";
    case MOE_ERANGE: return "weight value outside the layout's range";
    default: return "unknown status code";
    }
}

MOE_API int moe_version(void) { return 100; }

MOE_API int moe_create(int d, int ffn, int E, int k, moe_handle *out)
{
    if (!out) return MOE_EINVAL;
    *out = nullptr;
    if (d <= 0 || ffn <= 0 || E <= 0 || k <= 0 || k > E) return MOE_EINVAL;
    if (E != kExperts || k != kTopK) return MOE_EUNSUPPORTED;
    if (d % kBM || ffn % kBM || d < kBM || ffn < kBM || d > 65536 || ffn > 65536) return MOE_EUNSUPPORTED;
    moe_ctx *h = new (std::nothrow) moe_ctx();
    if (!h) return MOE_ENOMEM;
    h->d = d;
    h->F = ffn;
    h->E = E;
    h->k = k;
    *out = h;
    return MOE_OK;
}

MOE_API int moe_destroy(moe_handle h)
{
    if (!h) return MOE_OK;
    sync_last(h);
    for (DevBuf *b : {&h->b_route, &h->b_rperm, &h->b_xp, &h->b_h, &h->b_slots, &h->b_stage, &h->b_ep, &h->b_host[0],
                      &h->b_host[1]})
        if (b->ptr) cudaFree(b->ptr);
    for (int k = 0; k < 2; ++k) {
        if (h->ev_in[k]) cudaEventDestroy(h->ev_in[k]);
        if (h->ev_layer[k]) cudaEventDestroy(h->ev_layer[k]);
        if (h->ev_done[k]) cudaEventDestroy(h->ev_done[k]);
    }
    if (h->copy_in) cudaStreamDestroy(h->copy_in);
    if (h->copy_out) cudaStreamDestroy(h->copy_out);
    if (h->err) cudaFree(h->err);
    if (h->b_part.ptr) cudaFree(h->b_part.ptr);
    for (auto &p : h->pending) {
        cudaEventDestroy(p.a);
        cudaEventDestroy(p.b);
    }
    for (auto e : h->event_pool) cudaEventDestroy(e);
    delete h;
    return MOE_OK;
}

MOE_API int moe_set_router_bias(moe_handle h, const float *bias)
{
    if (!h) return MOE_EINVAL;
    if (bias && !aligned16(bias)) return MOE_EINVAL;
    h->bias = bias;
    return MOE_OK;
}

MOE_API int moe_set_padding_mask(moe_handle h, const uint8_t *mask)
{
    if (!h) return MOE_EINVAL;
    h->mask = mask;
    return MOE_OK;
}

MOE_API int moe_set_scale_block(moe_handle h, int kb)
{
    if (!h) return MOE_EINVAL;
    if (kb != 0 && kb != kScaleBlock) return MOE_EUNSUPPORTED;
    if (kb && (h->d % kb || h->F % kb)) return MOE_EINVAL;
    h->kblock = kb;
    return MOE_OK;
}

MOE_API int moe_set_timeout(moe_handle h, long long ns)
{
    if (!h || ns < 0) return MOE_EINVAL;
    h->timeout_ns = ns;
    return MOE_OK;
}

MOE_API int moe_set_cta_pairs(moe_handle h, int mode)
{
    if (!h || mode < 0 || mode > 3) return MOE_EINVAL;
    h->cta_pairs = mode;
    return MOE_OK;
}

MOE_API int moe_set_weight_layout(moe_handle h, int layout)
{
    if (!h || (layout != MOE_LAYOUT_IN_OUT && layout != MOE_LAYOUT_PACKED)) return MOE_EINVAL;
    h->layout = layout;
    return MOE_OK;
}

MOE_API int moe_pack_weight_n(moe_handle h, const int8_t *w, int8_t *w_packed, int which, int n_experts,
                              void *stream)
{
    if (!h || !w || !w_packed || !aligned16(w) || !aligned16(w_packed)) return MOE_EINVAL;
    if (which != 0 && which != 1) return MOE_EINVAL;
    if (n_experts < 1 || n_experts > h->E) return MOE_EINVAL;
    const size_t bytes = static_cast<size_t>(n_experts) * h->d * h->F;
    if (overlaps(w, bytes, w_packed, bytes)) return MOE_EINVAL;
    int rc = ensure_device(h);
    if (rc != MOE_OK) return rc;
    const int K = which == 0 ? h->d : h->F, M = which == 0 ? h->F : h->d;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int *flag = h->err + kCtlPackRange;
    int minus128 = 0;
    if (cudaMemsetAsync(flag, 0, sizeof(int), s) != cudaSuccess ||
        launch_pack_i8(w, w_packed, n_experts, K, M, flag, s) != cudaSuccess ||
        cudaMemcpyAsync(&minus128, flag, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return MOE_ECUDA;
    return minus128 ? MOE_ERANGE : MOE_OK;
}

MOE_API int moe_pack_weight(moe_handle h, const int8_t *w, int8_t *w_packed, int which, void *stream)
{
    return moe_pack_weight_n(h, w, w_packed, which, h ? h->E : 0, stream);
}

MOE_API int moe_plan(moe_handle h, int T, int *bn, int *splits)
{
    if (!h || T < 0 || T > MOE_MAX_TOKENS) return MOE_EINVAL;
    const int b = plan_bn(h, T);
    if (bn) *bn = b;
    if (splits) *splits = plan_splits(h, T, b);
    return MOE_OK;
}

MOE_API int moe_forward(moe_handle h, int T, const void *x, const float *router_w, const int8_t *w_lin,
                        const void *s_lin, const int8_t *w_v, const void *s_v, const int8_t *w_1, const void *s_1,
                        void *out, void *stream)
{
    if (!h || T < 0 || T > MOE_MAX_TOKENS) return MOE_EINVAL;
    if (T == 0) return MOE_OK;
    if (!x || !out || !aligned16(x) || !aligned16(out)) return MOE_EINVAL;
    int rc = check_weights(h, router_w, w_lin, s_lin, w_v, s_v, w_1, s_1);
    if (rc != MOE_OK) return rc;
    const size_t xb = static_cast<size_t>(T) * h->d * 2;
    if (overlaps(x, xb, out, xb)) return MOE_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((rc = begin_call(h, T, s)) != MOE_OK) return rc;
    return run_layer(h, T, x, router_w, w_lin, s_lin, w_v, s_v, w_1, s_1, out, nullptr, nullptr, nullptr, 0.f, s);
}

MOE_API int moe_forward_host(moe_handle h, int T, const void *x_host, const float *router_w, const int8_t *w_lin,
                             const void *s_lin, const int8_t *w_v, const void *s_v, const int8_t *w_1,
                             const void *s_1, void *out_host, void *stream)
{
    if (!h || T < 0 || T > MOE_MAX_TOKENS) return MOE_EINVAL;
    if (T == 0) return MOE_OK;
    if (!x_host || !out_host) return MOE_EINVAL;
    int rc = check_weights(h, router_w, w_lin, s_lin, w_v, s_v, w_1, s_1);
    if (rc != MOE_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((rc = begin_call(h, T, s)) != MOE_OK) return rc;
    const size_t xb = static_cast<size_t>(T) * h->d * 2;
    if (!h->host_overlap) {
        // output copies of earlier overlapped calls may still be running on copy_out: land them first
        // (this call may write the same host buffer)
        for (int k = 0; k < 2; ++k)
            if (h->slot_used[k] && cudaStreamWaitEvent(s, h->ev_done[k], 0) != cudaSuccess) return MOE_ECUDA;
        char *xs = static_cast<char *>(h->b_stage.ptr);
        char *os = xs + xb;
        if (cudaMemcpyAsync(xs, x_host, xb, cudaMemcpyHostToDevice, s) != cudaSuccess) return MOE_ECUDA;
        if ((rc = run_layer(h, T, xs, router_w, w_lin, s_lin, w_v, s_v, w_1, s_1, os, nullptr, nullptr, nullptr, 0.f,
                            s)) != MOE_OK)
            return rc;
        if (cudaMemcpyAsync(out_host, os, xb, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ECUDA;
        return MOE_OK;
    }
    // host overlap: slot k alternates between calls; the input copy runs on copy_in, the output
    // copy on copy_out
    if (!h->copy_in) {
        if (cudaStreamCreateWithFlags(&h->copy_in, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&h->copy_out, cudaStreamNonBlocking) != cudaSuccess)
            return MOE_ECUDA;
        for (int j = 0; j < 2; ++j)
            if (cudaEventCreateWithFlags(&h->ev_in[j], cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&h->ev_layer[j], cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&h->ev_done[j], cudaEventDisableTiming) != cudaSuccess)
                return MOE_ECUDA;
    }
    const int k = h->host_slot, o = k ^ 1;
    if ((rc = ensure(h, h->b_host[k], 2 * xb)) != MOE_OK) return rc;
    char *xs = static_cast<char *>(h->b_host[k].ptr);
    char *os = xs + xb;
    // the copy in waits for the slot's previous call, and for the other slot's pending output
    // when this input overlaps it (layers chained through host memory)
    const char *xh = static_cast<const char *>(x_host);
    const bool reads_pending = h->slot_used[o] && xh < h->slot_out[o] + h->slot_out_bytes[o] && h->slot_out[o] < xh + xb;
    if (h->slot_used[k] && cudaStreamWaitEvent(h->copy_in, h->ev_done[k], 0) != cudaSuccess) return MOE_ECUDA;
    if (reads_pending && cudaStreamWaitEvent(h->copy_in, h->ev_done[o], 0) != cudaSuccess) return MOE_ECUDA;
    if (cudaMemcpyAsync(xs, x_host, xb, cudaMemcpyHostToDevice, h->copy_in) != cudaSuccess ||
        cudaEventRecord(h->ev_in[k], h->copy_in) != cudaSuccess || cudaStreamWaitEvent(s, h->ev_in[k], 0) != cudaSuccess)
        return MOE_ECUDA;
    if ((rc = run_layer(h, T, xs, router_w, w_lin, s_lin, w_v, s_v, w_1, s_1, os, nullptr, nullptr, nullptr, 0.f, s)) !=
        MOE_OK)
        return rc;
    // the result goes out on copy_out once the layer has written it; the next call's layer on s does
    // not wait for it (it uses the other slot), and this slot's next input copy, on which the
    // layer that reuses the slot waits, waits for it (ev_done)
    if (cudaEventRecord(h->ev_layer[k], s) != cudaSuccess || cudaStreamWaitEvent(h->copy_out, h->ev_layer[k], 0) != cudaSuccess ||
        cudaMemcpyAsync(out_host, os, xb, cudaMemcpyDeviceToHost, h->copy_out) != cudaSuccess ||
        cudaEventRecord(h->ev_done[k], h->copy_out) != cudaSuccess)
        return MOE_ECUDA;
    h->slot_used[k] = true;
    h->slot_out[k] = static_cast<const char *>(out_host);
    h->slot_out_bytes[k] = xb;
    h->host_slot = o;
    return MOE_OK;
}

MOE_API int moe_set_host_overlap(moe_handle h, int on)
{
    if (!h || (on != 0 && on != 1)) return MOE_EINVAL;
    h->host_overlap = on != 0;
    return MOE_OK;
}

MOE_API int moe_host_wait(moe_handle h, void *stream)
{
    if (!h) return MOE_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    for (int k = 0; k < 2; ++k)
        if (h->slot_used[k] && cudaStreamWaitEvent(s, h->ev_done[k], 0) != cudaSuccess) return MOE_ECUDA;
    return MOE_OK;
}

MOE_API int moe_block_forward(moe_handle h, int T, void *h_io, const void *g_pre, const void *g_post, float eps,
                              const float *router_w, const int8_t *w_lin, const void *s_lin, const int8_t *w_v,
                              const void *s_v, const int8_t *w_1, const void *s_1, void *stream)
{
    if (!h || T < 0 || T > MOE_MAX_TOKENS) return MOE_EINVAL;
    if (T == 0) return MOE_OK;
    if (!h_io || !g_pre || !g_post || !aligned16(h_io) || !aligned16(g_pre) || !aligned16(g_post)) return MOE_EINVAL;
    if (!(eps >= 0.f)) return MOE_EINVAL;
    int rc = check_weights(h, router_w, w_lin, s_lin, w_v, s_v, w_1, s_1);
    if (rc != MOE_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((rc = begin_call(h, T, s)) != MOE_OK) return rc;
    return run_layer(h, T, h_io, router_w, w_lin, s_lin, w_v, s_v, w_1, s_1, nullptr, h_io, g_pre, g_post, eps, s);
}

MOE_API int moe_get_routing(moe_handle h, int32_t *idx, float *gate, int32_t *offsets, int32_t *perm, void *stream)
{
    if (!h || h->last_T < 0) return MOE_EINVAL;
    const int T = h->last_T;
    const RouteLayout L = route_layout(T, h->E);
    const int *rw = static_cast<const int *>(h->b_route.ptr);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    struct {
        void *dst;
        const void *src;
        size_t bytes;
    } cp[] = {{idx, rw + L.idx, 2 * static_cast<size_t>(T) * 4},
              {gate, rw + L.gate, 2 * static_cast<size_t>(T) * 4},
              {offsets, rw + L.offsets, static_cast<size_t>(h->E + 1) * 4},
              {perm, rw + L.perm, 2 * static_cast<size_t>(T) * 4}};
    for (auto &c : cp)
        if (c.dst && cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
            return MOE_ECUDA;
    return MOE_OK;
}

MOE_API int moe_get_block_input(moe_handle h, void *u, void *stream)
{
    if (!h || !u || !aligned16(u) || h->last_block_T < 0) return MOE_EINVAL;
    const size_t n = static_cast<size_t>(h->last_block_T) * h->d;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t e =
        h->stage_scaled
            ? launch_scale_rows(static_cast<const __nv_bfloat16 *>(h->b_stage.ptr), static_cast<__nv_bfloat16 *>(u), n,
                                kActUnscale, s)
            : cudaMemcpyAsync(u, h->b_stage.ptr, n * 2, cudaMemcpyDeviceToDevice, s);
    return e == cudaSuccess ? MOE_OK : MOE_ECUDA;
}

MOE_API int moe_sync_status(moe_handle h, void *stream)
{
    if (!h) return MOE_EINVAL;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ECUDA;
    // host-overlap copies run on the handle's own streams
    if (h->copy_in && cudaStreamSynchronize(h->copy_in) != cudaSuccess) return MOE_ECUDA;
    if (h->copy_out && cudaStreamSynchronize(h->copy_out) != cudaSuccess) return MOE_ECUDA;
    if (!h->err) return MOE_OK;
    int e = 0;
    if (cudaMemcpy(&e, h->err, sizeof e, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ECUDA;
    if (e == 0) return MOE_OK;
    // a kernel that gave up may have left tickets taken: clear the whole control block
    cudaMemset(h->err, 0, kCtlWords * 4);
    return e >= kErrTimeoutBase ? MOE_ETIMEOUT : MOE_ECUDA;
}

MOE_API int moe_set_profiling(moe_handle h, int on)
{
    if (!h) return MOE_EINVAL;
    h->prof = on != 0;
    return MOE_OK;
}

MOE_API int moe_get_kernel_times(moe_handle h, float *ms, int *launches, int n)
{
    if (!h || n < 0) return MOE_EINVAL;
    for (int i = 0; i < n; ++i) {
        if (ms) ms[i] = 0.f;
        if (launches) launches[i] = 0;
    }
    int rc = MOE_OK;
    for (auto &p : h->pending) {
        float t = 0.f;
        if (cudaEventSynchronize(p.b) != cudaSuccess || cudaEventElapsedTime(&t, p.a, p.b) != cudaSuccess) {
            cudaGetLastError();
            rc = MOE_ECUDA;
        } else if (p.id < n) {
            if (ms) ms[p.id] += t;
            if (launches) launches[p.id] += 1;
        }
        h->event_pool.push_back(p.a);
        h->event_pool.push_back(p.b);
    }
    h->pending.clear();
    return rc;
}

MOE_API int moe_ep_dispatch(moe_handle h, int T, const void *x, const float *router_w, void *send_rows,
                            int32_t *send_counts, void *stream)
{
    if (!h || T < 0 || T > MOE_MAX_TOKENS) return MOE_EINVAL;
    if (!send_counts || !aligned16(send_counts)) return MOE_EINVAL;
    if (T == 0) {   // nothing to route: every count is 0
        h->ep_T = 0;
        return cudaMemsetAsync(send_counts, 0, static_cast<size_t>(h->E) * 4, static_cast<cudaStream_t>(stream)) ==
                       cudaSuccess
                   ? MOE_OK
                   : MOE_ECUDA;
    }
    if (!x || !router_w || !send_rows) return MOE_EINVAL;
    if (!aligned16(x) || !aligned16(router_w) || !aligned16(send_rows) || !aligned16(send_counts)) return MOE_EINVAL;
    const size_t xb = static_cast<size_t>(T) * h->d * 2;
    if (overlaps(x, xb, send_rows, 2 * xb)) return MOE_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int rc = begin_call(h, T, s);
    if (rc != MOE_OK) return rc;
    return run_ep_dispatch(h, T, x, router_w, send_rows, send_counts, s);
}

MOE_API int moe_ep_experts(moe_handle h, int n_src, int E_local, const int32_t *recv_counts, const void *recv_rows,
                           const int8_t *w_lin, const void *s_lin, const int8_t *w_v, const void *s_v,
                           const int8_t *w_1, const void *s_1, float *y_rows, void *stream)
{
    if (!h || n_src < 1 || E_local < 1 || E_local > h->E || !recv_counts) return MOE_EINVAL;
    if (static_cast<long>(n_src) * E_local > kEpMaxRuns) return MOE_EUNSUPPORTED;
    long R = 0, max_rows = 0;
    for (int k = 0; k < E_local; ++k) {
        long n = 0;
        for (int src = 0; src < n_src; ++src) {
            const int c = recv_counts[src * E_local + k];
            if (c < 0) return MOE_EINVAL;
            n += c;
        }
        max_rows = n > max_rows ? n : max_rows;
        R += n;
    }
    if (R > 2L * MOE_MAX_TOKENS) return MOE_EINVAL;   // more rows than the workspace plans for
    if (R == 0) return MOE_OK;
    if (!recv_rows || !y_rows || !aligned16(recv_rows) || !aligned16(y_rows)) return MOE_EINVAL;
    const void *ws[] = {w_lin, s_lin, w_v, s_v, w_1, s_1};
    for (const void *p : ws)
        if (!p || !aligned16(p)) return MOE_EINVAL;
    int rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((rc = ensure_device(h)) != MOE_OK) return rc;
    if (h->used && s != h->last_stream && cudaStreamSynchronize(h->last_stream) != cudaSuccess) return MOE_ECUDA;
    h->last_stream = s;
    h->used = true;
    return run_ep_experts(h, n_src, E_local, recv_counts, static_cast<int>(R), static_cast<int>(max_rows), recv_rows,
                          w_lin, s_lin, w_v, s_v, w_1, s_1, y_rows, s);
}

MOE_API int moe_ep_combine(moe_handle h, int T, const float *y_back, void *out, void *stream)
{
    if (!h || T < 0 || T != h->ep_T) return MOE_EINVAL;
    if (T == 0) return MOE_OK;
    if (!y_back || !out || !aligned16(y_back) || !aligned16(out)) return MOE_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (s != h->last_stream && cudaStreamSynchronize(h->last_stream) != cudaSuccess) return MOE_ECUDA;
    h->last_stream = s;
    const RouteLayout L = route_layout(T, h->E);
    const int *rw = static_cast<const int *>(h->b_route.ptr);
    EpCombineArgs ca{T, h->d, rw + L.idx, reinterpret_cast<const float *>(rw + L.gate), rw + L.slot, y_back,
                     static_cast<__nv_bfloat16 *>(out)};
    return timed(h, K_COMBINE, s, [&] { return launch_ep_combine(ca, s); }) == cudaSuccess ? MOE_OK : MOE_ECUDA;
}

}  // extern "C"
