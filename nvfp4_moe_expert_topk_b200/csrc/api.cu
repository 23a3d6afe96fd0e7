// api.cu -- the C ABI of libnvfp4moe.so (declared in include/nvfp4moe.h):
// argument checks, workspace layout, tensor-map creation and the launch
// sequence of each entry point.  No allocation, no host synchronisation
// (except nvfp4_moe_get_error), everything on the caller's stream.
#include <mutex>

#include "internal.h"

using namespace nvfp4;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    int checked = 0;      // 1 ok, -1 unsupported
    int num_sms = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mutex;

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Current device must be sm_100 (B200).  Caches the SM count.
int device_check(int *num_sms)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return NVFP4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo &d = g_dev[dev];
    if (d.checked == 0) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        d.checked = (major == 10 && minor == 0) ? 1 : -1;
        d.num_sms = sms;
    }
    if (d.checked < 0)
        return NVFP4_ERR_UNSUPPORTED_DEVICE;
    if (num_sms)
        *num_sms = d.num_sms;
    if (g_encode == nullptr) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return NVFP4_ERR_CUDA;
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    return NVFP4_OK;
}

// 2-D uint8 tensor map over a row-major code matrix [rows, cols_bytes]
// (row stride cols_bytes), box box_rows rows x 128 bytes, 128-byte swizzle;
// rows and columns outside the matrix read as zero.
int make_code_map(CUtensorMap *map, const void *base, int64_t rows, int64_t cols_bytes, int box_rows)
{
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols_bytes), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols_bytes)};
    cuuint32_t box[2] = {128, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// bf16 output [rows, ldo] for the staged epilogue stores: 32 x 32 boxes,
// 64-byte swizzle (a box row is 64 bytes).
int make_out_map(CUtensorMap *map, void *base, int64_t rows, int64_t cols, int64_t ldo)
{
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldo * 2)};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? NVFP4_OK : NVFP4_ERR_CUDA;
}

bool aligned16(const void *p)
{
    return (reinterpret_cast<uintptr_t>(p) & 15) == 0;
}

int cuda_status(cudaError_t e)
{
    return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

int64_t round_up(int64_t v, int64_t m)
{
    return (v + m - 1) / m * m;
}

// ---------------------------------------------------------------- workspace
struct Layout {
    int64_t mt_max = 0, rpad = 0, sfa_block = 0;
    int64_t counts = 0, off = 0, poff = 0, mtiles = 0, pairs = 0, light = 0, ready = 0, inv = 0, yrow = 0, amax = 0;
    int64_t blk_hist = 0, blk_amax = 0;
    int64_t a_codes = 0, a_sf = 0, h_codes = 0, h_sf = 0, y = 0, total = 0;
};

// Header (256 B): int32 error word at 0, int32 m-tile count at 4, int32
// m-tile pair count at 8, fp32 global scale of x computed from the batch at
// 12, the front launch's grid ticket at 20, int32 light m-tile count at 24,
// the fused 1-CTA launch's tile claim counter at 28.
constexpr int kHdrNumMtiles = 4, kHdrNumPairs = 8, kHdrGs = 12, kHdrTicket = 20, kHdrNumLight = 24, kHdrClaim = 28;

Layout ws_layout(int64_t T, int k, int E, int64_t H, int64_t I)
{
    Layout L;
    const int64_t R = T * k;
    const int64_t ne = std::min<int64_t>(E, R);
    L.mt_max = (R + 127 * ne) / 128;          // >= sum_e ceil(count_e / 128)
    L.rpad = 128 * L.mt_max;
    L.sfa_block = ((H + 255) / 256) * 2048;  // x scales in row blocks: per 128 rows, 2 KB per k-tile
    int64_t o = 256;
    auto take = [&](int64_t bytes) {
        const int64_t at = o;
        o = round_up(o + bytes, 1024);
        return at;
    };
    L.counts = take(4 * E);
    L.off = take(4 * (E + 1));
    L.poff = take(4 * (E + 1));
    L.amax = take(4 * E);
    L.mtiles = take(16 * std::max<int64_t>(L.mt_max, 1));
    L.pairs = take(8 * std::max<int64_t>(L.mt_max, 1));
    L.light = take(4 * std::max<int64_t>(L.mt_max, 1));
    L.ready = take(4 * std::max<int64_t>(L.mt_max, 1));
    L.inv = take(4 * std::max<int64_t>(R, 1));
    L.yrow = take(4 * std::max<int64_t>(R, 1));
    L.blk_hist = take(4LL * kFrontMaxBlocks * ((E + 3) & ~3));
    L.blk_amax = take(4LL * kFrontMaxBlocks);
    L.a_codes = take(L.rpad * (H / 2));
    L.a_sf = take((L.rpad / 128) * L.sfa_block);
    L.h_codes = take(L.rpad * (I / 2));
    L.h_sf = take(L.rpad * (I / 16));
    L.y = take(R * H * 2);
    L.total = o;
    return L;
}

int check_moe_shape(int64_t T, int k, int E, int64_t H, int64_t I)
{
    if (T < 0 || H <= 0 || I <= 0 || E < 1 || k < 1)
        return NVFP4_ERR_INVALID_ARG;
    if (H % 128 != 0 || I % 128 != 0 || E > 1024 || k > 32 || T * k >= (1LL << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (H > (1LL << 20) || I > (1LL << 20) || static_cast<int64_t>(E) * 2 * I >= (1LL << 31) ||
        static_cast<int64_t>(E) * H >= (1LL << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    return NVFP4_OK;
}

// need_x false: the activations come pre-quantised (x is not read, x_gs is
// required instead).
int check_moe_args(const nvfp4_moe_args *a, bool need_out, bool need_x = true)
{
    if (a == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    int st = check_moe_shape(a->T, a->k, a->E, a->H, a->I);
    if (st != NVFP4_OK)
        return st;
    // an empty batch (T = 0) reads and writes nothing of the batch: its
    // pointers (x or x_gs, topk_ids, topk_weights, out) may then be NULL
    const bool batch = a->T > 0;
    const void *batch_ptrs[] = {need_x ? static_cast<const void *>(a->x) : static_cast<const void *>(a->x_gs),
                                a->topk_ids, a->topk_weights};
    for (const void *p : batch_ptrs)
        if (batch && p == nullptr)
            return NVFP4_ERR_INVALID_ARG;
    const void *weight_ptrs[] = {a->w13_codes, a->w13_scales, a->w13_gs, a->w2_codes, a->w2_scales, a->w2_gs};
    for (const void *p : weight_ptrs)
        if (p == nullptr)
            return NVFP4_ERR_INVALID_ARG;
    if (need_out && ((batch && a->out == nullptr) || a->inter_gs == nullptr))
        return NVFP4_ERR_INVALID_ARG;
    const void *al[] = {a->w13_codes, a->w13_scales, a->w2_codes, a->w2_scales};
    for (const void *p : al)
        if (!aligned16(p))
            return NVFP4_ERR_MISALIGNED;
    if (batch && ((need_x && !aligned16(a->x)) || (need_out && !aligned16(a->out))))
        return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}

// Routing + quantise/permute + L1 (given epilogue).  Shared by forward and calibrate.
// Records events[i] on s when events is non-null (per-stage timing).  While
// s is being captured into a CUDA graph the record becomes an external event
// node, so the event can still be timed after the graph is replayed.
int mark(void *const *events, int i, cudaStream_t s)
{
    if (events == nullptr)
        return NVFP4_OK;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    const unsigned flags = cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
    return cuda_status(cudaEventRecordWithFlags(static_cast<cudaEvent_t>(events[i]), s, flags));
}

// Pair tiles (clusters of two CTAs on 256-row tiles) fill a third less
// shared memory per MMA where both 128-row halves hold rows, but a pair whose
// second half is empty occupies two SMs for one m-tile's work.  Measured on
// the B200: dense GEMMs with M >= 256 gain ~6 %; the 384-expert prefill (64
// rows per expert on average, most experts one m-tile) runs 35 % slower with
// pairs.  So the grouped GEMMs use them only when experts average two full
// m-tiles or more.
int moe_cg(int64_t R, int E)
{
    return R >= 256LL * E ? 2 : 1;
}

// Batches of at least this many routed rows put the pairs of full m-tiles of
// experts with two or more m-tiles on pair tiles (pair mode 1): the pair
// launch costs a few microseconds even when no expert is that heavy.
constexpr int64_t kSplitMinRows = 2048;
// Pair mode 1 runs the pair launch on every cluster of two SMs that fits,
// then the 1-CTA launch, whose CTAs take over each SM as soon as the pair
// launch's CTA there has finished (the pair launch lets its dependent start
// at once; the 1-CTA launch claims tiles, so CTAs that start late just take
// fewer).  Measured on the B200 (prefill, CTA start / end stamps): running the
// pair launch on fewer clusters beside the 1-CTA launch gains nothing -- with
// both resident the pair of launches takes as long as one after the other
// (2.56 against 2.58 ms with two streams; as a dependent launch the second
// kernel's resident CTAs made no progress until the first kernel ended).

int gemm_grid(int cg, int64_t tiles, int num_sms)
{
    if (cg == 2)
        return 2 * static_cast<int>(std::min<int64_t>(std::max<int64_t>(tiles, 1), gemm_pair_clusters(num_sms)));
    return static_cast<int>(std::min<int64_t>(std::max<int64_t>(tiles, 1), num_sms));
}

// Global scale of x the GEMMs read: the caller's, or the one the front
// kernel computes from the batch into the workspace header.
const float *x_gs_ptr(const nvfp4_moe_args *a, uint8_t *ws)
{
    return a->x_gs != nullptr ? a->x_gs : reinterpret_cast<const float *>(ws + kHdrGs);
}

// Maps and arguments of the grouped L1 GEMM (gate_up, SwiGLU epilogue).
int l1_setup(const nvfp4_moe_args *a, uint8_t *ws, const Layout &L, CUtensorMap *ma, CUtensorMap *ma32,
             CUtensorMap *mb, GemmArgs *g)
{
    const int64_t H = a->H, I = a->I;
    const int E = a->E;
    int st = make_code_map(ma, ws + L.a_codes, L.rpad, H / 2, 128);
    if (st == NVFP4_OK)
        st = make_code_map(ma32, ws + L.a_codes, L.rpad, H / 2, 32);
    if (st == NVFP4_OK)
        st = make_code_map(mb, a->w13_codes, static_cast<int64_t>(E) * 2 * I, H / 2, 128);
    if (st != NVFP4_OK)
        return st;
    *g = GemmArgs{};
    g->sfa = ws + L.a_sf;
    g->sfa_rowmajor = 1;
    g->sfa_block_stride = L.sfa_block;
    g->sfb = a->w13_scales;
    g->sfb_block_stride = (H / 64) * 512;
    g->K = static_cast<int>(H);
    g->num_k_tiles = static_cast<int>((H + 255) / 256);
    g->num_mtiles_dev = reinterpret_cast<int32_t *>(ws + kHdrNumMtiles);
    g->mtiles = reinterpret_cast<int4 *>(ws + L.mtiles);
    g->num_pairs_dev = reinterpret_cast<int32_t *>(ws + kHdrNumPairs);
    g->pairs = reinterpret_cast<int2 *>(ws + L.pairs);
    g->num_light_dev = reinterpret_cast<int32_t *>(ws + kHdrNumLight);
    g->light = reinterpret_cast<int32_t *>(ws + L.light);
    g->ready = reinterpret_cast<int32_t *>(ws + L.ready);
    g->claim = reinterpret_cast<int32_t *>(ws + kHdrClaim);
    g->n_tiles = static_cast<int>(I / 128);
    g->b_rows_per_expert = 2 * I;
    g->b_tile_rows = 128;
    g->b_half_offset = static_cast<int>(I);
    g->a_gs = x_gs_ptr(a, ws);
    g->a_gs_per_expert = 0;
    g->b_gs = a->w13_gs;
    g->b_gs_stride = 2;
    g->nseg = 1;
    g->inter_gs = a->inter_gs;
    g->h_codes = ws + L.h_codes;
    g->h_ld_bytes = I / 2;
    g->h_sf = ws + L.h_sf;
    g->h_sf_block_stride = (I / 64) * 512;
    g->amax_bits = reinterpret_cast<unsigned int *>(ws + L.amax);
    g->err = reinterpret_cast<int32_t *>(ws);
    return NVFP4_OK;
}

// Maps and arguments of the grouped L2 GEMM (down, bf16 epilogue into y).
int l2_setup(const nvfp4_moe_args *a, uint8_t *ws, const Layout &L, int bn, CUtensorMap *ma, CUtensorMap *ma32,
             CUtensorMap *mb, GemmArgs *g)
{
    const int64_t H = a->H, I = a->I;
    const int E = a->E;
    int st = make_code_map(ma, ws + L.h_codes, L.rpad, I / 2, 128);
    if (st == NVFP4_OK)
        st = make_code_map(ma32, ws + L.h_codes, L.rpad, I / 2, 32);
    if (st == NVFP4_OK)
        st = make_code_map(mb, a->w2_codes, static_cast<int64_t>(E) * H, I / 2, 128);
    if (st != NVFP4_OK)
        return st;
    *g = GemmArgs{};
    g->sfa = ws + L.h_sf;
    g->sfa_block_stride = (I / 64) * 512;
    g->sfb = a->w2_scales;
    g->sfb_block_stride = (I / 64) * 512;
    g->K = static_cast<int>(I);
    g->num_k_tiles = static_cast<int>((I + 255) / 256);
    g->num_mtiles_dev = reinterpret_cast<int32_t *>(ws + kHdrNumMtiles);
    g->mtiles = reinterpret_cast<int4 *>(ws + L.mtiles);
    g->num_pairs_dev = reinterpret_cast<int32_t *>(ws + kHdrNumPairs);
    g->pairs = reinterpret_cast<int2 *>(ws + L.pairs);
    g->num_light_dev = reinterpret_cast<int32_t *>(ws + kHdrNumLight);
    g->light = reinterpret_cast<int32_t *>(ws + L.light);
    g->ready = reinterpret_cast<int32_t *>(ws + L.ready);
    g->n_tiles = static_cast<int>(H / bn);
    g->b_rows_per_expert = H;
    g->b_tile_rows = bn;
    g->b_half_offset = 128;
    g->a_gs = a->inter_gs;
    g->a_gs_per_expert = 1;
    g->b_gs = a->w2_gs;
    g->b_gs_stride = 1;
    g->nseg = 1;
    g->seg_end[0] = static_cast<int>(H);
    g->out = reinterpret_cast<__nv_bfloat16 *>(ws + L.y);
    g->ldo = H;
    g->err = reinterpret_cast<int32_t *>(ws);
    return NVFP4_OK;
}

// The front of the forward in one launch (front.cu): the global scale of x
// when the caller passes none, routing and tile tables for `pair_mode`, and
// quantise/permute; x == nullptr: routing only.  Events 0-2 when timing
// (0 before it, 1 and 2 after it).  (Earlier designs ran the global scale,
// the routing and the quantisation as three launches, the routing in one
// block; one launch with a grid-wide ticket between the histograms and the
// positions reads x once from HBM and once from L2.)
FrontArgs front_args(const nvfp4_moe_args *a, const int32_t *ids, int64_t T, int k, int E, uint8_t *ws,
                     const Layout &L, int pair_mode)
{
    FrontArgs f{};
    f.x = a != nullptr ? reinterpret_cast<const __nv_bfloat16 *>(a->x) : nullptr;
    f.ids = ids;
    f.T = T;
    f.H = a != nullptr ? a->H : 128;
    f.E = E;
    f.k = k;
    f.x_gs = a != nullptr ? a->x_gs : nullptr;
    f.gs_out = reinterpret_cast<float *>(ws + kHdrGs);
    f.pair_mode = pair_mode;
    f.counts = reinterpret_cast<int32_t *>(ws + L.counts);
    f.off = reinterpret_cast<int32_t *>(ws + L.off);
    f.poff = reinterpret_cast<int32_t *>(ws + L.poff);
    f.num_mtiles = reinterpret_cast<int32_t *>(ws + kHdrNumMtiles);
    f.mtiles = reinterpret_cast<int4 *>(ws + L.mtiles);
    f.num_pairs = reinterpret_cast<int32_t *>(ws + kHdrNumPairs);
    f.pairs = reinterpret_cast<int2 *>(ws + L.pairs);
    f.num_light = reinterpret_cast<int32_t *>(ws + kHdrNumLight);
    f.light = reinterpret_cast<int32_t *>(ws + L.light);
    f.ready = reinterpret_cast<int32_t *>(ws + L.ready);
    f.claim = reinterpret_cast<int32_t *>(ws + kHdrClaim);
    f.inv = reinterpret_cast<int32_t *>(ws + L.inv);
    f.yrow = reinterpret_cast<int32_t *>(ws + L.yrow);
    f.err = reinterpret_cast<int32_t *>(ws);
    f.a_codes = ws + L.a_codes;
    f.a_sf = ws + L.a_sf;
    f.blk_hist = reinterpret_cast<int32_t *>(ws + L.blk_hist);
    f.blk_amax = reinterpret_cast<float *>(ws + L.blk_amax);
    f.ticket = reinterpret_cast<unsigned int *>(ws + kHdrTicket);
    return f;
}

int run_front(const nvfp4_moe_args *a, uint8_t *ws, const Layout &L, int pair_mode, void *const *events,
              cudaStream_t s, int num_sms, const uint8_t *xq_codes = nullptr, const uint8_t *xq_scales = nullptr)
{
    if (mark(events, 0, s) != NVFP4_OK)
        return NVFP4_ERR_CUDA;
    FrontArgs f = front_args(a, a->topk_ids, a->T, a->k, a->E, ws, L, pair_mode);
    if (xq_codes != nullptr) {
        f.x = nullptr;
        f.xq_codes = xq_codes;
        f.xq_scales = xq_scales;
    }
    if (launch_front(f, num_sms, s) != cudaSuccess ||
        mark(events, 1, s) != NVFP4_OK || mark(events, 2, s) != NVFP4_OK)
        return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}

// The forward's execution plan: pair tiles for the grouped GEMMs, and
// whether L1 and L2 run as one fused launch (1-CTA tiles, 256-wide L2 tiles).
// pair_mode: 0 every m-tile a 1-CTA tile; 1 the heavy experts' full m-tile
// pairs on pair tiles (two launches: L1, L2) and the rest on 1-CTA tiles;
// 2 every m-tile on pair tiles.  fused: the 1-CTA tiles run L1 and L2 in one
// persistent launch (256-wide L2 tiles).
struct Plan {
    int pair_mode;
    int l2_bn;
    bool fused;
};

Plan moe_plan(int64_t T, int k, int E, int64_t H)
{
    Plan pl;
    const int64_t R = T * k;
    pl.l2_bn = (H % 256 == 0) ? 256 : 128;
    if (pl.l2_bn == 256 && moe_cg(R, E) == 2)
        pl.pair_mode = 2;
    else if (pl.l2_bn == 256 && R >= kSplitMinRows && E > 1)
        pl.pair_mode = 1;
    else
        pl.pair_mode = 0;
    pl.fused = pl.pair_mode != 2 && pl.l2_bn == 256;
    return pl;
}

} // namespace

int nvfp4::moe_args_status(const nvfp4_moe_args *args, bool need_out)
{
    return check_moe_args(args, need_out);
}

extern "C" {

const char *nvfp4_status_string(int status)
{
    switch (status) {
    case NVFP4_OK: return "NVFP4_OK";
    case NVFP4_ERR_INVALID_ARG: return "NVFP4_ERR_INVALID_ARG";
    case NVFP4_ERR_UNSUPPORTED_SHAPE: return "NVFP4_ERR_UNSUPPORTED_SHAPE";
    case NVFP4_ERR_MISALIGNED: return "NVFP4_ERR_MISALIGNED";
    case NVFP4_ERR_WORKSPACE_TOO_SMALL: return "NVFP4_ERR_WORKSPACE_TOO_SMALL";
    case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA";
    case NVFP4_ERR_UNSUPPORTED_DEVICE: return "NVFP4_ERR_UNSUPPORTED_DEVICE";
    case NVFP4_ERR_TIMEOUT: return "NVFP4_ERR_TIMEOUT";
    case NVFP4_ERR_BAD_EXPERT_ID: return "NVFP4_ERR_BAD_EXPERT_ID";
    default: return "NVFP4_ERR_UNKNOWN";
    }
}

int nvfp4_global_scale(const uint16_t *x, int64_t n, float *gs_out, void *stream)
{
    if (x == nullptr || gs_out == nullptr || n < 1)
        return NVFP4_ERR_INVALID_ARG;
    int sms = 0;
    int st = device_check(&sms);
    if (st != NVFP4_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(gs_out, 0, sizeof(float), s) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (launch_amax_bf16(reinterpret_cast<const __nv_bfloat16 *>(x), n, gs_out, sms, s) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return cuda_status(launch_finalize_gs(gs_out, s));
}

int nvfp4_amax(const uint16_t *x, int64_t n, float *amax_out, void *stream)
{
    if (x == nullptr || amax_out == nullptr || n < 1)
        return NVFP4_ERR_INVALID_ARG;
    int sms = 0;
    int st = device_check(&sms);
    if (st != NVFP4_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(amax_out, 0, sizeof(float), s) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return cuda_status(launch_amax_bf16(reinterpret_cast<const __nv_bfloat16 *>(x), n, amax_out, sms, s));
}

int64_t nvfp4_scales_bytes(int64_t rows, int64_t cols, int scale_layout)
{
    if (rows < 0 || cols < 0 || cols % 16 != 0)
        return -1;
    if (scale_layout == NVFP4_SCALES_ROWMAJOR)
        return rows * (cols / 16);
    if (scale_layout == NVFP4_SCALES_MMA) {
        if (cols % 64 != 0)
            return -1;
        return round_up(rows, 128) * (cols / 16);
    }
    return -1;
}

int nvfp4_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ldx, const float *gs, uint8_t *codes,
                   uint8_t *scales, int scale_layout, void *stream)
{
    if (x == nullptr || gs == nullptr || codes == nullptr || scales == nullptr || rows < 0 || cols <= 0 || ldx < cols)
        return NVFP4_ERR_INVALID_ARG;
    if (scale_layout != NVFP4_SCALES_ROWMAJOR && scale_layout != NVFP4_SCALES_MMA)
        return NVFP4_ERR_INVALID_ARG;
    if (cols % 16 != 0 || (scale_layout == NVFP4_SCALES_MMA && cols % 64 != 0))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || ldx % 8 != 0)
        return NVFP4_ERR_MISALIGNED;
    if (rows > (1LL << 31) / 8)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    int st = device_check(nullptr);
    if (st != NVFP4_OK)
        return st;
    if (rows == 0)
        return NVFP4_OK;
    return cuda_status(launch_quantize(reinterpret_cast<const __nv_bfloat16 *>(x), rows, cols, ldx, gs, codes, scales,
                                       scale_layout, static_cast<cudaStream_t>(stream)));
}

int nvfp4_swizzle_scales(const uint8_t *in, int64_t batch, int64_t rows, int64_t cols, uint8_t *out, void *stream)
{
    if (in == nullptr || out == nullptr || batch < 0 || rows < 0 || cols <= 0)
        return NVFP4_ERR_INVALID_ARG;
    if (cols % 64 != 0)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if ((reinterpret_cast<uintptr_t>(in) & 3) != 0 || (reinterpret_cast<uintptr_t>(out) & 3) != 0)
        return NVFP4_ERR_MISALIGNED;
    int st = device_check(nullptr);
    if (st != NVFP4_OK)
        return st;
    if (batch == 0 || rows == 0)
        return NVFP4_OK;
    return cuda_status(launch_swizzle(in, batch, rows, cols, out, static_cast<cudaStream_t>(stream)));
}

} // extern "C"

namespace {

// Dense GEMM tile plan: pair tiles when there are at least two m-tiles and
// the tiles are 256 wide, dealt round-robin over the resident units.  (A
// stream-K split of the (tile, k-tile) iterations was measured against this
// once the pair tiles stored their output through TMA: it lost on every shape
// tried: a partial last round runs its few tiles faster per SM than a full
// one, which the split's partial-sum traffic and waits do not beat.)
struct DensePlan {
    int bn, cg, grid;
};

DensePlan dense_plan(int64_t M, int64_t N, int sms)
{
    DensePlan d;
    d.bn = (N % 256 == 0) ? 256 : 128;
    d.cg = (M > 128 && d.bn == 256) ? 2 : 1;
    const int64_t m_units = d.cg == 2 ? (M + 255) / 256 : (M + 127) / 128;
    d.grid = gemm_grid(d.cg, m_units * (N / d.bn), sms);
    return d;
}

int gemm_impl(const uint8_t *a_codes, const uint8_t *a_scales, const float *a_gs, int64_t M, const uint8_t *b_codes,
              const uint8_t *b_scales, const float *b_gs, const int64_t *seg_end, int nseg, int64_t N, int64_t K,
              uint16_t *out, int64_t ldo, void *stream)
{
    if (a_codes == nullptr || a_scales == nullptr || a_gs == nullptr || b_codes == nullptr || b_scales == nullptr ||
        b_gs == nullptr || seg_end == nullptr || out == nullptr || M < 1 || N < 1 || K < 1 || nseg < 1 || ldo < N)
        return NVFP4_ERR_INVALID_ARG;
    if (N % 128 != 0 || K % 64 != 0 || nseg > 4 || M >= (1LL << 31) || N >= (1LL << 31) || K > (1LL << 20))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    int64_t prev = 0;
    for (int i = 0; i < nseg; ++i) {
        if (seg_end[i] <= prev || seg_end[i] % 32 != 0)
            return NVFP4_ERR_INVALID_ARG;
        prev = seg_end[i];
    }
    if (prev != N)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(b_codes) || !aligned16(b_scales) ||
        !aligned16(out) || ldo % 8 != 0)
        return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    int st = device_check(&sms);
    if (st != NVFP4_OK)
        return st;
    CUtensorMap ma, ma32, mb;
    st = make_code_map(&ma, a_codes, M, K / 2, 128);
    if (st == NVFP4_OK)
        st = make_code_map(&ma32, a_codes, M, K / 2, 32);
    if (st == NVFP4_OK)
        st = make_code_map(&mb, b_codes, N, K / 2, 128);
    if (st != NVFP4_OK)
        return st;
    const int bn = (N % 256 == 0) ? 256 : 128;
    GemmArgs g{};
    g.sfa = a_scales;
    g.sfa_block_stride = (K / 64) * 512;
    g.sfb = b_scales;
    g.sfb_block_stride = (K / 64) * 512;
    g.K = static_cast<int>(K);
    g.num_k_tiles = static_cast<int>((K + 255) / 256);
    g.num_mtiles_dev = nullptr;
    g.mtiles = nullptr;
    g.dense_m_tiles = static_cast<int>((M + 127) / 128);
    g.dense_M = static_cast<int>(M);
    g.n_tiles = static_cast<int>(N / bn);
    g.b_rows_per_expert = N;
    g.b_tile_rows = bn;
    g.b_half_offset = 128;
    g.a_gs = a_gs;
    g.a_gs_per_expert = 0;
    g.b_gs = b_gs;
    g.b_gs_stride = 0;
    g.nseg = nseg;
    for (int i = 0; i < nseg; ++i)
        g.seg_end[i] = static_cast<int>(seg_end[i]);
    g.out = reinterpret_cast<__nv_bfloat16 *>(out);
    g.ldo = ldo;
    g.err = nullptr;            // no workspace: a timed-out wait ends the kernel without a report
    const DensePlan d = dense_plan(M, N, sms);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // pair tiles write out through shared memory and TMA stores (rows >= M are not written)
    CUtensorMap mo;
    if (d.cg == 2) {
        st = make_out_map(&mo, out, M, N, ldo);
        if (st != NVFP4_OK)
            return st;
        g.out_tma = 1;
    }
    const CUtensorMap *mo_ptr = d.cg == 2 ? &mo : nullptr;
    return cuda_status(launch_gemm(d.bn, EPI_BF16, d.cg, ma, ma32, mb, g, d.grid, s, mo_ptr));
}

} // namespace

extern "C" {

int nvfp4_gemm(const uint8_t *a_codes, const uint8_t *a_scales, const float *a_gs, int64_t M, const uint8_t *b_codes,
               const uint8_t *b_scales, const float *b_gs, const int64_t *seg_end, int nseg, int64_t N, int64_t K,
               uint16_t *out, int64_t ldo, void *stream)
{
    return gemm_impl(a_codes, a_scales, a_gs, M, b_codes, b_scales, b_gs, seg_end, nseg, N, K, out, ldo, stream);
}

size_t nvfp4_moe_workspace_size(int64_t T, int k, int E, int64_t H, int64_t I)
{
    if (check_moe_shape(T, k, E, H, I) != NVFP4_OK)
        return 0;
    return static_cast<size_t>(ws_layout(T, k, E, H, I).total);
}

int nvfp4_moe_workspace_region(int64_t T, int k, int E, int64_t H, int64_t I, int region, int64_t *offset,
                               int64_t *bytes)
{
    if (offset == nullptr || bytes == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    int st = check_moe_shape(T, k, E, H, I);
    if (st != NVFP4_OK)
        return st;
    const Layout L = ws_layout(T, k, E, H, I);
    const int64_t R = T * k;
    switch (region) {
    case 0: *offset = L.a_codes; *bytes = L.rpad * (H / 2); break;
    case 1: *offset = L.a_sf; *bytes = (L.rpad / 128) * L.sfa_block; break;
    case 2: *offset = L.h_codes; *bytes = L.rpad * (I / 2); break;
    case 3: *offset = L.h_sf; *bytes = L.rpad * (I / 16); break;
    case 4: *offset = L.y; *bytes = R * H * 2; break;
    case 5: *offset = L.inv; *bytes = R * 4; break;
    case 6: *offset = L.counts; *bytes = 4LL * E; break;
    case 7: *offset = L.poff; *bytes = 4LL * (E + 1); break;
    case 8: *offset = kHdrGs; *bytes = 4; break;
    case 9: *offset = L.mtiles; *bytes = 16 * std::max<int64_t>(L.mt_max, 1); break;
    case 10: *offset = L.pairs; *bytes = 8 * std::max<int64_t>(L.mt_max, 1); break;
    case 11: *offset = L.light; *bytes = 4 * std::max<int64_t>(L.mt_max, 1); break;
    case 12: *offset = 0; *bytes = 256; break;
    default: return NVFP4_ERR_INVALID_ARG;
    }
    return NVFP4_OK;
}

static int moe_forward_impl(const nvfp4_moe_args *a, void *workspace, size_t ws_bytes, void *stream,
                            void *const *events, const uint8_t *xq_codes = nullptr, const uint8_t *xq_scales = nullptr)
{
    int st = check_moe_args(a, true, xq_codes == nullptr);
    if (st != NVFP4_OK)
        return st;
    if (a->T > 0 && xq_codes != nullptr && (!aligned16(xq_codes) || !aligned16(xq_scales)))
        return NVFP4_ERR_MISALIGNED;
    if (workspace == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(workspace))
        return NVFP4_ERR_MISALIGNED;
    const Layout L = ws_layout(a->T, a->k, a->E, a->H, a->I);
    if (ws_bytes < static_cast<size_t>(L.total))
        return NVFP4_ERR_WORKSPACE_TOO_SMALL;
    int sms = 0;
    st = device_check(&sms);
    if (st != NVFP4_OK)
        return st;
    if (a->T == 0)
        return NVFP4_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const Plan pl = moe_plan(a->T, a->k, a->E, a->H);
    st = run_front(a, ws, L, pl.pair_mode, events, s, sms, xq_codes, xq_scales);
    if (st != NVFP4_OK)
        return st;
    const int64_t H = a->H;
    CUtensorMap ma1, ma1_32, mb1, ma2, ma2_32, mb2;
    GemmArgs g1, g2;
    st = l1_setup(a, ws, L, &ma1, &ma1_32, &mb1, &g1);
    if (st == NVFP4_OK)
        st = l2_setup(a, ws, L, pl.l2_bn, &ma2, &ma2_32, &mb2, &g2);
    if (st != NVFP4_OK)
        return st;
    if (pl.pair_mode == 1) {
        // the heavy experts' pairs (fused L1 -> L2 on pair tiles), then the
        // fused 1-CTA launch over the light list: the pair launch lets its
        // dependent start at once, so 1-CTA CTAs move onto SMs as pair CTAs
        // finish; the 1-CTA launch reads only what the front wrote and waits
        // for the pair launch at its end, so that the combine sees both
        GemmArgs p1 = g1;
        p1.pdl_trigger_early = 1;
        const int pairs = gemm_pair_clusters(sms);
        GemmArgs l1 = g1;
        l1.pdl_wait_at_end = 1;
        // (timed: an event between the two launches separates their stages;
        // the 1-CTA launch then starts after the pair launch has ended)
        if (launch_moe_fused(2, ma1, ma1_32, mb1, p1, ma2, ma2_32, mb2, g2, 2 * pairs, s) != cudaSuccess ||
            mark(events, 3, s) != NVFP4_OK ||
            launch_moe_fused(1, ma1, ma1_32, mb1, l1, ma2, ma2_32, mb2, g2, sms, s) != cudaSuccess ||
            mark(events, 4, s) != NVFP4_OK)
            return NVFP4_ERR_CUDA;
    } else if (pl.pair_mode == 2) {
        // every m-tile on pair tiles: L1 launch, then L2 launch
        const int pair_grid = gemm_grid(2, 1LL << 30, sms);
        if (launch_gemm(256, EPI_SWIGLU_QUANT, 2, ma1, ma1_32, mb1, g1, pair_grid, s) != cudaSuccess ||
            mark(events, 3, s) != NVFP4_OK ||
            launch_gemm(256, EPI_BF16, 2, ma2, ma2_32, mb2, g2, pair_grid, s) != cudaSuccess ||
            mark(events, 4, s) != NVFP4_OK)
            return NVFP4_ERR_CUDA;
    } else if (pl.fused) {
        // every m-tile on 1-CTA tiles, L1 and L2 in one launch
        if (launch_moe_fused(1, ma1, ma1_32, mb1, g1, ma2, ma2_32, mb2, g2, sms, s) != cudaSuccess ||
            mark(events, 3, s) != NVFP4_OK || mark(events, 4, s) != NVFP4_OK)
            return NVFP4_ERR_CUDA;
    } else {
        // 128-wide L2 tiles: L1 launch, then L2 launch, 1-CTA tiles
        if (launch_gemm(256, EPI_SWIGLU_QUANT, 1, ma1, ma1_32, mb1, g1, gemm_grid(1, 1LL << 30, sms), s) !=
                cudaSuccess ||
            mark(events, 3, s) != NVFP4_OK ||
            launch_gemm(pl.l2_bn, EPI_BF16, 1, ma2, ma2_32, mb2, g2, gemm_grid(1, 1LL << 30, sms), s) !=
                cudaSuccess ||
            mark(events, 4, s) != NVFP4_OK)
            return NVFP4_ERR_CUDA;
    }

    if (launch_combine(reinterpret_cast<const __nv_bfloat16 *>(ws + L.y),
                       reinterpret_cast<const int32_t *>(ws + L.yrow), a->topk_weights, a->T, a->k, H,
                       reinterpret_cast<__nv_bfloat16 *>(a->out), s) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return mark(events, 5, s);
}

int nvfp4_debug_bounded_wait(const int32_t *flag, int32_t target, int32_t *err, void *stream)
{
    if (flag == nullptr || err == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    int st = device_check(nullptr);
    if (st != NVFP4_OK)
        return st;
    return cuda_status(launch_wait_probe(flag, target, err, static_cast<cudaStream_t>(stream)));
}

int nvfp4_moe_plan(int64_t T, int k, int E, int64_t H, int64_t I, int32_t *fused_l1_l2, int32_t *pair_tiles)
{
    if (fused_l1_l2 == nullptr || pair_tiles == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    const int st = check_moe_shape(T, k, E, H, I);
    if (st != NVFP4_OK)
        return st;
    const Plan pl = moe_plan(T, k, E, H);
    *fused_l1_l2 = pl.fused ? 1 : 0;
    *pair_tiles = pl.pair_mode;
    return NVFP4_OK;
}

int nvfp4_moe_forward(const nvfp4_moe_args *a, void *workspace, size_t ws_bytes, void *stream)
{
    return moe_forward_impl(a, workspace, ws_bytes, stream, nullptr);
}

int nvfp4_moe_forward_quantized(const nvfp4_moe_args *a, const uint8_t *x_codes, const uint8_t *x_scales,
                                void *workspace, size_t ws_bytes, void *stream)
{
    if (a == nullptr || (a->T > 0 && (x_codes == nullptr || x_scales == nullptr)))
        return NVFP4_ERR_INVALID_ARG;
    return moe_forward_impl(a, workspace, ws_bytes, stream, nullptr, x_codes, x_scales);
}

int nvfp4_moe_forward_timed(const nvfp4_moe_args *a, void *workspace, size_t ws_bytes, void *stream,
                            void *const *events)
{
    if (events == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    for (int i = 0; i < 6; ++i)
        if (events[i] == nullptr)
            return NVFP4_ERR_INVALID_ARG;
    return moe_forward_impl(a, workspace, ws_bytes, stream, events);
}

int nvfp4_moe_calibrate(const nvfp4_moe_args *a, float *inter_gs_out, void *workspace, size_t ws_bytes, void *stream)
{
    int st = check_moe_args(a, false);
    if (st != NVFP4_OK)
        return st;
    if (workspace == nullptr || inter_gs_out == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(workspace))
        return NVFP4_ERR_MISALIGNED;
    const Layout L = ws_layout(a->T, a->k, a->E, a->H, a->I);
    if (ws_bytes < static_cast<size_t>(L.total))
        return NVFP4_ERR_WORKSPACE_TOO_SMALL;
    int sms = 0;
    st = device_check(&sms);
    if (st != NVFP4_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    if (cudaMemsetAsync(ws + L.amax, 0, 4 * static_cast<size_t>(a->E), s) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (a->T > 0) {
        // every m-tile on one kind of tile: all pairs when experts average two
        // full m-tiles, else all 1-CTA tiles (the warmup epilogue runs once)
        const int cg = moe_cg(a->T * a->k, a->E);
        st = run_front(a, ws, L, cg == 2 ? 2 : 0, nullptr, s, sms);
        if (st != NVFP4_OK)
            return st;
        CUtensorMap ma, ma32, mb;
        GemmArgs g;
        st = l1_setup(a, ws, L, &ma, &ma32, &mb, &g);
        if (st != NVFP4_OK)
            return st;
        if (launch_gemm(256, EPI_SWIGLU_AMAX, cg, ma, ma32, mb, g, gemm_grid(cg, 1LL << 30, sms), s) !=
            cudaSuccess)
            return NVFP4_ERR_CUDA;
    }
    return cuda_status(
        launch_finalize_inter_gs(reinterpret_cast<const unsigned int *>(ws + L.amax), a->E, inter_gs_out, s));
}

int nvfp4_moe_route_debug(const int32_t *topk_ids, int64_t T, int k, int E, int32_t *counts, int32_t *padded_offsets,
                          int32_t *inv, void *workspace, size_t ws_bytes, void *stream)
{
    if (topk_ids == nullptr || counts == nullptr || padded_offsets == nullptr || inv == nullptr ||
        workspace == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    if (T < 0 || k < 1 || E < 1)
        return NVFP4_ERR_INVALID_ARG;
    if (E > 1024 || k > 32 || T * k >= (1LL << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const Layout L = ws_layout(T, k, E, 128, 128);
    if (ws_bytes < static_cast<size_t>(L.total))
        return NVFP4_ERR_WORKSPACE_TOO_SMALL;
    int st = NVFP4_OK;
    int sms = 0;
    st = device_check(&sms);
    if (st != NVFP4_OK)
        return st;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    FrontArgs f = front_args(nullptr, topk_ids, T, k, E, ws, L, 0);
    f.counts = counts;
    f.poff = padded_offsets;
    f.inv = inv;
    return cuda_status(launch_front(f, sms, static_cast<cudaStream_t>(stream)));
}

int nvfp4_moe_topk_shared(const float *logits, int64_t T, int E, int k, int scoring, int num_shared,
                          int32_t *topk_ids, float *topk_weights, void *stream)
{
    if (T < 0 || k < 1 || E < 1 || num_shared < 0)
        return NVFP4_ERR_INVALID_ARG;
    if (T > 0 && (logits == nullptr || topk_ids == nullptr || topk_weights == nullptr))
        return NVFP4_ERR_INVALID_ARG;
    if (scoring != NVFP4_SCORING_SOFTMAX && scoring != NVFP4_SCORING_SIGMOID)
        return NVFP4_ERR_INVALID_ARG;
    if (E > 1024 || k > E || k + num_shared > 32 || E + num_shared > 1024 || T * E >= (1LL << 40))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    int st = device_check(nullptr);
    if (st != NVFP4_OK)
        return st;
    return cuda_status(launch_topk(logits, T, E, k, num_shared, scoring, topk_ids, topk_weights,
                                   static_cast<cudaStream_t>(stream)));
}

int nvfp4_moe_topk(const float *logits, int64_t T, int E, int k, int scoring, int32_t *topk_ids, float *topk_weights,
                   void *stream)
{
    return nvfp4_moe_topk_shared(logits, T, E, k, scoring, 0, topk_ids, topk_weights, stream);
}

int nvfp4_fp4_mma_ceiling(int bn, int iters, int ctas, int64_t *cycles, int32_t *err, void *stream)
{
    if (cycles == nullptr || (bn != 128 && bn != 256) || iters < 1 || ctas < 1)
        return NVFP4_ERR_INVALID_ARG;
    if (iters > (1 << 24) || ctas > 65535)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    int st = device_check(nullptr);
    if (st != NVFP4_OK)
        return st;
    return cuda_status(launch_mma_ceiling(bn, iters, ctas, reinterpret_cast<long long *>(cycles), err,
                                          static_cast<cudaStream_t>(stream)));
}

int nvfp4_tma_stream_ceiling(const uint8_t *matrix, int64_t rows, int64_t row_bytes, int64_t work_tiles,
                             int stages, int32_t *err, void *stream)
{
    if (matrix == nullptr || rows < 256 || row_bytes < 128 || work_tiles < 1 || stages < 2)
        return NVFP4_ERR_INVALID_ARG;
    if (rows % 256 != 0 || row_bytes % 128 != 0 || stages > 6 || rows >= (1LL << 31) || row_bytes >= (1LL << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(matrix))
        return NVFP4_ERR_MISALIGNED;
    int sms = 0;
    int st = device_check(&sms);
    if (st != NVFP4_OK)
        return st;
    CUtensorMap map;
    st = make_code_map(&map, matrix, rows, row_bytes, 128);
    if (st != NVFP4_OK)
        return st;
    return cuda_status(launch_tma_stream(map, rows, row_bytes, work_tiles, stages, sms, err,
                                         static_cast<cudaStream_t>(stream)));
}

int nvfp4_moe_get_error(void *workspace, int32_t *err_host, void *stream)
{
    if (workspace == nullptr || err_host == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(err_host, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof(int32_t), s) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return cuda_status(cudaStreamSynchronize(s));
}

} // extern "C"
