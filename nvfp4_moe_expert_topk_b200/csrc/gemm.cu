// gemm.cu -- persistent block-scaled FP4 GEMM engine for sm_100a.
//
// D[128 x BN] tiles (BN = 256, or 128 when N is not a multiple of 256) of
// A (E2M1 codes, K-major) x B^T (E2M1 codes, K-major) with one E4M3 scale per
// 16 elements on both sides, on the 5th-generation tensor cores
// (tcgen05.mma kind::mxf4nvf4, block16 scaling), accumulating in fp32 in
// tensor memory.  This is the grouped GEMM of the expert chain
// ("nvfp4-megamoe-kernel / CURRENT_BUG.md", page 1 "Phase 1": L1 gate_up
// GEMM -> SiLU -> re-quantise -> L2 GEMM; with one group it is the plain
// NVFP4 GEMM of page 1 "Phase 2").
//
// Block of 14 warps, one block per SM, persistent over the tile list:
//   warp 0    TMA producer: per k-tile (256 elements) the valid 32-row boxes
//             (or one 128-row box) of A, the BN rows of B as 128-row boxes,
//             and the matching 512-byte scale atoms by bulk copy, into a
//             shared-memory ring guarded by mbarriers;
//   warps 10-13 scale stagers, one per TMEM lane quarter: move each stage's
//             E4M3 scales from shared memory into that stage's TMEM scale
//             slot with tcgen05.st (the layout the MMA reads: lane l, column
//             4*j + m holds the 4 scales of row 128*h + 32*m + l for k-block
//             j, B half h; replicated in all four quarters), then signal the
//             stage's sf_ready barrier (copying scales through the tensor
//             pipe with tcgen05.cp costs more pipe time than the MMAs);
//   warp 1    allocates TMEM; one thread issues the 4 tcgen05.mma (K=64) of
//             each k-tile once the stage's sf_ready barrier completes (which
//             implies its operand copies landed); tiles are 256 wide, which
//             halves the A bytes filled per FLOP against 128-wide tiles;
//   warps 2-9 epilogue, two per TMEM lane quarter (each owns one row of the
//             tile and half of its columns): TMEM -> registers in two waits,
//             release the accumulator to the MMA thread at once (the next
//             tile's MMAs wait only for this drain), then one of
//             EPI_SWIGLU_QUANT  h = SiLU(a_g*g) * (a_u*u), NVFP4-quantised
//                               with the expert's inter_gs (L1),
//             EPI_SWIGLU_AMAX   same h, max|h| per expert (warmup),
//             EPI_BF16          y = alpha * acc -> bf16 (L2, dense GEMM);
//             pair tiles write bf16 through shared memory: the dense GEMM
//             as 32 x 32 boxes with TMA stores, the grouped L2 (compact y
//             rows) as 128-byte row pieces of its valid rows.
// In the L1 tile the B tile is 128 gate rows stacked on the matching 128 up
// rows of the stacked [gate; up] weight (two boxes), so TMEM columns 0-127
// hold gate and 128-255 hold up of the same 128 h columns, and each
// 16-element block of h is produced and quantised by one thread.
//
// The tile list is either dense (m-tiles of M, n-major) or grouped: an
// m-tile table written on the device by the front launch (expert, first
// padded row, valid rows, first output row), so the launch needs no host
// sync and every expert's rows are covered by one tensor map over the padded
// A buffer and one over all experts' stacked weights.  Two variants of the
// same engine: pair tiles (CG = 2, clusters of two CTAs issuing
// cta_group::2 MMAs on 256-row tiles) and the fused grouped launch
// (FUSED = 1, every L1 tile then every L2 tile, L2 tiles gated per m-tile on
// counters the L1 epilogues publish).  See the template's comment.
//
// Every mbarrier wait is bounded (ptx.cuh): on a timeout the block records
// NVFP4_ERR_TIMEOUT in the error word, stops issuing, waits (bounded) for its
// copies and MMAs in flight, frees its TMEM and returns.
#include <mutex>

#include "internal.h"
#include "quant.cuh"

namespace nvfp4 {

constexpr int kBM = 128;
constexpr int kBK = 256;                        // elements per k-tile
constexpr int kBKBytes = 128;                   // bytes of codes per row per k-tile
constexpr int kTileBytes = 128 * kBKBytes;      // 16 KB: 128 rows of one k-tile
constexpr int kSFAtom = 512;                    // 128 rows x 4 scales (64 elements)
constexpr int kSFStage = 4 * kSFAtom;           // one 128-row block, 4 k-blocks
constexpr int kThreads = 448;
constexpr int kEpiWarps = 8;                    // warps 2-9
constexpr int kFirstSFWarp = 2 + kEpiWarps;     // warps 10-13
constexpr uint32_t kTmemCols = 512;
constexpr int kTileQ = 8;                       // dynamically claimed launch: queue of claimed tile indices

// CG = 1: one CTA computes a 128 x BN tile.  CG = 2: a cluster of two CTAs
// computes a 256 x 256 tile with pair MMAs; each CTA loads its own 128 A
// rows and one 128-row half of B (so per CTA a k-tile fills 32 KB of codes
// instead of 48 KB for the same MMA work) and holds the scales of all 256
// B rows.
template <int BN, int CG>
struct Cfg {
    static constexpr int kHalves = BN / 128;                 // 128-row halves of the B tile
    static constexpr int kBBoxes = CG == 2 ? 1 : kHalves;    // B boxes this CTA loads per k-tile
    static constexpr int kNumAcc = BN == 256 ? 1 : 2;        // TMEM accumulators
    static constexpr int kStages = CG == 2 ? 5 : (BN == 256 ? 4 : 6);
    static constexpr int kSFSlotCols = 16 + 16 * kHalves;    // A: 4 k-blocks x 4 cols; B: 4 x 4 per half
    static constexpr uint32_t kTmemSF = kNumAcc * BN;        // scale slots follow the accumulators
    static constexpr int kA = 0;
    static constexpr int kB = kA + kStages * kTileBytes;
    static constexpr int kSFA = kB + kStages * kTileBytes * kBBoxes;
    static constexpr int kSFB = kSFA + kStages * kSFStage;
    // pair tiles store their bf16 tiles through shared memory: 4 KB per
    // epilogue warp, two 2 KB boxes of 32 rows x 32 columns for TMA stores
    // (dense) or one block of 32 rows x 64 columns (grouped y)
    static constexpr bool kOutStage = CG == 2;
    static constexpr int kOutBuf = 32 * 32 * 2;
    static constexpr int kOut = kSFB + kStages * kSFStage * kHalves;
    static constexpr int kBars = kOut + (kOutStage ? kEpiWarps * 2 * kOutBuf : 0);
    static constexpr int kBarCount = 3 * kStages + 2 * kNumAcc + 1 + 2 * kTileQ;
    static constexpr int kMisc = kBars + kBarCount * 8;
    static constexpr int kSmem = kMisc + 16 + 4 * kTileQ + 1024;   // + tmem slot, abort flag, tile queue, slack
    static_assert(kTmemSF + kStages * kSFSlotCols <= kTmemCols, "TMEM budget");
    static_assert(kSmem <= 232448, "shared memory budget");
    static_assert(CG == 1 || BN == 256, "pair tiles are 256 wide");
    static_assert(kOut % 1024 == 0, "staging buffers on the 64-byte swizzle's 512-byte period");
};

struct TileInfo {
    int e, row0, valid, row0_out, nt;
    int mt;     // m-tile index in the grouped table
    int ph;     // fused launch: 0 = L1 tile, 1 = L2 tile
};

// Tile t of the launch's tile space, as seen by CTA `rank` of its cluster.
// CG = 1: m-tiles of 128 rows.  CG = 2: m-pairs; the even CTA takes the
// pair's first m-tile and the odd CTA the second (valid = 0 when the expert
// or matrix has no rows left for it).  FUSED: the L1 tiles of every m-tile
// (p.n_tiles per m-tile), then the L2 tiles (p2.n_tiles per m-tile).
template <int CG, int FUSED>
__device__ __forceinline__ TileInfo decode_tile(const GemmArgs &p, const GemmArgs &p2, int t, int m_units,
                                                uint32_t rank)
{
    TileInfo ti;
    ti.ph = 0;
    ti.mt = 0;
    if constexpr (FUSED) {
        // every L1 tile (m-unit-major), then every L2 tile; an m-unit is a
        // light m-tile (CG = 1) or a pair of m-tiles (CG = 2); the tables are
        // read from L2 (they were written by the front launch of this step)
        const int t1 = m_units * p.n_tiles;
        ti.ph = t >= t1 ? 1 : 0;
        const int n = ti.ph ? p2.n_tiles : p.n_tiles;
        const int tt = ti.ph ? t - t1 : t;
        const int u = tt / n;
        ti.nt = tt - u * n;
        int mt, mt_any;
        if constexpr (CG == 2) {
            const int2 pr = __ldcg(p.pairs + u);
            mt = rank == 0 ? pr.x : pr.y;
            mt_any = mt >= 0 ? mt : pr.x;
        } else {
            mt = __ldcg(p.light + u);
            mt_any = mt;
        }
        const int4 m = __ldcg(p.mtiles + mt_any);
        ti.mt = mt;
        ti.e = m.x;
        ti.row0 = mt >= 0 ? m.y : m.y + kBM;
        ti.valid = mt >= 0 ? m.z : 0;
        ti.row0_out = mt >= 0 ? m.w : m.w + kBM;
        return ti;
    }
    if constexpr (CG == 2) {
        if (p.mtiles != nullptr) {
            const int mp = t / p.n_tiles;
            ti.nt = t - mp * p.n_tiles;
            const int2 pr = p.pairs[mp];
            const int mt = rank == 0 ? pr.x : pr.y;
            const int4 m = p.mtiles[mt >= 0 ? mt : pr.x];
            ti.e = m.x;
            ti.row0 = mt >= 0 ? m.y : m.y + kBM;
            ti.valid = mt >= 0 ? m.z : 0;
            ti.row0_out = mt >= 0 ? m.w : m.w + kBM;
        } else {
            const int nt = t / m_units;
            const int mp = t - nt * m_units;
            ti.nt = nt;
            ti.e = 0;
            ti.row0 = mp * 2 * kBM + static_cast<int>(rank) * kBM;
            ti.valid = max(0, min(kBM, p.dense_M - ti.row0));
            ti.row0_out = ti.row0;
        }
        return ti;
    }
    if (p.mtiles != nullptr) {
        const int li = t / p.n_tiles;
        ti.nt = t - li * p.n_tiles;
        const int mt = p.light[li];
        ti.mt = mt;
        const int4 m = p.mtiles[mt];
        ti.e = m.x;
        ti.row0 = m.y;
        ti.valid = m.z;
        ti.row0_out = m.w;
    } else {
        const int nt = t / m_units;
        const int mt = t - nt * m_units;
        ti.nt = nt;
        ti.e = 0;
        ti.row0 = mt * kBM;
        ti.valid = min(kBM, p.dense_M - ti.row0);
        ti.row0_out = ti.row0;
    }
    return ti;
}

// One 32-row x 32-column bf16 box of a pair tile leaves through shared memory:
// each lane's row (16 words of packed bf16 pairs) goes into `buf` as four
// 16-byte chunks, chunk c at position c ^ ((row >> 1) & 3) (the 64-byte
// swizzle the output map names, so that no two lanes of a quarter-warp share
// a bank), then lane 0 stores the box at (x, y) with TMA.  The warp alternates
// two buffers: before filling one it waits until the store issued from it
// two boxes earlier has read it.
__device__ __forceinline__ void store_box_staged(uint8_t *buf, const uint32_t (&v)[16], int lane,
                                                 const CUtensorMap *map, int x, int y)
{
    if (lane == 0)
        bulk_wait_group_read<1>();
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4 *>(buf + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)) =
            make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(map, x, y, buf);
        bulk_commit_group();
    }
}

// v[i] for a run-time i < 4 without indexing a register array
__device__ __forceinline__ float pick4(const float (&v)[4], int i)
{
    return i == 0 ? v[0] : (i == 1 ? v[1] : (i == 2 ? v[2] : v[3]));
}

__device__ __forceinline__ void record_error(int32_t *err, int code)
{
    if (err != nullptr)
        atomicCAS(err, 0, code);
}

// SiLU(g) * u with the fast exponential and division (relative error a few
// ulp; h is re-quantised to 4 bits right after).
__device__ __forceinline__ float silu_mul(float g, float u)
{
    return __fdividef(g, 1.0f + __expf(-g)) * u;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Bounded wait (2 s) until the 32-bit counter reaches `target`; acquire at
// GPU scope, then order this thread's later async-proxy reads (TMA) after it.
__device__ __forceinline__ bool wait_counter(const int32_t *ctr, int target, volatile int *abort)
{
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 0; i < kWaitLimitSpins; ++i) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
        if (v >= target) {
            asm volatile("fence.proxy.async.global;" ::: "memory");
            return true;
        }
        if ((i & 15u) == 15u && (*abort || global_timer_ns() - t0 > kWaitLimitNs))
            return false;
        __nanosleep(64);
    }
    return false;
}

// Consumer side of the dynamically claimed launch's tile queue: the next
// tile the producer claimed, read in claim order from shared memory.
// Returns 1 with the tile in t, 0 at the end of the tiles, -1 when the wait
// gave up.  warp_wide: every lane of the warp calls it and lane 0 releases
// the slot after all lanes have read it; otherwise the calling thread does.
__device__ __forceinline__ int dyn_next(uint64_t *q_full, uint64_t *q_empty, const int *tile_q, int &qi, int &t,
                                        bool warp_wide, volatile int *abort)
{
    const int slot = qi % kTileQ;
    bool got = mbar_wait(&q_full[slot], static_cast<uint32_t>(qi / kTileQ) & 1u, abort);
    if (warp_wide)
        got = __all_sync(0xffffffffu, got);
    if (!got)
        return -1;
    t = *reinterpret_cast<const volatile int *>(tile_q + slot);
    if (warp_wide)
        __syncwarp();
    if (!warp_wide || (threadIdx.x & 31) == 0)
        mbar_arrive(&q_empty[slot]);
    ++qi;
    return t >= 0 ? 1 : 0;
}

// Work cursor of a CTA (or pair) that deals whole tiles round-robin:
// t = unit, unit + units, ...
struct Cursor {
    int it, end;
};

__device__ __forceinline__ bool cursor_next(Cursor &c, int units, int &t)
{
    if (c.it >= c.end)
        return false;
    t = c.it;
    c.it += units;
    return true;
}

// The fused launch's counter wait on its own: one thread waits until *flag
// >= target, or gives up after the bound and records NVFP4_ERR_TIMEOUT.
__global__ void wait_probe_kernel(const int32_t *flag, int target, int32_t *err)
{
    __shared__ int no_abort;
    if (threadIdx.x == 0) {
        no_abort = 0;
        if (!wait_counter(flag, target, &no_abort))
            record_error(err, NVFP4_ERR_TIMEOUT);
    }
}

cudaError_t launch_wait_probe(const int32_t *flag, int target, int32_t *err, cudaStream_t s)
{
    wait_probe_kernel<<<1, 32, 0, s>>>(flag, target, err);
    return cudaGetLastError();
}

// FUSED = 1 (grouped, BN = 256): one persistent launch runs the L1 tiles
// (arguments p, maps map_a / map_a32 / map_b, SwiGLU + re-quantisation
// epilogue) and then the L2 tiles (p2, map_a2 / map_a2_32 / map_b2, bf16
// epilogue).  Each L1 epilogue warp publishes its h rows by bumping the
// m-tile's counter; the producer starts an L2 tile once all L1 tiles of its
// m-tile have been published (a bounded wait).  CG = 1 claims tiles one at a
// time from a counter, so every tile a wait depends on was claimed earlier
// by a running CTA that reaches it without waiting (no residency
// requirement); CG = 2 deals tiles round-robin over clusters that are all
// resident (the launch follows the front on an idle GPU, one cluster per SM
// pair).
template <int BN, int EPI, int CG, int FUSED>
__global__ void __launch_bounds__(kThreads, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_a32,
                      const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap map_a2,
                      const __grid_constant__ CUtensorMap map_a2_32, const __grid_constant__ CUtensorMap map_b2,
                      const __grid_constant__ CUtensorMap map_out, const GemmArgs p, const GemmArgs p2)
{
    using C = Cfg<BN, CG>;
    static_assert(!FUSED || (BN == 256 && EPI == EPI_SWIGLU_QUANT), "fused launch: L1 quant + L2 bf16");
    // the fused 1-CTA launch claims its tiles one at a time (no residency
    // requirement); everything else deals tiles round-robin
    constexpr bool kDyn = FUSED && CG == 1;
    constexpr int kStages = C::kStages;
    constexpr int kHalves = C::kHalves;
    constexpr int kNumAcc = C::kNumAcc;
    constexpr bool kPair = CG == 2;
    static_assert(EPI == EPI_BF16 || BN == 256, "SwiGLU tiles are 128 gate + 128 up columns");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem + C::kA;
    uint8_t *sB = smem + C::kB;
    uint8_t *sSFA = smem + C::kSFA;
    uint8_t *sSFB = smem + C::kSFB;
    uint8_t *sOut = smem + C::kOut;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBars);
    uint64_t *empty = full + kStages;
    uint64_t *sf_ready = empty + kStages;
    uint64_t *acc_full = sf_ready + kStages;
    uint64_t *acc_empty = acc_full + kNumAcc;
    uint64_t *drain = acc_empty + kNumAcc;
    uint64_t *q_full = drain + 1;                // tile queue (kDyn): a claimed index is in the slot
    uint64_t *q_empty = q_full + kTileQ;         //                    every role has read the slot
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kMisc + 4);
    int *tile_q = reinterpret_cast<int *>(smem + C::kMisc + 16);
    __shared__ int never_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // pair tiles: the even CTA of the cluster issues the MMAs and owns the
    // sf_ready / acc_empty barriers both CTAs arrive on
    const uint32_t rank = kPair ? cluster_ctarank() : 0u;
    const int unit = kPair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int units = kPair ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sf_ready[s], 4 * CG);
        }
        for (int b = 0; b < kNumAcc; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kEpiWarps * CG);
        }
        mbar_init(drain, 1);
        for (int i = 0; i < kTileQ; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1 + 4 + kEpiWarps);   // MMA thread, stager warps, epilogue warps
        }
        *abort_flag = 0;
        never_abort = 0;
        fence_mbar_init();
        tma_prefetch_map(&map_a);
        tma_prefetch_map(&map_a32);
        tma_prefetch_map(&map_b);
        if (FUSED) {
            tma_prefetch_map(&map_a2);
            tma_prefetch_map(&map_a2_32);
            tma_prefetch_map(&map_b2);
        }
        if (C::kOutStage && p.out_tma)
            tma_prefetch_map(&map_out);
    }
    if (warp == 1) {
        if constexpr (kPair) {
            tmem_alloc_pair(tmem_slot, kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_slot, kTmemCols);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (kPair)
        cluster_sync();             // both CTAs' barriers exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // cluster addresses of the leader's sf_ready / acc_empty barriers
    const uint32_t sf_ready_lead = kPair ? map_shared_to_cta(smem_u32(sf_ready), 0) : 0u;
    const uint32_t acc_empty_lead = kPair ? map_shared_to_cta(smem_u32(acc_empty), 0) : 0u;
    // everything above overlaps the previous kernel's tail (dependent launch);
    // from here on the tile table, the operands and the outputs are touched.
    // A launch that may start while its predecessor still runs
    // (pdl_wait_at_end: it reads nothing that kernel writes; its own inputs
    // were complete before that kernel let it start) waits for the
    // predecessor only at its end, so that the next kernel sees both; a
    // launch that lets its successor start early triggers at once.
    if (!p.pdl_wait_at_end)
        pdl_wait();
    if (p.pdl_trigger_early)
        pdl_trigger();

    const int m_units = (p.mtiles != nullptr)
                            ? __ldcg(kPair ? p.num_pairs_dev : p.num_light_dev)
                            : (kPair ? (p.dense_M + 2 * kBM - 1) / (2 * kBM) : p.dense_m_tiles);
    const int total = m_units * (p.n_tiles + (FUSED ? p2.n_tiles : 0));

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------- producer
            int stage = 0;
            uint32_t phase = 0, pend_mask = 0, pend_par = 0;
            bool ok = true;
            Cursor cur{unit, total};
            int t = 0, pq = 0;
            while (ok) {
                if constexpr (kDyn) {
                    // claim the next tile just before loading it, and queue its index for the other roles
                    const int slot = pq % kTileQ;
                    if (pq >= kTileQ &&
                        !mbar_wait(&q_empty[slot], static_cast<uint32_t>(pq / kTileQ - 1) & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    int tc = atomicAdd(p.claim, 1);
                    if (tc >= total)
                        tc = -1;
                    tile_q[slot] = tc;
                    mbar_arrive(&q_full[slot]);
                    ++pq;
                    if (tc < 0)
                        break;
                    t = tc;
                } else if (!cursor_next(cur, units, t)) {
                    break;
                }
                const TileInfo ti = decode_tile<CG, FUSED>(p, p2, t, m_units, rank);
                const GemmArgs &q = (FUSED && ti.ph) ? p2 : p;
                const CUtensorMap *ma = (FUSED && ti.ph) ? &map_a2 : &map_a;
                const CUtensorMap *ma32 = (FUSED && ti.ph) ? &map_a2_32 : &map_a32;
                const CUtensorMap *mb = (FUSED && ti.ph) ? &map_b2 : &map_b;
                if (FUSED && ti.ph && ti.valid > 0 &&
                    !wait_counter(p2.ready + ti.mt, p.n_tiles * kEpiWarps, abort_flag)) {
                    ok = false;     // this m-tile's h never got published
                    break;
                }
                const int64_t brow0 = ti.e * q.b_rows_per_expert + static_cast<int64_t>(ti.nt) * q.b_tile_rows;
                const int64_t brow1 = brow0 + q.b_half_offset;
                // A: nothing for an empty pair half, else one 128-row box or the valid 32-row boxes
                const int a_boxes = ti.valid >= kBM ? 0 : (ti.valid + 31) / 32;
                const uint32_t a_bytes = ti.valid == 0 ? 0u : (a_boxes == 0 ? kTileBytes : a_boxes * (kTileBytes / 4));
                const uint8_t *sfa = q.sfa + static_cast<int64_t>(ti.row0 / kBM) * q.sfa_block_stride;
                const uint8_t *sfb0 = q.sfb + (brow0 / 128) * q.sfb_block_stride;
                const uint8_t *sfb1 = q.sfb + (brow1 / 128) * q.sfb_block_stride;
                for (int kt = 0; kt < q.num_k_tiles; ++kt) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int nkb = min(4, (q.K - kt * kBK) / 64);
                    const uint32_t sf_bytes = static_cast<uint32_t>(nkb * kSFAtom);
                    // A scales: row blocks hold a k-tile's scales as 16 bytes per row, so a
                    // partial m-tile copies only its 32-row groups; MMA atoms take nkb x 512
                    const uint32_t sfa_bytes =
                        ti.valid == 0 ? 0u
                                      : (q.sfa_rowmajor ? (a_boxes == 0 ? 128u * 16u : static_cast<uint32_t>(a_boxes) * 512u)
                                                        : sf_bytes);
                    mbar_arrive_expect_tx(&full[stage], a_bytes + C::kBBoxes * kTileBytes + sf_bytes * kHalves + sfa_bytes);
                    uint8_t *a_dst = sA + stage * kTileBytes;
                    if (ti.valid > 0) {
                        if (a_boxes == 0) {
                            tma_load_2d(a_dst, ma, kt * kBKBytes, ti.row0, &full[stage]);
                        } else {
                            for (int i = 0; i < a_boxes; ++i)
                                tma_load_2d(a_dst + i * (kTileBytes / 4), ma32, kt * kBKBytes, ti.row0 + 32 * i,
                                            &full[stage]);
                        }
                        bulk_load(sSFA + stage * kSFStage, sfa + kt * kSFStage, sfa_bytes, &full[stage]);
                    }
                    uint8_t *b_dst = sB + stage * C::kBBoxes * kTileBytes;
                    uint8_t *sfb_dst = sSFB + stage * kHalves * kSFStage;
                    if constexpr (kPair) {
                        // this CTA's half of the B rows; the scales of both halves
                        tma_load_2d(b_dst, mb, kt * kBKBytes, static_cast<int32_t>(rank == 0 ? brow0 : brow1),
                                    &full[stage]);
                    } else {
                        tma_load_2d(b_dst, mb, kt * kBKBytes, static_cast<int32_t>(brow0), &full[stage]);
                        if constexpr (kHalves == 2)
                            tma_load_2d(b_dst + kTileBytes, mb, kt * kBKBytes, static_cast<int32_t>(brow1),
                                        &full[stage]);
                    }
                    bulk_load(sfb_dst, sfb0 + kt * kSFStage, sf_bytes, &full[stage]);
                    if constexpr (kHalves == 2)
                        bulk_load(sfb_dst + kSFStage, sfb1 + kt * kSFStage, sf_bytes, &full[stage]);
                    pend_mask |= 1u << stage;
                    pend_par = (pend_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                *abort_flag = 1;
                record_error(p.err, NVFP4_ERR_TIMEOUT);
            }
            // every copy this thread issued has landed before the block exits
            for (int s = 0; s < kStages; ++s)
                if ((pend_mask >> s) & 1u)
                    mbar_wait(&full[s], (pend_par >> s) & 1u, &never_abort);
        }
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer
        // (pair tiles: the even CTA's thread issues for both CTAs)
        constexpr uint32_t idesc = idesc_nvf4(kBM * CG, BN);
        if (lane == 0 && rank == 0) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            Cursor cur{unit, total};
            int t = 0, qi = 0;
            while (ok) {
                if constexpr (kDyn) {
                    const int r = dyn_next(q_full, q_empty, tile_q, qi, t, false, abort_flag);
                    if (r < 0)
                        ok = false;
                    if (r <= 0)
                        break;
                } else if (!cursor_next(cur, units, t)) {
                    break;
                }
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * BN);
                const GemmArgs &q = (FUSED && t >= m_units * p.n_tiles) ? p2 : p;
                for (int kt = 0; kt < q.num_k_tiles; ++kt) {
                    // sf_ready completes only after every stager has seen its CTA's
                    // full barrier complete (all of the stage's copies landed), so
                    // one wait covers both the scales and the operand tiles
                    if (!mbar_wait(&sf_ready[stage], phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nkb = min(4, (q.K - kt * kBK) / 64);
                    const uint32_t a_addr = smem_u32(sA + stage * kTileBytes);
                    const uint32_t b_addr = smem_u32(sB + stage * C::kBBoxes * kTileBytes);
                    const uint32_t t_sfa = tmem + C::kTmemSF + static_cast<uint32_t>(stage * C::kSFSlotCols);
                    for (int kb = 0; kb < nkb; ++kb) {
                        const uint64_t ad = sdesc_kmajor_sw128(a_addr + kb * 32);
                        const uint64_t bd = sdesc_kmajor_sw128(b_addr + kb * 32);
                        const uint32_t acc_flag = (kt != 0 || kb != 0) ? 1u : 0u;
                        if constexpr (kPair)
                            tc_mma_nvf4_pair(d_tmem, ad, bd, idesc, t_sfa + kb * 4, t_sfa + 16 + kb * 4 * kHalves,
                                             acc_flag);
                        else
                            tc_mma_nvf4(d_tmem, ad, bd, idesc, t_sfa + kb * 4, t_sfa + 16 + kb * 4 * kHalves, acc_flag);
                    }
                    if constexpr (kPair)
                        tc_commit_pair(&empty[stage], 0x3);
                    else
                        tc_commit(&empty[stage]);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                if constexpr (kPair)
                    tc_commit_pair(&acc_full[acc], 0x3);
                else
                    tc_commit(&acc_full[acc]);
                if (++acc == kNumAcc) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            if (!ok) {
                *abort_flag = 1;
                record_error(p.err, NVFP4_ERR_TIMEOUT);
            }
            // all MMAs of this thread complete before TMEM is freed
            if constexpr (kPair)
                tc_commit_pair(drain, 0x1);
            else
                tc_commit(drain);
            mbar_wait(drain, 0, &never_abort);
        }
        __syncwarp();
    } else if (warp >= kFirstSFWarp) {
        // -------------------------------------------------------- scale stagers
        const int q = warp & 3;
        const uint32_t t_q = tmem + (static_cast<uint32_t>(q * 32) << 16) + C::kTmemSF;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        Cursor cur{unit, total};
        int t = 0, qi = 0;
        while (ok) {
            if constexpr (kDyn) {
                const int r = dyn_next(q_full, q_empty, tile_q, qi, t, true, abort_flag);
                if (r < 0)
                    ok = false;
                if (r <= 0)
                    break;
            } else if (!cursor_next(cur, units, t)) {
                break;
            }
            // an empty pair half has no A scales: its rows get scale 0
            const bool a_rows = !kPair || decode_tile<CG, FUSED>(p, p2, t, m_units, rank).valid > 0;
            const GemmArgs &q = (FUSED && t >= m_units * p.n_tiles) ? p2 : p;
            for (int kt = 0; kt < q.num_k_tiles; ++kt) {
                const bool got = mbar_wait(&full[stage], phase, abort_flag);
                if (!__all_sync(0xffffffffu, got)) {
                    ok = false;
                    break;
                }
                const int nkb = min(4, (q.K - kt * kBK) / 64);
                const uint32_t t_slot = t_q + static_cast<uint32_t>(stage * C::kSFSlotCols);
                // A: column 4*kb + m <- the 4 scales of row 32*m + lane for k-block kb:
                // row `lane` of atom kb (MMA layout), or word kb of row 32*m + lane
                // (row blocks, 16 bytes a row)
                uint32_t r[16];
                const uint8_t *src = sSFA + stage * kSFStage + lane * 16;
                if (q.sfa_rowmajor) {
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const uint4 v = a_rows ? *reinterpret_cast<const uint4 *>(src + m * 512) : make_uint4(0, 0, 0, 0);
                        r[m] = nkb > 0 ? v.x : 0u;
                        r[4 + m] = nkb > 1 ? v.y : 0u;
                        r[8 + m] = nkb > 2 ? v.z : 0u;
                        r[12 + m] = nkb > 3 ? v.w : 0u;
                    }
                } else {
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        const uint4 v = (kb < nkb && a_rows) ? *reinterpret_cast<const uint4 *>(src + kb * kSFAtom)
                                                             : make_uint4(0, 0, 0, 0);
                        r[4 * kb] = v.x, r[4 * kb + 1] = v.y, r[4 * kb + 2] = v.z, r[4 * kb + 3] = v.w;
                    }
                }
                tc_st_32x32b_x16(t_slot, r);
                // B: column 4*(kHalves*kb + h) + m <- row `lane` of atom kb of half h
                src = sSFB + stage * kHalves * kSFStage + lane * 16;
#pragma unroll
                for (int part = 0; part < kHalves; ++part) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int kb = (part * 4 + i) / kHalves, h = (part * 4 + i) % kHalves;
                        const uint4 v = kb < nkb ? *reinterpret_cast<const uint4 *>(src + h * kSFStage + kb * kSFAtom)
                                                 : make_uint4(0, 0, 0, 0);
                        r[4 * i] = v.x, r[4 * i + 1] = v.y, r[4 * i + 2] = v.z, r[4 * i + 3] = v.w;
                    }
                    tc_st_32x32b_x16(t_slot + 16 + 16 * part, r);
                }
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (kPair)
                        mbar_arrive_cluster(sf_ready_lead + stage * 8);
                    else
                        mbar_arrive(&sf_ready[stage]);
                }
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            record_error(p.err, NVFP4_ERR_TIMEOUT);
        }
    } else {
        // -------------------------------------------------------- epilogue
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int hf = (warp - 2) >> 2;         // which half of the tile's columns this warp owns
        const int row = q * 32 + lane;          // row of the tile owned by this thread
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(q * 32) << 16);
        int acc = 0;
        uint32_t acc_phase = 0;
        Cursor cur{unit, total};
        int t = 0, qi = 0;
        while (true) {
            if constexpr (kDyn) {
                const int r = dyn_next(q_full, q_empty, tile_q, qi, t, true, abort_flag);
                if (r < 0) {
                    if (lane == 0) {
                        *abort_flag = 1;
                        record_error(p.err, NVFP4_ERR_TIMEOUT);
                    }
                }
                if (r <= 0)
                    break;
            } else if (!cursor_next(cur, units, t)) {
                break;
            }
            // the tile's coordinates and global scales are read while its MMAs
            // run, so that the drain (which holds the accumulator) waits on no load:
            // dequantisation factors 1 / (a_gs * b_gs) per B segment (SwiGLU
            // tiles: gate, up) and the global scale of h
            const TileInfo ti = decode_tile<CG, FUSED>(p, p2, t, m_units, rank);
            const GemmArgs &ga = (FUSED && ti.ph) ? p2 : p;
            const bool valid = row < ti.valid;
            const uint32_t t_acc = t_lane + static_cast<uint32_t>(acc * BN);
            const bool swiglu_tile = FUSED ? ti.ph == 0 : EPI != EPI_BF16;
            float alpha_seg[4];
            {
                const float a = __ldcg(ga.a_gs + (ga.a_gs_per_expert ? ti.e : 0));
                const int n_seg = swiglu_tile ? 2 : ga.nseg;
                float b[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    b[i] = i < n_seg ? __ldcg(ga.b_gs + ti.e * ga.b_gs_stride + i) : 1.0f;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    alpha_seg[i] = __fdiv_rn(1.0f, __fmul_rn(a, b[i]));
            }
            const float h_gs = (EPI == EPI_SWIGLU_QUANT && swiglu_tile) ? __ldcg(ga.inter_gs + ti.e) : 0.0f;
            const bool got = mbar_wait(&acc_full[acc], acc_phase, abort_flag);
            if (!__all_sync(0xffffffffu, got)) {
                *abort_flag = 1;
                record_error(p.err, NVFP4_ERR_TIMEOUT);
                break;
            }
            tc_fence_after();

            if (swiglu_tile && BN == 256) {
                // drain gate columns [64hf, 64hf+64) and the matching up columns in two rounds of
                // 32 (one wait each), computing h as it arrives, then release the accumulator
                const float alpha_g = alpha_seg[0], alpha_u = alpha_seg[1];
                float h[64];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    uint32_t g[32], u[32];
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const uint32_t col = hf * 64 + r * 32 + c * 16;
                        tc_ld_32x32b_x16(t_acc + col, *reinterpret_cast<uint32_t(*)[16]>(&g[16 * c]));
                        tc_ld_32x32b_x16(t_acc + 128 + col, *reinterpret_cast<uint32_t(*)[16]>(&u[16 * c]));
                    }
                    tc_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        h[r * 32 + i] = silu_mul(__uint_as_float(g[i]) * alpha_g, __uint_as_float(u[i]) * alpha_u);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (kPair)
                        mbar_arrive_cluster(acc_empty_lead + acc * 8);
                    else
                        mbar_arrive(&acc_empty[acc]);
                }
                if constexpr (EPI == EPI_SWIGLU_AMAX) {
                    float amax = 0.0f;
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        amax = fmaxf(amax, fabsf(h[i]));
                    if (!valid)
                        amax = 0.0f;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1)
                        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                    if (lane == 0)
                        atomicMax(ga.amax_bits + ti.e, __float_as_uint(amax));
                } else {
                    const float hgs = h_gs;
                    uint32_t codes[8];
                    uint32_t sfw = 0;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float blk[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            blk[i] = h[c * 16 + i];
                        sfw |= quantize16(blk, hgs, codes[2 * c], codes[2 * c + 1]) << (8 * c);
                    }
                    if (valid) {
                        // 64 h columns: 32 bytes of codes and one 4-byte scale word (k-block 2nt + hf)
                        uint4 *hrow = reinterpret_cast<uint4 *>(ga.h_codes +
                                                                static_cast<int64_t>(ti.row0 + row) * ga.h_ld_bytes +
                                                                ti.nt * 64 + hf * 32);
                        hrow[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
                        hrow[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
                        *reinterpret_cast<uint32_t *>(ga.h_sf + static_cast<int64_t>(ti.row0 / kBM) * ga.h_sf_block_stride +
                                                      static_cast<int64_t>(2 * ti.nt + hf) * kSFAtom + lane * 16 +
                                                      q * 4) = sfw;
                    }
                    if (FUSED && ti.valid > 0) {
                        // publish this warp's h rows to the L2 tiles of this m-tile
                        __threadfence();
                        __syncwarp();
                        if (lane == 0) {
                            __threadfence();
                            atomicAdd(ga.ready + ti.mt, 1);
                        }
                    }
                }
            } else {
                constexpr int kCols = BN / 2;
                constexpr int kRound = kCols < 64 ? kCols : 64;
                // drain columns [hf*BN/2, (hf+1)*BN/2) in rounds of 64 (one wait each),
                // converting to bf16 as they arrive, then release the accumulator
                uint32_t o[kCols / 2];
#pragma unroll
                for (int r = 0; r < kCols / kRound; ++r) {
                    uint32_t v[kRound];
#pragma unroll
                    for (int c = 0; c < kRound / 16; ++c)
                        tc_ld_32x32b_x16(t_acc + hf * kCols + r * kRound + c * 16,
                                         *reinterpret_cast<uint32_t(*)[16]>(&v[16 * c]));
                    tc_wait_ld();
#pragma unroll
                    for (int c = 0; c < kRound / 16; ++c) {
                        const int col = ti.nt * BN + hf * kCols + r * kRound + c * 16;
                        int seg = 0;
#pragma unroll
                        for (int i = 0; i < 3; ++i)
                            if (i < ga.nseg - 1 && col >= ga.seg_end[i])
                                seg = i + 1;
                        const float alpha = pick4(alpha_seg, seg);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            o[(r * kRound + c * 16) / 2 + i] = pack_bf16x2(__uint_as_float(v[16 * c + 2 * i]) * alpha,
                                                                           __uint_as_float(v[16 * c + 2 * i + 1]) * alpha);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (kPair)
                        mbar_arrive_cluster(acc_empty_lead + acc * 8);
                    else
                        mbar_arrive(&acc_empty[acc]);
                }
                bool staged = false;
                if constexpr (C::kOutStage && kCols == 128) {
                    staged = true;
                    if (ga.out_tma) {
                        // four boxes of 32 rows x 32 columns through this warp's two
                        // buffers, written out by TMA stores (whole 64-byte row pieces
                        // instead of one 16-byte piece per row per store instruction)
                        if (q * 32 < ti.valid) {    // a box starts on a row the GEMM writes; rows past M are clipped
#pragma unroll
                            for (int b = 0; b < 4; ++b) {
                                uint32_t ob[16];
#pragma unroll
                                for (int i = 0; i < 16; ++i)
                                    ob[i] = o[16 * b + i];
                                store_box_staged(sOut + ((warp - 2) * 2 + (b & 1)) * C::kOutBuf, ob, lane, &map_out,
                                                 ti.nt * BN + hf * kCols + b * 32, ti.row0_out + q * 32);
                            }
                        }
                    } else if (q * 32 < ti.valid) {
                        // grouped tiles: y's rows are compact, so the rows past an m-tile's
                        // valid ones belong to the next expert and no box may cover them.
                        // The warp stages 32 rows x 64 columns at a time in its 4 KB
                        // (16-byte chunk c of row r at c ^ (r & 7): conflict-free both
                        // ways) and writes them back as 4 rows x 128 bytes per store
                        // instruction, each lane storing only for a valid row
                        uint8_t *wbuf = sOut + (warp - 2) * 2 * C::kOutBuf;
                        __nv_bfloat16 *ybase = ga.out + static_cast<int64_t>(ti.row0_out + q * 32) * ga.ldo +
                                               static_cast<int64_t>(ti.nt) * BN + hf * kCols;
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {
                            __syncwarp();           // the previous half has been read back
#pragma unroll
                            for (int c = 0; c < 8; ++c)
                                *reinterpret_cast<uint4 *>(wbuf + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                                    make_uint4(o[32 * h2 + 4 * c], o[32 * h2 + 4 * c + 1], o[32 * h2 + 4 * c + 2],
                                               o[32 * h2 + 4 * c + 3]);
                            __syncwarp();
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const int r = 4 * j + (lane >> 3), c = lane & 7;
                                const uint4 v = *reinterpret_cast<const uint4 *>(wbuf + r * 128 + ((c ^ (r & 7)) << 4));
                                if (q * 32 + r < ti.valid)
                                    *reinterpret_cast<uint4 *>(ybase + static_cast<int64_t>(r) * ga.ldo + h2 * 64 + c * 8) = v;
                            }
                        }
                    }
                }
                if (!staged && valid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(ga.out + static_cast<int64_t>(ti.row0_out + row) * ga.ldo +
                                                           static_cast<int64_t>(ti.nt) * BN + hf * kCols);
#pragma unroll
                    for (int i = 0; i < kCols / 8; ++i)
                        dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
                }
            }
            if (++acc == kNumAcc) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    if (C::kOutStage && warp >= 2 && warp < 2 + kEpiWarps) {
        if (lane == 0)
            bulk_wait_group_all();  // this warp's output stores have completed and read their buffers
        __syncwarp();
    }
    if (p.pdl_wait_at_end)
        pdl_wait();                 // the kernel this one overlapped has finished: the next sees both
    pdl_trigger();                  // the next kernel may start launching during the teardown
    tc_fence_before();
    __syncthreads();
    if constexpr (kPair)
        cluster_sync();             // no CTA leaves while the pair's MMAs or arrivals may touch it
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        if constexpr (kPair)
            tmem_dealloc_pair(tmem, kTmemCols);
        else
            tmem_dealloc(tmem, kTmemCols);
    }
}

template <int BN, int EPI, int CG, int FUSED>
static cudaError_t launch_one(const CUtensorMap &map_a, const CUtensorMap &map_a32, const CUtensorMap &map_b,
                              const GemmArgs &args, const CUtensorMap &map_a2, const CUtensorMap &map_a2_32,
                              const CUtensorMap &map_b2, const GemmArgs &args2, int grid, cudaStream_t stream,
                              const CUtensorMap *map_out = nullptr)
{
    if (args.out_tma && (map_out == nullptr || CG != 2 || EPI != EPI_BF16 || FUSED))
        return cudaErrorInvalidValue;
    const int smem = Cfg<BN, CG>::kSmem;
    static unsigned long long attr_done = 0;     // one bit per device
    const cudaError_t e =
        ensure_smem_limit(reinterpret_cast<const void *>(nvfp4_gemm_kernel<BN, EPI, CG, FUSED>), smem, &attr_done);
    if (e != cudaSuccess)
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    cfg.attrs = attr;
    cfg.numAttrs = 0;
    // the prologue (barriers, TMEM, tensor-map prefetch) overlaps the previous
    // kernel; a fused launch needs no cooperative launch: the 1-CTA one claims
    // its tiles (a wait only ever depends on tiles claimed before, by running
    // CTAs), and the pair one starts right after the front has finished, on an
    // empty GPU, with no more clusters than fit at once
    attr[cfg.numAttrs].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[cfg.numAttrs].val.programmaticStreamSerializationAllowed = 1;
    ++cfg.numAttrs;
    if constexpr (CG == 2) {
        attr[cfg.numAttrs].id = cudaLaunchAttributeClusterDimension;
        attr[cfg.numAttrs].val.clusterDim.x = 2;
        attr[cfg.numAttrs].val.clusterDim.y = 1;
        attr[cfg.numAttrs].val.clusterDim.z = 1;
        ++cfg.numAttrs;
    }
    // without staged stores the output map is never read: any valid map fills the slot
    return cudaLaunchKernelEx(&cfg, nvfp4_gemm_kernel<BN, EPI, CG, FUSED>, map_a, map_a32, map_b, map_a2,
                              map_a2_32, map_b2, map_out != nullptr ? *map_out : map_a, args, args2);
}

template <int BN, int EPI, int CG>
static cudaError_t launch_plain(const CUtensorMap &map_a, const CUtensorMap &map_a32, const CUtensorMap &map_b,
                                const GemmArgs &args, int grid, cudaStream_t stream, const CUtensorMap *map_out)
{
    return launch_one<BN, EPI, CG, 0>(map_a, map_a32, map_b, args, map_a, map_a32, map_b, args, grid, stream,
                                      map_out);
}

cudaError_t launch_gemm(int bn, int epi, int cg, const CUtensorMap &map_a, const CUtensorMap &map_a32,
                        const CUtensorMap &map_b, const GemmArgs &args, int grid, cudaStream_t stream,
                        const CUtensorMap *map_out)
{
#define NVFP4_PLAIN(BN_, EPI_, CG_) launch_plain<BN_, EPI_, CG_>(map_a, map_a32, map_b, args, grid, stream, map_out)
    if (cg == 2) {
        if (bn != 256 || grid % 2 != 0)
            return cudaErrorInvalidValue;
        switch (epi) {
        case EPI_SWIGLU_QUANT: return NVFP4_PLAIN(256, EPI_SWIGLU_QUANT, 2);
        case EPI_SWIGLU_AMAX: return NVFP4_PLAIN(256, EPI_SWIGLU_AMAX, 2);
        default: return NVFP4_PLAIN(256, EPI_BF16, 2);
        }
    }
    switch (epi) {
    case EPI_SWIGLU_QUANT: return NVFP4_PLAIN(256, EPI_SWIGLU_QUANT, 1);
    case EPI_SWIGLU_AMAX: return NVFP4_PLAIN(256, EPI_SWIGLU_AMAX, 1);
    default: return bn == 256 ? NVFP4_PLAIN(256, EPI_BF16, 1) : NVFP4_PLAIN(128, EPI_BF16, 1);
    }
#undef NVFP4_PLAIN
}

cudaError_t launch_moe_fused(int cg, const CUtensorMap &map_a1, const CUtensorMap &map_a1_32,
                             const CUtensorMap &map_b1, const GemmArgs &args1, const CUtensorMap &map_a2,
                             const CUtensorMap &map_a2_32, const CUtensorMap &map_b2, const GemmArgs &args2, int grid,
                             cudaStream_t stream)
{
    if (args1.mtiles == nullptr || args1.ready == nullptr || args2.ready != args1.ready)
        return cudaErrorInvalidValue;
    if (cg == 2)
        return grid % 2 != 0 ? cudaErrorInvalidValue
                             : launch_one<256, EPI_SWIGLU_QUANT, 2, 1>(map_a1, map_a1_32, map_b1, args1, map_a2,
                                                                        map_a2_32, map_b2, args2, grid, stream);
    if (args1.claim == nullptr)
        return cudaErrorInvalidValue;
    return launch_one<256, EPI_SWIGLU_QUANT, 1, 1>(map_a1, map_a1_32, map_b1, args1, map_a2, map_a2_32, map_b2, args2,
                                                    grid, stream);
}

// Clusters of two GEMM CTAs that can be resident at once on the current
// device (each CTA needs a whole SM's shared memory), cached per device.
int gemm_pair_clusters(int num_sms)
{
    constexpr int kMaxDev = 64;
    static int cached[kMaxDev];             // 0: not yet queried on that device
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return num_sms / 2;
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < kMaxDev && cached[dev] > 0)
        return cached[dev];
    const int smem = Cfg<256, 2>::kSmem;
    int n = 0;
    if (cudaFuncSetAttribute(nvfp4_gemm_kernel<256, EPI_BF16, 2, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(num_sms));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = static_cast<size_t>(smem);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, nvfp4_gemm_kernel<256, EPI_BF16, 2, 0>, &cfg) != cudaSuccess)
            n = 0;
    }
    (void)cudaGetLastError();
    if (n <= 0 || n > num_sms / 2)
        n = num_sms / 2;
    if (dev >= 0 && dev < kMaxDev)
        cached[dev] = n;
    return n;
}

} // namespace nvfp4
