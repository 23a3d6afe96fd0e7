// gemm.cu -- persistent block-scaled FP4 GEMM engine for sm_100a.
//
// D[128 x 128] tiles of  A (E2M1 codes, K-major) x B^T (E2M1 codes, K-major)
// with one E4M3 scale per 16 elements on both sides, on the 5th-generation
// tensor cores (tcgen05.mma kind::mxf4nvf4, block16 scaling), accumulating in
// fp32 in tensor memory.  This is the grouped GEMM of the expert chain
// ("nvfp4-megamoe-kernel / CURRENT_BUG.md", page 1 "Phase 1": L1 gate_up
// GEMM -> SiLU -> re-quantise -> L2 GEMM; with one group it is the plain
// NVFP4 GEMM of page 1 "Phase 2").
//
// Block of 10 warps, one block per SM, persistent over the tile list:
//   warp 0    TMA producer: per k-tile (256 elements) the valid 32-row boxes
//             (or one 128-row box) of A, the 128 rows of B, and the matching
//             512-byte scale atoms by bulk copy, into a 5- or 6-stage
//             shared-memory ring guarded by mbarriers;
//   warps 6-9 scale stagers, one per TMEM lane quarter: move each stage's
//             E4M3 scales from shared memory into that stage's TMEM scale
//             slot with tcgen05.st (the layout the MMA reads: lane l, column
//             4*kb + m holds the 4 scales of row 32*m + l, replicated in all
//             four quarters), then signal the stage's sf_ready barrier;
//             scale copies through the tensor pipe (tcgen05.cp) cost more
//             pipe time than the MMAs they feed at these tile sizes;
//   warp 1    allocates TMEM; one thread issues the 4 tcgen05.mma (K=64) of
//             each k-tile into one of two 128-column accumulators, so the
//             next tile's MMAs run while the epilogue drains the previous;
//   warps 2-5 epilogue: TMEM -> registers (each thread owns one row of the
//             tile), then one of
//             EPI_SWIGLU_QUANT  h = SiLU(a_g*g) * (a_u*u), NVFP4-quantised
//                               with the expert's inter_gs (L1),
//             EPI_SWIGLU_AMAX   same h, max|h| per expert (warmup),
//             EPI_BF16          y = alpha * acc -> bf16 (L2, dense GEMM).
// In the L1 tile the B tile is 64 gate rows stacked on the matching 64 up
// rows (the weight keeps its [gate; up] layout: two 64-row boxes), so TMEM
// columns 0-63 hold gate and 64-127 hold up of the same 64 h columns and each
// 16-element block of h is produced by one thread.  The scales of those two
// 64-row halves sit in two different 128-row scale atoms; the stagers pair
// their 32-row groups on the way into TMEM.
//
// The tile list is either dense (m-tiles of M, n-major) or grouped: an
// m-tile table written on the device by the routing kernel (expert, first
// padded row, valid rows, first output row), so the launch needs no host
// sync and every expert's rows are covered by one tensor map over the padded
// A buffer and one over all experts' stacked weights.
//
// Every mbarrier wait is bounded (ptx.cuh): on a timeout the block records
// NVFP4_ERR_TIMEOUT in the error word, stops issuing, waits (bounded) for its
// copies and MMAs in flight, frees its TMEM and returns.
#include "internal.h"
#include "quant.cuh"

namespace nvfp4 {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kBK = 256;                        // elements per k-tile
constexpr int kBKBytes = 128;                   // bytes of codes per row per k-tile
constexpr int kTileBytes = 128 * kBKBytes;      // 16 KB: 128 rows of one k-tile
constexpr int kSFAtom = 512;                    // 128 rows x 4 scales (64 elements)
constexpr int kSFStage = 4 * kSFAtom;           // one 128-row block, 4 k-blocks
constexpr int kNumAcc = 2;                      // TMEM accumulators
constexpr int kThreads = 320;
constexpr int kFirstSFWarp = 6;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemSF = kNumAcc * kBN;     // 256: per-stage scale slots follow the accumulators
constexpr uint32_t kSFSlotCols = 32;            // A: 4 k-blocks x 4 columns, then B: the same

template <int EPI>
struct Smem {
    static constexpr bool kPaired = EPI != EPI_BF16;
    static constexpr int kStages = kPaired ? 5 : 6;
    static constexpr int kA = 0;
    static constexpr int kB = kA + kStages * kTileBytes;
    static constexpr int kSFA = kB + kStages * kTileBytes;
    static constexpr int kSFB = kSFA + kStages * kSFStage;              // paired: gate atoms, then up atoms
    static constexpr int kBars = kSFB + kStages * kSFStage * (kPaired ? 2 : 1);
    static constexpr int kBarCount = 3 * kStages + 2 * kNumAcc + 1;
    static constexpr int kMisc = kBars + kBarCount * 8;
    static constexpr int kTotal = kMisc + 16 + 1024;   // + tmem slot, abort flag, alignment slack
    static_assert(kTmemSF + kStages * kSFSlotCols <= kTmemCols, "TMEM scale slots");
};

struct TileInfo {
    int e, row0, valid, row0_out, nt;
};

__device__ __forceinline__ TileInfo decode_tile(const GemmArgs &p, int t, int m_tiles)
{
    TileInfo ti;
    if (p.mtiles != nullptr) {
        const int mt = t / p.n_tiles;
        ti.nt = t - mt * p.n_tiles;
        const int4 m = p.mtiles[mt];
        ti.e = m.x;
        ti.row0 = m.y;
        ti.valid = m.z;
        ti.row0_out = m.w;
    } else {
        const int nt = t / m_tiles;
        const int mt = t - nt * m_tiles;
        ti.nt = nt;
        ti.e = 0;
        ti.row0 = mt * kBM;
        ti.valid = min(kBM, p.dense_M - ti.row0);
        ti.row0_out = ti.row0;
    }
    return ti;
}

__device__ __forceinline__ int tile_nt(const GemmArgs &p, int t, int m_tiles)
{
    return p.mtiles != nullptr ? t % p.n_tiles : t / m_tiles;
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

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_a32,
                      const __grid_constant__ CUtensorMap map_b, const GemmArgs p)
{
    using L = Smem<EPI>;
    constexpr bool kPaired = L::kPaired;
    constexpr int kStages = L::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem + L::kA;
    uint8_t *sB = smem + L::kB;
    uint8_t *sSFA = smem + L::kSFA;
    uint8_t *sSFB = smem + L::kSFB;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kBars);
    uint64_t *empty = full + kStages;
    uint64_t *sf_ready = empty + kStages;
    uint64_t *acc_full = sf_ready + kStages;
    uint64_t *acc_empty = acc_full + kNumAcc;
    uint64_t *drain = acc_empty + kNumAcc;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
    __shared__ int never_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sf_ready[s], 4);
        }
        for (int b = 0; b < kNumAcc; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        never_abort = 0;
        fence_mbar_init();
        tma_prefetch_map(&map_a);
        tma_prefetch_map(&map_a32);
        tma_prefetch_map(&map_b);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int m_tiles = (p.mtiles != nullptr) ? *reinterpret_cast<volatile const int32_t *>(p.num_mtiles_dev)
                                              : p.dense_m_tiles;
    const int total = m_tiles * p.n_tiles;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------- producer
            int stage = 0;
            uint32_t phase = 0, pend_mask = 0, pend_par = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const TileInfo ti = decode_tile(p, t, m_tiles);
                const int64_t brow0 = ti.e * p.b_rows_per_expert + static_cast<int64_t>(ti.nt) * p.b_tile_rows;
                const int64_t brow1 = brow0 + p.b_half_offset;
                const int a_boxes = ti.valid >= kBM ? 0 : (ti.valid + 31) / 32;   // 0: one 128-row box
                const uint32_t a_bytes = a_boxes == 0 ? kTileBytes : a_boxes * (kTileBytes / 4);
                const uint8_t *sfa = p.sfa + static_cast<int64_t>(ti.row0 / kBM) * p.sfa_block_stride;
                const uint8_t *sfb0 = p.sfb + (brow0 / 128) * p.sfb_block_stride;
                const uint8_t *sfb1 = p.sfb + (brow1 / 128) * p.sfb_block_stride;
                for (int kt = 0; kt < p.num_k_tiles; ++kt) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int nkb = min(4, (p.K - kt * kBK) / 64);
                    const uint32_t sf_bytes = static_cast<uint32_t>(nkb * kSFAtom);
                    mbar_arrive_expect_tx(&full[stage], a_bytes + kTileBytes + sf_bytes * (kPaired ? 3 : 2));
                    uint8_t *a_dst = sA + stage * kTileBytes;
                    if (a_boxes == 0) {
                        tma_load_2d(a_dst, &map_a, kt * kBKBytes, ti.row0, &full[stage]);
                    } else {
                        for (int i = 0; i < a_boxes; ++i)
                            tma_load_2d(a_dst + i * (kTileBytes / 4), &map_a32, kt * kBKBytes, ti.row0 + 32 * i,
                                        &full[stage]);
                    }
                    uint8_t *b_dst = sB + stage * kTileBytes;
                    if constexpr (kPaired) {
                        tma_load_2d(b_dst, &map_b, kt * kBKBytes, static_cast<int32_t>(brow0), &full[stage]);
                        tma_load_2d(b_dst + kTileBytes / 2, &map_b, kt * kBKBytes, static_cast<int32_t>(brow1),
                                    &full[stage]);
                        uint8_t *raw = sSFB + stage * 2 * kSFStage;
                        bulk_load(raw, sfb0 + kt * kSFStage, sf_bytes, &full[stage]);
                        bulk_load(raw + kSFStage, sfb1 + kt * kSFStage, sf_bytes, &full[stage]);
                    } else {
                        tma_load_2d(b_dst, &map_b, kt * kBKBytes, static_cast<int32_t>(brow0), &full[stage]);
                        bulk_load(sSFB + stage * kSFStage, sfb0 + kt * kSFStage, sf_bytes, &full[stage]);
                    }
                    bulk_load(sSFA + stage * kSFStage, sfa + kt * kSFStage, sf_bytes, &full[stage]);
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
        constexpr uint32_t idesc = idesc_nvf4(kBM, kBN);
        if (lane == 0) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * kBN);
                for (int kt = 0; kt < p.num_k_tiles; ++kt) {
                    if (!mbar_wait(&sf_ready[stage], phase, abort_flag) || !mbar_wait(&full[stage], phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nkb = min(4, (p.K - kt * kBK) / 64);
                    const uint32_t a_addr = smem_u32(sA + stage * kTileBytes);
                    const uint32_t b_addr = smem_u32(sB + stage * kTileBytes);
                    const uint32_t t_sfa = tmem + kTmemSF + static_cast<uint32_t>(stage) * kSFSlotCols;
                    for (int kb = 0; kb < nkb; ++kb)
                        tc_mma_nvf4(d_tmem, sdesc_kmajor_sw128(a_addr + kb * 32), sdesc_kmajor_sw128(b_addr + kb * 32),
                                    idesc, t_sfa + kb * 4, t_sfa + 16 + kb * 4, (kt | kb) != 0 ? 1u : 0u);
                    tc_commit(&empty[stage]);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
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
            tc_commit(drain);
            mbar_wait(drain, 0, &never_abort);
        }
        __syncwarp();
    } else if (warp >= kFirstSFWarp) {
        // -------------------------------------------------------- scale stagers
        const int q = warp & 3;
        const uint32_t t_q = tmem + (static_cast<uint32_t>(q * 32) << 16) + kTmemSF;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            // paired tiles: byte offset of this tile's two 32-row groups inside a 16-byte scale row
            const int pair_off = kPaired ? (tile_nt(p, t, m_tiles) & 1) * 8 : 0;
            for (int kt = 0; kt < p.num_k_tiles; ++kt) {
                const bool got = mbar_wait(&full[stage], phase, abort_flag);
                if (!__all_sync(0xffffffffu, got)) {
                    ok = false;
                    break;
                }
                const int nkb = min(4, (p.K - kt * kBK) / 64);
                uint32_t ra[16], rb[16];
                const uint8_t *sfa = sSFA + stage * kSFStage + lane * 16;
#pragma unroll
                for (int kb = 0; kb < 4; ++kb) {
                    uint4 va = make_uint4(0, 0, 0, 0), vb = make_uint4(0, 0, 0, 0);
                    if (kb < nkb) {
                        va = *reinterpret_cast<const uint4 *>(sfa + kb * kSFAtom);
                        if constexpr (kPaired) {
                            const uint8_t *raw = sSFB + stage * 2 * kSFStage + kb * kSFAtom + lane * 16 + pair_off;
                            const uint2 g = *reinterpret_cast<const uint2 *>(raw);
                            const uint2 u = *reinterpret_cast<const uint2 *>(raw + kSFStage);
                            vb = make_uint4(g.x, g.y, u.x, u.y);
                        } else {
                            vb = *reinterpret_cast<const uint4 *>(sSFB + stage * kSFStage + kb * kSFAtom + lane * 16);
                        }
                    }
                    ra[4 * kb] = va.x, ra[4 * kb + 1] = va.y, ra[4 * kb + 2] = va.z, ra[4 * kb + 3] = va.w;
                    rb[4 * kb] = vb.x, rb[4 * kb + 1] = vb.y, rb[4 * kb + 2] = vb.z, rb[4 * kb + 3] = vb.w;
                }
                const uint32_t t_slot = t_q + static_cast<uint32_t>(stage) * kSFSlotCols;
                tc_st_32x32b_x16(t_slot, ra);
                tc_st_32x32b_x16(t_slot + 16, rb);
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&sf_ready[stage]);
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
        const int row = q * 32 + lane;          // row of the tile owned by this thread
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(q * 32) << 16);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            const bool got = mbar_wait(&acc_full[acc], acc_phase, abort_flag);
            if (!__all_sync(0xffffffffu, got)) {
                *abort_flag = 1;
                record_error(p.err, NVFP4_ERR_TIMEOUT);
                break;
            }
            tc_fence_after();
            const TileInfo ti = decode_tile(p, t, m_tiles);
            const bool valid = row < ti.valid;
            const uint32_t t_acc = t_lane + static_cast<uint32_t>(acc * kBN);

            if constexpr (EPI == EPI_SWIGLU_QUANT || EPI == EPI_SWIGLU_AMAX) {
                const float a = p.a_gs[0];
                const float alpha_g = __fdiv_rn(1.0f, __fmul_rn(a, p.b_gs[ti.e * p.b_gs_stride + 0]));
                const float alpha_u = __fdiv_rn(1.0f, __fmul_rn(a, p.b_gs[ti.e * p.b_gs_stride + 1]));
                float amax = 0.0f;
                uint32_t sfword = 0;
                uint32_t codes[8];
                float hgs = 1.0f;
                if constexpr (EPI == EPI_SWIGLU_QUANT)
                    hgs = p.inter_gs[ti.e];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t g[16], u[16];
                    tc_ld_32x32b_x16(t_acc + c * 16, g);
                    tc_ld_32x32b_x16(t_acc + 64 + c * 16, u);
                    tc_wait_ld();
                    float h[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        h[i] = silu_mul(__uint_as_float(g[i]) * alpha_g, __uint_as_float(u[i]) * alpha_u);
                    if constexpr (EPI == EPI_SWIGLU_AMAX) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            amax = fmaxf(amax, fabsf(h[i]));
                    } else {
                        const uint32_t s = quantize16(h, hgs, codes[2 * c], codes[2 * c + 1]);
                        sfword |= s << (8 * c);
                    }
                }
                if constexpr (EPI == EPI_SWIGLU_AMAX) {
                    if (!valid)
                        amax = 0.0f;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1)
                        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                    if (lane == 0)
                        atomicMax(p.amax_bits + ti.e, __float_as_uint(amax));
                } else if (valid) {
                    // 64 h columns of this row: 32 bytes of codes and one 4-byte scale word (k-block nt)
                    uint4 *hrow = reinterpret_cast<uint4 *>(p.h_codes + static_cast<int64_t>(ti.row0 + row) * p.h_ld_bytes +
                                                            ti.nt * 32);
                    hrow[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
                    hrow[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
                    *reinterpret_cast<uint32_t *>(p.h_sf + static_cast<int64_t>(ti.row0 / kBM) * p.h_sf_block_stride +
                                                  static_cast<int64_t>(ti.nt) * kSFAtom + lane * 16 + q * 4) = sfword;
                }
            } else {
                const float a = p.a_gs[p.a_gs_per_expert ? ti.e : 0];
                __nv_bfloat16 *orow = p.out + static_cast<int64_t>(ti.row0_out + row) * p.ldo +
                                      static_cast<int64_t>(ti.nt) * kBN;
#pragma unroll
                for (int c = 0; c < kBN / 32; ++c) {
                    uint32_t v0[16], v1[16];
                    tc_ld_32x32b_x16(t_acc + c * 32, v0);
                    tc_ld_32x32b_x16(t_acc + c * 32 + 16, v1);
                    tc_wait_ld();
                    const int col = ti.nt * kBN + c * 32;
                    int seg = 0;
#pragma unroll
                    for (int i = 0; i < 3; ++i)
                        if (i < p.nseg - 1 && col >= p.seg_end[i])
                            seg = i + 1;
                    const float alpha = __fdiv_rn(1.0f, __fmul_rn(a, p.b_gs[ti.e * p.b_gs_stride + seg]));
                    if (valid) {
                        uint32_t ow[16];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(v0[2 * i]) * alpha,
                                                                     __uint_as_float(v0[2 * i + 1]) * alpha);
                            ow[i] = *reinterpret_cast<uint32_t *>(&b);
                            __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v1[2 * i]) * alpha,
                                                                      __uint_as_float(v1[2 * i + 1]) * alpha);
                            ow[8 + i] = *reinterpret_cast<uint32_t *>(&b2);
                        }
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(ow[4 * i], ow[4 * i + 1], ow[4 * i + 2], ow[4 * i + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&acc_empty[acc]);
            if (++acc == kNumAcc) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int EPI>
static cudaError_t launch_one(const CUtensorMap &map_a, const CUtensorMap &map_a32, const CUtensorMap &map_b,
                              const GemmArgs &args, int grid, cudaStream_t stream)
{
    const int smem = Smem<EPI>::kTotal;
    static int attr_done_device = -1;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (attr_done_device != dev) {
        e = cudaFuncSetAttribute(nvfp4_gemm_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess)
            return e;
        attr_done_device = dev;
    }
    nvfp4_gemm_kernel<EPI><<<grid, kThreads, smem, stream>>>(map_a, map_a32, map_b, args);
    return cudaGetLastError();
}

cudaError_t launch_gemm(int epi, const CUtensorMap &map_a, const CUtensorMap &map_a32, const CUtensorMap &map_b,
                        const GemmArgs &args, int grid, cudaStream_t stream)
{
    switch (epi) {
    case EPI_SWIGLU_QUANT: return launch_one<EPI_SWIGLU_QUANT>(map_a, map_a32, map_b, args, grid, stream);
    case EPI_SWIGLU_AMAX: return launch_one<EPI_SWIGLU_AMAX>(map_a, map_a32, map_b, args, grid, stream);
    default: return launch_one<EPI_BF16>(map_a, map_a32, map_b, args, grid, stream);
    }
}

} // namespace nvfp4
