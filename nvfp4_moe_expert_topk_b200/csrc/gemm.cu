// gemm.cu -- persistent block-scaled FP4 GEMM engine for sm_100a.
//
// D[128 x BN] tiles of  A (E2M1 codes, K-major) x B^T (E2M1 codes, K-major)
// with one E4M3 scale per 16 elements on both sides, on the 5th-generation
// tensor cores (tcgen05.mma kind::mxf4nvf4, block16 scaling), accumulating in
// fp32 in tensor memory.  This is the grouped GEMM of the expert chain
// ("nvfp4-megamoe-kernel / CURRENT_BUG.md", page 1 "Phase 1": L1 gate_up
// GEMM -> SiLU -> re-quantise -> L2 GEMM; with one group it is the plain
// NVFP4 GEMM of page 1 "Phase 2").
//
// Block of 6 warps, one block per SM, persistent over the tile list:
//   warp 0    TMA producer: per k-tile (256 elements) one 128x128-byte box
//             of A, one or two 128x128-byte boxes of B (128-byte swizzle),
//             and the matching 512-byte scale atoms by bulk copy, into a
//             4-stage shared-memory ring guarded by mbarriers;
//   warp 1    allocates TMEM, and one thread issues tcgen05.cp (scales ->
//             TMEM) and tcgen05.mma (4 instructions of K=64 per k-tile);
//   warps 2-5 epilogue: TMEM -> registers (each thread owns one row of the
//             128-row tile), then one of
//             EPI_SWIGLU_QUANT  h = SiLU(a_g*g) * (a_u*u), NVFP4-quantised
//                               with the expert's inter_gs (L1),
//             EPI_SWIGLU_AMAX   same h, max|h| per expert (warmup),
//             EPI_BF16          y = alpha * acc -> bf16 (L2, dense GEMM).
// In the L1 tile the B tile is 128 gate rows stacked on the 128 matching up
// rows, so TMEM columns 0-127 hold gate and 128-255 hold up of the same h
// columns, and every 16-element block of h is produced by one thread.
//
// The tile list is either dense (m-tiles of M) or grouped: an m-tile table
// written on the device by the routing kernel (expert, first padded row,
// valid rows, first output row), so the launch needs no host sync and every
// expert's rows are covered by one tensor map over the padded A buffer and
// one over all experts' stacked weights.
//
// Every mbarrier wait is bounded (ptx.cuh): on a timeout the block records
// NVFP4_ERR_TIMEOUT in the error word, stops issuing, waits (bounded) for its
// copies and MMAs in flight, frees its TMEM and returns.
#include "internal.h"
#include "quant.cuh"

namespace nvfp4 {

constexpr int kBM = 128;
constexpr int kBK = 256;                        // elements per k-tile
constexpr int kBKBytes = 128;                   // bytes of codes per row per k-tile
constexpr int kStages = 4;
constexpr int kATileBytes = kBM * kBKBytes;     // 16 KB
constexpr int kBHalfBytes = 128 * kBKBytes;     // 16 KB
constexpr int kSFAtom = 512;                    // 128 rows x 4 scales
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemSFA = 256;              // 4 k-blocks x 4 columns
constexpr uint32_t kTmemSFB = 272;              // 4 k-blocks x (4 or 8) columns

template <int BN>
struct Smem {
    static constexpr int kHalves = BN / 128;
    static constexpr int kBTileBytes = BN * kBKBytes;
    static constexpr int kSFBStageBytes = kHalves * 4 * kSFAtom;
    static constexpr int kA = 0;
    static constexpr int kB = kA + kStages * kATileBytes;
    static constexpr int kSFA = kB + kStages * kBTileBytes;
    static constexpr int kSFB = kSFA + kStages * 4 * kSFAtom;
    static constexpr int kBars = kSFB + kStages * kSFBStageBytes;
    static constexpr int kBarCount = 2 * kStages + 3;
    static constexpr int kMisc = kBars + kBarCount * 8;
    static constexpr int kTotal = kMisc + 16 + 1024;   // + tmem slot, abort flag, alignment slack
};

int gemm_smem_bytes(int bn)
{
    return bn == 256 ? Smem<256>::kTotal : Smem<128>::kTotal;
}

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

__device__ __forceinline__ void record_error(int32_t *err, int code)
{
    if (err != nullptr)
        atomicCAS(err, 0, code);
}

__device__ __forceinline__ float silu_mul(float g, float u)
{
    return g / (1.0f + __expf(-g)) * u;
}

template <int BN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                      const GemmArgs p)
{
    using L = Smem<BN>;
    constexpr int kHalves = L::kHalves;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem + L::kA;
    uint8_t *sB = smem + L::kB;
    uint8_t *sSFA = smem + L::kSFA;
    uint8_t *sSFB = smem + L::kSFB;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kBars);
    uint64_t *empty = full + kStages;
    uint64_t *acc_full = empty + kStages;
    uint64_t *acc_empty = acc_full + 1;
    uint64_t *drain = acc_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
    __shared__ int never_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 4);
        mbar_init(drain, 1);
        *abort_flag = 0;
        never_abort = 0;
        fence_mbar_init();
        tma_prefetch_map(&map_a);
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
                    mbar_arrive_expect_tx(&full[stage],
                                          kATileBytes + L::kBTileBytes + sf_bytes * (1 + kHalves));
                    tma_load_2d(sA + stage * kATileBytes, &map_a, kt * kBKBytes, ti.row0, &full[stage]);
                    tma_load_2d(sB + stage * L::kBTileBytes, &map_b, kt * kBKBytes, static_cast<int32_t>(brow0),
                                &full[stage]);
                    bulk_load(sSFA + stage * 4 * kSFAtom, sfa + kt * 4 * kSFAtom, sf_bytes, &full[stage]);
                    bulk_load(sSFB + stage * L::kSFBStageBytes, sfb0 + kt * 4 * kSFAtom, sf_bytes, &full[stage]);
                    if (kHalves == 2) {
                        tma_load_2d(sB + stage * L::kBTileBytes + kBHalfBytes, &map_b, kt * kBKBytes,
                                    static_cast<int32_t>(brow1), &full[stage]);
                        bulk_load(sSFB + stage * L::kSFBStageBytes + 4 * kSFAtom, sfb1 + kt * 4 * kSFAtom, sf_bytes,
                                  &full[stage]);
                    }
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
        if (lane == 0) {
            // ---------------------------------------------------- MMA issuer
            constexpr uint32_t idesc = idesc_nvf4(kBM, BN);
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                if (!mbar_wait(acc_empty, acc_phase ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kt = 0; kt < p.num_k_tiles; ++kt) {
                    if (!mbar_wait(&full[stage], phase, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nkb = min(4, (p.K - kt * kBK) / 64);
                    const uint32_t a_addr = smem_u32(sA + stage * kATileBytes);
                    const uint32_t b_addr = smem_u32(sB + stage * L::kBTileBytes);
                    const uint32_t sfa_addr = smem_u32(sSFA + stage * 4 * kSFAtom);
                    const uint32_t sfb_addr = smem_u32(sSFB + stage * L::kSFBStageBytes);
                    for (int kb = 0; kb < nkb; ++kb) {
                        tc_cp_32x128b_warpx4(tmem + kTmemSFA + kb * 4, sdesc_scale_block(sfa_addr + kb * kSFAtom));
#pragma unroll
                        for (int h = 0; h < kHalves; ++h)
                            tc_cp_32x128b_warpx4(tmem + kTmemSFB + kb * 4 * kHalves + h * 4,
                                                 sdesc_scale_block(sfb_addr + h * 4 * kSFAtom + kb * kSFAtom));
                    }
                    for (int kb = 0; kb < nkb; ++kb)
                        tc_mma_nvf4(tmem, sdesc_kmajor_sw128(a_addr + kb * 32), sdesc_kmajor_sw128(b_addr + kb * 32),
                                    idesc, tmem + kTmemSFA + kb * 4, tmem + kTmemSFB + kb * 4 * kHalves,
                                    (kt | kb) != 0 ? 1u : 0u);
                    tc_commit(&empty[stage]);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                tc_commit(acc_full);
                acc_phase ^= 1u;
            }
            if (!ok) {
                *abort_flag = 1;
                record_error(p.err, NVFP4_ERR_TIMEOUT);
            }
            // all MMAs and scale copies of this thread complete before TMEM is freed
            tc_commit(drain);
            mbar_wait(drain, 0, &never_abort);
        }
    } else {
        // -------------------------------------------------------- epilogue
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int row = q * 32 + lane;          // row of the tile owned by this thread
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(q * 32) << 16);
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x) {
            const bool got = mbar_wait(acc_full, acc_phase, abort_flag);
            if (!__all_sync(0xffffffffu, got)) {
                *abort_flag = 1;
                record_error(p.err, NVFP4_ERR_TIMEOUT);
                break;
            }
            tc_fence_after();
            const TileInfo ti = decode_tile(p, t, m_tiles);
            const bool valid = row < ti.valid;

            if constexpr (EPI == EPI_SWIGLU_QUANT || EPI == EPI_SWIGLU_AMAX) {
                const float a = p.a_gs[0];
                const float alpha_g = __fdiv_rn(1.0f, __fmul_rn(a, p.b_gs[ti.e * p.b_gs_stride + 0]));
                const float alpha_u = __fdiv_rn(1.0f, __fmul_rn(a, p.b_gs[ti.e * p.b_gs_stride + 1]));
                float hgs = 1.0f;
                uint8_t *hrow = nullptr;
                uint8_t *sfblk = nullptr;
                if constexpr (EPI == EPI_SWIGLU_QUANT) {
                    hgs = p.inter_gs[ti.e];
                    hrow = p.h_codes + static_cast<int64_t>(ti.row0 + row) * p.h_ld_bytes + ti.nt * 64;
                    sfblk = p.h_sf + static_cast<int64_t>(ti.row0 / kBM) * p.h_sf_block_stride + lane * 16 + q * 4;
                }
                float amax = 0.0f;
                uint32_t sfword = 0;
#pragma unroll 1
                for (int c = 0; c < 8; ++c) {
                    uint32_t g[16], u[16];
                    tc_ld_32x32b_x16(t_lane + c * 16, g);
                    tc_ld_32x32b_x16(t_lane + 128 + c * 16, u);
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
                        uint32_t lo, hi;
                        const uint32_t s = quantize16(h, hgs, lo, hi);
                        sfword |= s << (8 * (c & 3));
                        if (valid)
                            *reinterpret_cast<uint2 *>(hrow + c * 8) = make_uint2(lo, hi);
                        if ((c & 3) == 3) {
                            const int kb = ti.nt * 2 + (c >> 2);     // 64-column block of h
                            if (valid)
                                *reinterpret_cast<uint32_t *>(sfblk + static_cast<int64_t>(kb) * kSFAtom) = sfword;
                            sfword = 0;
                        }
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
                }
            } else {
                const float a = p.a_gs[p.a_gs_per_expert ? ti.e : 0];
                __nv_bfloat16 *orow = p.out + static_cast<int64_t>(ti.row0_out + row) * p.ldo +
                                      static_cast<int64_t>(ti.nt) * BN;
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    uint32_t v0[16], v1[16];
                    tc_ld_32x32b_x16(t_lane + c * 32, v0);
                    tc_ld_32x32b_x16(t_lane + c * 32 + 16, v1);
                    tc_wait_ld();
                    const int col = ti.nt * BN + c * 32;
                    int seg = 0;
#pragma unroll
                    for (int i = 0; i < 3; ++i)
                        if (i < p.nseg - 1 && col >= p.seg_end[i])
                            seg = i + 1;
                    const float alpha = __fdiv_rn(1.0f, __fmul_rn(a, p.b_gs[ti.e * p.b_gs_stride + seg]));
                    if (valid) {
                        uint4 o[4];
                        uint32_t *ow = reinterpret_cast<uint32_t *>(o);
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
                            dst[i] = o[i];
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(acc_empty);
            acc_phase ^= 1u;
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

template <int BN, int EPI>
static cudaError_t launch_one(const CUtensorMap &map_a, const CUtensorMap &map_b, const GemmArgs &args, int grid,
                              cudaStream_t stream)
{
    const int smem = Smem<BN>::kTotal;
    static int attr_done_device = -1;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (attr_done_device != dev) {
        e = cudaFuncSetAttribute(nvfp4_gemm_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess)
            return e;
        attr_done_device = dev;
    }
    nvfp4_gemm_kernel<BN, EPI><<<grid, kThreads, smem, stream>>>(map_a, map_b, args);
    return cudaGetLastError();
}

cudaError_t launch_gemm(int bn, int epi, const CUtensorMap &map_a, const CUtensorMap &map_b, const GemmArgs &args,
                        int grid, cudaStream_t stream)
{
    if (bn == 256) {
        switch (epi) {
        case EPI_SWIGLU_QUANT: return launch_one<256, EPI_SWIGLU_QUANT>(map_a, map_b, args, grid, stream);
        case EPI_SWIGLU_AMAX: return launch_one<256, EPI_SWIGLU_AMAX>(map_a, map_b, args, grid, stream);
        default: return launch_one<256, EPI_BF16>(map_a, map_b, args, grid, stream);
        }
    }
    return launch_one<128, EPI_BF16>(map_a, map_b, args, grid, stream);
}

} // namespace nvfp4
