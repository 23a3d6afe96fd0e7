// internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nvfp4moe.h"

namespace nvfp4 {

// Launches `kernel` with programmatic stream serialization: it may begin
// while the previous kernel on the stream finishes, and must call pdl_wait()
// before touching anything that kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Raises `kernel`'s dynamic shared-memory limit to `bytes` on the current
// device, once per (kernel, device): *done_mask keeps one bit per device id
// below 64 (larger ids set the attribute on every call).  Safe to call from
// several host threads driving different devices.
cudaError_t ensure_smem_limit(const void *kernel, int bytes, unsigned long long *done_mask);

// Host-side checks of nvfp4_moe_forward's arguments (shapes, null pointers,
// 16-byte alignment), as a status code; no device work (api.cu).
int moe_args_status(const nvfp4_moe_args *args, bool need_out);

// Arguments of the persistent block-scaled FP4 GEMM engine (gemm.cu).
struct GemmArgs {
    // scale factors, NVFP4_SCALES_MMA layout: one 128-row block = (K/64) atoms of 512 bytes
    const uint8_t *sfa;
    int64_t sfa_block_stride;
    const uint8_t *sfb;
    int64_t sfb_block_stride;
    // sfa_rowmajor: A's scales in row blocks instead: for each 128-row block
    // and k-tile, 2 KB holding 16 bytes per row (its 16 scales of the k-tile)
    // -- same addressing as the MMA atoms, row-major inside; a partial m-tile
    // copies only its first 32-row groups.  The permuted activations of the
    // grouped L1 use it (the front writes them one token row at a time).
    int sfa_rowmajor;
    int K;                    // reduction length in elements, multiple of 64
    int num_k_tiles;          // ceil(K / 256)
    // tile space: grouped (m-tile table written on the device) or dense
    const int32_t *num_mtiles_dev;
    const int4 *mtiles;       // {expert, first padded row, valid rows, first output row}
    const int32_t *num_pairs_dev;
    const int2 *pairs;        // pair tiles: {first m-tile, second m-tile of the same expert or -1}
    const int32_t *num_light_dev;
    const int32_t *light;     // 1-CTA tiles: the m-tiles not covered by pairs, by index into mtiles
    int32_t *ready;           // fused L1 -> L2 launch: per m-tile count of published L1 epilogue warps
    int dense_m_tiles;
    int dense_M;
    int n_tiles;
    int64_t b_rows_per_expert;
    int b_tile_rows;          // B rows advanced per n-tile (128 for the gate/up tiles of L1, else bn)
    int b_half_offset;        // row offset of the second 128-row box of a 256-wide tile (I for L1: the up half)
    // global scales: alpha = 1 / (a_gs * b_gs)
    const float *a_gs;
    int a_gs_per_expert;
    const float *b_gs;
    int b_gs_stride;          // b_gs index = expert * b_gs_stride + segment
    int nseg;
    int seg_end[4];           // column ends of the B segments (dense GEMM)
    // SwiGLU epilogues
    const float *inter_gs;
    uint8_t *h_codes;
    int64_t h_ld_bytes;
    uint8_t *h_sf;
    int64_t h_sf_block_stride;
    unsigned int *amax_bits;
    // bf16 epilogue
    __nv_bfloat16 *out;
    int64_t ldo;
    int out_tma;              // pair tiles: store through shared memory with the output tensor map
    int32_t *err;             // device error word
    // fused grouped launches: the 1-CTA launch claims its tiles one at a time
    // from this counter (zeroed by the front launch); in pair mode 1 the pair
    // launch lets its dependent start at once (pdl_trigger_early), so the
    // 1-CTA launch's CTAs take over SMs as pair CTAs finish, and the 1-CTA
    // launch waits for the pair launch only at its end (pdl_wait_at_end)
    int32_t *claim;
    int pdl_trigger_early;
    int pdl_wait_at_end;
};

enum Epilogue { EPI_SWIGLU_QUANT = 0, EPI_BF16 = 1, EPI_SWIGLU_AMAX = 2 };

// Launches the GEMM engine with 128 x bn tiles (bn 256, or 128 for EPI_BF16
// when N is not a multiple of 256), or with cg = 2 as clusters of two CTAs
// computing 256 x 256 tiles with pair MMAs (bn 256, grid even).  map_a /
// map_a32: 2-D uint8 tensor maps over the A code matrix with boxes of 128 and
// 32 rows; map_b: over the B code matrix with 128-row boxes; every box is 128
// bytes wide with 128-byte swizzle.  map_out (with args.out_tma = 1, bf16
// pair tiles only): 2-D bf16 tensor map over out ([rows, ldo], the rows the
// GEMM may write) with 32 x 32 boxes and 64-byte swizzle.
cudaError_t launch_gemm(int bn, int epi, int cg, const CUtensorMap &map_a, const CUtensorMap &map_a32,
                        const CUtensorMap &map_b, const GemmArgs &args, int grid, cudaStream_t stream,
                        const CUtensorMap *map_out = nullptr);
// One bounded counter wait (the fused launch's) in a one-thread kernel.
cudaError_t launch_wait_probe(const int32_t *flag, int target, int32_t *err, cudaStream_t s);
// Pair clusters that fit on the device at once (<= num_sms / 2).
int gemm_pair_clusters(int num_sms);
// One persistent launch of the grouped L1 (args1, maps *1, SwiGLU +
// re-quantisation epilogue) and L2 (args2, maps *2, bf16 epilogue) tiles:
// every L1 tile, then every L2 tile; an L2 tile starts once its m-tile's L1
// tiles are published in args1.ready / args2.ready (zeroed by the front).
// cg = 1: the light list on 1-CTA tiles, tiles claimed one at a time from
// args1.claim (no residency requirement: a tile waits only on tiles claimed
// before it, whose CTAs are running); cg = 2: the pair list on pair tiles,
// tiles dealt round-robin to the clusters (grid / 2 of them, all resident).
cudaError_t launch_moe_fused(int cg, const CUtensorMap &map_a1, const CUtensorMap &map_a1_32,
                             const CUtensorMap &map_b1, const GemmArgs &args1, const CUtensorMap &map_a2,
                             const CUtensorMap &map_a2_32, const CUtensorMap &map_b2, const GemmArgs &args2, int grid,
                             cudaStream_t stream);

// The forward's front in one launch (front.cu): the batch's global scale of
// x (x_gs == nullptr), routing and the tile tables, quantise + permute (x ==
// nullptr: routing only).  pair_mode 0: every m-tile is a 1-CTA ("light")
// tile; 1: experts with two or more m-tiles give their consecutive full
// pairs to the pair list and only the odd last m-tile to the light list;
// 2: every m-tile in a pair (the odd last one with an empty partner).
constexpr int kFrontMaxBlocks = 256;
struct FrontArgs {
    const __nv_bfloat16 *x;
    const int32_t *ids;
    int64_t T, H;
    int E, k;
    const float *x_gs;
    float *gs_out;
    int pair_mode;
    int32_t *counts, *off, *poff;
    int32_t *num_mtiles;
    int4 *mtiles;
    int32_t *num_pairs;
    int2 *pairs;
    int32_t *num_light;
    int32_t *light;
    int32_t *ready;           // may be null
    int32_t *claim;           // tile claim counter of the fused 1-CTA launch (zeroed here)
    int32_t *inv, *yrow;
    int32_t *err;
    uint8_t *a_codes, *a_sf;  // a_sf in row blocks: [rows/128][H/256 k-tiles][128 rows][16 bytes]
    // activations already in NVFP4 (x == nullptr, x_gs given): codes [T, H/2]
    // and row-major scales [T, H/16] that phase 3 only permutes
    const uint8_t *xq_codes, *xq_scales;
    int32_t *blk_hist;        // [kFrontMaxBlocks][(E + 3) & ~3]
    float *blk_amax;          // [kFrontMaxBlocks]
    unsigned int *ticket;     // zeroed once with the workspace
};
cudaError_t launch_front(const FrontArgs &args, int num_sms, cudaStream_t s);

// Memory-bound kernels (kernels.cu).
cudaError_t launch_amax_bf16(const __nv_bfloat16 *x, int64_t n, float *gs_out, int num_sms, cudaStream_t s);
cudaError_t launch_finalize_gs(float *gs, cudaStream_t s);
cudaError_t launch_quantize(const __nv_bfloat16 *x, int64_t rows, int64_t cols, int64_t ldx, const float *gs,
                            uint8_t *codes, uint8_t *scales, int layout, cudaStream_t s);
cudaError_t launch_swizzle(const uint8_t *in, int64_t batch, int64_t rows, int64_t cols, uint8_t *out,
                           cudaStream_t s);
cudaError_t launch_combine(const __nv_bfloat16 *y, const int32_t *yrow, const float *w, int64_t T, int k, int64_t H,
                           __nv_bfloat16 *out, cudaStream_t s);
cudaError_t launch_finalize_inter_gs(const unsigned int *amax_bits, int E, float *inter_gs, cudaStream_t s);
cudaError_t launch_mma_ceiling(int bn, int iters, int ctas, long long *cycles, int32_t *err, cudaStream_t s);
// TMA streaming probe (ceiling.cu): map = the GEMM's 128-row B-box map over
// a [rows, row_bytes] uint8 matrix (rows % 256 == 0, row_bytes % 128 == 0).
cudaError_t launch_tma_stream(const CUtensorMap &map, int64_t rows, int64_t row_bytes, int64_t work_tiles,
                              int stages, int ctas, int32_t *err, cudaStream_t s);
cudaError_t launch_topk(const float *logits, int64_t T, int E, int k, int ns, int scoring, int32_t *ids,
                        float *weights, cudaStream_t s);

} // namespace nvfp4
