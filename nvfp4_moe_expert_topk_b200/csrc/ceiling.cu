// ceiling.cu -- throughput probe of the block-scaled FP4 tensor-core
// instruction the GEMM engine issues (tcgen05.mma kind::mxf4nvf4, block16
// E4M3 scales, M = 128, K = 64, N = 256 or 128), with operands resident on
// chip: one CTA per SM fills a 128-row A tile and a BN-row B tile in shared
// memory (128-byte swizzled, K-major, pseudo-random E2M1 codes) and the
// scale slots in tensor memory once, then one thread issues `iters` k-tiles
// of four MMAs into one fp32 accumulator, the GEMM's own issue pattern
// without any memory traffic.  Its FLOP rate is the tensor-pipe ceiling the
// GEMMs are measured against; the per-CTA cycle count gives the pipe time of
// one instruction independent of the clock.
#include "internal.h"
#include "ptx.cuh"

namespace nvfp4 {

namespace {

constexpr int kCeilThreads = 128;
constexpr uint32_t kCeilTmemCols = 512;

template <int BN>
__global__ void __launch_bounds__(kCeilThreads, 1)
    mma_ceiling_kernel(int iters, long long *cycles, int32_t *err)
{
    constexpr int kABytes = 128 * 128;
    constexpr int kBBytes = BN * 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + kABytes;
    __shared__ uint64_t done;
    __shared__ uint32_t tmem_slot;
    __shared__ int never_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // pseudo-random codes (any nibble is a finite E2M1 value)
    uint32_t *words = reinterpret_cast<uint32_t *>(smem);
    for (int i = threadIdx.x; i < (kABytes + kBBytes) / 4; i += kCeilThreads) {
        uint32_t h = (static_cast<uint32_t>(i) + 0x9E3779B9u * (blockIdx.x + 1)) * 2654435761u;
        h ^= h >> 15;
        words[i] = h * 2246822519u;
    }
    if (threadIdx.x == 0) {
        mbar_init(&done, 1);
        never_abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, kCeilTmemCols);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;
    const uint32_t t_sf = tmem + 256;          // scale columns after the accumulator
    // every scale 1.0 (E4M3 0x38): A 16 columns, B 16 per 128-row half
    {
        uint32_t r[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            r[i] = 0x38383838u;
        const uint32_t t_q = t_sf + (static_cast<uint32_t>(warp * 32) << 16);
        tc_st_32x32b_x16(t_q, r);
        tc_st_32x32b_x16(t_q + 16, r);
        if (BN == 256)
            tc_st_32x32b_x16(t_q + 32, r);
        tc_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (threadIdx.x == 0) {
        constexpr uint32_t idesc = idesc_nvf4(128, BN);
        constexpr int kHalves = BN / 128;
        const uint32_t a_addr = smem_u32(sA), b_addr = smem_u32(sB);
        const long long t0 = clock64();
        for (int it = 0; it < iters; ++it) {
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)
                tc_mma_nvf4(tmem, sdesc_kmajor_sw128(a_addr + kb * 32), sdesc_kmajor_sw128(b_addr + kb * 32), idesc,
                            t_sf + kb * 4, t_sf + 16 + kb * 4 * kHalves, (it | kb) != 0 ? 1u : 0u);
        }
        tc_commit(&done);
        const bool ok = mbar_wait(&done, 0, &never_abort);
        const long long t1 = clock64();
        cycles[blockIdx.x] = ok ? t1 - t0 : -1;
        if (!ok && err != nullptr)
            atomicCAS(err, 0, NVFP4_ERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) {
        __syncwarp();
        tmem_dealloc(tmem, kCeilTmemCols);
    }
    (void)lane;
}

// TMA streaming probe: the GEMM engine's B-operand loads with nothing else.
// One CTA per SM; one thread loads, per step, two 128-row x 128-byte boxes
// (one k-tile of a 256-row weight tile, the map's 128-byte swizzle) into a
// `stages`-deep ring of 32 KB stages, and another thread releases each stage
// as soon as it has landed.  Tiles of 256 rows x (row_bytes / 128) steps are
// dealt round-robin; tile t reads rows of tile t mod (rows / 256), so a matrix
// larger than L2 measures the HBM read rate and a small one the L2 ->
// shared-memory rate.
constexpr int kStreamThreads = 64;
constexpr int kStreamStage = 2 * 128 * 128;

__global__ void __launch_bounds__(kStreamThreads, 1)
    tma_stream_kernel(const __grid_constant__ CUtensorMap map, int64_t work_tiles, int64_t tiles, int ksteps,
                      int stages, int32_t *err)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + stages * kStreamStage);
    uint64_t *empty = full + stages;
    __shared__ int abort_flag;
    __shared__ int never_abort;
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        abort_flag = 0;
        never_abort = 0;
        fence_mbar_init();
        tma_prefetch_map(&map);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int stage = 0;
        uint32_t phase = 0, pend = 0, pend_par = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < work_tiles && ok; t += gridDim.x) {
            const int64_t row0 = (t % tiles) * 256;
            for (int k = 0; k < ksteps; ++k) {
                if (!mbar_wait(&empty[stage], phase ^ 1u, &abort_flag)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&full[stage], kStreamStage);
                for (int h = 0; h < 2; ++h)
                    tma_load_2d(smem + stage * kStreamStage + h * (kStreamStage / 2), &map, k * 128,
                                static_cast<int32_t>(row0 + 128 * h), &full[stage]);
                pend |= 1u << stage;
                pend_par = (pend_par & ~(1u << stage)) | (phase << stage);
                if (++stage == stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok) {
            abort_flag = 1;
            if (err != nullptr)
                atomicCAS(err, 0, NVFP4_ERR_TIMEOUT);
        }
        for (int s = 0; s < stages; ++s)           // every copy has landed before the block exits
            if ((pend >> s) & 1u)
                mbar_wait(&full[s], (pend_par >> s) & 1u, &never_abort);
    } else if (threadIdx.x == 32) {
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; t < work_tiles && ok; t += gridDim.x) {
            for (int k = 0; k < ksteps; ++k) {
                if (!mbar_wait(&full[stage], phase, &abort_flag)) {
                    ok = false;
                    break;
                }
                mbar_arrive(&empty[stage]);
                if (++stage == stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok) {
            abort_flag = 1;
            if (err != nullptr)
                atomicCAS(err, 0, NVFP4_ERR_TIMEOUT);
        }
    }
    __syncthreads();
}

} // namespace

cudaError_t launch_tma_stream(const CUtensorMap &map, int64_t rows, int64_t row_bytes, int64_t work_tiles,
                              int stages, int ctas, int32_t *err, cudaStream_t s)
{
    auto smem_of = [](int n) { return n * kStreamStage + 2 * n * 8 + 1024; };
    const int smem = smem_of(stages);
    static unsigned long long attr_done = 0;     // one bit per device; the limit allows the deepest ring
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(tma_stream_kernel), smem_of(6), &attr_done);
    if (e != cudaSuccess)
        return e;
    tma_stream_kernel<<<ctas, kStreamThreads, smem, s>>>(map, work_tiles, rows / 256,
                                                         static_cast<int>(row_bytes / 128), stages, err);
    return cudaGetLastError();
}

cudaError_t launch_mma_ceiling(int bn, int iters, int ctas, long long *cycles, int32_t *err, cudaStream_t s)
{
    // 130 KB of dynamic shared memory (48 KB used) keeps one CTA per SM, so
    // `ctas` = the SM count puts one issuing thread on every SM.
    const int smem = 130 * 1024;
    if (bn == 256) {
        cudaError_t e = cudaFuncSetAttribute(mma_ceiling_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess)
            return e;
        mma_ceiling_kernel<256><<<ctas, kCeilThreads, smem, s>>>(iters, cycles, err);
    } else {
        cudaError_t e = cudaFuncSetAttribute(mma_ceiling_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess)
            return e;
        mma_ceiling_kernel<128><<<ctas, kCeilThreads, smem, s>>>(iters, cycles, err);
    }
    return cudaGetLastError();
}

} // namespace nvfp4
