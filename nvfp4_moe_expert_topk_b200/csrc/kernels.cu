// kernels.cu -- memory-bound kernels: global scale and max|x| of a tensor,
// plain NVFP4 quantisation, scale-layout conversion, the top-k weighted
// combine, the warmup scales and the top-k router.  (The forward's front --
// global scale, routing, quantise + permute -- is one launch, in front.cu.)
#include <algorithm>
#include <mutex>

#include "internal.h"
#include "quant.cuh"

namespace nvfp4 {

// ------------------------------------------------------------ global scale
// amax of a bf16 tensor, accumulated into *out_bits (the float bit pattern;
// non-negative floats order like their bits).  *out_bits must start at 0.
__global__ void __launch_bounds__(256) amax_bf16_kernel(const __nv_bfloat16 *__restrict__ x, int64_t n,
                                                        unsigned int *__restrict__ out_bits)
{
    pdl_wait();
    pdl_trigger();
    float m = 0.0f;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t nth = static_cast<int64_t>(gridDim.x) * blockDim.x;
    int64_t start_scalar = 0;
    if ((reinterpret_cast<uintptr_t>(x) & 15) == 0) {
        const int64_t n8 = n / 8;
        const uint4 *xv = reinterpret_cast<const uint4 *>(x);
        for (int64_t i0 = tid; i0 < n8; i0 += 4 * nth) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)     // four 16-byte loads in flight per thread
                v[u] = i0 + u * nth < n8 ? __ldg(xv + i0 + u * nth) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v[u]);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f = __bfloat1622float2(h[j]);
                    m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
                }
            }
        }
        start_scalar = n8 * 8;
    }
    for (int64_t i = start_scalar + tid; i < n; i += nth)
        m = fmaxf(m, fabsf(__bfloat162float(x[i])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float wmax[8];
    if ((threadIdx.x & 31) == 0)
        wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
            m = fmaxf(m, wmax[w]);
        atomicMax(out_bits, __float_as_uint(m));
    }
}

// gs = 2688 / amax (fp32, round to nearest), 1 if amax == 0; in place.
__global__ void finalize_gs_kernel(float *gs)
{
    pdl_wait();
    pdl_trigger();
    const float a = __uint_as_float(*reinterpret_cast<unsigned int *>(gs));
    *gs = (a == 0.0f) ? 1.0f : __fdiv_rn(2688.0f, a);
}

cudaError_t launch_amax_bf16(const __nv_bfloat16 *x, int64_t n, float *gs_out, int num_sms, cudaStream_t s)
{
    int64_t blocks = (n / 8 + 255) / 256;
    if (blocks < 1)
        blocks = 1;
    if (blocks > 8LL * num_sms)
        blocks = 8LL * num_sms;
    return launch_pdl(amax_bf16_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, x, n,
                      reinterpret_cast<unsigned int *>(gs_out));
}

cudaError_t launch_finalize_gs(float *gs, cudaStream_t s)
{
    return launch_pdl(finalize_gs_kernel, dim3(1), dim3(1), 0, s, gs);
}

// ------------------------------------------------------------ quantisation
// One warp per (row, 2048-column chunk); each lane handles 64 consecutive
// elements (4 blocks).  (The forward's quantisation of x, fused with the
// expert permutation, is in front.cu.)
constexpr int kQuantChunk = 2048;

// One (row, chunk) item by one whole warp (item < rows * chunks).
__device__ __forceinline__ void quantize_item(const __nv_bfloat16 *__restrict__ x, int64_t cols, int64_t ldx,
                                              float gs, uint8_t *__restrict__ codes, uint8_t *__restrict__ scales,
                                              int layout, int64_t item, int lane)
{
    const int64_t chunks = (cols + kQuantChunk - 1) / kQuantChunk;
    const int64_t row = item / chunks;
    const int64_t c0 = (item - row * chunks) * kQuantChunk + static_cast<int64_t>(lane) * 64;
    const bool active = c0 < cols;
    const int64_t kb_per_block = cols / 64;
    const __nv_bfloat16 *xr = x + row * ldx;
    const int64_t nb_left = active ? (cols - c0) / 16 : 0;
    const int nb = nb_left < 4 ? static_cast<int>(nb_left) : 4;
    uint32_t cw[8];
    uint32_t sw = 0;
    // all of this lane's loads first (up to 8 x 16 bytes in flight)
    uint4 ld[8];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const uint4 *src = reinterpret_cast<const uint4 *>(xr + c0 + 16 * b);
        ld[2 * b] = b < nb ? __ldg(src) : make_uint4(0, 0, 0, 0);
        ld[2 * b + 1] = b < nb ? __ldg(src + 1) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        cw[2 * b] = cw[2 * b + 1] = 0;
        if (b < nb) {
            const uint4 v0 = ld[2 * b], v1 = ld[2 * b + 1];
            const __nv_bfloat162 *h0 = reinterpret_cast<const __nv_bfloat162 *>(&v0);
            const __nv_bfloat162 *h1 = reinterpret_cast<const __nv_bfloat162 *>(&v1);
            float f[16];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 a = __bfloat1622float2(h0[j]);
                const float2 c = __bfloat1622float2(h1[j]);
                f[2 * j] = a.x;
                f[2 * j + 1] = a.y;
                f[8 + 2 * j] = c.x;
                f[8 + 2 * j + 1] = c.y;
            }
            const uint32_t sb = quantize16(f, gs, cw[2 * b], cw[2 * b + 1]);
            sw |= sb << (8 * b);
        }
    }
    if (active) {
        const int64_t dst = row;
        uint8_t *crow = codes + dst * (cols / 2) + c0 / 2;
        if (nb == 4) {
            reinterpret_cast<uint4 *>(crow)[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            reinterpret_cast<uint4 *>(crow)[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
        } else {
#pragma unroll
            for (int b = 0; b < 4; ++b)
                if (b < nb)
                    reinterpret_cast<uint2 *>(crow)[b] = make_uint2(cw[2 * b], cw[2 * b + 1]);
        }
        if (layout == NVFP4_SCALES_MMA) {
            *reinterpret_cast<uint32_t *>(scales + mma_scale_offset(dst, c0 / 64, kb_per_block)) = sw;
        } else {
            uint8_t *srow = scales + dst * (cols / 16) + c0 / 16;
            if (nb == 4 && (cols % 64) == 0)
                *reinterpret_cast<uint32_t *>(srow) = sw;
            else
                for (int b = 0; b < nb; ++b)
                    srow[b] = static_cast<uint8_t>(sw >> (8 * b));
        }
    }
}

__global__ void __launch_bounds__(256) quantize_rows_kernel(const __nv_bfloat16 *__restrict__ x, int64_t rows,
                                                            int64_t cols, int64_t ldx, const float *__restrict__ gs_ptr,
                                                            uint8_t *__restrict__ codes, uint8_t *__restrict__ scales,
                                                            int layout)
{
    pdl_wait();
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t chunks = (cols + kQuantChunk - 1) / kQuantChunk;
    const int64_t item = static_cast<int64_t>(blockIdx.x) * 8 + warp;
    if (item >= rows * chunks)
        return;
    quantize_item(x, cols, ldx, __ldg(gs_ptr), codes, scales, layout, item, lane);
}

cudaError_t launch_quantize(const __nv_bfloat16 *x, int64_t rows, int64_t cols, int64_t ldx, const float *gs,
                            uint8_t *codes, uint8_t *scales, int layout, cudaStream_t s)
{
    const int64_t items = rows * ((cols + kQuantChunk - 1) / kQuantChunk);
    const int64_t blocks = (items + 7) / 8;
    return launch_pdl(quantize_rows_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, x, rows, cols, ldx, gs,
                      codes, scales, layout);
}

// ------------------------------------------------------------ scale layout
// One thread per 4-byte word of the MMA layout: row r, 64-element block kb.
__global__ void swizzle_scales_kernel(const uint8_t *__restrict__ in, int64_t batch, int64_t rows, int64_t cols,
                                      uint8_t *__restrict__ out)
{
    const int64_t kbs = cols / 64;
    const int64_t rblocks = (rows + 127) / 128;
    const int64_t per_batch_words = rblocks * kbs * 128;
    const int64_t total = batch * per_batch_words;
    for (int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; w < total;
         w += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t b = w / per_batch_words;
        int64_t rem = w - b * per_batch_words;
        const int64_t atom = rem / 128;
        const int64_t word = rem - atom * 128;
        const int64_t rb = atom / kbs, kb = atom - rb * kbs;
        const int64_t r = rb * 128 + (word & 3) * 32 + (word >> 2);
        uint32_t v = 0;
        if (r < rows)
            v = *reinterpret_cast<const uint32_t *>(in + (b * rows + r) * (cols / 16) + kb * 4);
        reinterpret_cast<uint32_t *>(out)[w] = v;
    }
}

cudaError_t launch_swizzle(const uint8_t *in, int64_t batch, int64_t rows, int64_t cols, uint8_t *out,
                           cudaStream_t s)
{
    const int64_t words = batch * ((rows + 127) / 128) * (cols / 64) * 128;
    int64_t blocks = (words + 255) / 256;
    if (blocks > 65535)
        blocks = 65535;
    if (blocks < 1)
        blocks = 1;
    swizzle_scales_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(in, batch, rows, cols, out);
    return cudaGetLastError();
}

// ------------------------------------------------------------ kernel attributes
cudaError_t ensure_smem_limit(const void *kernel, int bytes, unsigned long long *done_mask)
{
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
    std::lock_guard<std::mutex> lock(mu);
    if (bit != 0 && (*done_mask & bit) != 0)
        return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
        *done_mask |= bit;
    return e;
}

// ------------------------------------------------------------ combine
// out[t] = bf16( sum_{j ascending} w[t,j] * y[yrow[t*k+j]] ) in fp32, where
// yrow is the slot's row in the unpadded expert-major y buffer (-1: skipped).
// One block per (token, 2048-column chunk); each thread owns 8 columns (16
// bytes) and issues the loads of up to eight slots before accumulating them in
// order.
constexpr int kCombineThreads = 256;
constexpr int kCombineCols = 8 * kCombineThreads;

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const __nv_bfloat16 *__restrict__ y,
                                                                  const int32_t *__restrict__ yrow,
                                                                  const float *__restrict__ w, int k, int64_t H,
                                                                  __nv_bfloat16 *__restrict__ out)
{
    __shared__ int64_t s_row[32];
    __shared__ float s_w[32];
    pdl_wait();
    pdl_trigger();
    const int64_t t = blockIdx.x;
    if (threadIdx.x < k) {
        const int64_t f = t * k + threadIdx.x;
        s_row[threadIdx.x] = yrow[f];
        s_w[threadIdx.x] = w[f];
    }
    __syncthreads();
    const int64_t c = static_cast<int64_t>(blockIdx.y) * kCombineCols + static_cast<int64_t>(threadIdx.x) * 8;
    if (c < H) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            acc[i] = 0.0f;
        for (int j0 = 0; j0 < k; j0 += 8) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t row = j0 + u < k ? s_row[j0 + u] : -1;
                v[u] = row >= 0 ? __ldg(reinterpret_cast<const uint4 *>(y + row * H + c)) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (j0 + u >= k || s_row[j0 + u] < 0)
                    continue;
                const float wj = s_w[j0 + u];
                const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v[u]);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = __bfloat1622float2(h[i]);
                    acc[2 * i] = __fadd_rn(acc[2 * i], __fmul_rn(wj, f.x));
                    acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], __fmul_rn(wj, f.y));
                }
            }
        }
        uint4 o;
        __nv_bfloat162 *oh = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            oh[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        *reinterpret_cast<uint4 *>(out + t * H + c) = o;
    }
}

cudaError_t launch_combine(const __nv_bfloat16 *y, const int32_t *yrow, const float *w, int64_t T, int k, int64_t H,
                           __nv_bfloat16 *out, cudaStream_t s)
{
    const dim3 grid(static_cast<unsigned>(T), static_cast<unsigned>((H + kCombineCols - 1) / kCombineCols));
    return launch_pdl(combine_kernel, grid, dim3(kCombineThreads), 0, s, y, yrow, w, k, H, out);
}

// ------------------------------------------------------------ warmup scales
// inter_gs[e] = 2688 / amax_e; experts with amax 0 use the largest amax.
__global__ void finalize_inter_gs_kernel(const unsigned int *__restrict__ amax_bits, int E, float *inter_gs)
{
    __shared__ float wmax[32];
    const int tid = threadIdx.x;
    const float a = tid < E ? __uint_as_float(amax_bits[tid]) : 0.0f;
    float m = a;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0)
        wmax[tid >> 5] = m;
    __syncthreads();
    if (tid < 32) {
        m = tid < static_cast<int>(blockDim.x >> 5) ? wmax[tid] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (tid == 0)
            wmax[0] = m;
    }
    __syncthreads();
    const float gmax = wmax[0];
    if (tid < E) {
        const float use = a > 0.0f ? a : gmax;
        inter_gs[tid] = use == 0.0f ? 1.0f : __fdiv_rn(2688.0f, use);
    }
}

cudaError_t launch_finalize_inter_gs(const unsigned int *amax_bits, int E, float *inter_gs, cudaStream_t s)
{
    finalize_inter_gs_kernel<<<1, 1024, 0, s>>>(amax_bits, E, inter_gs);
    return cudaGetLastError();
}

// ------------------------------------------------------------ top-k router
// One warp per token.  Every logit becomes a 32-bit key, its fp32 value
// mapped to an unsigned integer of the same order (-0 folded into +0); lane l
// holds experts l, l + 32, ... and keeps its largest key and, among equal
// keys, its lowest expert.  Each of the k rounds takes two warp reductions
// (redux.sync): the largest key, then the lowest expert holding it; the
// owning lane retires that key (to 0, below every real key) and rescans.
// With ns shared experts, lanes k .. k + ns - 1 write the shared slots.
constexpr int kTopkWarps = 8;

__device__ __forceinline__ uint32_t order_bits(float x)
{
    const uint32_t u = __float_as_uint(x == 0.0f ? 0.0f : x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float from_order_bits(uint32_t o)
{
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

template <int P>
__global__ void __launch_bounds__(32 * kTopkWarps) topk_kernel(const float *__restrict__ logits, int64_t T, int E,
                                                               int k, int ns, int scoring, int32_t *__restrict__ ids,
                                                               float *__restrict__ weights)
{
    const int lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * kTopkWarps + (threadIdx.x >> 5);
    if (t >= T)
        return;   // whole warp leaves together
    const float *row = logits + t * E;
    uint32_t key[P];
#pragma unroll
    for (int i = 0; i < P; i++) {
        const int e = lane + 32 * i;
        key[i] = e < E ? order_bits(__ldg(row + e)) : 0u;
    }
    // this lane's best key and the lowest i holding it
    uint32_t best = 0;
    int best_i = 0;
#pragma unroll
    for (int i = 0; i < P; i++)
        if (key[i] > best) {
            best = key[i];
            best_i = i;
        }
    uint32_t alive = P >= 32 ? 0xffffffffu : (1u << P) - 1u;   // bit i: key[i] not yet taken
    float mine = 0.0f;   // lane j < k: logit of the j-th winner
    int mine_id = 0;
    for (int j = 0; j < k; j++) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, best);
        const uint32_t cand = best == m ? static_cast<uint32_t>(lane + 32 * best_i) : 0xffffffffu;
        const uint32_t w = __reduce_min_sync(0xffffffffu, cand);
        if (lane == j) {
            mine = from_order_bits(m);
            mine_id = static_cast<int>(w);
        }
        if (lane == static_cast<int>(w & 31u)) {   // the winner was this lane's best: retire it, rescan
            alive &= ~(1u << best_i);
            best = 0;
            best_i = 0;
#pragma unroll
            for (int i = 0; i < P; i++) {
                const uint32_t kv = ((alive >> i) & 1u) ? key[i] : 0u;
                if (kv > best) {
                    best = kv;
                    best_i = i;
                }
            }
        }
    }
    // Weights over the selection: softmax (shifted by the top logit) or
    // sigmoid, then divided by their sum.
    const float top = __shfl_sync(0xffffffffu, mine, 0);
    float v = 0.0f;
    if (lane < k)
        v = scoring == 0 ? expf(mine - top) : __frcp_rn(1.0f + expf(-mine));
    float sum = v;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
    // Row stride k + ns: the routed slots, then one slot per shared expert
    // (ids E .. E + ns - 1, weight 1), so that the forward runs the shared
    // experts as extra groups of the same grouped GEMMs.
    const int64_t ld = k + ns;
    if (lane < k) {
        ids[t * ld + lane] = mine_id;
        weights[t * ld + lane] = __fdiv_rn(v, sum);
    } else if (lane < ld) {
        ids[t * ld + lane] = E + (lane - k);
        weights[t * ld + lane] = 1.0f;
    }
}

cudaError_t launch_topk(const float *logits, int64_t T, int E, int k, int ns, int scoring, int32_t *ids,
                        float *weights, cudaStream_t s)
{
    if (T == 0)
        return cudaSuccess;
    const unsigned grid = static_cast<unsigned>((T + kTopkWarps - 1) / kTopkWarps);
    const int per_lane = (E + 31) / 32;
#define NVFP4_TOPK_CASE(P)                                                                                       \
    if (per_lane <= P) {                                                                                         \
        topk_kernel<P><<<grid, 32 * kTopkWarps, 0, s>>>(logits, T, E, k, ns, scoring, ids, weights);             \
        return cudaGetLastError();                                                                               \
    }
    NVFP4_TOPK_CASE(2)
    NVFP4_TOPK_CASE(4)
    NVFP4_TOPK_CASE(8)
    NVFP4_TOPK_CASE(12)
    NVFP4_TOPK_CASE(16)
    NVFP4_TOPK_CASE(24)
    NVFP4_TOPK_CASE(32)
#undef NVFP4_TOPK_CASE
    return cudaErrorInvalidValue;
}

} // namespace nvfp4
