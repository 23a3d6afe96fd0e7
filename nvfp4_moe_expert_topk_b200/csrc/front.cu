// front.cu -- the front of the routed-expert forward in one launch: the
// batch's activation global scale, the routing (per-expert histogram, prefix
// sums, stable permutation, the m-tile / pair / light tile tables) and the
// NVFP4 quantisation of x fused with the expert permutation.
//
// ("nvfp4-megamoe-kernel / CURRENT_BUG.md": page 3 "Architecture Notes" --
// every token goes to 6 of 384 experts and the experts run as one grouped
// GEMM; page 2 "What the quant method does" -- the activation global scale
// multiplies x before the FP4 conversion.)
//
// Grid: G blocks of 1024 threads (G <= the SM count, so every block is
// resident once the previous kernel on the stream has drained; it waits for
// nothing but the other blocks of this grid).  Block b owns the contiguous
// tokens [T*b/G, T*(b+1)/G) and their k slots each.
//   phase 1  max|x| over its rows (when the caller passes no global scale)
//            and per-warp histograms of its slots' expert ids; publishes its
//            amax and its per-expert counts, then arrives on a grid ticket;
//   barrier  one arrival per block on a 32-bit ticket: every launch adds
//            exactly 1024 in total (block 0 adds 1025 - G, the others 1), so
//            the ticket (zero in a fresh workspace) is a multiple of 1024
//            between launches and a block waits until it reaches the next
//            multiple -- nothing to reset between launches;
//   phase 2  every block reads all blocks' counts (L2), forms per expert the
//            total and the count of earlier blocks, scans the experts (row
//            offsets, 128-row padded offsets, tile tables; block 0 writes the
//            tables) and gives each of its slots its stable position:
//            padded_offset[e] + #earlier slots of e in slot order;
//   phase 3  quantises its tokens (x re-read from L2) with the global scale
//            and writes codes and scales to each slot's padded row.
// The barrier wait is bounded (2 s): a block that gives up records
// NVFP4_ERR_TIMEOUT, empties the tile tables so that the GEMMs do nothing,
// and returns.
#include "internal.h"
#include "quant.cuh"

namespace nvfp4 {

constexpr int kFrontThreads = 1024;
constexpr int kFrontWarps = kFrontThreads / 32;
constexpr int kRouteWarps = 16;             // warps that own slot chunks (per-warp histograms)
constexpr int kQuantCols = 1024;            // columns per quantisation item: 32 per lane
constexpr int kIdsCache = 4096;             // a block's slot ids kept in shared memory between phases 1 and 2

__device__ __forceinline__ int block_count(int64_t T, int b, int G)
{
    return static_cast<int>(T * b / G);
}

// Exclusive block-wide scan (1024 threads, one value set per thread) of four
// int values; returns the exclusive prefixes and, in total[], the sums.
__device__ __forceinline__ void block_scan4(int (&v)[4], int (&excl)[4], int (&total)[4], int *scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        inc[i] = v[i];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int n = __shfl_up_sync(0xffffffffu, inc[i], o);
            if (lane >= o)
                inc[i] += n;
        }
    }
    if (lane == 31) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            scratch[i * 32 + warp] = inc[i];
    }
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int w = scratch[i * 32 + lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o)
                    w += n;
            }
            scratch[128 + i * 32 + lane] = w;        // inclusive over warps
        }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        excl[i] = (warp > 0 ? scratch[128 + i * 32 + warp - 1] : 0) + inc[i] - v[i];
        total[i] = scratch[128 + i * 32 + 31];
    }
    __syncthreads();
}

// Bounded wait (2 s) until the ticket reaches `target` (wrap-around safe),
// acquire at GPU scope.
__device__ __forceinline__ bool wait_ticket(const unsigned int *ticket, unsigned int target)
{
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 0; i < kWaitLimitSpins; ++i) {
        unsigned int v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ticket) : "memory");
        if (static_cast<int>(v - target) >= 0)
            return true;
        if ((i & 15u) == 15u && global_timer_ns() - t0 > kWaitLimitNs)
            return false;
        __nanosleep(32);
    }
    return false;
}

__global__ void __launch_bounds__(kFrontThreads, 1) front_kernel(const FrontArgs a)
{
    extern __shared__ int32_t sm[];
    const int E = a.E, k = a.k;
    const int Epad = (E + 3) & ~3;
    int32_t *wcnt = sm;                               // [kRouteWarps][E]: per-warp counts, then prefixes
    int32_t *tot_s = wcnt + kRouteWarps * E;          // [Epad] total per expert
    int32_t *pre_s = tot_s + Epad;                    // [Epad] slots of e in earlier blocks
    int32_t *poff_s = pre_s + Epad;                   // [Epad] padded row offset of e
    int32_t *off_s = poff_s + Epad;                   // [Epad] row offset of e
    int32_t *ids_s = off_s + Epad;                    // [kIdsCache] this block's slot ids (when they fit)
    __shared__ int scan_scratch[256];
    __shared__ float red[kFrontWarps];
    __shared__ int abort_s;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = gridDim.x, b = blockIdx.x;
    const int64_t T = a.T;
    const int t0 = block_count(T, b, G), t1 = block_count(T, b + 1, G);
    const int64_t f0 = static_cast<int64_t>(t0) * k, f1 = static_cast<int64_t>(t1) * k;
    const bool do_amax = a.x != nullptr && a.x_gs == nullptr;

    for (int i = tid; i < kRouteWarps * E; i += kFrontThreads)
        wcnt[i] = 0;
    for (int i = tid; i < Epad; i += kFrontThreads)
        tot_s[i] = pre_s[i] = 0;
    if (tid == 0)
        abort_s = 0;
    pdl_wait();
    __syncthreads();

    // ------------------------------------------------ phase 1: amax, histograms
    if (do_amax) {
        const int64_t n8 = static_cast<int64_t>(t1 - t0) * a.H / 8;     // H % 128 == 0
        const uint4 *xv = reinterpret_cast<const uint4 *>(a.x + static_cast<int64_t>(t0) * a.H);
        float m = 0.0f;
        for (int64_t i0 = tid; i0 < n8; i0 += 8 * kFrontThreads) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)            // eight 16-byte loads in flight per thread (128 KB per block)
                v[u] = i0 + u * kFrontThreads < n8 ? __ldg(xv + i0 + u * kFrontThreads) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v[u]);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f = __bfloat1622float2(h[j]);
                    m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0)
            red[warp] = m;
    }
    const int64_t nslots = f1 - f0;
    const int64_t chunk = (nslots + kRouteWarps - 1) / kRouteWarps;
    const int64_t c0 = f0 + (nslots < warp * chunk ? nslots : warp * chunk);
    const int64_t c1 = f0 + (nslots < (warp + 1) * chunk ? nslots : (warp + 1) * chunk);
    const bool ids_cached = nslots <= kIdsCache;
    if (warp < kRouteWarps) {
        int bad = 0;
        for (int64_t base = c0; base < c1; base += 4 * 32) {
            int ev[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)            // four loads in flight per lane
                ev[u] = base + lane + 32 * u < c1 ? __ldg(a.ids + base + lane + 32 * u) : -1;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (ids_cached && base + lane + 32 * u < c1)
                    ids_s[base + lane + 32 * u - f0] = ev[u];
                if (ev[u] >= E)
                    bad = 1;
                else if (ev[u] >= 0)
                    atomicAdd(&wcnt[warp * E + ev[u]], 1);
            }
        }
        if (bad)
            atomicCAS(a.err, 0, NVFP4_ERR_BAD_EXPERT_ID);
    }
    __syncthreads();
    // per expert: exclusive prefix over the route warps (in place), block total
    for (int e = tid; e < Epad; e += kFrontThreads) {
        int c = 0;
        if (e < E) {
#pragma unroll 4
            for (int w = 0; w < kRouteWarps; ++w) {
                const int v = wcnt[w * E + e];
                wcnt[w * E + e] = c;
                c += v;
            }
        }
        a.blk_hist[static_cast<int64_t>(b) * Epad + e] = c;     // pad columns: 0
    }
    if (do_amax && tid == 0) {
        float m = red[0];
        for (int w = 1; w < kFrontWarps; ++w)
            m = fmaxf(m, red[w]);
        a.blk_amax[b] = m;
    }
    __threadfence();
    __syncthreads();

    // ------------------------------------------------ grid barrier
    if (tid == 0) {
        const unsigned int add = b == 0 ? static_cast<unsigned int>(1025 - G) : 1u;
        const unsigned int old = atomicAdd(a.ticket, add);
        const unsigned int target = (old & ~1023u) + 1024u;
        if (!wait_ticket(a.ticket, target)) {
            abort_s = 1;
            atomicCAS(a.err, 0, NVFP4_ERR_TIMEOUT);
            *a.num_mtiles = 0;                  // the GEMMs then have no tiles to wait on
            *a.num_pairs = 0;
            *a.num_light = 0;
            atomicExch(a.ticket, 0u);           // a multiple of 1024 again for the next launch
        }
    }
    __syncthreads();
    if (abort_s)
        return;

    // ------------------------------------------------ phase 2: scans, positions
    // One pass over what the blocks published, every load issued before any
    // result is used: the blocks' max|x| (one per thread) and their expert
    // counts -- nq column blocks of 32 int4 (128 experts) and ng = 32 / nq
    // row groups of warps; warp (g, q) sums block rows g, g + ng, ... of its
    // column block, eight rows in flight, then adds its sums into shared
    // memory.
    float gs = 1.0f;
    float amax_part = 0.0f;
    if (do_amax && tid < G)
        amax_part = __ldcg(a.blk_amax + tid);
    {
        const int E4 = Epad / 4;
        const int nq = (E4 + 31) / 32;
        const int ng = kFrontWarps / nq;
        const int q = warp / ng, g = warp - (warp / ng) * ng;
        const int c4 = 32 * q + lane;
        int4 tot = make_int4(0, 0, 0, 0), pre = make_int4(0, 0, 0, 0);
        if (q < nq && c4 < E4) {
            for (int r0 = g; r0 < G; r0 += 8 * ng) {
                int4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int r = r0 + u * ng;
                    v[u] = r < G ? __ldcg(reinterpret_cast<const int4 *>(a.blk_hist + static_cast<int64_t>(r) * Epad) + c4)
                                 : make_int4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    tot.x += v[u].x, tot.y += v[u].y, tot.z += v[u].z, tot.w += v[u].w;
                    if (r0 + u * ng < b)
                        pre.x += v[u].x, pre.y += v[u].y, pre.z += v[u].z, pre.w += v[u].w;
                }
            }
            const int e = 4 * c4;
            const int tv[4] = {tot.x, tot.y, tot.z, tot.w};
            const int pv[4] = {pre.x, pre.y, pre.z, pre.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (tv[i])
                    atomicAdd(&tot_s[e + i], tv[i]);
                if (pv[i])
                    atomicAdd(&pre_s[e + i], pv[i]);
            }
        }
    }
    if (do_amax) {
        float m = amax_part;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0)
            red[warp] = m;
    }
    __syncthreads();
    if (do_amax) {
        float m = red[0];
        for (int w = 1; w < kFrontWarps; ++w)
            m = fmaxf(m, red[w]);
        gs = m == 0.0f ? 1.0f : __fdiv_rn(2688.0f, m);
        if (b == 0 && tid == 0)
            *a.gs_out = gs;
    } else if (a.x != nullptr) {
        gs = __ldg(a.x_gs);
    }
    // expert scans: thread e owns expert e (E <= 1024)
    {
        const int e = tid;
        const int cnt = e < E ? tot_s[e] : 0;
        const int tiles = (cnt + 127) / 128;
        int npair = 0, nlight = tiles;
        if (a.pair_mode == 1) {
            npair = tiles >= 2 ? tiles / 2 : 0;
            nlight = tiles - 2 * npair;
        } else if (a.pair_mode == 2) {
            npair = (tiles + 1) / 2;
            nlight = 0;
        }
        int v[4] = {cnt, tiles, npair, nlight}, ex[4], total[4];
        block_scan4(v, ex, total, scan_scratch);
        if (e < E) {
            off_s[e] = ex[0];
            poff_s[e] = ex[1] * 128;
        }
        if (b == 0) {
            if (e < E) {
                a.counts[e] = cnt;
                a.off[e] = ex[0];
                a.poff[e] = ex[1] * 128;
                for (int i = 0; i < tiles; ++i) {
                    a.mtiles[ex[1] + i] =
                        make_int4(e, (ex[1] + i) * 128, min(128, cnt - 128 * i), ex[0] + 128 * i);
                    if (a.ready != nullptr)
                        a.ready[ex[1] + i] = 0;
                }
                for (int i = 0; i < npair; ++i) {
                    const int second = 2 * i + 1 < tiles ? ex[1] + 2 * i + 1 : -1;
                    a.pairs[ex[2] + i] = make_int2(ex[1] + 2 * i, second);
                }
                for (int i = 0; i < nlight; ++i)
                    a.light[ex[3] + i] = ex[1] + (tiles - nlight) + i;
            }
            if (tid == 0) {
                if (a.claim != nullptr)
                    *a.claim = 0;
                a.off[E] = total[0];
                a.poff[E] = total[1] * 128;
                *a.num_mtiles = total[1];
                *a.num_pairs = total[2];
                *a.num_light = total[3];
            }
        }
    }
    __syncthreads();
    // stable positions of this block's slots (each route warp walks its chunk in order)
    if (warp < kRouteWarps) {
        const unsigned lt_mask = (1u << lane) - 1u;
        for (int64_t base = c0; base < c1; base += 4 * 32) {
            int ev[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t f = base + 32 * u + lane;
                ev[u] = f < c1 ? (ids_cached ? ids_s[f - f0] : __ldg(a.ids + f)) : -1;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t f = base + 32 * u + lane;
                const bool act = f < c1;
                const int e = ev[u];
                const bool valid = act && e >= 0 && e < E;
                const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
                const int rank = __popc(peers & lt_mask);
                if (valid) {
                    const int r = pre_s[e] + wcnt[warp * E + e] + rank;
                    a.inv[f] = poff_s[e] + r;
                    a.yrow[f] = off_s[e] + r;
                    if (ids_cached)             // the slot's id is read: keep its padded row there
                        ids_s[f - f0] = poff_s[e] + r;
                } else if (act) {
                    a.inv[f] = -1;
                    a.yrow[f] = -1;
                    if (ids_cached)
                        ids_s[f - f0] = -1;
                }
                __syncwarp();
                if (valid && rank == 0)
                    wcnt[warp * E + e] += __popc(peers);
                __syncwarp();
            }
        }
    }
    const bool pre_quantised = a.xq_codes != nullptr;
    if (a.x == nullptr && !pre_quantised)
        return;
    __syncthreads();                            // this block's inv is written

    // ------------------------------------------------ phase 3: quantise + permute
    // item = (token, 1024-column chunk); lane l quantises columns
    // [32 l, 32 l + 32) of the chunk (two 16-element blocks) and writes 16
    // bytes of codes per destination row; lanes 2m, 2m + 1 join their scales
    // into the 4-byte word of one 64-column group of the MMA scale layout.
    const int64_t H = a.H;
    const int nchunks = static_cast<int>((H + kQuantCols - 1) / kQuantCols);
    const int64_t nkt = (H + 255) / 256;        // k-tiles of 256 columns per row block
    const int items = (t1 - t0) * nchunks;
    for (int it = warp; it < items; it += kFrontWarps) {
        const int t = t0 + it / nchunks;
        const int c = it - (it / nchunks) * nchunks;
        const int64_t col0 = static_cast<int64_t>(c) * kQuantCols + 32 * lane;
        const bool active = col0 < H;
        int my_dst = -1;                          // lane j < k: destination row of slot j
        if (lane < k)
            my_dst = ids_cached ? ids_s[static_cast<int64_t>(t) * k + lane - f0]
                                : __ldcg(a.inv + static_cast<int64_t>(t) * k + lane);
        uint32_t cw[4] = {0u, 0u, 0u, 0u};
        uint32_t s2 = 0;
        if (pre_quantised) {
            // NVFP4 rows quantised elsewhere (e.g. before an expert-parallel
            // dispatch): this lane's 16 bytes of codes and two scales
            if (active) {
                const uint4 c4 = __ldg(reinterpret_cast<const uint4 *>(a.xq_codes + static_cast<int64_t>(t) * (H / 2) +
                                                                       col0 / 2));
                cw[0] = c4.x, cw[1] = c4.y, cw[2] = c4.z, cw[3] = c4.w;
                s2 = __ldg(reinterpret_cast<const unsigned short *>(a.xq_scales + static_cast<int64_t>(t) * (H / 16) +
                                                                   col0 / 16));
            }
        } else if (active) {
            uint4 ld[4];
            const uint4 *src = reinterpret_cast<const uint4 *>(a.x + static_cast<int64_t>(t) * H + col0);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                ld[i] = __ldg(src + i);
#pragma unroll
            for (int blk = 0; blk < 2; ++blk) {
                const __nv_bfloat162 *h0 = reinterpret_cast<const __nv_bfloat162 *>(&ld[2 * blk]);
                const __nv_bfloat162 *h1 = reinterpret_cast<const __nv_bfloat162 *>(&ld[2 * blk + 1]);
                float f[16];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 p = __bfloat1622float2(h0[j]);
                    const float2 q = __bfloat1622float2(h1[j]);
                    f[2 * j] = p.x;
                    f[2 * j + 1] = p.y;
                    f[8 + 2 * j] = q.x;
                    f[8 + 2 * j + 1] = q.y;
                }
                s2 |= quantize16(f, gs, cw[2 * blk], cw[2 * blk + 1]) << (8 * blk);
            }
        }
        const uint32_t s_hi = __shfl_xor_sync(0xffffffffu, s2, 1);
        const uint32_t sword = s2 | (s_hi << 16);          // valid on even lanes: 4 scales, 64 columns
        for (int d = 0; d < k; ++d) {
            const int dst = __shfl_sync(0xffffffffu, my_dst, d);
            if (!active || dst < 0)
                continue;
            *reinterpret_cast<uint4 *>(a.a_codes + static_cast<int64_t>(dst) * (H / 2) + col0 / 2) =
                make_uint4(cw[0], cw[1], cw[2], cw[3]);
            // row blocks: the row's 16 scale bytes of a k-tile are contiguous, so
            // four lane pairs write one 16-byte piece per k-tile of the chunk
            if ((lane & 1) == 0)
                *reinterpret_cast<uint32_t *>(a.a_sf + ((static_cast<int64_t>(dst) >> 7) * nkt + (col0 >> 8)) * 2048 +
                                              (dst & 127) * 16 + ((col0 & 255) >> 4)) = sword;
        }
    }
}

size_t front_smem_bytes(int E)
{
    const int Epad = (E + 3) & ~3;
    return sizeof(int32_t) * (static_cast<size_t>(kRouteWarps) * E + 4 * static_cast<size_t>(Epad) + kIdsCache);
}

int front_blocks(int64_t T, int num_sms)
{
    int64_t g = T < num_sms ? T : num_sms;
    if (g > kFrontMaxBlocks)
        g = kFrontMaxBlocks;
    return g < 1 ? 1 : static_cast<int>(g);
}

cudaError_t launch_front(const FrontArgs &args, int num_sms, cudaStream_t s)
{
    static unsigned long long attr_done = 0;
    const size_t smem = front_smem_bytes(args.E);
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(front_kernel),
                                      static_cast<int>(front_smem_bytes(1024)), &attr_done);
    if (e != cudaSuccess)
        return e;
    return launch_pdl(front_kernel, dim3(static_cast<unsigned>(front_blocks(args.T, num_sms))), dim3(kFrontThreads),
                      smem, s, args);
}

} // namespace nvfp4
