/*
 * nvfp4moe.h -- C ABI of libnvfp4moe.so: the NVFP4 (W4A4) routed-expert MoE
 * block of a DeepSeek-V4-style layer on one B200 (sm_100a).
 *
 * Source of the operations: "nvfp4-megamoe-kernel / CURRENT_BUG.md" (three
 * snapshots of one page).  Page 1 "Phase 1: CuTeDSL Shared Expert Kernel"
 * gives the chain L1 gate_up GEMM -> SiLU -> re-quantise -> L2 GEMM with the
 * gate and up weights stacked; page 1 "Phase 2" gives the dual global scales
 * of a stacked projection; page 2 "What the quant method does" gives the
 * global-scale convention; page 3 "Architecture Notes" gives 384 experts,
 * top-6 and expert intermediate 3072; page 1 "Phase 1" asks for a
 * cudagraph-safe runner with pre-allocated buffers and warmup global scales.
 *
 * Conventions for every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller, unless a
 *    parameter says "host".  The library allocates no memory, never
 *    synchronises the device (except nvfp4_moe_get_error) and launches only
 *    on the given stream (a cudaStream_t passed as void*; NULL = legacy
 *    default stream).  Nothing is JIT-compiled at run time.
 *  - Launches are asynchronous: the return code reports argument checks and
 *    launch errors only.  Faults inside a kernel surface later, as CUDA
 *    errors on the stream.
 *  - bf16 tensors are passed as uint16_t bit patterns.
 *  - NVFP4 tensor = codes + scales + one fp32 global scale gs:
 *      codes  [rows, cols/2] uint8, row-major; element 2i of a row in the low
 *             nibble of byte i, element 2i+1 in the high nibble; each nibble is
 *             an E2M1 value (sign bit 3, magnitudes 0,.5,1,1.5,2,3,4,6).
 *      scales one E4M3 byte per 16 consecutive elements of a row, in one of
 *             two layouts:
 *             NVFP4_SCALES_ROWMAJOR  [rows, cols/16] row-major;
 *             NVFP4_SCALES_MMA       the tensor-core tile layout: rows padded
 *             to a multiple of 128, stored as [rows/128][cols/64][512 bytes]
 *             where byte (r % 32)*16 + ((r % 128)/32)*4 + j of a 512-byte
 *             atom holds the scale of row r, 16-column block 4*kb + j.
 *      value  = e2m1(code) * e4m3(scale) / gs.
 *  - Quantisation of a 16-element block (bit-exact contract):
 *      a = max|x_i| (fp32); v = (a / 6) * gs; s = E4M3(v) (round to nearest
 *      even, saturating at 448); r = (s == 0) ? 0 : gs / value(s);
 *      q_i = E2M1(x_i * r) (round to nearest even, saturating at 6, sign of
 *      zero kept).  Every fp32 step rounds to nearest.
 *  - Global scale: gs = 2688 / amax (= 448 * 6 / amax) in fp32; 1 if amax = 0.
 *  - Inputs must be finite.
 */
#ifndef NVFP4MOE_H
#define NVFP4MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every int-valued entry point. */
#define NVFP4_OK                       0
#define NVFP4_ERR_INVALID_ARG         -1  /* null pointer, negative size, bad enum   */
#define NVFP4_ERR_UNSUPPORTED_SHAPE   -2  /* size outside the documented constraints */
#define NVFP4_ERR_MISALIGNED          -3  /* pointer or leading dim not 16-B aligned */
#define NVFP4_ERR_WORKSPACE_TOO_SMALL -4
#define NVFP4_ERR_CUDA                -5  /* a CUDA runtime or driver call failed   */
#define NVFP4_ERR_UNSUPPORTED_DEVICE  -6  /* current device is not sm_100           */
#define NVFP4_ERR_TIMEOUT             -7  /* device error word: a bounded wait gave up */
#define NVFP4_ERR_BAD_EXPERT_ID       -8  /* device error word: a top-k id >= E      */

#define NVFP4_SCALES_ROWMAJOR 0
#define NVFP4_SCALES_MMA      1

/* Human-readable name of a status code (static string; never NULL). */
const char *nvfp4_status_string(int status);

/* Global scale of a bf16 tensor (page 2, "What the quant method does": the
 * global scale is a multiplier applied before FP4 conversion).
 * x: [n] bf16; gs_out: device float, receives 2688 / max|x| (1 if all zero).
 * gs_out is also used as the reduction's scratch word.  n >= 1. */
int nvfp4_global_scale(const uint16_t *x, int64_t n, float *gs_out, void *stream);

/* max|x| of a bf16 tensor: x [n] bf16; amax_out: device float (also the
 * reduction's scratch word).  n >= 1.  The global scale of a tensor split
 * over several devices is 2688 / (max over the devices of this value), as
 * for one tensor. */
int nvfp4_amax(const uint16_t *x, int64_t n, float *amax_out, void *stream);

/* Bytes needed for the scales of a [rows, cols] NVFP4 tensor in a layout. */
int64_t nvfp4_scales_bytes(int64_t rows, int64_t cols, int scale_layout);

/* NVFP4 quantisation of a bf16 matrix (page 3 test table: activation
 * quantisation; page 1 "Confirmed working": NVFP4 weights).
 * x: [rows, ldx] bf16, ldx >= cols, ldx % 8 == 0; gs: device float [1];
 * codes: [rows, cols/2]; scales: see scale_layout (NVFP4_SCALES_MMA needs
 * cols % 64 == 0 and nvfp4_scales_bytes() bytes; pad rows of the last
 * 128-row block are not written).  cols % 16 == 0.  x, codes, scales 16-B
 * aligned. */
int nvfp4_quantize(const uint16_t *x, int64_t rows, int64_t cols, int64_t ldx, const float *gs,
                   uint8_t *codes, uint8_t *scales, int scale_layout, void *stream);

/* Row-major scales [batch, rows, cols/16] -> NVFP4_SCALES_MMA layout, per
 * batch entry (weight preparation, page 3 "Next Steps" 2: weight packing).
 * cols % 64 == 0.  Pad rows of the last 128-row block are written as 0.
 * out: batch * nvfp4_scales_bytes(rows, cols, NVFP4_SCALES_MMA) bytes. */
int nvfp4_swizzle_scales(const uint8_t *in, int64_t batch, int64_t rows, int64_t cols,
                         uint8_t *out, void *stream);

/* Dense NVFP4 GEMM, out[m, n] = bf16( sum_k A[m,k] * B[n,k] ), i.e. the
 * grouped engine with one group (page 1 "Phase 1": ScaledGroupedGemm with
 * num_groups=1 is a regular GEMM; page 1 "Phase 2": one NVFP4 GEMM per
 * attention projection, with two global scales for fused_wqa_wkv).
 * a_codes [M, K/2], a_scales NVFP4_SCALES_MMA, a_gs device [1];
 * b_codes [N, K/2], b_scales NVFP4_SCALES_MMA, b_gs device [nseg];
 * seg_end HOST [nseg]: increasing column ends of the B segments, the last
 * equal to N, each a multiple of 32; rows of B in segment s use b_gs[s].
 * out [M, ldo] bf16, ldo >= N, ldo % 8 == 0; only the [M, N] window is
 * written.  Each output element is one fp32 sum in a fixed k order, so
 * repeated calls give identical results.
 * Constraints: M >= 1, N % 128 == 0, K % 64 == 0, 1 <= nseg <= 4. */
int nvfp4_gemm(const uint8_t *a_codes, const uint8_t *a_scales, const float *a_gs, int64_t M,
               const uint8_t *b_codes, const uint8_t *b_scales, const float *b_gs,
               const int64_t *seg_end, int nseg, int64_t N, int64_t K,
               uint16_t *out, int64_t ldo, void *stream);

/* The routed-expert MoE block (page 1 "Phase 1" chain; page 3
 * "Architecture Notes" routing).  Shapes: T tokens, hidden H, expert
 * intermediate I, E experts, top-k.
 * Constraints: T >= 0, H % 128 == 0, I % 128 == 0, 1 <= E <= 1024,
 * 1 <= k <= 32, T*k < 2^31.  All pointers 16-B aligned.  With T = 0 the
 * batch's pointers (x, x_gs when it is required, topk_ids, topk_weights,
 * out) may be NULL: nothing of the batch is read or written. */
typedef struct {
    const uint16_t *x;            /* [T, H] bf16 activations                          */
    int64_t T, H, I;
    int32_t E, k;
    const int32_t *topk_ids;      /* [T, k]; id < 0: slot skipped; id >= E: error word set, slot skipped */
    const float *topk_weights;    /* [T, k] fp32                                      */
    const float *x_gs;            /* [1] global scale of x (nvfp4_global_scale, or warmup); NULL:
                                     the call computes 2688 / max|x| of this batch itself (kept in
                                     workspace region 8) */
    const uint8_t *w13_codes;     /* [E, 2I, H/2]: rows 0..I-1 gate, rows I..2I-1 up   */
    const uint8_t *w13_scales;    /* NVFP4_SCALES_MMA of [E*2I, H]                     */
    const float *w13_gs;          /* [E, 2]: global scale of (gate, up) of each expert */
    const uint8_t *w2_codes;      /* [E, H, I/2]                                       */
    const uint8_t *w2_scales;     /* NVFP4_SCALES_MMA of [E*H, I]                      */
    const float *w2_gs;           /* [E]                                               */
    const float *inter_gs;        /* [E] global scale of h = SiLU(gate)*up, from warmup */
    uint16_t *out;                /* [T, H] bf16 output                                */
} nvfp4_moe_args;

/* Workspace bytes nvfp4_moe_forward / nvfp4_moe_calibrate need (page 1
 * "Phase 1": a cudagraph-safe runner works on pre-allocated buffers, so the
 * caller allocates this once and every call reuses it).  The workspace is
 * caller-owned device memory; zero it once after allocation.  It holds the
 * sticky device error word and the front launch's grid ticket, which every
 * call leaves at a multiple of 1024 and which the launch's grid barrier
 * relies on: in a workspace that was not zeroed the barrier may release
 * blocks early (wrong routing) or time out (NVFP4_ERR_TIMEOUT).  Calls
 * sharing a workspace must not overlap on the device.  Host only; 0 for a
 * shape outside the constraints of nvfp4_moe_forward. */
size_t nvfp4_moe_workspace_size(int64_t T, int k, int E, int64_t H, int64_t I);

/* out = sum_j topk_weights[t,j] * Expert_{ids[t,j]}(x[t]) with
 * Expert_e(x) = W2_e . q(SiLU(W13g_e . q(x)) * (W13u_e . q(x))), all GEMMs
 * in NVFP4 on the tensor cores, q() the NVFP4 quantiser (x with x_gs, h with
 * inter_gs[e]).  Launches on `stream`: the front (one kernel: the global
 * scale of x when x_gs is NULL, routing, quantise+permute), L1 (fused
 * SiLU*up re-quantise epilogue) and L2 (one to three launches, see
 * nvfp4_moe_plan) and the combine; no memset, no host sync, no
 * allocation, so the call can be captured in a CUDA graph (make one eager
 * call per device first: it sets per-kernel attributes). */
int nvfp4_moe_forward(const nvfp4_moe_args *args, void *workspace, size_t ws_bytes, void *stream);

/* nvfp4_moe_forward on activations that are already NVFP4 -- for expert
 * parallelism (page 1 "Config values": 48 of the 384 experts per rank), where
 * a rank quantises its tokens once and sends 4-bit rows (H/2 + H/16 bytes
 * each) to the ranks owning their experts.  x_codes [T, H/2] and x_scales
 * [T, H/16] (NVFP4_SCALES_ROWMAJOR, as nvfp4_quantize writes them), both
 * 16-byte aligned (NULL allowed only when T = 0), quantised with the global
 * scale args->x_gs (required when T > 0);
 * args->x is not read (may be NULL).  The front launch copies each row to its
 * slots' padded rows instead of quantising it; everything else is
 * nvfp4_moe_forward, so given the codes nvfp4_quantize makes from x with
 * x_gs, the output equals nvfp4_moe_forward's on x with x_gs bit for bit. */
int nvfp4_moe_forward_quantized(const nvfp4_moe_args *args, const uint8_t *x_codes, const uint8_t *x_scales,
                                void *workspace, size_t ws_bytes, void *stream);

/* Measurement hook, not a step of the method: nvfp4_moe_forward with CUDA
 * events recorded on `stream` at its stage boundaries: events = 6
 * cudaEvent_t handles created by the caller; event 0 before the front
 * launch, 1 and 2 after it, 3 and 4 after the first and the second GEMM
 * stage of the plan (nvfp4_moe_plan says which launches each holds; a stage
 * may be empty) and 5 after the combine.  Otherwise identical; for
 * per-stage timing.  While `stream` is being captured into a
 * CUDA graph the records become external event nodes, so the events can be
 * timed after each replay. */
int nvfp4_moe_forward_timed(const nvfp4_moe_args *args, void *workspace, size_t ws_bytes, void *stream,
                            void *const *events);

/* Warmup (page 1 "Phase 1": warmup-based gs; page 2 "Option A": compute the
 * scale from a warmup pass): runs the chain up to h on args (a warmup batch;
 * inter_gs and out are ignored) and writes inter_gs_out[e] = 2688 / max|h|
 * over expert e's rows; experts without rows get 2688 / (max over experts),
 * and every expert 1.0 when no expert has a row (e.g. T = 0).
 * inter_gs_out: device [E]. */
int nvfp4_moe_calibrate(const nvfp4_moe_args *args, float *inter_gs_out, void *workspace,
                        size_t ws_bytes, void *stream);

/* The routing step alone (page 3 "Architecture Notes": each token's top-6
 * expert ids decide which expert's grouped-GEMM segment its row joins), for
 * inspection and tests: counts [E], padded_offsets [E+1]
 * (expert segments padded to 128 rows), inv [T*k] (padded row of each slot,
 * -1 if skipped).  Slot f = t*k + j of expert e lands at
 * padded_offsets[e] + #{f' < f : ids[f'] == e} (a stable counting sort). */
int nvfp4_moe_route_debug(const int32_t *topk_ids, int64_t T, int k, int E, int32_t *counts,
                          int32_t *padded_offsets, int32_t *inv, void *workspace, size_t ws_bytes,
                          void *stream);

/* Byte offset and size of a workspace region (build helper for inspection
 * and tests, no passage on the pages; host only).
 * region: 0 A codes, 1 A scales (row blocks: for each 128-row block and
 * each 256-column k-tile, 2 KB holding the row's 16 scale bytes of that
 * k-tile at (row % 128) * 16), 2 h codes, 3 h scales
 * (MMA layout), 4 y (bf16 [T*k, H], rows in expert-major routing order),
 * 5 inv, 6 counts, 7 padded offsets, 8 the fp32 global scale of x computed
 * by the last call made with x_gs = NULL, 9 the m-tile table (int32 x 4 per
 * m-tile: expert, first padded row, rows, first y row), 10 the pair table
 * (int32 x 2 per pair: first m-tile, second m-tile or -1), 11 the light list
 * (int32 m-tile indices run on 1-CTA tiles), 12 the 256-byte header (int32
 * error word at byte 0, m-tile count at 4, pair count at 8, light count at
 * 24). */
int nvfp4_moe_workspace_region(int64_t T, int k, int E, int64_t H, int64_t I, int region,
                               int64_t *offset, int64_t *bytes);

/* nvfp4_moe_forward without a caller-supplied workspace, for callers that
 * cannot allocate device memory: a plug-in inside a host framework that owns
 * all device memory through its own pool and forbids side allocations, a
 * serving loop that cannot take cudaMalloc's implicit device-wide
 * synchronisation on its latency path, an embedded deployment whose memory
 * budget is fixed at start-up.  The pages have no counterpart of this entry
 * point; it is a deployment convenience.
 * Scratch: one static device array of NVFP4_NOALLOC_SCRATCH_BYTES (32 MiB).
 * With lazy module loading (the CUDA 12 default) a device holds it from the
 * first call of this entry point on that device; with
 * CUDA_MODULE_LOADING=EAGER every device the process initialises holds it;
 * in both cases until the process exits.  Shapes whose
 * nvfp4_moe_workspace_size() exceeds it return
 * NVFP4_ERR_WORKSPACE_TOO_SMALL; like every other argument error, that is
 * reported before any device work is queued.  The call allocates nothing
 * (no cudaMalloc, no cudaFree, no allocating library routine).  Its first
 * call on a device looks up the array's device address with that device
 * current (cudaGetSymbolAddress) and caches it: make that first call before
 * any stream capture, and do not use this entry point across a
 * cudaDeviceReset.  All calls on a device share the array (it keeps the last
 * call's contents; each call clears the error word, and the forward rewrites
 * every other word it reads), so calls that overlap on the GPU race:
 * serialise them (one stream, or events).  Device-side errors (a top-k id
 * >= E) skip the slot as in nvfp4_moe_forward but cannot be read back. */
#define NVFP4_NOALLOC_SCRATCH_BYTES (32u << 20)
int nvfp4_moe_forward_noalloc(const nvfp4_moe_args *args, void *stream);

/* Test hook for failure detection, not a step of the method (no
 * counterpart on the pages): launches one
 * thread that runs the fused launch's bounded device wait -- until the
 * device int *flag >= target -- and, when the wait gives up (after 2 s),
 * writes NVFP4_ERR_TIMEOUT into the device int *err if it is still 0.  No
 * fault and no trap: the context stays usable.  flag, err: device pointers. */
int nvfp4_debug_bounded_wait(const int32_t *flag, int32_t target, int32_t *err, void *stream);

/* Execution plan nvfp4_moe_forward uses for a shape (host only, no GPU
 * work; page 3 "Architecture Notes": a persistent grouped GEMM over skewed
 * expert loads).  Each expert's routed rows form 128-row m-tiles.
 * *pair_tiles (the pair mode):
 *   0  every m-tile runs on 1-CTA tiles (128 x 256);
 *   1  batches of >= 2048 routed rows: an expert with two or more m-tiles
 *      runs its consecutive full pairs of m-tiles on pair tiles (256 x 256,
 *      a cluster of two CTAs sharing each weight tile), in an L1 launch and
 *      an L2 launch of their own; its odd last m-tile and every other expert
 *      run on 1-CTA tiles;
 *   2  experts average two full m-tiles or more (T*k >= 256*E): every m-tile
 *      on pair tiles (an odd last m-tile with an empty partner).
 * *fused_l1_l2 = 1 when the 1-CTA tiles run L1 and L2 in one persistent
 * launch (the L2 tiles of an m-tile start as soon as that m-tile's L1 tiles
 * have written h).  Stages between the events of nvfp4_moe_forward_timed:
 * 0-1 the front launch (1-2 empty); then pair mode 0 fused: 2-3 the fused
 * launch (3-4 empty); pair mode 1: 2-3 the fused pair launch, 3-4 the fused
 * 1-CTA launch (with the event between them the 1-CTA launch starts only
 * when the pair launch has ended; without events its CTAs take over SMs as
 * pair CTAs finish); otherwise 2-3 L1, 3-4 L2; 4-5 the combine.  Both
 * outputs are host ints. */
int nvfp4_moe_plan(int64_t T, int k, int E, int64_t H, int64_t I, int32_t *fused_l1_l2, int32_t *pair_tiles);

/* Reads and clears the sticky device error word of a workspace (build
 * helper: the pages' NaN hunt, page 3 "Root Cause Investigation", checked
 * every stage for bad values by hand; here the kernels record a top-k id
 * >= E or a bounded wait that gave up in this word).  Host err_host receives
 * NVFP4_OK or a device error code.  The only call that synchronises
 * `stream`. */
int nvfp4_moe_get_error(void *workspace, int32_t *err_host, void *stream);

/* Measurement hook, not a step of the method (the pages have no
 * counterpart): tensor-core ceiling probe.
 * Launches `ctas` blocks (one per SM when ctas <= the SM count), each
 * issuing `iters` k-tiles of four block-scaled FP4 MMAs (M = 128, N = bn,
 * K = 64, the GEMM engine's instruction) from one thread into one TMEM
 * accumulator with operands already on chip: the rate the GEMMs cannot
 * exceed.  FLOPs = ctas * iters * 4 * 2 * 128 * bn * 64.  cycles: device
 * int64 [ctas], SM clock cycles from first issue to completion per block
 * (-1 if the bounded completion wait gave up, which also writes
 * NVFP4_ERR_TIMEOUT to *err when err is not NULL).  bn is 128 or 256;
 * 1 <= iters <= 1 << 24; 1 <= ctas <= 65535. */
int nvfp4_fp4_mma_ceiling(int bn, int iters, int ctas, int64_t *cycles, int32_t *err, void *stream);

/* Measurement hook, not a step of the method (the pages have no
 * counterpart): TMA streaming probe.  The GEMM engine's weight-tile loads
 * alone: one block per SM loads, per step, two 128-row x 128-byte boxes of
 * the row-major uint8 matrix [rows, row_bytes] (device, 16-byte aligned; one
 * k-tile of a 256-row weight tile, the GEMM's tensor map) into a `stages`-deep
 * ring of 32 KB stages that another thread releases as soon as each lands.
 * work_tiles tiles of 256 rows x row_bytes / 128 steps are dealt round-robin
 * over the blocks; tile t reads the rows of tile t mod (rows / 256).  Bytes
 * moved into shared memory = work_tiles * 256 * row_bytes: with a matrix
 * larger than L2 the rate is the HBM read rate of the GEMM's access pattern,
 * with a small one the L2 -> shared-memory rate.  Constraints: rows % 256 == 0,
 * row_bytes % 128 == 0, 2 <= stages <= 6, work_tiles >= 1.  A bounded wait
 * that gives up writes NVFP4_ERR_TIMEOUT to *err when err is not NULL. */
int nvfp4_tma_stream_ceiling(const uint8_t *matrix, int64_t rows, int64_t row_bytes, int64_t work_tiles,
                             int stages, int32_t *err, void *stream);

/* Top-k router: the step that produces topk_ids / topk_weights for
 * nvfp4_moe_forward (page 3 "Architecture Notes": every token is routed to
 * 6 of 384 experts).  The pages name the routing but not the score function;
 * this entry point takes router logits and offers both usual ones.
 * logits [T, E] fp32 row-major (finite).  For each token the k experts with
 * the largest logits, in descending order, ties to the lower expert id
 * (softmax and sigmoid preserve order, so these are also the k largest
 * scores).  topk_ids [T, k] int32.  topk_weights [T, k] fp32, renormalised
 * over the selection:
 *   NVFP4_SCORING_SOFTMAX  w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0)
 *   NVFP4_SCORING_SIGMOID  w_j = sigmoid(l_j) / sum_i sigmoid(l_i)
 * Ids are exact; weights are fp32 evaluations of these formulas (relative
 * error a few units in the last place).  1 <= k <= min(E, 32), E <= 1024,
 * T >= 0 (T = 0 launches nothing, and the pointers may then be NULL).
 * Allocates nothing. */
#define NVFP4_SCORING_SOFTMAX 0
#define NVFP4_SCORING_SIGMOID 1
int nvfp4_moe_topk(const float *logits, int64_t T, int E, int k, int scoring, int32_t *topk_ids,
                   float *topk_weights, void *stream);

/* The router with the shared experts folded in as extra groups.  Page 1
 * "Phase 1" describes the shared expert as the routed chain with one expert
 * and no routing (L1, SiLU, re-quantisation, L2, same stacked weights), so
 * it can run as one more group of the routed launches.  Identical to
 * nvfp4_moe_topk for the k routed slots, except that rows have
 * k + num_shared slots: topk_ids / topk_weights are [T, k + num_shared],
 * slot k + i holding expert id E + i with weight exactly 1.0f.  Fed to
 * nvfp4_moe_forward with E + num_shared experts (the shared experts' NVFP4
 * weights stored after the E routed ones, their inter_gs calibrated like
 * any other expert's), the output is
 *   out[t] = sum_j<k w[t,j] * Expert_{ids[t,j]}(x[t]) + sum_i Shared_i(x[t]),
 * summed in fp32 in slot order and rounded once to bf16: the routed and
 * shared contributions in one set of launches instead of two chains.
 * 0 <= num_shared, k + num_shared <= 32, E + num_shared <= 1024; the other
 * arguments and errors are nvfp4_moe_topk's (which is this call with
 * num_shared = 0).  Allocates nothing. */
int nvfp4_moe_topk_shared(const float *logits, int64_t T, int E, int k, int scoring, int num_shared,
                          int32_t *topk_ids, float *topk_weights, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4MOE_H */
