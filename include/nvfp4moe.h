/*
 * nvfp4moe.h -- C ABI of the NVFP4 block-scaled Mixture-of-Experts library
 * for NVIDIA B200 (sm_100a).
 *
 * The library implements the MoE FFN hot path that the pages "Peering into the
 * CUTLASS Kernel Cache", "Peering into the CUTLASS Kernel", "Peering into the
 * CUTLASS Kernel Scheduler" and "Peering into the CUTLASS SharedStorage" turn
 * on: an FP4 block-scaled grouped GEMM in which each expert's weight matrix
 * multiplies only the 16-256 tokens routed to it.
 *
 * Data format (NVFP4). Elements are E2M1 4-bit codes, two per byte, the even
 * element of each pair in the low nibble; every 16 consecutive elements along K
 * share one E4M3 block scale byte; each tensor carries one FP32 global scale
 * ("Peering into the CUTLASS SharedStorage", Input Knowledge Required, item 3;
 * "Peering into the CUTLASS Kernel Cache", Knowledge Required, last item). The
 * stored global scale is the dequantisation multiplier g_dec = amax / (6*448);
 * a value decodes as E2M1(code) * E4M3(scale) * g_dec.
 *
 * Conventions for every call:
 *  - Ownership: the caller owns every buffer. The library never allocates or
 *    frees device memory. Buffers marked "device" must be device (or managed)
 *    memory of the current device; sizes are in elements unless stated.
 *  - Streams: every call is asynchronous on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream). No call synchronises with the host except
 *    nvfp4_get_device_status().
 *  - Concurrency of the grouped GEMM (and of the layer calls that run it):
 *    each launch hands out its work items from a counter in the library's
 *    device memory. Launches draw 64 such counters in turn and the last CTA
 *    of a launch leaves its counter at zero, so up to 64 grouped GEMMs may be
 *    in flight on one device at once (any streams). A CUDA graph that
 *    captured a grouped GEMM keeps the counter its capture drew: replays of
 *    such a graph must run one after another (one stream, or ordered by
 *    events) and must not overlap direct launches; two launches that share a
 *    counter at the same time hand out tiles twice or not at all.
 *  - Errors: argument, alignment, shape and capability problems are reported
 *    synchronously, before anything is launched. Launch failures map to
 *    NVFP4_ERR_CUDA. Problems only visible on the device (expert ids out of
 *    range, inconsistent expert offsets, a pipeline wait that ran out) are
 *    latched in a device status word read by nvfp4_get_device_status().
 *  - Layouts: matrices are row-major. GEMM operands are K-major: activations
 *    [rows, K], weights [N, K] per expert (like nn.Linear), so a packed row is
 *    K/2 bytes and a row of block scales is K/16 bytes.
 *  - BF16 tensors are passed as uint16_t bit patterns.
 */
#ifndef NVFP4MOE_H
#define NVFP4MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t. */
typedef struct CUstream_st* nvfp4_stream_t;

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,       /* null pointer, negative or zero size, bad enum */
    NVFP4_ERR_MISALIGNED = 2,        /* a pointer is not 16-byte aligned */
    NVFP4_ERR_UNSUPPORTED_SHAPE = 3, /* K, N, E, k outside what the kernels implement */
    NVFP4_ERR_WORKSPACE = 4,         /* workspace missing or smaller than required */
    NVFP4_ERR_SMEM_BUDGET = 5,       /* the device cannot give the kernel its shared memory */
    NVFP4_ERR_CUDA = 6,              /* a CUDA runtime call or launch failed */
    NVFP4_ERR_DEVICE_TIMEOUT = 7,    /* (device) a bounded pipeline wait ran out */
    NVFP4_ERR_DEVICE_INPUT = 8       /* (device) expert id out of range, duplicate id in a
                                        token's top-k, inconsistent expert offsets, or a
                                        combine row index past y */
} nvfp4_status;

typedef enum { NVFP4_EPI_NONE = 0, NVFP4_EPI_SWIGLU = 1 } nvfp4_epilogue;

/* Block-scale layouts.
 * NVFP4_SF_ROWMAJOR: sf[r * (K/16) + b] is the scale of elements [16b, 16b+16) of row r.
 * NVFP4_SF_MMA_TILED: the same bytes permuted for the tensor-core scale path. Rows
 *   are grouped in 128-row blocks and K in 64-element steps (4 scales); each
 *   (row block rb, step kc) pair is a 512-byte atom at ((rb * (K/64)) + kc) * 512,
 *   and inside it the scale of row r, block b sits at
 *   (r % 32) * 16 + ((r % 128) / 32) * 4 + (b % 4).
 *   Requires rows % 128 == 0 and K % 64 == 0.
 * NVFP4_SF_KSTAGE: one [rows x 16 bytes] slab per 256-element K step: the scale
 *   of row r, block b sits at ((b / 16) * rows + r) * 16 + (b % 16). The 16
 *   scales of a K step are one 16-byte piece per row, and the pieces of
 *   consecutive rows are adjacent, so any run of rows of one K step is one
 *   contiguous copy. Requires K % 128 == 0 and a 16-byte aligned buffer of
 *   ceil(K/256) * rows * 16 bytes: when K % 256 == 128 the last slab holds
 *   8 scales per row and 8 zero bytes (zero scales) after them. The grouped
 *   GEMM reads its activation scales in this layout. */
typedef enum { NVFP4_SF_ROWMAJOR = 0, NVFP4_SF_MMA_TILED = 1, NVFP4_SF_KSTAGE = 2 } nvfp4_sf_layout;

/* ------------------------------------------------------------------------ */
/* nvfp4_quantize: BF16 -> packed E2M1 codes + E4M3 block scales + FP32      */
/* global scale, for one tensor X [rows, K].                                 */
/*                                                                           */
/* Computes (format of "Peering into the CUTLASS SharedStorage", Input       */
/* Knowledge Required, item 3), with IEEE FP32 round-to-nearest-even steps:  */
/*   amax = max|x|; g_enc = 2688/amax, g_dec = amax/2688 (both 1 if amax=0); */
/*   if global_scale_in != NULL it is g_dec and g_enc = 1/g_dec (no amax);   */
/*   per 16-block: S = E4M3_satfinite((amax_b / 6) * g_enc);                 */
/*   S == 0 -> codes +0, else code = E2M1_satfinite(x * (g_enc / S)), the    */
/*   sign kept on zero.                                                      */
/* Arguments:                                                                */
/*   x                [rows, K] BF16 bits, device, 16-byte aligned           */
/*   rows, K          rows >= 1, K % 16 == 0 (MMA_TILED: rows % 128 == 0,    */
/*                    K % 64 == 0; KSTAGE: K % 128 == 0)                     */
/*   global_scale_in  device FP32 scalar or NULL (dynamic amax)             */
/*   q                [rows, K/2] bytes, device, 8-byte aligned              */
/*   sf               rows*K/16 bytes (KSTAGE: ceil(K/256)*rows*16, 16-byte  */
/*                    aligned), device, in `layout`                          */
/*   global_scale_out device FP32 scalar receiving g_dec (may equal         */
/*                    global_scale_in)                                       */
/*   ws, ws_bytes     device scratch of nvfp4_quantize_workspace_size() bytes*/
/*                    (the per-block amax partials); NULL/0 allowed when     */
/*                    global_scale_in is given                               */
/* ------------------------------------------------------------------------ */
NVFP4_API size_t nvfp4_quantize_workspace_size(int64_t rows, int64_t K);
NVFP4_API nvfp4_status nvfp4_quantize(const uint16_t* x, int64_t rows, int64_t K, const float* global_scale_in,
                            uint8_t* q, uint8_t* sf, float* global_scale_out, nvfp4_sf_layout layout,
                            void* ws, size_t ws_bytes, nvfp4_stream_t stream);

/* nvfp4_amax: raises *amax_bits (device uint32, 4-byte aligned; the caller  */
/* sets it to 0 first) to max |x| over x [rows, K] BF16 (device, 16-byte    */
/* aligned, K % 8 == 0), as the BF16 bit pattern in the low 16 bits -- the   */
/* amax nvfp4_quantize derives its dynamic scale from. Several calls (or     */
/* ranks combining their words with an integer max) accumulate one amax.     */
NVFP4_API nvfp4_status nvfp4_amax(const uint16_t* x, int64_t rows, int64_t K, uint32_t* amax_bits,
                        nvfp4_stream_t stream);

/* nvfp4_quantize_from_amax: nvfp4_quantize with a dynamic global scale whose */
/* amax is already known (amax_bits: device uint32 holding max |x| as the    */
/* BF16 bit pattern in its low 16 bits, e.g. written by                      */
/* moe_grouped_gemm_nvfp4_amax). Identical output to nvfp4_quantize(x, ...,  */
/* global_scale_in = NULL, ...) for the same amax; one pass over x, no       */
/* workspace. Same shape, layout and alignment rules; amax_bits 4-byte       */
/* aligned.                                                                  */
NVFP4_API nvfp4_status nvfp4_quantize_from_amax(const uint16_t* x, int64_t rows, int64_t K, const uint32_t* amax_bits,
                                      uint8_t* q, uint8_t* sf, float* global_scale_out, nvfp4_sf_layout layout,
                                      nvfp4_stream_t stream);
/* nvfp4_quantize_from_amax_prefetch: the same, and while it runs it pulls  */
/* the first l2_next_bytes bytes at l2_next (device memory that no kernel   */
/* in flight writes, e.g. the next GEMM's packed expert weights, taken by   */
/* its schedule in address order) into L2: bulk L2 prefetches of 64 KB from */
/* one thread per CTA (the kernel lasts until they land). A hint: the       */
/* outputs do not depend on it; l2_next NULL or 0 bytes prefetches nothing. */
/* Otherwise l2_next is 16-byte aligned (else NVFP4_ERR_MISALIGNED) and the */
/* whole range lies inside one device allocation (not checked).             */
NVFP4_API nvfp4_status nvfp4_quantize_from_amax_prefetch(const uint16_t* x, int64_t rows, int64_t K,
                                               const uint32_t* amax_bits, uint8_t* q, uint8_t* sf,
                                               float* global_scale_out, nvfp4_sf_layout layout,
                                               const void* l2_next, size_t l2_next_bytes,
                                               nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* moe_permute: group routed (token, slot) pairs by expert and gather the    */
/* quantised activation rows into expert order ("Peering into the CUTLASS   */
/* Kernel Cache", Knowledge Required: each expert's weight matrix multiplies */
/* the subset of tokens routed to it).                                       */
/*   expert_offsets[e] = number of pairs routed to experts < e; [E] = T*k.   */
/*   Inside expert e, pairs are ordered by token t ascending, then slot j.   */
/*   perm_src[p] = source token of permuted row p;                           */
/*   inv_perm[t*k + j] = permuted row of pair (t, j);                        */
/*   q_perm[p] = q[perm_src[p]] (K/2 bytes); the K/16 scale bytes of row p   */
/*   are those of row perm_src[p] of sf, written in sf_perm_layout:          */
/*   NVFP4_SF_KSTAGE (what the grouped GEMM reads; T*k rows per slab) or     */
/*   NVFP4_SF_ROWMAJOR (sf_perm[p] = sf[perm_src[p]], e.g. for sending rows  */
/*   to other ranks).                                                        */
/* Arguments: topk_ids [T, k] int32 (device) with ids in [0, E), distinct   */
/*   within a token (violations latch NVFP4_ERR_DEVICE_INPUT); 1 <= T,       */
/*   1 <= k <= 32, 1 <= E <= 1024, T*k < 2^31; q [T, K/2],                  */
/*   sf [T, K/16] row-major; outputs q_perm [T*k, K/2], sf_perm (T*k*K/16    */
/*   bytes; KSTAGE: ceil(K/256)*T*k*16), expert_offsets [E+1], perm_src      */
/*   [T*k], inv_perm [T*k]; all device, 16-byte aligned. K % 128 == 0.       */
/*   ws of moe_permute_workspace_size() bytes.                               */
/*   Any other sf_perm_layout returns NVFP4_ERR_INVALID_ARG.                 */
/* ------------------------------------------------------------------------ */
NVFP4_API size_t moe_permute_workspace_size(int32_t T, int32_t k, int32_t E);
NVFP4_API nvfp4_status moe_permute(const int32_t* topk_ids, int32_t T, int32_t k, int32_t E,
                         const uint8_t* q, const uint8_t* sf, int64_t K,
                         uint8_t* q_perm, uint8_t* sf_perm, nvfp4_sf_layout sf_perm_layout,
                         int32_t* expert_offsets, int32_t* perm_src, int32_t* inv_perm,
                         void* ws, size_t ws_bytes, nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* moe_quantize_permute: nvfp4_quantize(x) followed by moe_permute of the    */
/* result, in one call: the same outputs, byte for byte (q_perm, sf_perm,    */
/* g_x = the global scale nvfp4_quantize would return, expert_offsets,       */
/* perm_src, inv_perm). Up to 32,768 pairs (and E * ceil(T/32) <= 20,480)   */
/* it runs as two kernels -- the ranking beside the amax of x, then one that */
/* quantises each token's row once and writes it to the token's k permuted */
/* rows -- and never writes x's codes in token order; larger batches       */
/* quantise into the workspace first. With an invalid expert id the rows   */
/* past expert_offsets[E] are left unspecified (no pair maps to them).     */
/* Arguments: x [T, H] BF16 (device, 16-byte aligned), H % 128 == 0; the     */
/*   rest as moe_permute with K = H; g_x one FP32 (4-byte aligned); ws of    */
/*   moe_quantize_permute_workspace_size() bytes (16-byte aligned).         */
/* ------------------------------------------------------------------------ */
NVFP4_API size_t moe_quantize_permute_workspace_size(int32_t T, int32_t k, int32_t E, int64_t H);
NVFP4_API nvfp4_status moe_quantize_permute(const uint16_t* x, int32_t T, int64_t H, const int32_t* topk_ids,
                                  int32_t k, int32_t E, uint8_t* q_perm, uint8_t* sf_perm,
                                  nvfp4_sf_layout sf_perm_layout, float* g_x, int32_t* expert_offsets,
                                  int32_t* perm_src, int32_t* inv_perm, void* ws, size_t ws_bytes,
                                  nvfp4_stream_t stream);
/* moe_quantize_permute_prefetch: the same, with the L2 prefetch hint of     */
/* nvfp4_quantize_from_amax_prefetch and its rules (issued by the           */
/* two-kernel path only).                                                   */
NVFP4_API nvfp4_status moe_quantize_permute_prefetch(const uint16_t* x, int32_t T, int64_t H,
                                           const int32_t* topk_ids, int32_t k, int32_t E, uint8_t* q_perm,
                                           uint8_t* sf_perm, nvfp4_sf_layout sf_perm_layout, float* g_x,
                                           int32_t* expert_offsets, int32_t* perm_src, int32_t* inv_perm,
                                           void* ws, size_t ws_bytes, const void* l2_next,
                                           size_t l2_next_bytes, nvfp4_stream_t stream);
/* moe_layer_l2_prefetch_bytes: the prefetch hints moe_layer_nvfp4 gives    */
/* (bytes of the gate/up and of the down weights: 96 MB and 48 MB, or the   */
/* whole tensor when smaller; 0 when the experts average 32 rows or more,   */
/* where the GEMMs do not stream their weights at HBM rate). Host only.     */
NVFP4_API void moe_layer_l2_prefetch_bytes(int32_t T, int32_t k, int32_t E, int64_t H, int64_t I, size_t* gate_up,
                                 size_t* down);

/* ------------------------------------------------------------------------ */
/* moe_permute_noalloc: moe_permute without a caller workspace. No passage   */
/* of the pages corresponds to it; it exists for callers that cannot hand    */
/* the library any device memory of their own -- code running where         */
/* cudaMalloc is not allowed (inside a CUDA stream capture, on a real-time   */
/* path that forbids allocation, or in a host framework that owns every     */
/* device byte through a fixed pool it does not expose).                    */
/* Same arguments, results and errors as moe_permute, minus ws / ws_bytes.  */
/* Its per-(token chunk, expert) count table lives in a fixed array of      */
/* NVFP4_PERMUTE_NOALLOC_SCRATCH_ENTRIES int32 (256 KiB) in the library's   */
/* own device memory, which every GPU that loads the library holds until    */
/* the process exits. Shapes with ceil(T/256) * E above that limit return   */
/* NVFP4_ERR_UNSUPPORTED_SHAPE before anything is launched.                  */
/* The first call on a device looks up the array's device address (with    */
/* that device current); make that first call before any stream capture.   */
/* All calls share the one array and leave their counts in it; every entry  */
/* a call reads is written earlier in the same call, so nothing needs       */
/* clearing, but calls whose kernels overlap on the GPU (different streams  */
/* without ordering) race on the array and give wrong results.              */
/* ------------------------------------------------------------------------ */
#define NVFP4_PERMUTE_NOALLOC_SCRATCH_ENTRIES 65536
NVFP4_API nvfp4_status moe_permute_noalloc(const int32_t* topk_ids, int32_t T, int32_t k, int32_t E,
                                 const uint8_t* q, const uint8_t* sf, int64_t K,
                                 uint8_t* q_perm, uint8_t* sf_perm, nvfp4_sf_layout sf_perm_layout,
                                 int32_t* expert_offsets, int32_t* perm_src, int32_t* inv_perm,
                                 nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* moe_grouped_gemm_nvfp4: one launch for every expert's FP4 block-scaled    */
/* GEMM ("Peering into the CUTLASS Kernel Cache": TMA warp-specialised       */
/* grouped GEMM; "Peering into the CUTLASS Kernel Scheduler": producer /     */
/* MMA / epilogue warp roles).                                               */
/* For expert e and activation rows m in [off[e], off[e+1]):                 */
/*   acc[m, n] = sum_k A(m,k) W_e(n,k)   (block-scaled E2M1 x E2M1, FP32)    */
/*   alpha_e   = a_gscale[0] * w_gscale[e]                                   */
/*   NONE:   out[m, n] = BF16(alpha_e * acc[m, n]),            out [rows, N] */
/*   SWIGLU: out[m, n] = BF16(silu(alpha_e acc[m, n]) * alpha_e acc[m, N/2+n])*/
/*           (rows [0, N/2) of each W_e are the gate, [N/2, N) the up        */
/*           projection),                                     out [rows, N/2]*/
/* Arguments:                                                                */
/*   a_q [max_rows, K/2]; a_sf: ceil(K/256)*max_rows*16 bytes in            */
/*     NVFP4_SF_KSTAGE with max_rows rows per slab (as moe_permute writes   */
/*     it for T*k rows); a_gscale scalar                                     */
/*   w_packed: the weights [E, N, K] packed by nvfp4_pack_weights() as one   */
/*     [E*N, K] matrix (nvfp4_packed_weight_bytes(E*N, K) bytes);           */
/*     w_gscale [E]                                                          */
/*   expert_offsets [E+1] (device; non-decreasing, off[0] >= 0,              */
/*   off[E] <= max_rows, else NVFP4_ERR_DEVICE_INPUT is latched and the      */
/*   offending experts are skipped)                                          */
/*   Shapes: 1 <= E <= 1024, K % 128 == 0, max_rows >= 0; NONE: N % 128 == 0;*/
/*   SWIGLU: N % 256 == 0 (N / 2 % 128 == 0: the gate and the up rows of an  */
/*   output column sit in the same TMEM lane of two 128-row weight blocks,  */
/*   so half-blocks of gate rows are not offered: a SwiGLU N / 2 % 64      */
/*   is narrowed to this). K % 256 == 128 runs a last stage of 128 K-       */
/*   elements; NONE with N % 256 == 128 a last column tile of 128 rows.     */
/*   All pointers device, 16-byte aligned. Rows outside every expert's range */
/*   are not written.                                                        */
/* ------------------------------------------------------------------------ */
NVFP4_API nvfp4_status moe_grouped_gemm_nvfp4(const uint8_t* a_q, const uint8_t* a_sf, const float* a_gscale,
                                    const uint8_t* w_packed, const float* w_gscale,
                                    const int32_t* expert_offsets, int32_t E, int64_t max_rows,
                                    int64_t N, int64_t K, nvfp4_epilogue epi, uint16_t* out,
                                    nvfp4_stream_t stream);

/* moe_grouped_gemm_nvfp4_amax: the same GEMM, and also the amax of its      */
/* output for the next quantisation (nvfp4_quantize_from_amax), so that step */
/* needs no separate pass over out.                                          */
/*   out_amax: device uint32, 4-byte aligned, or NULL (= the call above).    */
/*   The kernel raises *out_amax (atomic max) to max |out| over every stored */
/*   element, as the BF16 bit pattern of |out| in the low 16 bits; the       */
/*   caller sets it to 0 before the call. Same value as the amax pass of     */
/*   nvfp4_quantize on out (NaN sorts above +inf in both).                   */
NVFP4_API nvfp4_status moe_grouped_gemm_nvfp4_amax(const uint8_t* a_q, const uint8_t* a_sf, const float* a_gscale,
                                         const uint8_t* w_packed, const float* w_gscale,
                                         const int32_t* expert_offsets, int32_t E, int64_t max_rows,
                                         int64_t N, int64_t K, nvfp4_epilogue epi, uint16_t* out,
                                         uint32_t* out_amax, nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* moe_grouped_gemm_nvfp4_quant: the gate/up GEMM (SWIGLU) with its output  */
/* h quantised to NVFP4 in the epilogue, by a static (calibrated) global    */
/* scale, in place of BF16 h -- the producer-side fusion that leaves no h   */
/* in memory for the down GEMM's activations ("Peering into the CUTLASS     */
/* Kernel Cache", Knowledge Required: the grouped GEMM of a                 */
/* Mixture-of-Experts layer; the format of "Peering into the CUTLASS        */
/* SharedStorage", Input Knowledge Required, item 3).                        */
/*   q_h, sf_h = nvfp4_quantize(h, global_scale_in = h_gscale,              */
/*               layout = NVFP4_SF_KSTAGE) bit for bit, where h [max_rows,  */
/*               N/2] is what moe_grouped_gemm_nvfp4(..., SWIGLU) writes;   */
/*   h_amax (nullable, zeroed by the caller) is raised to max |h| as BF16   */
/*   bits -- the amax a dynamic scale would use, to calibrate the next call */
/*   (g_dec = amax / 2688).                                                 */
/* Arguments: as moe_grouped_gemm_nvfp4 with the SWIGLU epilogue, plus      */
/*   h_gscale (device FP32 scalar, g_dec of h), q_h [max_rows, N/4] and     */
/*   sf_h (ceil((N/2)/256) * max_rows * 16 bytes, K-stage slabs of max_rows */
/*   rows), both device, 16-byte aligned. Rows outside every expert are not */
/*   written.                                                                */
/* ------------------------------------------------------------------------ */
NVFP4_API nvfp4_status moe_grouped_gemm_nvfp4_quant(const uint8_t* a_q, const uint8_t* a_sf, const float* a_gscale,
                                          const uint8_t* w_packed, const float* w_gscale,
                                          const int32_t* expert_offsets, int32_t E, int64_t max_rows,
                                          int64_t N, int64_t K, const float* h_gscale, uint8_t* q_h,
                                          uint8_t* sf_h, uint32_t* h_amax, nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* moe_grouped_gemm_nvfp4_finalize: the down GEMM with the top-k combine     */
/* fused into its epilogue -- the FINALIZE epilogue that performs the final */
/* MoE output write ("Peering into the CUTLASS Kernel", Input Knowledge     */
/* Required, item 5).                                                        */
/*   The GEMM (NONE epilogue) writes y [max_rows, N] as moe_grouped_gemm_    */
/*   nvfp4 does, and out [T, N] = moe_unpermute_combine(y, inv_perm,        */
/*   topk_w) -- the same bits: for every (token, 128-column block) the CTA  */
/*   that writes the token's k-th row of that block sums the k rows in FP64 */
/*   in slot order with one final rounding, whichever rows came first.      */
/* Arguments: the GEMM's as in moe_grouped_gemm_nvfp4 (NONE epilogue, y is   */
/*   its output); perm_src [max_rows] (row -> token), inv_perm [T*k]         */
/*   ((token, slot) -> row) as moe_permute writes them, topk_w [T, k] FP32,  */
/*   T * k <= max_rows, k <= 32; counters: moe_finalize_counters_size(T, N)  */
/*   bytes of device memory, zero before the first call (each call leaves   */
/*   it zero again; re-zero it after a call that reported an error);        */
/*   out [T, N] BF16. All device, 4-byte aligned (y and out as for the       */
/*   GEMM). Calls sharing one counters buffer must not overlap.              */
/* ------------------------------------------------------------------------ */
NVFP4_API size_t moe_finalize_counters_size(int32_t T, int64_t N);
NVFP4_API nvfp4_status moe_grouped_gemm_nvfp4_finalize(const uint8_t* a_q, const uint8_t* a_sf,
                                             const float* a_gscale, const uint8_t* w_packed,
                                             const float* w_gscale, const int32_t* expert_offsets,
                                             int32_t E, int64_t max_rows, int64_t N, int64_t K,
                                             uint16_t* y, const int32_t* perm_src, const int32_t* inv_perm,
                                             const float* topk_w, int32_t T, int32_t k, uint32_t* counters,
                                             uint16_t* out, nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* nvfp4_pack_weights: one-time packing of a quantised weight matrix         */
/* [rows, K] (codes q [rows, K/2], row-major scales sf [rows, K/16]) into   */
/* the tiles the grouped GEMM streams. Tile (rb, kt) = rows [128 rb, +128) x */
/* K [256 kt, +256) is 18432 contiguous bytes at (rb*ceil(K/256) + kt) *     */
/* 18432 (K % 256 == 128: the last tile of a row block holds 128 K-elements  */
/* and zero codes and zero scales in place of the other 128):                */
/*   [0, 16384): code bytes, row r at r*128, its 16-byte piece c (K bytes    */
/*   16c..16c+15 of the tile row) at (c XOR (r % 8)) * 16 (the 128-byte      */
/*   swizzle the tensor core reads);                                         */
/*   [16384, 18432): scales, K step kc (64 elements) at kc*512, row r's 4    */
/*   scale bytes of that step at (r % 32)*16 + (r / 32)*4.                   */
/* rows % 128 == 0, K % 128 == 0; all pointers device, 16-byte aligned;      */
/* packed holds nvfp4_packed_weight_bytes(rows, K) bytes                     */
/* (= rows * ceil(K/256) * 144: rows*(K/2+K/16) when K % 256 == 0).          */
/* ------------------------------------------------------------------------ */
NVFP4_API size_t nvfp4_packed_weight_bytes(int64_t rows, int64_t K);
NVFP4_API nvfp4_status nvfp4_pack_weights(const uint8_t* q, const uint8_t* sf, int64_t rows, int64_t K,
                                uint8_t* packed, nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* moe_unpermute_combine: top-k weighted sum of the expert outputs back in   */
/* token order -- the final MoE output write of the FINALIZE epilogue       */
/* ("Peering into the CUTLASS Kernel", Input Knowledge Required, item 5).    */
/*   out[t, h] = BF16( sum_{j=0..k-1} topk_w[t, j] * y[inv_perm[t*k+j], h] ) */
/*   accumulated in FP64 over j ascending (each FP32 x BF16 product is exact */
/*   in FP64) and rounded once to BF16 (nearest even); a negative inv_perm   */
/*   entry is skipped, and so is an entry >= T*k (past the last row of y),  */
/*   which also latches NVFP4_ERR_DEVICE_INPUT.                              */
/* Arguments: y [T*k, H] BF16, inv_perm [T*k], topk_w [T, k] FP32, out [T, H]*/
/*   BF16; y and out 16-byte aligned, inv_perm and topk_w 4-byte aligned;   */
/*   all device; H % 8 == 0, 1 <= k <= 32, T >= 1.                           */
/* ------------------------------------------------------------------------ */
NVFP4_API nvfp4_status moe_unpermute_combine(const uint16_t* y, const int32_t* inv_perm, const float* topk_w,
                                   int32_t T, int32_t k, int64_t H, uint16_t* out,
                                   nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* moe_route_topk: the router -- for each token, the k experts with the     */
/* largest logits and their weights. The grouped GEMM multiplies each       */
/* expert's weights by "the subset of tokens routed to it" ("Peering into   */
/* the CUTLASS Kernel Cache", Knowledge Required); the pages do not describe */
/* the router, so this is the plainest reading of top-k softmax routing:    */
/*   topk_ids[t, j] = index of the j-th largest logits[t, :] (equal values: */
/*     the lower index first; -0 equals +0);                                */
/*   topk_w[t, j]   = exp(z_j - z_0) / sum_{i<k} exp(z_i - z_0) with        */
/*     z_j = logits[t, topk_ids[t, j]] -- the softmax over all E restricted */
/*     to the chosen k and renormalised -- computed in FP64 (the sum over i */
/*     ascending) and rounded once to FP32; 1/k each when z_0 is -inf.      */
/* Arguments: logits [T, E] FP32 (device, 4-byte aligned; finite or -inf,   */
/*   no NaN or +inf); topk_ids [T, k] int32 and topk_w [T, k] FP32 (device, */
/*   4-byte aligned). 1 <= T, 1 <= E <= 1024, 1 <= k <= min(E, 32). The ids  */
/*   of a token are distinct, as moe_permute requires.                      */
/* ------------------------------------------------------------------------ */
NVFP4_API nvfp4_status moe_route_topk(const float* logits, int32_t T, int32_t E, int32_t k, int32_t* topk_ids,
                            float* topk_w, nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* moe_layer_nvfp4: the whole MoE FFN in one call, every step in this        */
/* library's kernels, in this order: quantize(x) -> moe_permute ->           */
/* grouped GEMM gate/up (SWIGLU, N = 2I, K = H, amax of h as a side output)  */
/* -> quantize(h) from that amax -> grouped GEMM down (NONE, N = H, K = I)   */
/* -> moe_unpermute_combine. Results equal the four calls above run one by   */
/* one (nvfp4_quantize of h with a dynamic scale). With fewer than 32 rows   */
/* per expert, the kernels before each GEMM carry the L2 prefetch hints of   */
/* moe_layer_l2_prefetch_bytes (the *_prefetch calls): same results.         */
/* Arguments: x [T, H] BF16, topk_ids [T, k], topk_w [T, k];                 */
/*   w13_packed (W13 [E, 2I, H] packed as an [E*2I, H] matrix), w13_gscale   */
/*   [E]; w2_packed (W2 [E, H, I] packed as [E*H, I]), w2_gscale [E];        */
/*   out [T, H] BF16.                                                        */
/*   H % 128 == 0, I % 128 == 0, plus the limits of the calls above. ws of   */
/*   moe_layer_workspace_size() bytes holds every intermediate; its layout   */
/*   is reported by moe_layer_workspace_layout().                            */
/* ------------------------------------------------------------------------ */
typedef struct {
    size_t q_x, sf_x, g_x;                 /* quantised x [T, H/2], [T, H/16], scalar */
    size_t q_perm, sf_perm;                /* [T*k, H/2]; ceil(H/256)*T*k*16 bytes, NVFP4_SF_KSTAGE */
    size_t offsets, perm_src, inv_perm;    /* [E+1], [T*k], [T*k] int32 */
    size_t h;                              /* [T*k, I] BF16 */
    size_t q_h, sf_h, g_h;                 /* [T*k, I/2]; ceil(I/256)*T*k*16 bytes, NVFP4_SF_KSTAGE; scalar */
    size_t amax_h;                         /* uint32: max |h| (BF16 bits), from the gate/up GEMM */
    size_t fin_counters;                   /* the down GEMM's fused-combine counters, right after amax_h
                                              (both zeroed by one memset at the start of each call) */
    size_t y;                              /* [T*k, H] BF16 */
    size_t scratch;                        /* quantize / permute scratch */
    size_t topk_ids, topk_w;               /* [T, k] int32 / FP32: the router's output
                                              (moe_layer_nvfp4_from_logits only) */
    size_t total;
} nvfp4_layer_workspace;

NVFP4_API nvfp4_status moe_layer_workspace_layout(int32_t T, int32_t k, int32_t E, int64_t H, int64_t I,
                                        nvfp4_layer_workspace* layout);
NVFP4_API size_t moe_layer_workspace_size(int32_t T, int32_t k, int32_t E, int64_t H, int64_t I);
NVFP4_API nvfp4_status moe_layer_nvfp4(const uint16_t* x, const int32_t* topk_ids, const float* topk_w,
                             int32_t T, int32_t k, int32_t E, int64_t H, int64_t I,
                             const uint8_t* w13_packed, const float* w13_gscale,
                             const uint8_t* w2_packed, const float* w2_gscale,
                             uint16_t* out, void* ws, size_t ws_bytes, nvfp4_stream_t stream);
/* moe_layer_nvfp4_from_logits: moe_route_topk(logits [T, E] FP32, k) into   */
/* the workspace's topk_ids / topk_w, then moe_layer_nvfp4 on them. Same     */
/* results as the two calls in sequence; same arguments as moe_layer_nvfp4   */
/* with the router logits (device, 4-byte aligned) in place of the routing, */
/* and the router's limits (k <= 32, E <= 1024, finite or -inf logits).      */
NVFP4_API nvfp4_status moe_layer_nvfp4_from_logits(const uint16_t* x, const float* logits,
                                         int32_t T, int32_t k, int32_t E, int64_t H, int64_t I,
                                         const uint8_t* w13_packed, const float* w13_gscale,
                                         const uint8_t* w2_packed, const float* w2_gscale,
                                         uint16_t* out, void* ws, size_t ws_bytes, nvfp4_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Capability and pipeline plan of the grouped GEMM.                         */
/* The launch succeeds iff nvfp4_can_implement() returns NVFP4_OK for the    */
/* current device ("Peering into the CUTLASS SharedStorage", Why This        */
/* Message Was Written: initialize() failed after can_implement() passed --  */
/* this check is the same one the launcher performs, so they cannot          */
/* disagree).                                                                */
/* Per-stage transaction bytes follow the mainloop accounting of that page's */
/* Message excerpt: bytes of the A tile plus its scales, plus bytes of the B */
/* tile plus its scales.                                                     */
/* ------------------------------------------------------------------------ */
typedef struct {                 /* fields up to `threads` describe the narrow (decode) tile shape */
    int32_t tile_weight_rows;    /* weight rows (GEMM N) per tile: 256 */
    int32_t tile_tokens_max;     /* activation rows (GEMM M) per tile, at most */
    int32_t stage_k;             /* K elements per pipeline stage */
    int32_t stages;              /* pipeline depth */
    int32_t stage_bytes_weights; /* packed weight bytes per stage */
    int32_t stage_bytes_weight_sf;
    int32_t stage_bytes_act_max; /* packed activation bytes per stage at tile_tokens_max */
    int32_t stage_bytes_act_sf;  /* activation scale bytes staged per stage */
    int32_t smem_bytes;          /* dynamic shared memory per CTA */
    int32_t tmem_columns;        /* tensor-memory columns allocated per CTA */
    int32_t threads;             /* threads per CTA */
    /* The wide tile shape, used when the experts average at least
     * wide_min_avg_rows rows (max_rows >= wide_min_avg_rows * E): up to
     * wide_tile_tokens_max activation rows per tile, one accumulator buffer. */
    int32_t wide_tile_tokens_max;
    int32_t wide_stage_bytes_act_max;
    int32_t wide_smem_bytes;
    int32_t wide_min_avg_rows;
    /* The CTA-pair tile (two SMs, tcgen05 cta_group::2: 256 weight rows x up to
     * pair_tile_tokens_max activation rows), used when the experts average at
     * least pair_min_avg_rows rows. */
    int32_t pair_tile_tokens_max;
    int32_t pair_smem_bytes;
    int32_t pair_min_avg_rows;
} nvfp4_gemm_plan;

NVFP4_API nvfp4_status nvfp4_gemm_get_plan(nvfp4_gemm_plan* plan);
/* Expect-tx bytes one stage's TMA and bulk copies deliver for a tile of `tokens` rows
 * (wide != 0: the wide tile shape): both packed weight tiles, the activation rows
 * rounded up to 16 and the `tokens` rows' 16 scale bytes of the K step. -1 when
 * tokens is outside [1, tile maximum]. */
NVFP4_API int64_t nvfp4_gemm_stage_tx_bytes(int32_t tokens, int32_t wide);
/* Pure host check against a given opt-in shared-memory budget (bytes per block). */
NVFP4_API nvfp4_status nvfp4_can_implement_with_budget(int64_t N, int64_t K, int32_t E, nvfp4_epilogue epi,
                                             int64_t smem_optin_bytes);
/* The same check against the current device. */
NVFP4_API nvfp4_status nvfp4_can_implement(int64_t N, int64_t K, int32_t E, nvfp4_epilogue epi);

/* ------------------------------------------------------------------------ */
/* Device status and diagnostics.                                            */
/* ------------------------------------------------------------------------ */
/* Synchronises `stream`, reads the device status word of the current device,
 * clears it and returns NVFP4_OK, NVFP4_ERR_DEVICE_TIMEOUT or
 * NVFP4_ERR_DEVICE_INPUT (timeout wins when both are latched). */
NVFP4_API nvfp4_status nvfp4_get_device_status(nvfp4_stream_t stream);
/* Upper bound, in nanoseconds, on any single pipeline wait inside the GEMM
 * (default 1 s). After it the kernel latches NVFP4_ERR_DEVICE_TIMEOUT, drains
 * its own copies, frees its tensor memory and returns. */
NVFP4_API void nvfp4_set_wait_timeout_ns(uint64_t ns);
NVFP4_API uint64_t nvfp4_get_wait_timeout_ns(void);
/* Test hook for the failure-detection test only; 0 (the default) on every
 * normal call. Bit 0: the grouped GEMM's producer warp issues no loads, so each
 * consumer's bounded wait runs out after the wait timeout and the kernel
 * latches NVFP4_ERR_DEVICE_TIMEOUT and returns (nothing is in flight, the
 * context stays usable). Other bits are ignored. */
NVFP4_API void nvfp4_debug_set_flags(uint32_t flags);
/* Number of kernel launches made by this library in this process. */
NVFP4_API uint64_t nvfp4_launch_count(void);
NVFP4_API const char* nvfp4_status_string(nvfp4_status status);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4MOE_H */
