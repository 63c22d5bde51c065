/*
 * nvfp4moe.h - C ABI of the NVFP4 W4A4 routed mixture-of-experts feed-forward layer
 * for NVIDIA B200 (sm_100a).  Library: libnvfp4moe.so.
 *
 * What the layer computes.  The pages describe routed experts stored and run as
 * "NVFP4 W4A4" (Qwen3.8-Flash-Next-NVFP4-SSD-Stream model card, "What this model is"),
 * two NVFP4 values per packed byte (same card, "Why Hugging Face shows 68B parameters and
 * 8-bit precision"), 512 routed experts and prefill batches of up to 512 tokens that reuse
 * the routed expert weights (Eider, "Qwen3.8 Flash Next", "Performance"), and grouped
 * routed kernels for many decode rows (DwarfStar CUDA multi-GPU doc).  The pages do not
 * define the arithmetic; this library implements the standard NVFP4 format:
 *
 *   value = e2m1(code) * e4m3(block scale) * fp32 tensor scale,
 *   one E4M3 block scale per 16 consecutive elements along K,
 *   dynamic tensor scale = amax / (6 * 448),
 *
 * and the routed feed-forward layer
 *
 *   ids, w   = top-k of the router logits (ties -> lower expert index),
 *              w = softmax over the k selected logits
 *   xq       = NVFP4(x)                      (one tensor scale for the layer input)
 *   g, u     = xq . Wg[e]^T, xq . Wu[e]^T     (per selected expert e)
 *   h        = NVFP4(silu(g) * u)            (per-expert tensor scale s_h[e], given)
 *   y        = h . Wd[e]^T
 *   out[t]   = bf16( sum_j w[t][j] * y[t][j] )
 *
 * Conventions (all entry points):
 *  - Every pointer argument is a DEVICE pointer owned by the caller unless stated.
 *    The library never allocates device memory: scratch comes from a caller-provided
 *    workspace whose size is given by the matching *_workspace_size() query.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default).
 *  - Argument checks are synchronous and return an error status before any launch.
 *    Problems only the device can see (an expert id out of range, a duplicate id in a
 *    token) set a sticky device status word; nvfp4moe_device_status() reads it.
 *    Kernels never trap and never spin.
 *  - nvfp4moe_last_error() returns a message for the last failing call of this thread.
 *
 * Layouts:
 *  - codes: row-major [rows][K/2] bytes; element 2i in the low nibble of byte i,
 *    element 2i+1 in the high nibble.  Rows start every K/2 bytes.
 *  - block scales (SF), one E4M3 byte per 16 elements, in one of two layouts:
 *      NVFP4MOE_SF_ROWMAJOR: [rows][K/16];
 *      NVFP4MOE_SF_MMA: the tcgen05 block-scaled MMA layout.  Rows are grouped in
 *        blocks of 128, K in atoms of 64 elements (4 scales).  The scale of row r,
 *        16-element block b sits at byte
 *          ((r/128) * (K/64) + b/4) * 512 + (r%32) * 16 + ((r%128)/32) * 4 + b%4.
 *        The buffer spans ceil(rows/128)*128 rows; K must be a multiple of 64.
 *  - gate/up weights of one expert are stored as ONE matrix W13 [2I][H]: its row 32c+j
 *    is gate row 16c+j for j < 16 and up row 16c+j-16 for j >= 16 (groups of 16 rows).
 *    Requires I % 64 == 0.
 */
#ifndef NVFP4MOE_H
#define NVFP4MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Every declaration below is exported from the shared library, whatever the default
 * symbol visibility of the translation unit that includes this header. */
#if defined(__GNUC__)
#pragma GCC visibility push(default)
#endif

typedef struct CUstream_st* nvfp4moe_stream_t; /* == cudaStream_t */

typedef enum {
  NVFP4MOE_OK = 0,
  NVFP4MOE_INVALID_ARG = 1,       /* null pointer, negative size, bad enum, misalignment */
  NVFP4MOE_UNSUPPORTED_SHAPE = 2, /* a size the kernels do not implement */
  NVFP4MOE_WORKSPACE_TOO_SMALL = 3,
  NVFP4MOE_CUDA_ERROR = 4,        /* a CUDA runtime call or launch failed */
  NVFP4MOE_DEVICE_FAULT = 5       /* the device status word is non-zero */
} nvfp4moe_status;

enum { NVFP4MOE_SF_ROWMAJOR = 0, NVFP4MOE_SF_MMA = 1 };
enum { NVFP4MOE_SCALE_GIVEN = 0, NVFP4MOE_SCALE_DYNAMIC = 1 };
enum { NVFP4MOE_DTYPE_BF16 = 0, NVFP4MOE_DTYPE_F32 = 1 };

/* Device status bits (nvfp4moe_device_status). */
enum {
  NVFP4MOE_DEV_BAD_EXPERT_ID = 1u << 0,  /* a routing id outside [0, E) was skipped */
  NVFP4MOE_DEV_DUPLICATE_ID = 1u << 1,   /* a token listed the same expert twice */
  NVFP4MOE_DEV_ROW_OVERFLOW = 1u << 2,   /* permuted rows exceeded the stated capacity */
  NVFP4MOE_DEV_TIMEOUT = 1u << 3,        /* a bounded wait inside a kernel gave up */
  NVFP4MOE_DEV_BAD_GATHER = 1u << 4      /* a row_gather entry past the input rows was skipped */
};

/* Message for the last failing call on this host thread ("" if none). */
const char* nvfp4moe_last_error(void);

/* Library version, e.g. 0x000400 = 0.4.0. */
int32_t nvfp4moe_version(void);

/* Waits for `stream`, then returns the sticky device status word of the current device
 * in *status (0 = no fault).  If `clear` is non-zero the word is reset to 0 afterwards.
 * Returns NVFP4MOE_OK or NVFP4MOE_CUDA_ERROR. */
nvfp4moe_status nvfp4moe_device_status(nvfp4moe_stream_t stream, int32_t clear,
                                       uint32_t* status);

/* ------------------------------------------------------------------------------
 * nvfp4_codec_convert - the element encoders every kernel uses, exposed for checking.
 * in: fp32 [n].  e2m1: one code per byte in the low nibble (round to nearest, ties to
 * the even code, saturate to +-6, sign kept).  e4m3: one E4M3 byte (round to nearest
 * even, saturate to +-448).  Either output may be NULL.
 * ---------------------------------------------------------------------------- */
nvfp4moe_status nvfp4_codec_convert(const float* in, int64_t n, uint8_t* e2m1,
                                    uint8_t* e4m3, nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------------
 * nvfp4_quantize - bf16/fp32 -> NVFP4 block quantiser (the "A4" of W4A4 and the weight
 * preparation step).
 *
 * x: [batch][rows][K] of dtype x_dtype, row stride ldx elements, batch stride
 *    x_batch_stride elements.  x must be 16-byte aligned and ldx*elt, x_batch_stride*elt
 *    multiples of 16 bytes.
 * row_gather (nullable): [out_rows]; output row r of every batch item reads input row
 *    row_gather[r] of the same item; a negative entry leaves output row r unwritten.
 *    NULL means out_rows == rows and row r reads row r.
 * scale_mode: GIVEN reads tensor_scale[b] for batch item b; DYNAMIC computes
 *    tensor_scale[b] = amax(|x[b]|) / 2688 over the item's `rows` input rows and writes it.
 * codes: [batch][out_rows][K/2] with batch stride codes_batch_stride bytes.
 * sf: block scales in sf_layout with batch stride sf_batch_stride bytes (ROWMAJOR:
 *    out_rows*K/16 at least; MMA: ceil(out_rows/128)*128*K/16 at least).
 * Per 16-element block (every step one IEEE fp32 operation, round to nearest):
 *    sf = e4m3(amax_b / (6*s_t)); if e4m3 value is 0 all codes are 0; otherwise
 *    inv = 1 / (e4m3val(sf) * s_t) and code_i = e2m1(x_i * inv).  s_t == 0 gives
 *    all-zero codes and scales.  Requires K % 16 == 0 (K % 64 == 0 for the MMA layout).
 * workspace: DYNAMIC mode needs nvfp4_quantize_workspace_size() bytes; GIVEN needs none.
 * ---------------------------------------------------------------------------- */
size_t nvfp4_quantize_workspace_size(int64_t batch, int64_t rows, int64_t K);
nvfp4moe_status nvfp4_quantize(const void* x, int32_t x_dtype, int64_t batch, int64_t rows,
                               int64_t K, int64_t ldx, int64_t x_batch_stride,
                               const int32_t* row_gather, int64_t out_rows, int32_t scale_mode,
                               float* tensor_scale, uint8_t* codes, int64_t codes_batch_stride,
                               uint8_t* sf, int64_t sf_batch_stride, int32_t sf_layout,
                               void* workspace, size_t workspace_bytes,
                               nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------------
 * nvfp4_quantize_dynamic_noalloc - nvfp4_quantize in DYNAMIC scale mode for callers that
 * cannot allocate device memory.  (The pages have no counterpart: this is a packaging
 * variant of the quantiser above, not a step of the method.)
 *
 * Some callers cannot hand the library a workspace or call cudaMalloc: plug-ins running
 * inside a host framework that owns the device allocator and forbids side allocations, and
 * deployments that fix their whole device-memory footprint up front.  This entry point
 * takes no workspace.  Its scratch (the per-CTA amax partials of the dynamic scale) is a
 * 64 KiB array compiled into the library, which every GPU that loads the library keeps
 * until the process exits.  Arguments, layouts and results are those of nvfp4_quantize with
 * scale_mode = NVFP4MOE_SCALE_DYNAMIC (tensor_scale is written).
 *  - Sizes whose scratch need (nvfp4_quantize_workspace_size(batch, rows, K)) exceeds
 *    65536 bytes are rejected with NVFP4MOE_UNSUPPORTED_SHAPE before any work.
 *  - The first call on a device looks up the device address of the array (once per
 *    device, with that device current); make that first call before any stream capture.
 *  - Every call on a device shares the array and it keeps the last call's contents; each
 *    call overwrites every partial it reads, so nothing has to be cleared.  Calls whose
 *    kernels overlap on the GPU (unordered streams) race on the array: order them.
 *  - The call itself allocates nothing.  The array is part of the library's device module:
 *    the driver places it in device memory when it loads that module on a device, which
 *    under CUDA's default lazy module loading can be the first call into the library on
 *    that device.  A host that must see no device allocation after its set-up makes one
 *    warm-up call of this entry point at set-up (or runs with CUDA_MODULE_LOADING=EAGER).
 * ---------------------------------------------------------------------------- */
nvfp4moe_status nvfp4_quantize_dynamic_noalloc(const void* x, int32_t x_dtype, int64_t batch,
                                               int64_t rows, int64_t K, int64_t ldx,
                                               int64_t x_batch_stride, const int32_t* row_gather,
                                               int64_t out_rows, float* tensor_scale,
                                               uint8_t* codes, int64_t codes_batch_stride,
                                               uint8_t* sf, int64_t sf_batch_stride,
                                               int32_t sf_layout, nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------------
 * nvfp4_from_mxfp4 - the exact NVFP4 form of MXFP4 weight matrices, so that MXFP4 weights
 * run on every path of the layer.  MXFP4 (the DwarfStar CUDA multi-GPU doc's launcher default,
 * read as the OCP microscaling definition): E2M1 codes packed as NVFP4's (element 2i in the
 * low nibble of byte i) and one E8M0 scale 2^(E-127) per 32 elements along K.  A power of two
 * 2^j is an E4M3 value for j in [-9, 8]: both 16-element halves of a block get the E4M3 scale
 * 2^(E-127-shift) and the matrix the fp32 tensor scale 2^shift, shift = (largest E of a
 * block with a nonzero code) - 135; a zero block gets scale 0.
 *
 * codes [batch][rows][K/2], e8m0 [batch][rows][K/32] (device).  Out row r of each matrix
 * takes input row row_gather[r] (nullable: r; -1: the row is left untouched, for building
 * the interleaved W13 from gate and up in two calls; an entry >= rows is NVFP4MOE_INVALID_ARG),
 * out_rows rows.  Writes
 * sf_out [batch][sf_mma_bytes(out_rows, K)] (MMA layout), tensor_scale [batch], and, when
 * codes_out is non-null, the codes [batch][out_rows][K/2].  K % 64 == 0; codes 16-byte
 * aligned.  Workspace: nvfp4_from_mxfp4_workspace_size(batch) bytes.  Synchronous (a setup
 * step): returns NVFP4MOE_UNSUPPORTED_SHAPE, naming the matrices, when the scales of a
 * matrix's nonzero blocks span more than 18 binades (no exact NVFP4 form).
 * ---------------------------------------------------------------------------- */
size_t nvfp4_from_mxfp4_workspace_size(int64_t batch);
nvfp4moe_status nvfp4_from_mxfp4(const uint8_t* codes, const uint8_t* e8m0, int64_t batch, int64_t rows,
                                 int64_t K, const int32_t* row_gather, int64_t out_rows,
                                 uint8_t* codes_out, uint8_t* sf_out, float* tensor_scale,
                                 void* workspace, size_t workspace_bytes, nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------------
 * nvfp4_prep_weights - weights that arrive already quantised to NVFP4 (E2M1 codes, E4M3 block
 * scales, fp32 tensor scales: the form the Qwen3.8-Flash-Next-NVFP4-SSD-Stream model card's
 * checkpoint keeps its routed experts in, two codes per byte) into the layout the layer reads.
 * Bytes only, nothing is recomputed:
 *  - out row r of each matrix takes input row row_gather[r] (nullable: row r); a negative
 *    entry leaves out row r untouched, so the interleaved W13 is built from gate and up in
 *    two calls (see the gate/up layout above); an entry >= rows also leaves it untouched and
 *    sets NVFP4MOE_DEV_BAD_GATHER in the device status word;
 *  - the row's block scales are written in sf_out_layout (the layer needs NVFP4MOE_SF_MMA);
 *  - the row's codes are copied to codes_out, unless codes_out is NULL: the call then only
 *    converts the scales between the two layouts (either direction).
 * Tensor scales are used as they are (moe_ffn_desc.w13_scale keeps gate's and up's apart).
 * codes [batch][rows][K/2] (16-byte aligned when codes_out is given), sf [batch][...] in
 * sf_layout (ROWMAJOR: rows*K/16 bytes per matrix; MMA: ceil(rows/128)*128*K/16), 4-byte
 * aligned; codes_out [batch][out_rows][K/2]; sf_out like sf for out_rows rows.
 * K % 64 == 0.  Asynchronous on `stream`; allocates nothing.
 * ---------------------------------------------------------------------------- */
nvfp4moe_status nvfp4_prep_weights(const uint8_t* codes, const uint8_t* sf, int32_t sf_layout, int64_t batch,
                                   int64_t rows, int64_t K, const int32_t* row_gather, int64_t out_rows,
                                   uint8_t* codes_out, uint8_t* sf_out, int32_t sf_out_layout,
                                   nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------------
 * moe_route - router top-k (DwarfStar CUDA multi-GPU doc: routers run replicated next to
 * the routed experts).
 * logits: fp32 [T][E] (finite).  ids: int32 [T][k], experts in descending logit order,
 * equal logits (including +0 / -0) in ascending expert index.  w: fp32 [T][k], the
 * softmax of the k selected logits.  1 <= k <= min(E, 32), 1 <= E <= 1024.
 * ---------------------------------------------------------------------------- */
nvfp4moe_status moe_route(const float* logits, int32_t T, int32_t E, int32_t k, int32_t* ids,
                          float* w, nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------------
 * moe_permute - expert histogram and prefix-scan permutation into per-expert row groups
 * (the grouped routed kernels of the DwarfStar doc and Eider's grouped MoE prefill).
 *
 * ids: int32 [T][k].  m_tile: row padding of each expert group (1 = none; 64 for the
 * tensor-core layer path; 32 and 128 are also accepted).  Rows of expert e occupy [padded_offsets[e], padded_offsets[e] +
 * counts[e]) in ascending token order; experts in ascending index.  Outputs:
 *   counts [E], offsets [E+1] (exclusive scan of counts), padded_offsets [E+1]
 *   (exclusive scan of counts rounded up to m_tile), pair_to_row [T*k] (pair t*k+j ->
 *   padded row), row_token [rows_cap] and row_pair [rows_cap] (padded row -> token /
 *   pair; -1 on padding rows), tile_expert [rows_cap/m_tile] (expert of each m_tile-row
 *   tile), active [E+1] (active[0] = number of experts with rows, then their indices in
 *   ascending order), and zero_f32 (nullable, [E] floats set to 0; used for the optional
 *   per-expert amax output of moe_ffn_forward).
 * rows_cap must be >= moe_permute_rows_capacity(T, E, k, m_tile).  Out-of-range or
 * duplicate ids are skipped (pair_to_row = -1) and flag the device status word.
 * T*k <= 2^24, E <= 1024, k <= 32, m_tile in {1, 32, 64, 128}.
 * ---------------------------------------------------------------------------- */
int64_t moe_permute_rows_capacity(int32_t T, int32_t E, int32_t k, int32_t m_tile);
nvfp4moe_status moe_permute(const int32_t* ids, int32_t T, int32_t E, int32_t k,
                            int32_t m_tile, int64_t rows_cap, int32_t* counts,
                            int32_t* offsets, int32_t* padded_offsets, int32_t* pair_to_row,
                            int32_t* row_token, int32_t* row_pair, int32_t* tile_expert,
                            int32_t* active, float* zero_f32, nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------------
 * nvfp4_gemm - one NVFP4 x NVFP4 GEMM, D[M][N] = (A . B^T) * a_scale[0] * b_scale[0].
 * A: codes [M][K/2] + SF (MMA layout over M rows); B: codes [N][K/2] + SF (MMA layout
 * over N rows); both K-major.  D: [M][N] row-major, d_dtype BF16 or F32.
 * M <= 16 runs the split-K GEMV kernel, larger M the tcgen05 block-scaled MMA kernel.
 * Requires K % 128 == 0, N % 128 == 0, 16-byte aligned pointers.
 * ---------------------------------------------------------------------------- */
size_t nvfp4_gemm_workspace_size(int64_t M, int64_t N, int64_t K);
nvfp4moe_status nvfp4_gemm(const uint8_t* A, const uint8_t* A_sf, const float* a_scale,
                           const uint8_t* B, const uint8_t* B_sf, const float* b_scale,
                           int64_t M, int64_t N, int64_t K, void* D, int32_t d_dtype,
                           void* workspace, size_t workspace_bytes, nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------------
 * moe_ffn_forward - the whole routed feed-forward layer.
 * ---------------------------------------------------------------------------- */
enum { NVFP4MOE_PATH_AUTO = 0, NVFP4MOE_PATH_GEMV = 1, NVFP4MOE_PATH_GEMM = 2 };
/* How the k weighted expert rows of a token are combined:
 *   ORDERED     each row is kept in fp32 and a token's rows are summed in slot order, one
 *               rounding to bf16 (deterministic);
 *   ACCUMULATE  the down GEMM adds each row into an fp32 [T][H] accumulator (reduction order
 *               not fixed, so the last bits of an fp32 sum may differ between calls), then one
 *               rounding to bf16; no per-slot rows, far less memory traffic for large batches
 *               (tensor-core path only);
 *   AUTO        ORDERED; ACCUMULATE when top_k == 1 on the tensor-core path (one term per
 *               output: exact and deterministic). */
enum { NVFP4MOE_COMBINE_AUTO = 0, NVFP4MOE_COMBINE_ORDERED = 1, NVFP4MOE_COMBINE_ACCUMULATE = 2 };
/* Activation format of the expert products:
 *   NVFP4  W4A4: x and the intermediate h are quantised to NVFP4 (the layer the model cards
 *          describe as "NVFP4 W4A4", Qwen3.8-Flash-Next-NVFP4-SSD-Stream card);
 *   BF16   W4A16, weight-only: x enters the products in bf16 and h is rounded to bf16 (no
 *          activation-quantisation site, as the Qwen3.8-27B-nvfp4full-dflash2-NInfer card's
 *          "Limits" names it); x_scale, h_scale, h_scale_mode and h_amax are unused.  Runs the
 *          split-K GEMV path (PATH_AUTO resolves to it; PATH_GEMM is UNSUPPORTED_SHAPE). */
enum { NVFP4MOE_ACT_NVFP4 = 0, NVFP4MOE_ACT_BF16 = 1 };

typedef struct {
  int32_t T, H, I, E, top_k;
  int32_t path;               /* NVFP4MOE_PATH_*; AUTO: tensor cores when I % 128 == 0, else GEMV */
  int32_t x_scale_mode;       /* NVFP4MOE_SCALE_GIVEN or _DYNAMIC */
  const float* x_scale;       /* [1], read when GIVEN */
  const uint8_t* w13_codes;   /* [E][2I][H/2], gate/up rows interleaved (see above) */
  const uint8_t* w13_sf;      /* [E][2I*H/16], MMA layout per expert */
  const float* w13_scale;     /* [E][2]: tensor scales of gate and up */
  const uint8_t* w2_codes;    /* [E][H][I/2] */
  const uint8_t* w2_sf;       /* [E][H*I/16], MMA layout per expert */
  const float* w2_scale;      /* [E] */
  const float* h_scale;       /* [E]: requantisation tensor scale of h per expert */
  float* h_amax;              /* nullable [E]: receives amax|h| per expert (calibration) */
  /* nullable: NVFP4MOE_STAGES cudaEvent_t handles (created by the caller) that the call
   * records on `stream` at its stage boundaries, for per-stage timing: [0] start,
   * [1] after routing, [2] after the permutation, [3] after quantising x, [4] after the
   * gate/up GEMM, [5] after the down GEMM, [6] after the combine. */
  void* const* stage_events;
  int32_t combine;            /* NVFP4MOE_COMBINE_* */
  /* NVFP4MOE_SCALE_GIVEN: h is requantised with h_scale[e] (a calibrated constant);
   * NVFP4MOE_SCALE_DYNAMIC: with amax(h of expert e in this call) / 2688 (1 for an expert
   * without tokens), h_scale unused; the scales used are left in the workspace at
   * layout.h_stats + 4*E (tensor-core path only, else NVFP4MOE_UNSUPPORTED_SHAPE; h_amax,
   * when given, receives the maxima as well). */
  int32_t h_scale_mode;
  int32_t act_mode;           /* NVFP4MOE_ACT_* */
  /* Optional shared expert, a dense BF16 SwiGLU MLP beside the routed experts (the SSD-Stream
   * card: "shared experts ... remain BF16"): shared_I = its intermediate size (0: none;
   * else a positive multiple of 64), shared_w13 bf16 [2*shared_I][H] with gate and up rows
   * interleaved like w13_codes (rows 32c+j: gate row 16c+j for j < 16, up row 16c+j-16
   * otherwise), shared_w2 bf16 [H][shared_I].  out = bf16(routed + w2 . bf16(silu(g) * u)),
   * one rounding of the fp32 sum; the shared expert's products are fp32. */
  int32_t shared_I;
  const uint16_t* shared_w13;
  const uint16_t* shared_w2;
  /* NVFP4MOE_LAUNCH_*: how a batch that the single-launch layer supports (tensor-core path,
   * at most 16 tokens, ordered combine, given h scales, no shared expert) is run:
   *   SINGLE  one persistent, cooperative launch for the whole layer (after a small launch
   *           that resets its counters): every CTA routes the batch and keeps x quantised in
   *           shared memory, then runs one of two schedules, chosen per call from the routing
   *           (every CTA takes the same decision):
   *             expert-local: units of (active expert, 256, 512 or 1024 columns of h); a CTA
   *               runs a unit's gate/up tiles, keeps its h chunk in shared memory and runs the
   *               unit's down tiles from it.  Taken when I % 256 == 0 and the units fill the
   *               grid's rounds to at least 80 % (the widest such chunk is used);
   *             tile-level: gate/up and down tiles spread over all CTAs, h through global
   *               memory, the down tiles of an expert waiting on counters of its gate/up tiles;
   *           then, after a grid-wide barrier, every CTA sums a slice of the outputs over the
   *           k x K-chunk slot rows in slot order;
   *   SINGLE_TILE, SINGLE_LOCAL  SINGLE with that schedule (SINGLE_LOCAL needs I % 256 == 0 and
   *           I <= 63 * 256, else NVFP4MOE_UNSUPPORTED_SHAPE);
   *   MULTI   the routing/permutation/quantisation prologue, then the grouped GEMMs, then the
   *           combine (the path every larger batch takes);
   *   AUTO    the faster of SINGLE and MULTI for the shape (see moe_ffn_workspace_layout's
   *           single_launch).
   * All give the same routing, permutation and codes, and outputs within the stated tolerance
   * (the schedules differ only in the order of the fp32 sums over K). */
  int32_t launch_mode;
} moe_ffn_desc;

enum {
  NVFP4MOE_LAUNCH_AUTO = 0,
  NVFP4MOE_LAUNCH_SINGLE = 1,
  NVFP4MOE_LAUNCH_MULTI = 2,
  NVFP4MOE_LAUNCH_SINGLE_TILE = 3,
  NVFP4MOE_LAUNCH_SINGLE_LOCAL = 4
};

enum { NVFP4MOE_STAGES = 7 };

/* Byte offsets of the intermediates inside the workspace (for inspection and tests). */
typedef struct {
  int64_t topk_ids, topk_w, counts, offsets, padded_offsets, pair_to_row, row_token,
      row_pair, tile_expert, active, x_scale, x_codes, x_sf, h_codes, h_sf, slots,
      amax_partials, total;
  int64_t x_rows;   /* rows of x_codes / x_sf (T on the GEMV path, rows_cap otherwise) */
  int64_t h_rows;   /* rows of h_codes / h_sf */
  int64_t items;    /* small batches on the GEMM path: the grouped GEMMs' work lists, written by
                       the routing step (int4 entries; see csrc/ffn_grouped.cu); else unused */
  int32_t m_tile;   /* 1 on the GEMV path, 64 on the GEMM path */
  int32_t path;     /* resolved path */
  int32_t combine;  /* resolved combine mode; ACCUMULATE: the accumulator is at `slots` */
  int32_t single_launch; /* 1: the whole layer runs as one persistent launch (batches of at most
                            16 tokens on the GEMM path, ordered combine, given h scales, no
                            shared expert); `items` then holds its counters, `slots` its fp32
                            rows by (pair, K chunk): chunks of 256 under the expert-local
                            schedule, of at most 2048 under the tile-level one */
  int64_t h_f32;    /* dynamic h scale: fp32 h [h_rows][I] before requantisation */
  int64_t h_stats;  /* dynamic h scale: amax[E] then the scales used, s_h[E] (fp32) */
  int64_t h_bf16;   /* weight-only layer: h in bf16 [T*k][I], permuted rows (x_codes, x_sf,
                       h_codes, h_sf are empty then) */
  int64_t shared_h; /* shared expert: its h in bf16 [T][shared_I] */
  int64_t shared_y; /* shared expert: its output rows in fp32 [T][H] */
} moe_ffn_ws_layout;

nvfp4moe_status moe_ffn_workspace_layout(const moe_ffn_desc* d, moe_ffn_ws_layout* layout);
size_t moe_ffn_workspace_size(const moe_ffn_desc* d);

/* x: bf16 [T][H]; logits: fp32 [T][E]; out: bf16 [T][H]; desc is a HOST pointer.
 * Requires H % 256 == 0, I % 64 == 0, E <= 1024, 1 <= top_k <= min(E, 32). */
nvfp4moe_status moe_ffn_forward(const moe_ffn_desc* desc, const void* x, const float* logits,
                                void* out, void* workspace, size_t workspace_bytes,
                                nvfp4moe_stream_t stream);

/* ------------------------------------------------------------------------------
 * Measurement and self-test entry points.  The pages have no counterpart of these: they
 * measure the device and exercise the library's failure reporting, and compute nothing of
 * the layer.
 *
 * nvfp4moe_mma_peak_probe - the block-scaled FP4 tensor-core ceiling of this device.  One
 * CTA per SM issues iters x 4 tcgen05.mma kind::mxf4nvf4 (M=128, N=256, K=64, E4M3 scales
 * per 16 elements) on operands resident in shared memory; time the launch on `stream` and
 * divide nvfp4moe_mma_peak_probe_flops(iters) by it.  1 <= iters <= 2^24.  Writes nothing
 * but the device status word (NVFP4MOE_DEV_TIMEOUT if a bounded wait gave up).
 *
 * nvfp4moe_wait_selftest - one thread waits, at most `polls` polls (1 <= polls <= 2^20),
 * on an mbarrier phase that never completes, with the bounded wait every tcgen05 kernel of
 * the library uses.  When the polls run out it sets NVFP4MOE_DEV_TIMEOUT in the device
 * status word and stores 0 in *result (device int32; 1 if the wait had completed), then
 * returns.  Nothing faults: the context and later calls stay usable.
 * ---------------------------------------------------------------------------- */
nvfp4moe_status nvfp4moe_mma_peak_probe(int64_t iters, nvfp4moe_stream_t stream);
int64_t nvfp4moe_mma_peak_probe_flops(int64_t iters);
nvfp4moe_status nvfp4moe_wait_selftest(uint32_t polls, int32_t* result, nvfp4moe_stream_t stream);

#if defined(__GNUC__)
#pragma GCC visibility pop
#endif

#ifdef __cplusplus
}
#endif
#endif /* NVFP4MOE_H */
