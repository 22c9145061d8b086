/*
 * fp8q.h -- C ABI of the FP8 E4M3 quantization library for B200 (sm_100a).
 *
 * Three operations of an LLM inference engine's FP8 path:
 *   1. per-token 1x128-group activation quantization (fp8_group_quant);
 *   2. the paged KV-cache quantize-and-scatter, reshape_and_cache_fp8
 *      semantics (fp8_kv_write);
 *   3. online calibration of the per-tensor KV scales over a window of
 *      tokens: device absmax (fp8_kv_amax_observe), staging of the window's
 *      bf16 K/V, the freeze and the chronological replay
 *      (fp8_kv_calib_* and fp8_kv_freeze_replay).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Arithmetic.  bf16 in; E4M3 ("FN": bias 7, max finite 448, no infinity)
 *    out.  A code is E4M3(fp32(x / scale)): the quotient is the IEEE fp32
 *    division of x by the scale, then rounded to E4M3 to nearest-even,
 *    saturating to +-448, keeping the sign of zero.  Results are bit-identical
 *    to a plain CPU restatement of these definitions.  Inputs must be finite
 *    (no NaN, no infinity).
 *  - Memory.  Every pointer except the calibration handle is DEVICE memory
 *    owned by the caller; the library allocates no device memory and frees
 *    none.  Sizes and strides are in ELEMENTS unless the name says bytes.
 *  - Streams.  `stream` is a cudaStream_t passed as void*; NULL is the legacy
 *    default stream.  All device work is enqueued on it and nothing
 *    synchronizes the host, except the calls documented as synchronizing.
 *  - Errors.  Arguments are checked before anything is enqueued: a bad
 *    argument returns FP8Q_EINVAL and touches no memory.  A failed launch
 *    returns FP8Q_ECUDA.  Conditions only the device can see (a slot past the
 *    end of the pool, a device-resident scale that is not a positive number)
 *    skip the affected writes and set a bit in a sticky per-device error word
 *    read by fp8q_device_error().  Nothing traps, nothing waits.
 *  - Alignment.  bf16 buffers and staging buffers: 16-byte aligned, row
 *    strides multiples of 8 elements.  Code buffers and pools: 8-byte aligned.
 *    fp32 and int64 arrays: naturally aligned.
 *
 * Citations name the source page's title and the item on it.
 */
#ifndef FP8Q_H
#define FP8Q_H

#include <stdint.h>

#if defined(_WIN32)
#define FP8Q_API __declspec(dllexport)
#else
#define FP8Q_API __attribute__((visibility("default")))
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t fp8q_status;

#define FP8Q_OK 0
#define FP8Q_EINVAL (-1)      /* bad argument; nothing was enqueued         */
#define FP8Q_ECUDA (-2)       /* a CUDA call failed                          */
#define FP8Q_ESTATE (-3)      /* calibration call out of order               */
#define FP8Q_ENOMEM (-4)      /* host memory for a handle could not be had   */
#define FP8Q_ETOOBIG (-5)     /* needs more than the library's fixed scratch */

/* Bits of the sticky per-device error word. */
#define FP8Q_DEVERR_SLOT_OUT_OF_RANGE 0x1u  /* slot >= num_blocks*block_size: token skipped */
#define FP8Q_DEVERR_BAD_SCALE 0x2u          /* device scale NaN or <= 0: tensor not written */

/* E4M3 saturation value and the group width of the activation quantizer. */
#define FP8Q_E4M3_MAX 448.0f
#define FP8Q_GROUP 128

/* Largest number of tokens a calibration window stages; a longer requested
 * window is clamped to it.  Source: "spark_model/layers/fp8_calibration/
 * staging.rs", MAX_STAGED_TOKENS. */
#define FP8Q_MAX_STAGED_TOKENS 4096

/* Scale of the entries written inside the window, before the freeze
 * (2.0 * 448 covers |x| <= 896).  Source: "metrale_model_layers/layers/
 * fp8_calibration.rs", PROVISIONAL_SCALE. */
#define FP8Q_PROVISIONAL_SCALE 2.0f

/* ------------------------------------------------------------------------ */
/* 1. Activation quantization                                               */
/* ------------------------------------------------------------------------ */

/*
 * fp8_group_quant -- per-token 1x128-group quantization.
 *
 * Source: "spark_model/layers/ops/fp8_act_quant.rs", module doc (a bf16
 * [M, K] activation, one fp32 scale per 128-element K-group, E4M3 codes) and
 * fp8_quant_grid (K/128 groups per row; M may exceed 65535);
 * "spark_model/layers/ops/dispatch_proj_decode.rs", DecodeW8a8Scratch::fits
 * and decode_w8a8_quant_act (codes rows*k bytes; scales rows*(k/128) fp32 in
 * the quantizer's [M, K/128] order).
 *
 * For each row r < m and group g < k/128:
 *   amax  = max_j |x[r, 128g + j]|                  (fp32, exact from bf16)
 *   s     = max(amax, 1e-12f) / 448.0f              (IEEE fp32 division)
 *   scales[r * (k/128) + g] = s
 *   q[r * k + 128g + j]     = E4M3(fp32(x[r, 128g + j] / s))
 *
 *   x            device bf16, row r at x + r * x_row_stride; 16-byte aligned
 *   x_row_stride elements between rows; >= k, multiple of 8
 *   q            device E4M3 [m, k], packed rows; 8-byte aligned
 *   scales       device fp32 [m, k/128], row-major
 *   m            rows (tokens), >= 0; 0 is a no-op
 *   k            row width, a positive multiple of 128
 * Returns FP8Q_OK, FP8Q_EINVAL (sizes, alignment, null pointers),
 * FP8Q_ECUDA.
 */
FP8Q_API fp8q_status fp8_group_quant(const void *x, int64_t x_row_stride,
                                     void *q, float *scales, int64_t m,
                                     int64_t k, void *stream);

/*
 * fp8_group_quant_kmajor -- the same quantization, laid out for a padded FP8
 * GEMM: phantom rows zeroed and the scales transposed K-major, in one launch.
 *
 * Source: "spark_model/layers/ops/dispatch_proj_decode.rs",
 * decode_w8a8_quant_act (quantize the rows, zero the codes of the phantom
 * rows rows..ceil16(rows), re-lay the 1x128 scales out K-major over all m_pad
 * rows, pad rows included), DecodeW8a8Plan (the cuBLASLt GEMM is handed
 * m_pad = ceil16(M) rows) and the scale-layout clause of its doc (the GEMM
 * reads the activation scales token-contiguous; the quantizer's [M, K/128]
 * order gives wrong results on the same codes).  The pages do this as three
 * launches (quantize, memset, transpose); here it is one pass.
 *
 * For r < m and g < k/128, with s and the codes exactly as fp8_group_quant:
 *   q[r * k + 128g + j]       = E4M3(fp32(x[r, 128g + j] / s))
 *   scales_km[g * m_pad + r]  = s
 * and for m <= r < m_pad (phantom rows; x is not read):
 *   q[r * k + 128g + j] = 0,  scales_km[g * m_pad + r] = 0.0f
 *
 *   x            device bf16, row r at x + r * x_row_stride; 16-byte aligned
 *                (may be NULL when m == 0)
 *   x_row_stride elements between rows; >= k, multiple of 8
 *   q            device E4M3 [m_pad, k], packed rows; 8-byte aligned
 *   scales_km    device fp32 [k/128, m_pad] (K-major); 4-byte aligned
 *   m            live rows, >= 0
 *   m_pad        rows of q and columns of scales_km, >= m (ceil16(m) for a
 *                GEMM padded to 16 rows); 0 is a no-op
 *   k            row width, a positive multiple of 128
 * Returns FP8Q_OK, FP8Q_EINVAL (sizes, alignment, null pointers),
 * FP8Q_ECUDA.
 */
FP8Q_API fp8q_status fp8_group_quant_kmajor(const void *x, int64_t x_row_stride,
                                            void *q, float *scales_km,
                                            int64_t m, int64_t m_pad, int64_t k,
                                            void *stream);

/* ------------------------------------------------------------------------ */
/* 2. Paged KV-cache quantize-and-scatter                                   */
/* ------------------------------------------------------------------------ */

/*
 * fp8_kv_write -- reshape_and_cache_fp8.
 *
 * Source: "spark_model/layers/fp8_calibration/staging.rs", Fp8KvWriteTarget
 * (k_pool, v_pool, block_size, cache_stride = block_size * num_kv_heads *
 * head_dim elements between blocks, key_stride / value_stride source row
 * strides, an int64 slot per token) and KvStaging::replay_and_release (the
 * call's argument list); "metrale_model_layers/layers/fp8_calibration.rs",
 * module doc (one k_scale / v_scale per tensor).
 *
 * For each token t < num_tokens with slot = slot_mapping[t]:
 *   slot < 0                         -> skipped (padding token)
 *   slot >= num_blocks * block_size  -> skipped, FP8Q_DEVERR_SLOT_OUT_OF_RANGE
 *   otherwise, with E = num_kv_heads * head_dim, blk = slot / block_size,
 *   off = slot % block_size, for e < E:
 *     k_pool[blk * cache_stride + off * E + e] = E4M3(fp32(k[t*key_stride + e] / k_scale))
 *     v_pool[...same...]                       = E4M3(fp32(v[t*value_stride + e] / v_scale))
 * i.e. the pool layout is [num_blocks][block_size][num_kv_heads][head_dim]
 * with an optional pad between blocks.  Slots must be distinct within one
 * call (two tokens of one call writing one slot race); across calls stream
 * order decides, the later call wins.
 *
 *   k, v           device bf16 [num_tokens, num_kv_heads, head_dim] rows;
 *                  16-byte aligned
 *   key_stride,
 *   value_stride   elements between token rows; >= E, multiples of 8
 *   slot_mapping   device int64 [num_tokens]
 *   num_tokens     >= 0; 0 is a no-op
 *   num_kv_heads,
 *   head_dim       E = num_kv_heads * head_dim must be a multiple of 8
 *   k_pool, v_pool device E4M3 pools, num_blocks * cache_stride bytes each;
 *                  8-byte aligned
 *   block_size     tokens per block, > 0
 *   cache_stride   elements between blocks, >= block_size * E, multiple of 8
 *   num_blocks     blocks in each pool, >= 0
 *   scale_dev      NULL: use k_scale / v_scale (finite, > 0).  Otherwise a
 *                  device fp32 [2] = {k_scale, v_scale} read by the kernel
 *                  (what a calibrator publishes; keeps the call free of host
 *                  values so a captured graph stays valid across the freeze)
 * Returns FP8Q_OK, FP8Q_EINVAL, FP8Q_ECUDA.
 */
FP8Q_API fp8q_status fp8_kv_write(const void *k, const void *v,
                                  int64_t key_stride, int64_t value_stride,
                                  const int64_t *slot_mapping,
                                  int64_t num_tokens, int32_t num_kv_heads,
                                  int32_t head_dim, void *k_pool, void *v_pool,
                                  int32_t block_size, int64_t cache_stride,
                                  int64_t num_blocks, float k_scale,
                                  float v_scale, const float *scale_dev,
                                  void *stream);

/* One layer's arguments of fp8_kv_write_layers. */
typedef struct fp8q_kv_layer {
    const void *k;                /* device bf16 rows, as for fp8_kv_write      */
    const void *v;
    const int64_t *slot_mapping;  /* device int64 [num_tokens]                  */
    void *k_pool;                 /* this layer's pools                         */
    void *v_pool;
    const float *scale_dev;       /* device {k_scale, v_scale}, or NULL         */
    float k_scale;                /* used when scale_dev is NULL                */
    float v_scale;
} fp8q_kv_layer;

#define FP8Q_MAX_LAYERS 128

/*
 * fp8_kv_write_layers -- reshape_and_cache_fp8 for several layers in one launch.
 *
 * Source: as fp8_kv_write ("spark_model/layers/fp8_calibration/staging.rs",
 * Fp8KvWriteTarget; "metrale_model_layers/layers/fp8_calibration.rs",
 * module doc).  The pages write one layer per call; this performs exactly
 * fp8_kv_write(layers[i], ...) for every i, as one grid (blockIdx.y = layer),
 * for callers that hold all layers' K/V of a set of tokens at once (KV
 * restored from host memory or a prefix cache, KV received from another
 * device).  Layers are independent, so their order does not matter.
 *
 *   layers         HOST array [num_layers] of per-layer pointers and scales;
 *                  alignment and scale rules as for fp8_kv_write
 *   num_layers     0..FP8Q_MAX_LAYERS (0 is a no-op)
 *   key_stride, value_stride, num_tokens, num_kv_heads, head_dim,
 *   block_size, cache_stride, num_blocks
 *                  shared by all layers, as for fp8_kv_write
 * Returns FP8Q_OK, FP8Q_EINVAL, FP8Q_ECUDA.
 */
FP8Q_API fp8q_status fp8_kv_write_layers(const fp8q_kv_layer *layers,
                                         int32_t num_layers, int64_t key_stride,
                                         int64_t value_stride, int64_t num_tokens,
                                         int32_t num_kv_heads, int32_t head_dim,
                                         int32_t block_size, int64_t cache_stride,
                                         int64_t num_blocks, void *stream);

/* ------------------------------------------------------------------------ */
/* 3. Calibration                                                           */
/* ------------------------------------------------------------------------ */

/*
 * fp8_kv_amax_observe -- max-accumulate |K| and |V| of one batch on the device.
 *
 * Source: "metrale_model_layers/layers/fp8_calibration.rs",
 * Fp8KvCalibration::absmax (bf16_absmax max-accumulates into an
 * 8-byte [k_absmax, v_absmax] fp32 buffer the caller zeroes first).
 *
 *   amax_dev[0] = max(amax_dev[0], max_{t,e} |k[t*key_stride + e]|)
 *   amax_dev[1] = max(amax_dev[1], max_{t,e} |v[t*value_stride + e]|)
 * amax_dev holds non-negative fp32 values (zero it to start a new maximum).
 * Row strides are honoured (padding between rows is not read).  Stream
 * ordered; the host is not synchronized.
 *
 *   k, v, key_stride, value_stride, num_tokens, num_kv_heads, head_dim:
 *                as for fp8_kv_write
 *   amax_dev     device fp32 [2], 8-byte aligned
 * Returns FP8Q_OK, FP8Q_EINVAL, FP8Q_ECUDA.
 */
FP8Q_API fp8q_status fp8_kv_amax_observe(const void *k, const void *v,
                                         int64_t key_stride,
                                         int64_t value_stride,
                                         int64_t num_tokens,
                                         int32_t num_kv_heads,
                                         int32_t head_dim, float *amax_dev,
                                         void *stream);

/* Opaque per-layer calibrator (host memory, owned by the library). */
typedef struct fp8_kv_calib fp8_kv_calib;

/* Size of the fixed device scratch array behind fp8_kv_calib_window_noalloc. */
#define FP8Q_NOALLOC_SCRATCH_BYTES (1 << 20)

/* Step reported by an observe. */
#define FP8Q_STEP_STAGE 1           /* in the window, batch staged           */
#define FP8Q_STEP_STAGE_DECLINED 2  /* in the window, staging declined it    */
#define FP8Q_STEP_FREEZE 3          /* this batch reached the window         */
#define FP8Q_STEP_FROZEN 4          /* after the freeze                      */

/* Bytes of device memory the calibrator needs: state_dev and, per staged
 * token, a bf16 K row, a bf16 V row and an int64 slot. */
#define FP8Q_CALIB_STATE_BYTES 16

/*
 * fp8_kv_calib_create -- build the calibrator of one attention layer.
 *
 * Source: "metrale_model_layers/layers/fp8_calibration.rs",
 * Fp8KvCalibration::new (headroom below 1.0 is clamped to 1.0; the window is
 * clamped to MAX_STAGED_TOKENS; a window of 1 freezes on the first observe
 * and stages nothing; no calibrator exists for a window of 0) and module doc;
 * "spark_model/layers/fp8_calibration/staging.rs", module doc (the staging
 * cost is window * num_kv_heads * head_dim * 2 bytes * 2 per layer) and
 * KvStaging::stage.
 *
 *   window_tokens   requested window, >= 1 (clamped to FP8Q_MAX_STAGED_TOKENS)
 *   headroom        multiplier of the frozen amax; < 1 or NaN becomes 1
 *   num_kv_heads,
 *   head_dim        the row shape staging is laid out for (E = product,
 *                   a multiple of 8)
 *   stage_k,
 *   stage_v         device bf16 [stage_capacity_tokens, E] each, 16-byte
 *                   aligned; may be NULL when stage_capacity_tokens is 0
 *   stage_slots     device int64 [stage_capacity_tokens]
 *   stage_capacity_tokens
 *                   rows of staging provided; the effective capacity is
 *                   min(this, clamped window).  Batches that do not fit are
 *                   declined: written at the provisional scale and never
 *                   rewritten.  Pass the clamped window to stage everything.
 *   state_dev       device, FP8Q_CALIB_STATE_BYTES bytes, 16-byte aligned:
 *                   {k_amax, v_amax, k_scale, v_scale} fp32; the create call
 *                   enqueues its initialisation {0, 0, 2.0, 2.0} on `stream`.
 *                   While calibrating, [2..3] hold the provisional scale; the
 *                   freeze replaces them; pass state_dev + 2 as the scale_dev
 *                   of fp8_kv_write (see fp8_kv_calib_scale_dev).
 *   out             receives the handle
 * All device buffers stay owned by the caller and must outlive the handle
 * (staging may be released once the freeze has been replayed).
 * Returns FP8Q_OK, FP8Q_EINVAL, FP8Q_ENOMEM, FP8Q_ECUDA.
 */
FP8Q_API fp8q_status fp8_kv_calib_create(int64_t window_tokens, float headroom,
                                         int32_t num_kv_heads, int32_t head_dim,
                                         void *stage_k, void *stage_v,
                                         int64_t *stage_slots,
                                         int64_t stage_capacity_tokens,
                                         float *state_dev, void *stream,
                                         fp8_kv_calib **out);

/*
 * fp8_kv_calib_observe -- fold one batch into the window.
 *
 * Source: "metrale_model_layers/layers/fp8_calibration.rs",
 * Fp8KvCalibration::observe and module doc; "spark_model/layers/
 * fp8_calibration/staging.rs", KvStaging::stage.
 *
 * Before the freeze: adds num_tokens to the running count and max-accumulates
 * |K|, |V| into state_dev on the device.  If the count stays below the window
 * the batch's rows (strided -> packed) and slots are copied into staging at
 * the next free row (FP8Q_STEP_STAGE), or declined when the row shape
 * differs from the handle's or the rows do not fit
 * (FP8Q_STEP_STAGE_DECLINED).  Either way the caller then writes the batch
 * with fp8_kv_write at the provisional scale (scale_dev = state_dev + 2).
 * If the count reaches the window the step is FP8Q_STEP_FREEZE and nothing
 * is staged: the caller must call fp8_kv_freeze_replay next, then write the
 * batch at the frozen scale.  After the freeze: FP8Q_STEP_FROZEN, no device
 * work.  The decision uses only token counts, so the host never waits for
 * the device.
 *
 *   k, v, key_stride, value_stride, slot_mapping, num_tokens,
 *   num_kv_heads, head_dim   the batch, as for fp8_kv_write
 *   step_out                 receives FP8Q_STEP_*
 * Returns FP8Q_OK, FP8Q_EINVAL, FP8Q_ESTATE (a freeze is pending: call
 * fp8_kv_freeze_replay first), FP8Q_ECUDA.
 */
FP8Q_API fp8q_status fp8_kv_calib_observe(fp8_kv_calib *calib, const void *k,
                                          const void *v, int64_t key_stride,
                                          int64_t value_stride,
                                          const int64_t *slot_mapping,
                                          int64_t num_tokens,
                                          int32_t num_kv_heads,
                                          int32_t head_dim, void *stream,
                                          int32_t *step_out);

/*
 * fp8_kv_freeze_replay -- freeze the scales and rewrite the window.
 *
 * Source: "metrale_model_layers/layers/fp8_calibration.rs", module doc
 * (scale = amax * headroom / 448 over every token observed up to and
 * including the batch that reached the window) and observe (the Freeze arm);
 * "spark_model/layers/fp8_calibration/staging.rs", module doc (replay is
 * chronological, so the last writer of each slot is the original one even
 * when a block was freed and re-allocated inside the window; the crossing
 * batch is written by the caller afterwards) and
 * KvStaging::replay_and_release.
 *
 * On the device: k_scale = max(k_amax * headroom, 1e-12f) / 448.0f (the
 * product rounded to fp32 first), likewise v_scale, stored in state_dev[2..3];
 * then each staged batch, in the order it was staged, is written with
 * reshape_and_cache_fp8 semantics from the packed staging rows at those
 * scales into the given pools.  Staging is then empty and may be released.
 *
 *   k_pool, v_pool, block_size, cache_stride, num_blocks
 *                      the layer's pools, as for fp8_kv_write
 *   replayed_tokens    optional; receives the number of tokens rewritten
 * Returns FP8Q_OK, FP8Q_EINVAL, FP8Q_ESTATE (no freeze pending), FP8Q_ECUDA.
 */
FP8Q_API fp8q_status fp8_kv_freeze_replay(fp8_kv_calib *calib, void *k_pool,
                                          void *v_pool, int32_t block_size,
                                          int64_t cache_stride,
                                          int64_t num_blocks, void *stream,
                                          int64_t *replayed_tokens);

/*
 * fp8_kv_calib_observe_write -- observe and write in the fewest passes.
 *
 * The same contract as fp8_kv_calib_observe followed by the caller's
 * fp8_kv_write at the scales the step calls for (and, on FP8Q_STEP_FREEZE,
 * fp8_kv_freeze_replay in between), with identical results.  In the window
 * the absmax, the staging copy and the provisional-scale write share one
 * read of K and V; on the freeze the absmax comes first, then the replay,
 * whose last launch also writes the crossing batch when it fits (a crossing
 * batch above 8192 tokens gets a launch of its own after it); after the
 * freeze, one write.
 * Returns as fp8_kv_calib_observe and fp8_kv_freeze_replay.
 */
FP8Q_API fp8q_status fp8_kv_calib_observe_write(
    fp8_kv_calib *calib, const void *k, const void *v, int64_t key_stride,
    int64_t value_stride, const int64_t *slot_mapping, int64_t num_tokens,
    int32_t num_kv_heads, int32_t head_dim, void *k_pool, void *v_pool,
    int32_t block_size, int64_t cache_stride, int64_t num_blocks, void *stream,
    int32_t *step_out);

/*
 * fp8_kv_calib_restore -- start a calibrator frozen at saved scales.
 *
 * The pages keep the calibration state in memory only.  A server that
 * restarts would otherwise calibrate every layer again (and keep CUDA graphs
 * suppressed for the whole window).  A calibrator that has observed nothing
 * yet can instead be frozen at scales saved earlier, e.g. read with
 * fp8_kv_calib_read_state after a previous freeze: the call enqueues
 * state_dev = {k_scale, v_scale, k_scale, v_scale} (the saved scales also
 * stand in as the maxima) and every later observe is FP8Q_STEP_FROZEN.
 *
 *   k_scale, v_scale  finite and > 0
 * Returns FP8Q_OK, FP8Q_EINVAL, FP8Q_ESTATE (the calibrator has already
 * observed a batch), FP8Q_ECUDA.
 */
FP8Q_API fp8q_status fp8_kv_calib_restore(fp8_kv_calib *calib, float k_scale,
                                          float v_scale, void *stream);

/* Device pointer to {k_scale, v_scale} of the calibrator (state_dev + 2):
 * the provisional scale until the freeze, the frozen scales after it. */
FP8Q_API const float *fp8_kv_calib_scale_dev(const fp8_kv_calib *calib);

/* Host-side counters of the calibrator; the fields of the freeze log
 * ("metrale_model_layers/layers/fp8_calibration.rs", observe, Freeze arm),
 * without the device-resident values (read those with
 * fp8_kv_calib_read_state). */
typedef struct fp8_kv_calib_stats {
    int64_t requested_tokens;  /* window asked for                          */
    int64_t window_tokens;     /* after the MAX_STAGED_TOKENS clamp         */
    int64_t capacity_tokens;   /* effective staging capacity                */
    int64_t tokens_seen;       /* tokens observed (after the freeze too)    */
    int64_t staged_tokens;     /* rows currently staged                     */
    int64_t staged_batches;    /* STAGE steps (staged or declined)          */
    int64_t unstaged_tokens;   /* tokens of declined batches                */
    int64_t freeze_tokens;     /* tokens_seen at the freeze, 0 before it    */
    int64_t replayed_tokens;   /* tokens rewritten by the replay            */
    int64_t replayed_batches;  /* batches rewritten by the replay           */
    float headroom;            /* after the clamp                           */
    int32_t state;             /* 0 calibrating, 1 freeze pending, 2 frozen */
} fp8_kv_calib_stats;

FP8Q_API fp8q_status fp8_kv_calib_stats_get(const fp8_kv_calib *calib,
                                            fp8_kv_calib_stats *out);

/* Synchronizes `stream` and copies state_dev to out[4] = {k_amax, v_amax,
 * k_scale, v_scale}.  SYNCHRONIZING; for logs and tests, not the hot path. */
FP8Q_API fp8q_status fp8_kv_calib_read_state(const fp8_kv_calib *calib,
                                             void *stream, float *out);

/* Frees the host handle (no device memory is owned). NULL is ignored. */
FP8Q_API void fp8_kv_calib_destroy(fp8_kv_calib *calib);

/*
 * fp8_kv_calib_window_noalloc -- one layer's calibration window in one call,
 * for callers that cannot allocate device memory.
 *
 * The source pages have no counterpart of this call: their calibrator
 * allocates its staging on first use.  Some callers cannot do that -- an
 * engine that gives all device memory to its KV pool at start-up and
 * forbids later cudaMalloc, code that must not risk the device-wide
 * synchronization an allocation or free can cause, a host that gives the
 * library no allocator.  This call needs no device memory from anyone: its
 * scratch (the window's staged bf16 K/V rows and slots, and the 16-byte
 * calibration state) is a fixed array of FP8Q_NOALLOC_SCRATCH_BYTES inside
 * the library, which every device that loads the library holds until the
 * process exits.  The call allocates nothing, host or device.
 *
 * Result: exactly what a calibrator made by fp8_kv_calib_create(window_tokens,
 * headroom, ...) with staging for the whole window produces when it is fed
 * the batches in order through fp8_kv_calib_observe_write: batches before the
 * one that reaches the window are written at the provisional scale (and
 * staged), that batch's arrival freezes the scales and replays the staged
 * batches in order, and it and every later batch are written at the frozen
 * scales.  If the batches end before the window is reached nothing is frozen
 * or replayed (the staging does not outlive the call).
 *
 *   k, v, key_stride, value_stride, slot_mapping
 *                  all batches' rows, one after another (batch b starts at
 *                  the row after batch b-1's last), as for fp8_kv_write
 *   batch_tokens   HOST int64 [num_batches], tokens of each batch (>= 0)
 *   num_batches    >= 0
 *   num_kv_heads, head_dim, window_tokens, headroom
 *                  as for fp8_kv_calib_create (clamps included)
 *   k_pool, v_pool, block_size, cache_stride, num_blocks
 *                  the layer's pools, as for fp8_kv_write
 *   scales_out     optional device fp32 [2]: receives {k_scale, v_scale}
 *                  after the last batch (2.0 if the window was not reached)
 * Limit: the rows staged before the freeze need staged * (4 * E + 8) bytes,
 * E = num_kv_heads * head_dim; more than FP8Q_NOALLOC_SCRATCH_BYTES - 256
 * returns FP8Q_ETOOBIG before anything is enqueued.  At most window - 1 rows
 * are ever staged, so with 4 x 128 rows every window of up to 510 tokens fits.
 * Sharing: every call uses the same array and leaves its contents there;
 * the call initialises what must start from zero.  Calls whose work overlaps
 * on the GPU (two streams, two threads) race on the array: serialize them.
 * Set-up: the first call on each device looks up the array's device address
 * (with that device current) and caches it; make that first call before any
 * stream capture.
 * Returns FP8Q_OK, FP8Q_EINVAL, FP8Q_ETOOBIG, FP8Q_ECUDA.
 */
FP8Q_API fp8q_status fp8_kv_calib_window_noalloc(
    const void *k, const void *v, int64_t key_stride, int64_t value_stride,
    const int64_t *slot_mapping, const int64_t *batch_tokens, int32_t num_batches,
    int32_t num_kv_heads, int32_t head_dim, int64_t window_tokens, float headroom,
    void *k_pool, void *v_pool, int32_t block_size, int64_t cache_stride,
    int64_t num_blocks, float *scales_out, void *stream);

/*
 * fp8_kv_graphs_ready -- whether CUDA graphs may be captured again.
 *
 * Source: "metrale_model_layers/layers/fp8_calibration.rs",
 * graphs_ready_after_fp8_kv_cal.  states[i] per layer: -1 no calibrator,
 * 0 still inside the window, 1 frozen.  Returns 1 when no layer is inside
 * its window (also for n == 0), else 0; -1 if states is NULL with n > 0.
 */
FP8Q_API int32_t fp8_kv_graphs_ready(const int8_t *states, int64_t n);

/* ------------------------------------------------------------------------ */
/* Diagnostics                                                              */
/* ------------------------------------------------------------------------ */

/* Reads (and with clear != 0 resets) the sticky error word of the current
 * device.  SYNCHRONIZING: waits for all work on the device first. */
FP8Q_API fp8q_status fp8q_device_error(uint32_t *bits_out, int32_t clear);

/* Static description of a status code. */
FP8Q_API const char *fp8q_status_string(fp8q_status status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
FP8Q_API int32_t fp8q_version(void);

/* Number of kernels this library has enqueued in this process (every
 * successful launch, including ones recorded into a CUDA graph capture). */
FP8Q_API int64_t fp8q_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8Q_H */
