// Internal interface between the C ABI (fp8q_api.cpp) and the kernels
// (fp8q_kernels.cu).  Not installed; the public surface is include/fp8q.h.
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

namespace fp8q {

// One pass of the KV kernel over a batch of tokens.  Which of the three jobs
// it does is chosen by the flags; every job reads each K/V row once.
//   amax   max-accumulate |K|, |V| (fp32 bit patterns) into amax_bits[0..1]
//   stage  copy the rows, packed, to stage_k/stage_v at row stage_offset + t,
//          and the slot to stage_slots[stage_offset + t]
//   write  quantize the rows and scatter them into the pools
struct KvPass {
    const uint16_t *k = nullptr;
    const uint16_t *v = nullptr;
    int64_t key_stride = 0;
    int64_t value_stride = 0;
    const int64_t *slot_mapping = nullptr;
    int64_t num_tokens = 0;
    int32_t elems = 0;  // num_kv_heads * head_dim, a multiple of 8

    // write
    uint8_t *k_pool = nullptr;
    uint8_t *v_pool = nullptr;
    int32_t block_size = 0;
    int32_t block_shift = -1;   // log2(block_size) when it is a power of two
    int64_t cache_stride = 0;
    int64_t num_slots = 0;
    // Scale source, first match wins:
    //   freeze_amax != null: scale = max(amax*headroom, 1e-12)/448 from the
    //                        accumulated maxima; block 0 stores it to scale_out
    //   scale_dev   != null: {k_scale, v_scale} read from device memory
    //   otherwise           k_scale / v_scale by value
    const uint32_t *freeze_amax = nullptr;
    float headroom = 1.0f;
    float *scale_out = nullptr;
    const float *scale_dev = nullptr;
    float k_scale = 1.0f;
    float v_scale = 1.0f;

    // Crossing batch written by the same launch after a replayed staged
    // batch (write passes only): tokens [num_tokens, num_tokens + x_tokens)
    // come from xk / xv / x_slots.  A staged token whose slot the crossing
    // batch also writes is skipped, so the crossing token is the last writer,
    // as if the two had been written by two launches in that order.
    const uint16_t *xk = nullptr;
    const uint16_t *xv = nullptr;
    int64_t x_key_stride = 0;
    int64_t x_value_stride = 0;
    const int64_t *x_slots = nullptr;
    int64_t x_tokens = 0;

    // amax
    uint32_t *amax_bits = nullptr;

    // stage
    uint16_t *stage_k = nullptr;
    uint16_t *stage_v = nullptr;
    int64_t *stage_slots = nullptr;
    int64_t stage_offset = 0;

    bool do_amax = false;
    bool do_stage = false;
    bool do_write = false;
    // The launch directly before this one on the stream is a kernel of this
    // library, and nothing this pass reads (rows, slots, crossing slots) is
    // written by it.  Every kernel here passes its dependency wait before it
    // lets its dependents start, so everything enqueued before that kernel has
    // completed by the time this pass starts: the pass may then load its rows
    // and build its crossing-slot table before its own wait.  Only scales
    // produced by the previous kernel and the stores wait.  Set only where a
    // call enqueues that whole chain itself.
    bool early_loads = false;
    // Replay of a whole window in one launch: rows [0, num_tokens) are every
    // staged batch in arrival order and the crossing rows follow; a row is
    // written only if no later row of the launch has the same slot.  Needs
    // num_tokens + x_tokens <= kMaxLastWriterTokens.
    bool last_writer = false;
};

// Several layers' writes in one launch (fp8_kv_write_layers): row strides,
// shapes and pool geometry are shared, pointers and scales are per layer.
constexpr int kMaxLayers = 128;

struct KvLayer {
    const uint16_t *k;
    const uint16_t *v;
    const int64_t *slot_mapping;
    uint8_t *k_pool;
    uint8_t *v_pool;
    const float *scale_dev;   // {k_scale, v_scale} on the device, or null
    float k_scale;
    float v_scale;
};

struct KvLayers {
    int64_t key_stride = 0;
    int64_t value_stride = 0;
    int64_t num_tokens = 0;
    int32_t elems = 0;
    int32_t block_size = 0;
    int32_t block_shift = -1;
    int32_t num_layers = 0;
    int64_t cache_stride = 0;
    int64_t num_slots = 0;
    KvLayer layer[kMaxLayers];
};

cudaError_t launch_kv_write_layers(const KvLayers &p, cudaStream_t stream);

cudaError_t launch_group_quant(const uint16_t *x, int64_t x_row_stride, uint8_t *q,
                               float *scales, int64_t m, int64_t k, cudaStream_t stream);

// Launches one KV pass.  A pass with no tokens still launches when it must
// publish a frozen scale (freeze_amax and scale_out set).
cudaError_t launch_kv_pass(const KvPass &p, cudaStream_t stream);

// Largest crossing batch a single launch can merge with a replay (its slots
// go into a hash set in shared memory); larger ones use two launches.
constexpr int64_t kMaxMergedCrossing = 8192;
constexpr int64_t kMaxLastWriterTokens = 2048;
bool can_merge_crossing(const KvPass &p);

// The device work of a freeze: every staged batch (packed rows in arrival
// order, counts[i] rows for batch i, at stage_k / stage_v / stage_slots) is
// rewritten at the scales frozen from the device maxima, the first launch also
// publishing them; then `crossing` (the batch that reached the window, a
// write pass that reads the published scales), if given.  When the window is
// small enough, every staged row and the crossing batch share one launch that
// writes each slot only from its last writer; otherwise the batches replay one
// launch each in arrival order, the last one sharing its launch with the
// crossing batch when that fits.  Either way each slot ends with its last
// writer in arrival order.  `base` carries the pools, their geometry,
// freeze_amax, headroom and scale_out.  `chained`: the launch before this
// sequence on the stream is a kernel of this library enqueued by the same
// call (see KvPass::early_loads).  Used by the calibrator and by the
// allocation-free window call, so both issue the same launches.
cudaError_t enqueue_freeze_replay(const KvPass &base, const uint16_t *stage_k,
                                  const uint16_t *stage_v, const int64_t *stage_slots,
                                  const int64_t *counts, int64_t num_batches,
                                  const KvPass *crossing, bool chained, cudaStream_t stream,
                                  int64_t *rewritten);

// Group quantization with phantom rows m..m_pad-1 zeroed and the scales
// written K-major, scales_km[g * m_pad + r].
cudaError_t launch_group_quant_kmajor(const uint16_t *x, int64_t x_row_stride, uint8_t *q,
                                      float *scales_km, int64_t m, int64_t m_pad, int64_t k,
                                      cudaStream_t stream);

// Enqueues state_dev = {0, 0, 2.0, 2.0} (bit patterns of the fp32 values).
cudaError_t launch_calib_init(float *state_dev, cudaStream_t stream);

// Enqueues state_dev = {a, b, c, d}.
cudaError_t launch_calib_set(float *state_dev, float a, float b, float c, float d,
                             cudaStream_t stream);

// Number of kernels this library has launched in this process.
int64_t launch_count();

// Sticky device error word of the current device.
cudaError_t read_device_error(uint32_t *bits, bool clear);

}  // namespace fp8q
