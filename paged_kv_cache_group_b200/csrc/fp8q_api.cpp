// fp8q_api.cpp -- the C ABI of include/fp8q.h: argument checks, the
// calibrator's host state machine, and dispatch to the kernels.
//
// The calibrator follows "metrale_model_layers/layers/fp8_calibration.rs"
// (Fp8KvCalibration::new / observe) and "spark_model/layers/fp8_calibration/
// staging.rs" (KvStaging::stage / replay_and_release), with one structural
// change for the GPU: the running maxima and the frozen scales live in device
// memory (state_dev) and are never read back on the hot path.  The freeze
// decision needs only token counts, which the host has, so an observe never
// waits for the device; the scale is computed by the replay kernel from the
// device maxima.
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <new>
#include <vector>

#include <cuda_runtime.h>

#include "fp8q.h"
#include "fp8q_internal.h"

namespace {

using fp8q::KvPass;

constexpr int32_t kVersion = 10100;  // 1.1.0: fp8_group_quant_kmajor, fp8_kv_calib_restore

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

fp8q_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FP8Q_OK : FP8Q_ECUDA; }

cudaStream_t as_stream(void *s) { return static_cast<cudaStream_t>(s); }

// Shape and alignment of a batch of K/V rows (shared by write, amax, observe).
bool valid_rows(const void *k, const void *v, int64_t key_stride, int64_t value_stride,
                int64_t num_tokens, int32_t num_kv_heads, int32_t head_dim, int64_t *elems) {
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0) return false;
    const int64_t e = static_cast<int64_t>(num_kv_heads) * head_dim;
    if (e % 8 != 0 || e > (int64_t{1} << 30)) return false;
    if (key_stride < e || value_stride < e || key_stride % 8 || value_stride % 8) return false;
    if (num_tokens > 0) {
        if (k == nullptr || v == nullptr) return false;
        if (!aligned(k, 16) || !aligned(v, 16)) return false;
    }
    *elems = e;
    return true;
}

int32_t pow2_shift(int32_t v) {
    if (v <= 0 || (v & (v - 1)) != 0) return -1;
    int32_t s = 0;
    while ((1 << s) != v) ++s;
    return s;
}

bool valid_pools(const void *k_pool, const void *v_pool, int32_t block_size,
                 int64_t cache_stride, int64_t num_blocks, int64_t elems) {
    if (block_size <= 0 || num_blocks < 0) return false;
    if (cache_stride < static_cast<int64_t>(block_size) * elems || cache_stride % 8) return false;
    if (num_blocks > 0 && (k_pool == nullptr || v_pool == nullptr)) return false;
    if (!aligned(k_pool, 8) || !aligned(v_pool, 8)) return false;
    if (num_blocks > INT64_MAX / block_size) return false;
    return true;
}

}  // namespace

// ---------------------------------------------------------------------------
// calibrator

enum CalibPhase : int32_t { kCalibrating = 0, kFreezePending = 1, kFrozen = 2 };

struct fp8_kv_calib {
    int64_t requested_tokens = 0;
    int64_t window_tokens = 0;
    float headroom = 1.0f;
    int32_t num_kv_heads = 0;
    int32_t head_dim = 0;
    int64_t elems = 0;
    uint16_t *stage_k = nullptr;
    uint16_t *stage_v = nullptr;
    int64_t *stage_slots = nullptr;
    int64_t capacity_tokens = 0;
    float *state_dev = nullptr;   // {k_amax, v_amax, k_scale, v_scale}

    int32_t phase = kCalibrating;
    int64_t tokens_seen = 0;
    int64_t used_tokens = 0;
    int64_t staged_batches = 0;
    int64_t unstaged_tokens = 0;
    int64_t freeze_tokens = 0;
    int64_t replayed_tokens = 0;
    int64_t replayed_batches = 0;
    // rows of each staged batch, in arrival order (packed in staging)
    std::vector<int64_t> staged_counts;
};

namespace {

uint32_t *amax_bits(fp8_kv_calib *c) { return reinterpret_cast<uint32_t *>(c->state_dev); }
float *scale_dev(fp8_kv_calib *c) { return c->state_dev + 2; }

// Host half of an observe: counts tokens, decides the step and whether the
// batch is staged; fills the device pass (amax, and stage when staged).
fp8q_status plan_observe(fp8_kv_calib *c, const void *k, const void *v, int64_t key_stride,
                         int64_t value_stride, const int64_t *slot_mapping, int64_t num_tokens,
                         int32_t num_kv_heads, int32_t head_dim, KvPass *pass, int32_t *step) {
    int64_t elems = 0;
    if (!valid_rows(k, v, key_stride, value_stride, num_tokens, num_kv_heads, head_dim, &elems))
        return FP8Q_EINVAL;
    if (num_tokens > 0 && slot_mapping == nullptr) return FP8Q_EINVAL;
    if (c->phase == kFreezePending) return FP8Q_ESTATE;
    if (c->phase == kFrozen) {
        c->tokens_seen += num_tokens;
        *step = FP8Q_STEP_FROZEN;
        return FP8Q_OK;
    }
    pass->k = static_cast<const uint16_t *>(k);
    pass->v = static_cast<const uint16_t *>(v);
    pass->key_stride = key_stride;
    pass->value_stride = value_stride;
    pass->slot_mapping = slot_mapping;
    pass->num_tokens = num_tokens;
    pass->elems = static_cast<int32_t>(elems);
    pass->do_amax = true;
    pass->amax_bits = amax_bits(c);

    c->tokens_seen += num_tokens;
    if (c->tokens_seen >= c->window_tokens) {
        c->phase = kFreezePending;
        c->freeze_tokens = c->tokens_seen;
        *step = FP8Q_STEP_FREEZE;
        return FP8Q_OK;
    }
    c->staged_batches += 1;
    if (elems == c->elems && c->used_tokens + num_tokens <= c->capacity_tokens) {
        pass->do_stage = num_tokens > 0;
        pass->stage_k = c->stage_k;
        pass->stage_v = c->stage_v;
        pass->stage_slots = c->stage_slots;
        pass->stage_offset = c->used_tokens;
        c->staged_counts.push_back(num_tokens);
        c->used_tokens += num_tokens;
        *step = FP8Q_STEP_STAGE;
    } else {
        c->unstaged_tokens += num_tokens;
        *step = FP8Q_STEP_STAGE_DECLINED;
    }
    return FP8Q_OK;
}

// The freeze's device work (fp8q::enqueue_freeze_replay): every staged batch
// rewritten, in arrival order, at the scales frozen from the device maxima,
// the scales published to state_dev, then `crossing` (the batch that reached
// the window, as a write pass reading the published scales) if given.  Each
// slot ends with its last writer in arrival order.
fp8q_status run_replay(fp8_kv_calib *c, void *k_pool, void *v_pool, int32_t block_size,
                       int64_t cache_stride, int64_t num_blocks, cudaStream_t stream,
                       int64_t *replayed, const KvPass *crossing, bool chained = false) {
    if (c->phase != kFreezePending) return FP8Q_ESTATE;
    if (!valid_pools(k_pool, v_pool, block_size, cache_stride, num_blocks, c->elems))
        return FP8Q_EINVAL;
    KvPass p;
    p.do_write = true;
    p.elems = static_cast<int32_t>(c->elems);
    p.k_pool = static_cast<uint8_t *>(k_pool);
    p.v_pool = static_cast<uint8_t *>(v_pool);
    p.block_size = block_size;
    p.block_shift = pow2_shift(block_size);
    p.cache_stride = cache_stride;
    p.num_slots = num_blocks * block_size;
    p.freeze_amax = amax_bits(c);
    p.headroom = c->headroom;
    p.scale_out = scale_dev(c);
    int64_t rewritten = 0;
    // chained: the previous launch on the stream is this call's own amax pass;
    // the staged rows and the crossing batch were all written before it.
    const cudaError_t e = fp8q::enqueue_freeze_replay(
        p, c->stage_k, c->stage_v, c->stage_slots, c->staged_counts.data(),
        static_cast<int64_t>(c->staged_counts.size()), crossing, chained, stream, &rewritten);
    if (e != cudaSuccess) return FP8Q_ECUDA;
    c->replayed_tokens = rewritten;
    c->replayed_batches = static_cast<int64_t>(c->staged_counts.size());
    c->staged_counts.clear();
    c->used_tokens = 0;
    c->phase = kFrozen;
    if (replayed) *replayed = rewritten;
    return FP8Q_OK;
}

KvPass write_pass(const void *k, const void *v, int64_t key_stride, int64_t value_stride,
                  const int64_t *slot_mapping, int64_t num_tokens, int64_t elems, void *k_pool,
                  void *v_pool, int32_t block_size, int64_t cache_stride, int64_t num_blocks) {
    KvPass p;
    p.k = static_cast<const uint16_t *>(k);
    p.v = static_cast<const uint16_t *>(v);
    p.key_stride = key_stride;
    p.value_stride = value_stride;
    p.slot_mapping = slot_mapping;
    p.num_tokens = num_tokens;
    p.elems = static_cast<int32_t>(elems);
    p.k_pool = static_cast<uint8_t *>(k_pool);
    p.v_pool = static_cast<uint8_t *>(v_pool);
    p.block_size = block_size;
    p.block_shift = pow2_shift(block_size);
    p.cache_stride = cache_stride;
    p.num_slots = num_blocks * block_size;
    p.do_write = true;
    return p;
}

}  // namespace

extern "C" {

FP8Q_API fp8q_status fp8_group_quant(const void *x, int64_t x_row_stride, void *q, float *scales,
                                     int64_t m, int64_t k, void *stream) {
    if (m < 0 || k <= 0 || k % FP8Q_GROUP != 0) return FP8Q_EINVAL;
    if (x_row_stride < k || x_row_stride % 8 != 0) return FP8Q_EINVAL;
    if (m == 0) return FP8Q_OK;
    if (x == nullptr || q == nullptr || scales == nullptr) return FP8Q_EINVAL;
    if (!aligned(x, 16) || !aligned(q, 8) || !aligned(scales, 4)) return FP8Q_EINVAL;
    if (m > INT64_MAX / k) return FP8Q_EINVAL;
    return from_cuda(fp8q::launch_group_quant(static_cast<const uint16_t *>(x), x_row_stride,
                                              static_cast<uint8_t *>(q), scales, m, k,
                                              as_stream(stream)));
}

FP8Q_API fp8q_status fp8_group_quant_kmajor(const void *x, int64_t x_row_stride, void *q,
                                            float *scales_km, int64_t m, int64_t m_pad,
                                            int64_t k, void *stream) {
    if (m < 0 || m_pad < m || k <= 0 || k % FP8Q_GROUP != 0) return FP8Q_EINVAL;
    if (x_row_stride < k || x_row_stride % 8 != 0) return FP8Q_EINVAL;
    if (m_pad == 0) return FP8Q_OK;
    if (q == nullptr || scales_km == nullptr || (m > 0 && x == nullptr)) return FP8Q_EINVAL;
    if (!aligned(x, 16) || !aligned(q, 8) || !aligned(scales_km, 4)) return FP8Q_EINVAL;
    if (m_pad > INT64_MAX / x_row_stride || k / FP8Q_GROUP > 0xFFFFFFFF) return FP8Q_EINVAL;
    return from_cuda(fp8q::launch_group_quant_kmajor(
        static_cast<const uint16_t *>(x), x_row_stride, static_cast<uint8_t *>(q), scales_km, m,
        m_pad, k, as_stream(stream)));
}

FP8Q_API fp8q_status fp8_kv_write(const void *k, const void *v, int64_t key_stride,
                                  int64_t value_stride, const int64_t *slot_mapping,
                                  int64_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                                  void *k_pool, void *v_pool, int32_t block_size,
                                  int64_t cache_stride, int64_t num_blocks, float k_scale,
                                  float v_scale, const float *scale_dev_ptr, void *stream) {
    int64_t elems = 0;
    if (!valid_rows(k, v, key_stride, value_stride, num_tokens, num_kv_heads, head_dim, &elems))
        return FP8Q_EINVAL;
    if (!valid_pools(k_pool, v_pool, block_size, cache_stride, num_blocks, elems))
        return FP8Q_EINVAL;
    if (scale_dev_ptr == nullptr) {
        if (!(k_scale > 0.0f) || !(v_scale > 0.0f) || std::isinf(k_scale) || std::isinf(v_scale))
            return FP8Q_EINVAL;
    } else if (!aligned(scale_dev_ptr, 8)) {
        return FP8Q_EINVAL;
    }
    if (num_tokens == 0) return FP8Q_OK;
    if (slot_mapping == nullptr || !aligned(slot_mapping, 8)) return FP8Q_EINVAL;
    KvPass p = write_pass(k, v, key_stride, value_stride, slot_mapping, num_tokens, elems, k_pool,
                          v_pool, block_size, cache_stride, num_blocks);
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.scale_dev = scale_dev_ptr;
    return from_cuda(fp8q::launch_kv_pass(p, as_stream(stream)));
}

FP8Q_API fp8q_status fp8_kv_write_layers(const fp8q_kv_layer *layers, int32_t num_layers,
                                         int64_t key_stride, int64_t value_stride,
                                         int64_t num_tokens, int32_t num_kv_heads,
                                         int32_t head_dim, int32_t block_size,
                                         int64_t cache_stride, int64_t num_blocks, void *stream) {
    if (num_layers < 0 || num_layers > FP8Q_MAX_LAYERS) return FP8Q_EINVAL;
    if (num_layers > 0 && layers == nullptr) return FP8Q_EINVAL;
    int64_t elems = 0;
    // shapes are checked once; pointers per layer
    if (!valid_rows(nullptr, nullptr, key_stride, value_stride, 0, num_kv_heads, head_dim, &elems))
        return FP8Q_EINVAL;
    if (num_tokens < 0) return FP8Q_EINVAL;
    static_assert(FP8Q_MAX_LAYERS == fp8q::kMaxLayers, "layer limit");
    fp8q::KvLayers L;
    for (int32_t i = 0; i < num_layers; ++i) {
        const fp8q_kv_layer &a = layers[i];
        int64_t e = 0;
        if (!valid_rows(a.k, a.v, key_stride, value_stride, num_tokens, num_kv_heads, head_dim, &e))
            return FP8Q_EINVAL;
        if (!valid_pools(a.k_pool, a.v_pool, block_size, cache_stride, num_blocks, elems))
            return FP8Q_EINVAL;
        if (num_tokens > 0 && (a.slot_mapping == nullptr || !aligned(a.slot_mapping, 8)))
            return FP8Q_EINVAL;
        if (a.scale_dev == nullptr) {
            if (!(a.k_scale > 0.0f) || !(a.v_scale > 0.0f) || std::isinf(a.k_scale) ||
                std::isinf(a.v_scale))
                return FP8Q_EINVAL;
        } else if (!aligned(a.scale_dev, 8)) {
            return FP8Q_EINVAL;
        }
        fp8q::KvLayer &d = L.layer[i];
        d.k = static_cast<const uint16_t *>(a.k);
        d.v = static_cast<const uint16_t *>(a.v);
        d.slot_mapping = a.slot_mapping;
        d.k_pool = static_cast<uint8_t *>(a.k_pool);
        d.v_pool = static_cast<uint8_t *>(a.v_pool);
        d.scale_dev = a.scale_dev;
        d.k_scale = a.k_scale;
        d.v_scale = a.v_scale;
    }
    if (num_tokens == 0 || num_layers == 0) return FP8Q_OK;
    L.key_stride = key_stride;
    L.value_stride = value_stride;
    L.num_tokens = num_tokens;
    L.elems = static_cast<int32_t>(elems);
    L.block_size = block_size;
    L.block_shift = pow2_shift(block_size);
    L.num_layers = num_layers;
    L.cache_stride = cache_stride;
    L.num_slots = num_blocks * block_size;
    return from_cuda(fp8q::launch_kv_write_layers(L, as_stream(stream)));
}

FP8Q_API fp8q_status fp8_kv_amax_observe(const void *k, const void *v, int64_t key_stride,
                                         int64_t value_stride, int64_t num_tokens,
                                         int32_t num_kv_heads, int32_t head_dim, float *amax_dev,
                                         void *stream) {
    int64_t elems = 0;
    if (!valid_rows(k, v, key_stride, value_stride, num_tokens, num_kv_heads, head_dim, &elems))
        return FP8Q_EINVAL;
    if (amax_dev == nullptr || !aligned(amax_dev, 8)) return FP8Q_EINVAL;
    if (num_tokens == 0) return FP8Q_OK;
    KvPass p;
    p.k = static_cast<const uint16_t *>(k);
    p.v = static_cast<const uint16_t *>(v);
    p.key_stride = key_stride;
    p.value_stride = value_stride;
    p.num_tokens = num_tokens;
    p.elems = static_cast<int32_t>(elems);
    p.do_amax = true;
    p.amax_bits = reinterpret_cast<uint32_t *>(amax_dev);
    return from_cuda(fp8q::launch_kv_pass(p, as_stream(stream)));
}

FP8Q_API fp8q_status fp8_kv_calib_create(int64_t window_tokens, float headroom,
                                         int32_t num_kv_heads, int32_t head_dim, void *stage_k,
                                         void *stage_v, int64_t *stage_slots,
                                         int64_t stage_capacity_tokens, float *state_dev,
                                         void *stream, fp8_kv_calib **out) {
    if (out == nullptr) return FP8Q_EINVAL;
    *out = nullptr;
    if (window_tokens <= 0 || num_kv_heads <= 0 || head_dim <= 0) return FP8Q_EINVAL;
    const int64_t elems = static_cast<int64_t>(num_kv_heads) * head_dim;
    if (elems % 8 != 0 || elems > (int64_t{1} << 30)) return FP8Q_EINVAL;
    if (stage_capacity_tokens < 0) return FP8Q_EINVAL;
    if (stage_capacity_tokens > 0) {
        if (stage_k == nullptr || stage_v == nullptr || stage_slots == nullptr) return FP8Q_EINVAL;
        if (!aligned(stage_k, 16) || !aligned(stage_v, 16) || !aligned(stage_slots, 8))
            return FP8Q_EINVAL;
    }
    if (state_dev == nullptr || !aligned(state_dev, 16)) return FP8Q_EINVAL;

    fp8_kv_calib *c = new (std::nothrow) fp8_kv_calib();
    if (c == nullptr) return FP8Q_ENOMEM;
    c->requested_tokens = window_tokens;
    c->window_tokens = window_tokens < FP8Q_MAX_STAGED_TOKENS ? window_tokens
                                                              : FP8Q_MAX_STAGED_TOKENS;
    c->headroom = headroom >= 1.0f ? headroom : 1.0f;   // NaN -> 1.0 as well
    c->num_kv_heads = num_kv_heads;
    c->head_dim = head_dim;
    c->elems = elems;
    c->stage_k = static_cast<uint16_t *>(stage_k);
    c->stage_v = static_cast<uint16_t *>(stage_v);
    c->stage_slots = stage_slots;
    c->capacity_tokens = stage_capacity_tokens < c->window_tokens ? stage_capacity_tokens
                                                                  : c->window_tokens;
    c->state_dev = state_dev;
    cudaError_t e = fp8q::launch_calib_init(state_dev, as_stream(stream));
    if (e != cudaSuccess) {
        delete c;
        return FP8Q_ECUDA;
    }
    *out = c;
    return FP8Q_OK;
}

FP8Q_API fp8q_status fp8_kv_calib_observe(fp8_kv_calib *calib, const void *k, const void *v,
                                          int64_t key_stride, int64_t value_stride,
                                          const int64_t *slot_mapping, int64_t num_tokens,
                                          int32_t num_kv_heads, int32_t head_dim, void *stream,
                                          int32_t *step_out) {
    if (calib == nullptr || step_out == nullptr) return FP8Q_EINVAL;
    KvPass p;
    int32_t step = 0;
    fp8q_status st = plan_observe(calib, k, v, key_stride, value_stride, slot_mapping, num_tokens,
                                  num_kv_heads, head_dim, &p, &step);
    if (st != FP8Q_OK) return st;
    *step_out = step;
    if (step == FP8Q_STEP_FROZEN) return FP8Q_OK;
    return from_cuda(fp8q::launch_kv_pass(p, as_stream(stream)));
}

FP8Q_API fp8q_status fp8_kv_freeze_replay(fp8_kv_calib *calib, void *k_pool, void *v_pool,
                                          int32_t block_size, int64_t cache_stride,
                                          int64_t num_blocks, void *stream,
                                          int64_t *replayed_tokens) {
    if (calib == nullptr) return FP8Q_EINVAL;
    return run_replay(calib, k_pool, v_pool, block_size, cache_stride, num_blocks,
                      as_stream(stream), replayed_tokens, nullptr);
}

FP8Q_API fp8q_status fp8_kv_calib_observe_write(
    fp8_kv_calib *calib, const void *k, const void *v, int64_t key_stride, int64_t value_stride,
    const int64_t *slot_mapping, int64_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
    void *k_pool, void *v_pool, int32_t block_size, int64_t cache_stride, int64_t num_blocks,
    void *stream, int32_t *step_out) {
    if (calib == nullptr || step_out == nullptr) return FP8Q_EINVAL;
    int64_t elems = 0;
    if (!valid_rows(k, v, key_stride, value_stride, num_tokens, num_kv_heads, head_dim, &elems))
        return FP8Q_EINVAL;
    if (!valid_pools(k_pool, v_pool, block_size, cache_stride, num_blocks, elems))
        return FP8Q_EINVAL;
    if (num_tokens > 0 && (slot_mapping == nullptr || !aligned(slot_mapping, 8)))
        return FP8Q_EINVAL;
    if (calib->phase == kFreezePending) return FP8Q_ESTATE;
    cudaStream_t s = as_stream(stream);

    KvPass p;
    int32_t step = 0;
    fp8q_status st = plan_observe(calib, k, v, key_stride, value_stride, slot_mapping, num_tokens,
                                  num_kv_heads, head_dim, &p, &step);
    if (st != FP8Q_OK) return st;
    *step_out = step;

    KvPass w = write_pass(k, v, key_stride, value_stride, slot_mapping, num_tokens, elems,
                          k_pool, v_pool, block_size, cache_stride, num_blocks);
    if (step == FP8Q_STEP_FROZEN) {
        w.scale_dev = scale_dev(calib);
        return from_cuda(fp8q::launch_kv_pass(w, s));
    }
    if (step == FP8Q_STEP_STAGE || step == FP8Q_STEP_STAGE_DECLINED) {
        // one read of K and V: absmax (+ staging copy) + provisional write
        p.do_write = true;
        p.k_pool = w.k_pool;
        p.v_pool = w.v_pool;
        p.block_size = block_size;
        p.block_shift = w.block_shift;
        p.cache_stride = cache_stride;
        p.num_slots = w.num_slots;
        p.k_scale = FP8Q_PROVISIONAL_SCALE;
        p.v_scale = FP8Q_PROVISIONAL_SCALE;
        return from_cuda(fp8q::launch_kv_pass(p, s));
    }
    // FREEZE: the maxima must include this batch before any write; then the
    // replay, with the crossing batch written at the frozen scales last
    cudaError_t e = fp8q::launch_kv_pass(p, s);
    if (e != cudaSuccess) return FP8Q_ECUDA;
    w.scale_dev = scale_dev(calib);
    // the amax pass above is enqueued only when the batch has tokens
    return run_replay(calib, k_pool, v_pool, block_size, cache_stride, num_blocks, s, nullptr,
                      &w, /*chained=*/p.num_tokens > 0);
}

FP8Q_API fp8q_status fp8_kv_calib_restore(fp8_kv_calib *c, float k_scale, float v_scale,
                                          void *stream) {
    if (c == nullptr) return FP8Q_EINVAL;
    if (!(k_scale > 0.0f) || !(v_scale > 0.0f) || std::isinf(k_scale) || std::isinf(v_scale))
        return FP8Q_EINVAL;
    if (c->phase != kCalibrating || c->tokens_seen != 0 || c->staged_batches != 0)
        return FP8Q_ESTATE;
    cudaError_t e = fp8q::launch_calib_set(c->state_dev, k_scale, v_scale, k_scale, v_scale,
                                           as_stream(stream));
    if (e != cudaSuccess) return FP8Q_ECUDA;
    c->phase = kFrozen;
    c->staged_counts.clear();
    c->used_tokens = 0;
    return FP8Q_OK;
}

FP8Q_API const float *fp8_kv_calib_scale_dev(const fp8_kv_calib *calib) {
    return calib == nullptr ? nullptr : calib->state_dev + 2;
}

FP8Q_API fp8q_status fp8_kv_calib_stats_get(const fp8_kv_calib *c, fp8_kv_calib_stats *out) {
    if (c == nullptr || out == nullptr) return FP8Q_EINVAL;
    out->requested_tokens = c->requested_tokens;
    out->window_tokens = c->window_tokens;
    out->capacity_tokens = c->capacity_tokens;
    out->tokens_seen = c->tokens_seen;
    out->staged_tokens = c->used_tokens;
    out->staged_batches = c->staged_batches;
    out->unstaged_tokens = c->unstaged_tokens;
    out->freeze_tokens = c->freeze_tokens;
    out->replayed_tokens = c->replayed_tokens;
    out->replayed_batches = c->replayed_batches;
    out->headroom = c->headroom;
    out->state = c->phase;
    return FP8Q_OK;
}

FP8Q_API fp8q_status fp8_kv_calib_read_state(const fp8_kv_calib *c, void *stream, float *out) {
    if (c == nullptr || out == nullptr) return FP8Q_EINVAL;
    cudaError_t e = cudaStreamSynchronize(as_stream(stream));
    if (e != cudaSuccess) return FP8Q_ECUDA;
    e = cudaMemcpy(out, c->state_dev, 4 * sizeof(float), cudaMemcpyDeviceToHost);
    return from_cuda(e);
}

FP8Q_API void fp8_kv_calib_destroy(fp8_kv_calib *c) { delete c; }

FP8Q_API int32_t fp8_kv_graphs_ready(const int8_t *states, int64_t n) {
    if (n < 0 || (n > 0 && states == nullptr)) return -1;
    for (int64_t i = 0; i < n; ++i)
        if (states[i] == 0) return 0;
    return 1;
}

FP8Q_API fp8q_status fp8q_device_error(uint32_t *bits_out, int32_t clear) {
    if (bits_out == nullptr) return FP8Q_EINVAL;
    return from_cuda(fp8q::read_device_error(bits_out, clear != 0));
}

FP8Q_API const char *fp8q_status_string(fp8q_status status) {
    switch (status) {
    case FP8Q_OK: return "ok";
    case FP8Q_EINVAL: return "invalid argument";
    case FP8Q_ECUDA: return "CUDA error";
    case FP8Q_ESTATE: return "calibration call out of order";
    case FP8Q_ENOMEM: return "out of host memory";
    case FP8Q_ETOOBIG: return "request exceeds the fixed scratch of the allocation-free call";
    default: return "unknown status";
    }
}

FP8Q_API int32_t fp8q_version(void) { return kVersion; }

FP8Q_API int64_t fp8q_launch_count(void) { return fp8q::launch_count(); }

}  // extern "C"
