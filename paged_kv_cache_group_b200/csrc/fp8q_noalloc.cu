// fp8q_noalloc.cu -- the calibration window of one layer in a single call,
// with its scratch in a fixed device array of the library instead of memory
// the caller provides.
//
// Who needs this: a caller that cannot allocate device memory when the
// window runs.  Typical cases are an engine that hands all device memory to
// its KV pool at start-up and forbids later cudaMalloc, code that must not
// trigger the implicit device synchronization a cudaMalloc/cudaFree can
// cause, and hosts (plugins, sandboxes) that give a library no allocator.
//
// The scratch is the window's staging (the bf16 K and V rows and the int64
// slots of the batches written before the freeze) plus the 16-byte
// calibration state {k_amax, v_amax, k_scale, v_scale}.  It lives in
// `g_noalloc_scratch`, FP8Q_NOALLOC_SCRATCH_BYTES bytes that every device
// which loads the library holds until the process exits.
//
// Layout inside the array: state at byte 0, staged K rows at byte 256, then
// the staged V rows, then the staged slots.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "fp8q.h"
#include "fp8q_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[FP8Q_NOALLOC_SCRATCH_BYTES];

constexpr int64_t kStageOffset = 256;
constexpr int kMaxDevices = 64;

std::mutex g_addr_mutex;
void *g_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device.  In host code
// the name g_noalloc_scratch is only a host-side stand-in, so the address is
// looked up once per device (with that device current) and cached.
cudaError_t scratch_address(unsigned char **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_addr_mutex);
    if (g_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_addr[dev] = p;
    }
    *out = static_cast<unsigned char *>(g_addr[dev]);
    return cudaSuccess;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int32_t pow2_shift(int32_t v) {
    if (v <= 0 || (v & (v - 1)) != 0) return -1;
    int32_t s = 0;
    while ((1 << s) != v) ++s;
    return s;
}

}  // namespace

extern "C" FP8Q_API fp8q_status fp8_kv_calib_window_noalloc(
    const void *k, const void *v, int64_t key_stride, int64_t value_stride,
    const int64_t *slot_mapping, const int64_t *batch_tokens, int32_t num_batches,
    int32_t num_kv_heads, int32_t head_dim, int64_t window_tokens, float headroom,
    void *k_pool, void *v_pool, int32_t block_size, int64_t cache_stride, int64_t num_blocks,
    float *scales_out, void *stream_ptr) {
    // ---- arguments (host only; nothing is enqueued on failure) ----
    if (num_batches < 0 || (num_batches > 0 && batch_tokens == nullptr)) return FP8Q_EINVAL;
    if (window_tokens <= 0 || num_kv_heads <= 0 || head_dim <= 0) return FP8Q_EINVAL;
    const int64_t elems = static_cast<int64_t>(num_kv_heads) * head_dim;
    if (elems % 8 != 0 || elems > (int64_t{1} << 30)) return FP8Q_EINVAL;
    if (key_stride < elems || value_stride < elems || key_stride % 8 || value_stride % 8)
        return FP8Q_EINVAL;
    if (block_size <= 0 || num_blocks < 0 || num_blocks > INT64_MAX / block_size)
        return FP8Q_EINVAL;
    if (cache_stride < static_cast<int64_t>(block_size) * elems || cache_stride % 8)
        return FP8Q_EINVAL;
    if (num_blocks > 0 && (k_pool == nullptr || v_pool == nullptr)) return FP8Q_EINVAL;
    if (!aligned(k_pool, 8) || !aligned(v_pool, 8)) return FP8Q_EINVAL;
    if (scales_out != nullptr && !aligned(scales_out, 8)) return FP8Q_EINVAL;
    int64_t total = 0;
    for (int32_t b = 0; b < num_batches; ++b) {
        if (batch_tokens[b] < 0) return FP8Q_EINVAL;
        total += batch_tokens[b];
    }
    if (total > 0) {
        if (k == nullptr || v == nullptr || slot_mapping == nullptr) return FP8Q_EINVAL;
        if (!aligned(k, 16) || !aligned(v, 16) || !aligned(slot_mapping, 8)) return FP8Q_EINVAL;
    }

    // ---- plan: the calibrator's token counting, on the host ----
    const int64_t window = window_tokens < FP8Q_MAX_STAGED_TOKENS ? window_tokens
                                                                  : FP8Q_MAX_STAGED_TOKENS;
    const float h = headroom >= 1.0f ? headroom : 1.0f;   // NaN -> 1 as well
    int32_t freeze_at = -1;   // batch that reaches the window
    int64_t staged = 0;       // rows staged before it
    {
        int64_t seen = 0;
        for (int32_t b = 0; b < num_batches; ++b) {
            seen += batch_tokens[b];
            if (seen >= window) {
                freeze_at = b;
                break;
            }
            staged += batch_tokens[b];
        }
    }
    const int64_t stage_bytes = staged * (4 * elems + 8);
    if (stage_bytes > FP8Q_NOALLOC_SCRATCH_BYTES - kStageOffset) return FP8Q_ETOOBIG;

    // ---- device ----
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    unsigned char *base = nullptr;
    if (scratch_address(&base) != cudaSuccess) return FP8Q_ECUDA;
    float *state = reinterpret_cast<float *>(base);
    uint16_t *stage_k = reinterpret_cast<uint16_t *>(base + kStageOffset);
    uint16_t *stage_v = stage_k + staged * elems;
    int64_t *stage_slots = reinterpret_cast<int64_t *>(stage_v + staged * elems);

    if (fp8q::launch_calib_init(state, stream) != cudaSuccess) return FP8Q_ECUDA;

    fp8q::KvPass w;   // the write half, common to every batch
    w.key_stride = key_stride;
    w.value_stride = value_stride;
    w.elems = static_cast<int32_t>(elems);
    w.k_pool = static_cast<uint8_t *>(k_pool);
    w.v_pool = static_cast<uint8_t *>(v_pool);
    w.block_size = block_size;
    w.block_shift = pow2_shift(block_size);
    w.cache_stride = cache_stride;
    w.num_slots = num_blocks * block_size;
    w.do_write = true;
    // every pass below follows a launch of this call (calib_init first), and
    // none reads what the launch before it writes
    w.early_loads = true;

    const uint16_t *k16 = static_cast<const uint16_t *>(k);
    const uint16_t *v16 = static_cast<const uint16_t *>(v);
    int64_t row = 0;          // first row of the current batch
    int64_t stage_row = 0;    // next free staging row
    for (int32_t b = 0; b < num_batches; ++b) {
        const int64_t n = batch_tokens[b];
        fp8q::KvPass p = w;
        p.k = k16 + row * key_stride;
        p.v = v16 + row * value_stride;
        p.slot_mapping = slot_mapping + row;
        p.num_tokens = n;
        if (freeze_at < 0 || b < freeze_at) {
            // in the window: absmax + staging copy + write at the provisional scale
            p.do_amax = true;
            p.amax_bits = reinterpret_cast<uint32_t *>(state);
            p.do_stage = true;
            p.stage_k = stage_k;
            p.stage_v = stage_v;
            p.stage_slots = stage_slots;
            p.stage_offset = stage_row;
            p.k_scale = FP8Q_PROVISIONAL_SCALE;
            p.v_scale = FP8Q_PROVISIONAL_SCALE;
            if (fp8q::launch_kv_pass(p, stream) != cudaSuccess) return FP8Q_ECUDA;
            stage_row += n;
        } else if (b == freeze_at) {
            // the batch that reaches the window: its absmax first, then the
            // freeze with the crossing batch written last, exactly as the
            // calibrator's fused observe issues them
            fp8q::KvPass a = p;
            a.do_write = false;
            a.do_amax = true;
            a.amax_bits = reinterpret_cast<uint32_t *>(state);
            if (fp8q::launch_kv_pass(a, stream) != cudaSuccess) return FP8Q_ECUDA;
            fp8q::KvPass r = w;
            r.freeze_amax = reinterpret_cast<uint32_t *>(state);
            r.headroom = h;
            r.scale_out = state + 2;
            p.scale_dev = state + 2;
            int64_t rewritten = 0;
            if (fp8q::enqueue_freeze_replay(r, stage_k, stage_v, stage_slots, batch_tokens, b, &p,
                                            true, stream, &rewritten) != cudaSuccess)
                return FP8Q_ECUDA;
        } else {
            p.scale_dev = state + 2;
            if (fp8q::launch_kv_pass(p, stream) != cudaSuccess) return FP8Q_ECUDA;
        }
        row += n;
    }
    if (scales_out != nullptr &&
        cudaMemcpyAsync(scales_out, state + 2, 2 * sizeof(float), cudaMemcpyDeviceToDevice,
                        stream) != cudaSuccess)
        return FP8Q_ECUDA;
    return FP8Q_OK;
}
