// fp8q_kernels.cu -- sm_100a kernels of the FP8 E4M3 quantization path.
//
// All three kernels are bound by HBM bandwidth: every element is read once
// (bf16, 2 B) and written once (E4M3, 1 B) with a handful of ALU operations in
// between.  Nothing here is a contraction, so there are no tensor-core paths;
// the design goals are fully coalesced 128-bit loads, enough bytes in flight
// per SM to cover HBM latency, and an encode that is exact yet cheap.
//
// Exact arithmetic.  A code is E4M3(fp32(x / s)).  The fp32 quotient is
// formed from r = RN(1/s) (one IEEE reciprocal per group or per tensor) with
// one product and one FMA correction:
//     q0 = RN(x * r);  e = x - q0*s (exact in an FMA);  q = RN(q0 + e*r)
// By Markstein's theorem (r within half an ulp of 1/s, q0 within one ulp of
// x/s, no underflow or overflow) q is the correctly rounded x/s.  The three
// steps run on pairs of values (fma.rn.f32x2, two independent IEEE
// operations per instruction).  The residual step is rounded toward -inf: a
// nonzero residual is exact, so the mode changes nothing but the sign of an
// exact zero, and with it x = -0 (and a negative x whose quotient underflows)
// keeps its sign through q = q0 + e*r, as IEEE division does.  When s is a
// power of two, r = 1/s exactly and RN(x * r) is already the quotient: one
// product.  A per-tensor scale may be small enough that x * r overflows for
// huge x, so there the product uses r' = r * 2^-k in [0.5, 1) (and s' =
// s * 2^k) and is scaled back by an exact multiply by 2^k before the
// correction; a product that overflows there is infinite and saturates to
// +-448, the code of the (equally huge) quotient.  Both forms were checked
// on the CPU against IEEE division: the group form over every pair of bf16 x
// and bf16 group maximum, the per-tensor form over every bf16 x at 2400
// scales in [2^-64, 2^64]; codes agree everywhere.  Scales outside that
// range use __fdiv_rn.  The quotient is then rounded by the hardware
// conversion cvt.rn.satfinite.e4m3x2.f32: nearest-even, saturating to +-448.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>
#include <utility>

#include "fp8q_internal.h"

namespace fp8q {

// Kernels launched by this library in this process (diagnostics).
std::atomic<int64_t> g_launch_count{0};

// Sticky error word of this device (one per device that loads the library).
__device__ uint32_t g_error_word;

namespace {

constexpr float kScaleFloor = 1e-12f;
constexpr uint32_t kErrSlot = 0x1u;
constexpr uint32_t kErrScale = 0x2u;

// ---------------------------------------------------------------------------
// device helpers

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 128-bit load of data read exactly once: no L1 allocation.  volatile: the
// load must never be hoisted above the bounds test that guards it.
__device__ __forceinline__ uint4 ld_once(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p));
    return v;
}

// Programmatic dependent launch.  Every kernel here is launched with
// programmatic stream serialization: it may be scheduled while the previous
// kernel in the stream is still running, so it first waits until that kernel
// has completed and its writes are visible, and then lets the next kernel
// start its own launch.  Launched without the attribute, both are no-ops.
__device__ __forceinline__ void wait_for_previous_grid() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void allow_next_grid() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Warm L2 with bytes this thread is about to read.  Issued before
// wait_for_previous_grid(), so the DRAM reads overlap the previous kernel's
// tail.  It is only a hint: L2 is where the GPU's writes become coherent, so
// a later load still returns whatever the previous kernel wrote.
__device__ __forceinline__ void prefetch_l2_bulk(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(p), "r"(bytes) : "memory");
}

// Per-half max of |a| and |b| for two bf16x2 words (the sign bits of the
// result carry no meaning and are cleared by the caller).
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t absmax_uint4(uint32_t acc, const uint4 &c) {
    acc = absmax_bf16x2(acc, c.x);
    acc = absmax_bf16x2(acc, c.y);
    acc = absmax_bf16x2(acc, c.z);
    acc = absmax_bf16x2(acc, c.w);
    return acc;
}

// Largest |value| of a bf16x2 accumulator, as the 16-bit magnitude pattern.
__device__ __forceinline__ uint32_t absmax_bits16(uint32_t acc) {
    acc &= 0x7FFF7FFFu;
    return max(acc & 0xFFFFu, acc >> 16);
}

// Two fp32 values to two E4M3 codes: byte 0 <- lo, byte 1 <- hi.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    unsigned short d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return d;
}

struct Divisor {
    float s;     // the scale
    float r;     // RN(1/s)
};

// A pair of fp32 values in one 64-bit register, as the f32x2 instructions take.
__device__ __forceinline__ uint64_t pair(float lo, float hi) {
    uint64_t v;
    asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(lo), "f"(hi));
    return v;
}
__device__ __forceinline__ uint64_t pair_of_bf16x2(uint32_t w) { return pair(bf16_lo(w), bf16_hi(w)); }
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
// Two fp32 values (a pair) to two E4M3 codes: byte 0 <- lo, byte 1 <- hi.
__device__ __forceinline__ uint32_t e4m3x2_pair(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return e4m3x2(lo, hi);
}

// The divisor as pairs: {r, r} and {-s, -s}.
struct PairDivisor {
    uint64_t r2, ns2;
};
__device__ __forceinline__ PairDivisor pair_divisor(const Divisor &d) {
    return PairDivisor{pair(d.r, d.r), pair(-d.s, -d.s)};
}

__device__ __forceinline__ uint64_t fma2_rm(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rm.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// Correctly rounded quotients of a pair, signs of zero included (see the
// file comment).
__device__ __forceinline__ uint64_t quotient2(uint64_t x, const PairDivisor &d) {
    const uint64_t q0 = mul2(x, d.r2);
    const uint64_t e = fma2_rm(q0, d.ns2, x);
    return fma2(e, d.r2, q0);
}

// Codes of four values (bf16x2 words w0, w1).
__device__ __forceinline__ uint32_t encode4(uint32_t w0, uint32_t w1, const PairDivisor &d) {
    return e4m3x2_pair(quotient2(pair_of_bf16x2(w0), d)) |
           (e4m3x2_pair(quotient2(pair_of_bf16x2(w1), d)) << 16);
}

// Codes of four values for a power-of-two scale: r is exact, one product.
__device__ __forceinline__ uint32_t encode4_pow2(uint32_t w0, uint32_t w1, uint64_t r2) {
    return e4m3x2_pair(mul2(pair_of_bf16x2(w0), r2)) |
           (e4m3x2_pair(mul2(pair_of_bf16x2(w1), r2)) << 16);
}

// Group scale RN(y / 448) for y >= 1e-12.  448 = 7 * 64, so the quotient is
// RN(y / 7) * 2^-6 exactly (no underflow in that range), and RN(y / 7) is the
// correctly rounded division by the constant 7 from RN(1/7), by the same
// Markstein step as above.  Checked against IEEE division for every fp32 y
// from 1e-12 to the largest finite value.
__device__ __forceinline__ float group_scale(float y) {
    constexpr float kRecip7 = 0x1.24924ap-3f;   // RN(1/7)
    const float q0 = __fmul_rn(y, kRecip7);
    const float e = __fmaf_rn(q0, 7.0f, -y);
    return __fmul_rn(__fmaf_rn(-e, kRecip7, q0), 0x1p-6f);
}

__device__ __forceinline__ uint2 encode8(const uint4 &w, const PairDivisor &d) {
    return make_uint2(encode4(w.x, w.y, d), encode4(w.z, w.w, d));
}

__device__ __forceinline__ uint2 encode8_pow2(const uint4 &w, uint64_t r2) {
    return make_uint2(encode4_pow2(w.x, w.y, r2), encode4_pow2(w.z, w.w, r2));
}

// IEEE division per element, for scales outside the fast range.
__device__ __forceinline__ uint2 encode8_div(const uint4 &w, float s) {
    uint2 o;
    o.x = e4m3x2(__fdiv_rn(bf16_lo(w.x), s), __fdiv_rn(bf16_hi(w.x), s)) |
          (e4m3x2(__fdiv_rn(bf16_lo(w.y), s), __fdiv_rn(bf16_hi(w.y), s)) << 16);
    o.y = e4m3x2(__fdiv_rn(bf16_lo(w.z), s), __fdiv_rn(bf16_hi(w.z), s)) |
          (e4m3x2(__fdiv_rn(bf16_lo(w.w), s), __fdiv_rn(bf16_hi(w.w), s)) << 16);
    return o;
}

// Per-tensor quotients of a pair with the product taken on r' = r * 2^-k and
// scaled back by c = 2^k (see the file comment): no overflow before the
// correction, an infinite result only where the quotient itself is huge.
struct ScaledDivisor {
    uint64_t rs2;    // {r', r'}
    uint64_t nss2;   // {-s', -s'}
    uint64_t c2;     // {2^k, 2^k}
    uint64_t r2;     // {r, r}
};

__device__ __forceinline__ uint64_t quotient2_scaled(uint64_t x, const ScaledDivisor &d) {
    const uint64_t q0 = mul2(x, d.rs2);
    const uint64_t e = fma2_rm(q0, d.nss2, x);
    return fma2(e, d.r2, mul2(q0, d.c2));
}

__device__ __forceinline__ uint2 encode8_scaled(const uint4 &w, const ScaledDivisor &d) {
    uint2 o;
    o.x = e4m3x2_pair(quotient2_scaled(pair_of_bf16x2(w.x), d)) |
          (e4m3x2_pair(quotient2_scaled(pair_of_bf16x2(w.y), d)) << 16);
    o.y = e4m3x2_pair(quotient2_scaled(pair_of_bf16x2(w.z), d)) |
          (e4m3x2_pair(quotient2_scaled(pair_of_bf16x2(w.w), d)) << 16);
    return o;
}

// Per-tensor encoder.  Scales in [2^-64, 2^64]: the reciprocal form, plain
// when r < 1 (no bf16 value can overflow x * r) and scaled otherwise; a
// power-of-two scale takes one product.  Other scales: IEEE division per
// element.
struct TensorEncoder {
    float s;
    PairDivisor pd;      // {r, r}, {-s, -s}
    ScaledDivisor sd;
    bool fast;
    bool pow2;           // s is a power of two: RN(x * r) is the quotient
    bool scaled;         // r >= 1: take the product on r' and scale back
    bool ok;             // scale is a positive number

    // `bounded`: the caller knows |x| / s <= 448 for every x it encodes (the
    // maxima the scale comes from cover them), so x * r cannot overflow and
    // the plain form serves.
    __device__ __forceinline__ void init(float scale, bool bounded = false) {
        s = scale;
        ok = s > 0.0f;   // false for NaN
        fast = (s >= 0x1p-64f) && (s <= 0x1p64f);
        pow2 = fast && (__float_as_uint(s) & 0x7FFFFFu) == 0;
        const float r = __frcp_rn(s);
        pd.r2 = pair(r, r);
        pd.ns2 = pair(-s, -s);
        scaled = !bounded && fast && !pow2 && r >= 1.0f;
        if (scaled) {
            // r' = r * 2^-k in [0.5, 1), s' = s * 2^k, c = 2^k: exponent-field
            // arithmetic, exact for the normal r and s of the fast range
            const uint32_t k = ((__float_as_uint(r) >> 23) & 0xFF) - 126;
            const float rs = __uint_as_float(__float_as_uint(r) - (k << 23));
            const float ss = __uint_as_float(__float_as_uint(s) + (k << 23));
            const float c = __uint_as_float((127 + k) << 23);
            sd.rs2 = pair(rs, rs);
            sd.nss2 = pair(-ss, -ss);
            sd.c2 = pair(c, c);
            sd.r2 = pd.r2;
        }
    }

    // The calibrator's provisional scale 2.0 (in-window writes): a power of
    // two, r = 0.5 exactly, no reciprocal to compute.
    __device__ __forceinline__ void init_provisional() {
        s = 2.0f;
        ok = fast = pow2 = true;
        scaled = false;
        pd.r2 = pair(0.5f, 0.5f);
        pd.ns2 = pair(-2.0f, -2.0f);
    }

    // Two chunks of a row.
    __device__ __forceinline__ void encode2(const uint4 &a, const uint4 &b, uint2 &oa,
                                            uint2 &ob) const {
        if (pow2) {
            oa = encode8_pow2(a, pd.r2);
            ob = encode8_pow2(b, pd.r2);
        } else if (fast) {
            if (scaled) {
                oa = encode8_scaled(a, sd);
                ob = encode8_scaled(b, sd);
            } else {
                oa = encode8(a, pd);
                ob = encode8(b, pd);
            }
        } else {
            oa = encode8_div(a, s);
            ob = encode8_div(b, s);
        }
    }
};

// Frozen scale: max(amax * headroom, 1e-12) / 448, product rounded first.
// The division is group_scale's exact RN(y / 448) (y is a normal fp32 here);
// an infinite product stays infinite, as in IEEE division.
__device__ __forceinline__ float freeze_scale(uint32_t amax_bits, float headroom) {
    const float y = fmaxf(__fmul_rn(__uint_as_float(amax_bits), headroom), kScaleFloor);
    return y < INFINITY ? group_scale(y) : y;
}

// ---------------------------------------------------------------------------
// 1. per-token 1x128-group quantization
//
// Four lanes own one 128-element group (32 elements each); a warp covers
// eight consecutive groups (2 KB of input).  Lane q of a group loads chunks
// q, q+4, q+8, q+12 of 16 bytes, so each of the four load instructions of a
// warp reads eight fully used 64-byte runs, and each store writes eight full
// 32-byte sectors.  The group maximum needs two shuffles.

constexpr int kGqThreads = 256;

// One group of four lanes: load the 128 elements (zeros when !load), reduce
// the group maximum and return the group's scale; the codes are left in c.
__device__ __forceinline__ Divisor quant_group_load(const uint16_t *src, bool load, int ql,
                                                   uint4 (&c)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
        c[j] = load ? ld_once(src + (ql + 4 * j) * 8) : make_uint4(0, 0, 0, 0);

    uint32_t acc = c[0].x;
    acc = absmax_bf16x2(acc, c[0].y);
    acc = absmax_bf16x2(acc, c[0].z);
    acc = absmax_bf16x2(acc, c[0].w);
#pragma unroll
    for (int j = 1; j < 4; ++j) acc = absmax_uint4(acc, c[j]);
    uint32_t m = absmax_bits16(acc);
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));

    const float amax = __uint_as_float(m << 16);
    Divisor d;
    d.s = group_scale(fmaxf(amax, kScaleFloor));
    d.r = __frcp_rn(d.s);
    return d;
}

template <bool kPacked>
__global__ void __launch_bounds__(kGqThreads)
group_quant_kernel(const uint16_t *__restrict__ x, int64_t x_row_stride,
                   uint8_t *__restrict__ q, float *__restrict__ scales,
                   int64_t total_groups, uint32_t groups_per_row) {
    const int lane = threadIdx.x & 31;
    const int sub = lane >> 2;   // group within the warp's eight
    const int ql = lane & 3;     // lane within the group
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kGqThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kGqThreads) >> 5;
    const int64_t octets = (total_groups + 7) >> 3;
    // Strided rows: this lane's group as (row, column), advanced by the grid's
    // stride without a division per step.
    const int64_t g0 = warp * 8 + sub;
    int64_t row = kPacked ? 0 : g0 / groups_per_row;
    int64_t col = kPacked ? 0 : g0 - row * groups_per_row;
    const int64_t step = nwarps * 8;
    const int64_t drow = kPacked ? 0 : step / groups_per_row;
    const int64_t dcol = kPacked ? 0 : step - drow * groups_per_row;
    auto group_src = [&](int64_t g) -> const uint16_t * {
        if (kPacked) return x + g * 128;
        return x + row * x_row_stride + col * 128;
    };
    // the first eight groups this warp reads: one 256-byte group per lane 0..7
    if (kPacked && lane < 8 && warp < octets && warp * 8 + lane < total_groups)
        prefetch_l2_bulk(x + (warp * 8 + lane) * 128, 256);
    if (!kPacked && (lane & 3) == 0 && warp < octets && g0 < total_groups)
        prefetch_l2_bulk(group_src(g0), 256);
    wait_for_previous_grid();
    allow_next_grid();

    for (int64_t o = warp; o < octets; o += nwarps) {
        const int64_t g = o * 8 + sub;
        const bool valid = g < total_groups;
        uint4 c[4];
        const Divisor d = quant_group_load(valid ? group_src(g) : x, valid, ql, c);
        const PairDivisor pd = pair_divisor(d);
        if (valid) {
            uint8_t *dst = q + g * 128;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                *reinterpret_cast<uint2 *>(dst + (ql + 4 * j) * 8) = encode8(c[j], pd);
            if (ql == 0) scales[g] = d.s;
        }
        if (!kPacked) {
            row += drow;
            col += dcol;
            if (col >= groups_per_row) {
                col -= groups_per_row;
                ++row;
            }
        }
    }
}

// K-major variant.  A warp's eight groups are one column g of eight
// consecutive rows, so their eight scales are adjacent in scales_km (one
// 32-byte sector); consecutive warps take the next column of the same eight
// rows, which keeps the grid's reads inside one slab of rows at a time.
// Rows m..m_pad-1 are phantom: nothing is read, zeros are written.
__global__ void __launch_bounds__(kGqThreads)
group_quant_kmajor_kernel(const uint16_t *__restrict__ x, int64_t x_row_stride,
                          uint8_t *__restrict__ q, float *__restrict__ scales_km,
                          int64_t m, int64_t m_pad, uint32_t groups_per_row) {
    const int lane = threadIdx.x & 31;
    const int sub = lane >> 2;
    const int ql = lane & 3;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kGqThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kGqThreads) >> 5;
    const int64_t octets = ((m_pad + 7) >> 3) * groups_per_row;
    const int64_t k = static_cast<int64_t>(groups_per_row) * 128;
    // this warp's (row octet, column), advanced by the grid's stride without
    // a division per step
    int64_t ro = warp / groups_per_row;
    int64_t col = warp - ro * groups_per_row;
    const int64_t dro = nwarps / groups_per_row;
    const int64_t dcol = nwarps - dro * groups_per_row;
    if (lane < 8 && warp < octets) {
        const int64_t row = ro * 8 + lane;
        if (row < m) prefetch_l2_bulk(x + row * x_row_stride + col * 128, 256);
    }
    wait_for_previous_grid();
    allow_next_grid();

    for (int64_t o = warp; o < octets; o += nwarps) {
        const int64_t row = ro * 8 + sub;
        const bool live = row < m;
        uint4 c[4];
        const Divisor d =
            quant_group_load(x + (live ? row * x_row_stride + col * 128 : 0), live, ql, c);
        const PairDivisor pd = pair_divisor(d);
        if (row < m_pad) {
            uint8_t *dst = q + row * k + col * 128;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                *reinterpret_cast<uint2 *>(dst + (ql + 4 * j) * 8) =
                    live ? encode8(c[j], pd) : make_uint2(0, 0);
            if (ql == 0) scales_km[col * m_pad + row] = live ? d.s : 0.0f;
        }
        ro += dro;
        col += dcol;
        if (col >= groups_per_row) {
            col -= groups_per_row;
            ++ro;
        }
    }
}

// ---------------------------------------------------------------------------
// 2./3. KV pass: absmax, staging copy and quantize-and-scatter
//
// One warp per token.  Lane l owns 16-byte chunks l and l+32 of the K row and
// of the V row, so every load and store instruction of the warp is one
// contiguous run (512 B of bf16 in, 256 B of codes out).  The slot decides
// where the codes land: one token's entry is E contiguous bytes of the pool,
// written as 32 8-byte stores per instruction.
//
// Each warp issues its token's loads before anything else, then resolves the
// scales itself (a dependent 8-byte load; for a freeze the frozen scale from
// the device maxima) while those loads are in flight.  CTAs are 256 threads,
// 512 for the merged freeze launch.  Rows of 4 x 128 elements (the pages'
// shape) take kernels of their own for the three passes of the calibrating
// write path (kv_stage512_kernel, kv_freeze512_kernel, kv_write512_kernel);
// kv_pass_kernel serves every other shape and job (grid-stride when the
// batch is larger than the resident grid).

constexpr int kKvThreads = 256;
constexpr int kKvWarps = kKvThreads / 32;
constexpr uint32_t kEmptySlot = 0xFFFFFFFFu;

// Shared-memory hash set of the crossing batch's slots (open addressing,
// linear probing, 2^log2 entries, at most half full).
__device__ __forceinline__ uint32_t slot_hash(uint32_t key, int log2) {
    return (key * 2654435761u) >> (32 - log2);
}

__device__ __forceinline__ void table_insert(uint32_t *tab, int log2, uint32_t key) {
    const uint32_t mask = (1u << log2) - 1u;
    uint32_t h = slot_hash(key, log2);
    for (uint32_t probe = 0; probe <= mask; ++probe) {   // bounded: the table is never full
        const uint32_t prev = atomicCAS(&tab[h], kEmptySlot, key);
        if (prev == kEmptySlot || prev == key) return;
        h = (h + 1u) & mask;
    }
}

__device__ __forceinline__ bool table_contains(const uint32_t *tab, int log2, uint32_t key) {
    const uint32_t mask = (1u << log2) - 1u;
    uint32_t h = slot_hash(key, log2);
    for (uint32_t probe = 0; probe <= mask; ++probe) {
        const uint32_t v = tab[h];
        if (v == key) return true;
        if (v == kEmptySlot) return false;
        h = (h + 1u) & mask;
    }
    return false;
}

// Pools of at most this many slots take an exact bitmap of the crossing slots
// (one bit per slot, 32 KB of shared memory at most) instead of the hash set.
constexpr int64_t kBitmapMaxSlots = int64_t{1} << 18;

// Hash-set size for `entries` crossing slots: load factor at most 1/4 up to
// 4096 entries, at most 1/2 above (64 KB at the 8192-slot merge limit).
__host__ __device__ __forceinline__ int table_log2(int64_t entries) {
    const int64_t want = entries <= 4096 ? 4 * entries : 2 * entries;
    int log2 = 6;
    while ((int64_t{1} << log2) < want) ++log2;
    return log2;
}

// Shared-memory bytes of the crossing set of a merged launch.
__host__ __device__ __forceinline__ int64_t crossing_set_bytes(int64_t num_slots,
                                                              int64_t x_tokens) {
    if (num_slots <= kBitmapMaxSlots) return ((num_slots + 127) >> 7) * 16;
    return int64_t{4} << table_log2(x_tokens);
}

// Membership in the crossing set: log2 == 0 is the slot bitmap.
__device__ __forceinline__ bool crossing_contains(const uint32_t *tab, int log2, uint32_t key) {
    if (log2 == 0) return (tab[key >> 5] >> (key & 31u)) & 1u;
    return table_contains(tab, log2, key);
}

// Last-writer table of a whole-window replay: 2^L slot keys followed by 2^L
// values, the value of a slot being 1 + the highest row index that writes it
// (open addressing, linear probing, at most half full).
__host__ __device__ __forceinline__ int last_writer_log2(int64_t rows) {
    int log2 = 6;
    while ((int64_t{1} << log2) < 2 * rows) ++log2;
    return log2;
}

__device__ __forceinline__ void last_writer_insert(uint32_t *tab, int log2, uint32_t key,
                                                   uint32_t row1) {
    const uint32_t mask = (1u << log2) - 1u;
    uint32_t h = slot_hash(key, log2);
    for (uint32_t probe = 0; probe <= mask; ++probe) {   // bounded: the table is never full
        const uint32_t prev = atomicCAS(&tab[h], kEmptySlot, key);
        if (prev == kEmptySlot || prev == key) {
            atomicMax(&tab[(1u << log2) + h], row1);
            return;
        }
        h = (h + 1u) & mask;
    }
}

__device__ __forceinline__ uint32_t last_writer_of(const uint32_t *tab, int log2, uint32_t key) {
    const uint32_t mask = (1u << log2) - 1u;
    uint32_t h = slot_hash(key, log2);
    for (uint32_t probe = 0; probe <= mask; ++probe) {
        const uint32_t v = tab[h];
        if (v == key) return tab[(1u << log2) + h];
        if (v == kEmptySlot) return 0;
        h = (h + 1u) & mask;
    }
    return 0;
}

// Whether a later row of the launch writes this row's slot.  log2 < 0: the
// last-writer table of a whole-window replay (2^-log2 entries); otherwise the
// crossing set, which only staged rows consult.
__device__ __forceinline__ bool superseded(const uint32_t *tab, int log2, uint32_t key, int64_t t,
                                           int64_t num_tokens) {
    if (log2 < 0) return last_writer_of(tab, -log2, key) != static_cast<uint32_t>(t + 1);
    return t < num_tokens && crossing_contains(tab, log2, key);
}

// Scales of a write pass (see KvPass).  Every warp resolves them itself from
// two loads issued together with its row loads; a CTA-wide broadcast through
// shared memory would put a barrier behind the slowest of those loads.  Lane 0
// of the grid's first warp reports a bad scale and, for a freeze, publishes
// the frozen scales.
__device__ __forceinline__ void resolve_scales(const KvPass &p, TensorEncoder &kenc,
                                               TensorEncoder &venc) {
    float ks, vs;
    if (p.freeze_amax != nullptr) {
        const uint2 a = *reinterpret_cast<const uint2 *>(p.freeze_amax);
        ks = freeze_scale(a.x, p.headroom);
        vs = freeze_scale(a.y, p.headroom);
        if (p.scale_out != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
            p.scale_out[0] = ks;
            p.scale_out[1] = vs;
        }
    } else if (p.scale_dev != nullptr) {
        const float2 sd = *reinterpret_cast<const float2 *>(p.scale_dev);
        ks = sd.x;
        vs = sd.y;
    } else {
        ks = p.k_scale;
        vs = p.v_scale;
    }
    // Every row a freeze pass writes (staged or crossing) went into the maxima
    // the scale comes from, so |x| / s <= 448 / headroom <= 448.
    kenc.init(ks, p.freeze_amax != nullptr);
    venc.init(vs, p.freeze_amax != nullptr);
    if (!(kenc.ok && venc.ok) && blockIdx.x == 0 && threadIdx.x == 0)
        atomicOr(&g_error_word, kErrScale);
}

// Per-layer variant: a bad scale is reported by the first CTA of each layer.
__device__ __forceinline__ void resolve_layer_scales(const KvPass &p, TensorEncoder &kenc,
                                                     TensorEncoder &venc) {
    float ks = p.k_scale, vs = p.v_scale;
    if (p.scale_dev != nullptr) {
        const float2 sd = *reinterpret_cast<const float2 *>(p.scale_dev);
        ks = sd.x;
        vs = sd.y;
    }
    kenc.init(ks);
    venc.init(vs);
    if (!(kenc.ok && venc.ok) && blockIdx.x == 0 && threadIdx.x == 0)
        atomicOr(&g_error_word, kErrScale);
}

// A token's row pointers (staged or crossing) and its first 64 chunks.
struct Row {
    const uint16_t *k;
    const uint16_t *v;
    int64_t slot;
    uint4 ka, kb, va, vb;
};

template <bool kCross, bool kSlot, int kChunks>
__device__ __forceinline__ void load_row(const KvPass &p, int64_t t, int lane, int nchunks,
                                         Row &r) {
    if (kCross && t >= p.num_tokens) {
        const int64_t u = t - p.num_tokens;
        r.k = p.xk + u * p.x_key_stride;
        r.v = p.xv + u * p.x_value_stride;
        r.slot = __ldg(p.x_slots + u);
    } else {
        r.k = p.k + t * p.key_stride;
        r.v = p.v + t * p.value_stride;
        r.slot = kSlot ? __ldg(p.slot_mapping + t) : -1;
    }
    const uint4 z = make_uint4(0, 0, 0, 0);
    const bool ha = lane < nchunks;
    const bool hb = 32 + lane < nchunks;
    r.ka = ha ? ld_once(r.k + lane * 8) : z;
    r.kb = hb ? ld_once(r.k + (32 + lane) * 8) : z;
    r.va = ha ? ld_once(r.v + lane * 8) : z;
    r.vb = hb ? ld_once(r.v + (32 + lane) * 8) : z;
}

// One row of a pass: absmax, staging copy, and the quantized write into the
// pool entry of its slot.
template <bool kAmax, bool kStage, bool kWrite, bool kCross, int kChunks>
__device__ __forceinline__ void process_row(const KvPass &p, Row &r, int64_t t, int lane,
                                            int nchunks, const TensorEncoder &kenc,
                                            const TensorEncoder &venc, const uint32_t *table,
                                            int log2, bool small_slots, uint32_t &kacc,
                                            uint32_t &vacc) {
    const uint4 z = make_uint4(0, 0, 0, 0);
    const int64_t slot = r.slot;
    bool write_row = false;
    int64_t dst = 0;
    if (kWrite && slot >= 0) {
        if (slot >= p.num_slots) {
            if (lane == 0) atomicOr(&g_error_word, kErrSlot);
        } else if (!(kCross && superseded(table, log2, static_cast<uint32_t>(slot), t,
                                          p.num_tokens))) {
            int64_t blk, off;
            if (p.block_shift >= 0) {
                blk = slot >> p.block_shift;
                off = slot & ((int64_t{1} << p.block_shift) - 1);
            } else if (small_slots) {
                const uint32_t s32 = static_cast<uint32_t>(slot);
                const uint32_t b32 = s32 / static_cast<uint32_t>(p.block_size);
                blk = b32;
                off = s32 - b32 * static_cast<uint32_t>(p.block_size);
            } else {
                blk = slot / p.block_size;
                off = slot - blk * p.block_size;
            }
            dst = blk * p.cache_stride + off * p.elems;
            write_row = true;
        }
    }

    for (int c0 = 0; c0 < nchunks; c0 += 64) {
        const int ca = c0 + lane;
        const int cb = c0 + 32 + lane;
        const bool ha = ca < nchunks;
        const bool hb = cb < nchunks;
        if (c0 > 0) {   // rows wider than 512 elements: next 64 chunks
            r.ka = ha ? ld_once(r.k + ca * 8) : z;
            r.kb = hb ? ld_once(r.k + cb * 8) : z;
            r.va = ha ? ld_once(r.v + ca * 8) : z;
            r.vb = hb ? ld_once(r.v + cb * 8) : z;
        }
        if (kAmax) {
            kacc = absmax_uint4(absmax_uint4(kacc, r.ka), r.kb);
            vacc = absmax_uint4(absmax_uint4(vacc, r.va), r.vb);
        }
        if (kStage) {
            const int64_t row = (p.stage_offset + t) * p.elems;
            if (ha) {
                *reinterpret_cast<uint4 *>(p.stage_k + row + ca * 8) = r.ka;
                *reinterpret_cast<uint4 *>(p.stage_v + row + ca * 8) = r.va;
            }
            if (hb) {
                *reinterpret_cast<uint4 *>(p.stage_k + row + cb * 8) = r.kb;
                *reinterpret_cast<uint4 *>(p.stage_v + row + cb * 8) = r.vb;
            }
        }
        if (kWrite && write_row) {
            uint2 oa, ob;
            if (kenc.ok) {
                kenc.encode2(r.ka, r.kb, oa, ob);
                if (ha) *reinterpret_cast<uint2 *>(p.k_pool + dst + ca * 8) = oa;
                if (hb) *reinterpret_cast<uint2 *>(p.k_pool + dst + cb * 8) = ob;
            }
            if (venc.ok) {
                venc.encode2(r.va, r.vb, oa, ob);
                if (ha) *reinterpret_cast<uint2 *>(p.v_pool + dst + ca * 8) = oa;
                if (hb) *reinterpret_cast<uint2 *>(p.v_pool + dst + cb * 8) = ob;
            }
        }
    }
    if (kStage && lane == 0) p.stage_slots[p.stage_offset + t] = slot;
}

// Warm L2 with the K row (lane 0) or the V row (lane 1) of token t; pointers
// are chosen by selects, so the two lanes do not diverge.
template <bool kCross>
__device__ __forceinline__ void prefetch_row(const KvPass &p, int64_t t, int lane) {
    const bool crossing = kCross && t >= p.num_tokens;
    const int64_t u = crossing ? t - p.num_tokens : t;
    const uint16_t *base = lane ? p.v : p.k;
    int64_t stride = lane ? p.value_stride : p.key_stride;
    if (kCross && crossing) {
        base = lane ? p.xv : p.xk;
        stride = lane ? p.x_value_stride : p.x_key_stride;
    }
    prefetch_l2_bulk(base + u * stride, static_cast<uint32_t>(p.elems) * 2u);
}

// kChunks: 16-byte chunks per row when fixed at compile time (64 for the
// common 4 x 128 rows), or 0 for any multiple of 8 elements.
//
// kThreads: 256, or 512 for the merged freeze launch (kCross), where half as
// many CTAs build the crossing slots' table (measured: 4.81 -> 4.44 us per
// 4593-token replay; the other passes are faster with 256).
template <bool kAmax, bool kStage, bool kWrite, bool kCross, int kChunks,
          int kThreads = kKvThreads>
__global__ void __launch_bounds__(kThreads, 1024 / kThreads) kv_pass_kernel(const KvPass p) {
    constexpr int kWarps = kThreads / 32;
    extern __shared__ uint32_t s_table[];        // crossing slots (kCross)

    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
    const int nchunks = kChunks > 0 ? kChunks : (p.elems >> 3);
    const int64_t total = p.num_tokens + (kCross ? p.x_tokens : 0);
    constexpr bool kSlot = kWrite || kStage;

    // Only CTAs that rewrite staged tokens consult the crossing slots.  With
    // the grid-stride loop a CTA's tokens are blockIdx.x*8 + k*nwarps + w, so
    // a CTA whose first token is a crossing token never sees a staged one.
    // A whole-window replay checks every row against its last-writer table.
    const bool need_table =
        kCross && (p.last_writer || static_cast<int64_t>(blockIdx.x) * kWarps < p.num_tokens);
    const bool early = p.early_loads;
    if (!early) {
        // the first token's K row, V row and slot into L2 while the previous
        // kernel finishes (and, for a merged crossing batch, its slot list)
        if (warp < total && lane < 2) prefetch_row<kCross>(p, warp, lane);
        if (need_table && threadIdx.x == 32) {
            const int64_t bytes = p.x_tokens * 8;
            if ((reinterpret_cast<uintptr_t>(p.x_slots) & 15) == 0 && bytes % 16 == 0 &&
                bytes > 0)
                prefetch_l2_bulk(p.x_slots, static_cast<uint32_t>(bytes));
        }
        if (kCross && p.last_writer && threadIdx.x == 64) {
            const int64_t bytes = p.num_tokens * 8;
            if ((reinterpret_cast<uintptr_t>(p.slot_mapping) & 15) == 0 && bytes % 16 == 0 &&
                bytes > 0)
                prefetch_l2_bulk(p.slot_mapping, static_cast<uint32_t>(bytes));
        }
        wait_for_previous_grid();
        allow_next_grid();
    }

    // 1. this warp's first token: loads out first
    Row r;
    int64_t t = warp;
    if (t < total) load_row<kCross, kSlot, kChunks>(p, t, lane, nchunks, r);

    // 2. per CTA: the crossing slots, as a bitmap over the pool's slots or,
    // for larger pools, a hash set
    int log2 = 0;
    if (need_table && p.last_writer) {
        const int lw = last_writer_log2(total);
        log2 = -lw;
        uint4 *tab4 = reinterpret_cast<uint4 *>(s_table);
        const int keys4 = (1 << lw) / 4;
        const uint4 empty = make_uint4(kEmptySlot, kEmptySlot, kEmptySlot, kEmptySlot);
        for (int i = threadIdx.x; i < 2 * keys4; i += kThreads)
            tab4[i] = i < keys4 ? empty : make_uint4(0, 0, 0, 0);
        __syncthreads();
        for (int64_t i = threadIdx.x; i < total; i += kThreads) {
            const int64_t sl = i < p.num_tokens ? __ldg(p.slot_mapping + i)
                                                : __ldg(p.x_slots + (i - p.num_tokens));
            if (sl >= 0 && sl < p.num_slots)
                last_writer_insert(s_table, lw, static_cast<uint32_t>(sl),
                                   static_cast<uint32_t>(i + 1));
        }
        __syncthreads();
    } else if (need_table) {
        const bool bitmap = p.num_slots <= kBitmapMaxSlots;
        log2 = bitmap ? 0 : table_log2(p.x_tokens);
        uint4 *tab4 = reinterpret_cast<uint4 *>(s_table);
        const int n4 = static_cast<int>(crossing_set_bytes(p.num_slots, p.x_tokens) >> 4);
        const uint32_t f = bitmap ? 0u : kEmptySlot;
        const uint4 fill = make_uint4(f, f, f, f);
        for (int i = threadIdx.x; i < n4; i += kThreads) tab4[i] = fill;
        __syncthreads();
        for (int64_t i = threadIdx.x; i < p.x_tokens; i += kThreads) {
            const int64_t sl = __ldg(p.x_slots + i);
            if (sl >= 0 && sl < p.num_slots) {
                const uint32_t key = static_cast<uint32_t>(sl);
                if (bitmap)
                    atomicOr(&s_table[key >> 5], 1u << (key & 31u));
                else
                    table_insert(s_table, log2, key);
            }
        }
        __syncthreads();
    }
    if (early) {
        // rows and table are in; the scales and every store wait
        wait_for_previous_grid();
        allow_next_grid();
    }
    TensorEncoder kenc, venc;
    if (kWrite && kAmax) {
        // a write in the same pass as the absmax is an in-window write, always
        // at the provisional scale (launch_kv_pass checks it)
        kenc.init_provisional();
        venc.init_provisional();
    } else if (kWrite) {
        resolve_scales(p, kenc, venc);
    }

    const bool small_slots = p.num_slots <= 0x7FFFFFFF;
    uint32_t kacc = 0, vacc = 0;

    // the first token (the only one unless the grid is smaller than the
    // batch), then the rest of the grid-stride loop
    if (t < total) {
        process_row<kAmax, kStage, kWrite, kCross, kChunks>(p, r, t, lane, nchunks, kenc, venc,
                                                            s_table, log2, small_slots, kacc,
                                                            vacc);
    }
    for (t += nwarps; t < total; t += nwarps) {
        load_row<kCross, kSlot, kChunks>(p, t, lane, nchunks, r);
        process_row<kAmax, kStage, kWrite, kCross, kChunks>(p, r, t, lane, nchunks, kenc, venc,
                                                            s_table, log2, small_slots, kacc,
                                                            vacc);
    }

    if (kAmax) {
        __shared__ uint32_t red[2][kWarps];
        uint32_t km = __reduce_max_sync(0xFFFFFFFFu, absmax_bits16(kacc));
        uint32_t vm = __reduce_max_sync(0xFFFFFFFFu, absmax_bits16(vacc));
        const int w = threadIdx.x >> 5;
        if (lane == 0) {
            red[0][w] = km;
            red[1][w] = vm;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
#pragma unroll
            for (int i = 1; i < kWarps; ++i) {
                km = max(km, red[0][i]);
                vm = max(vm, red[1][i]);
            }
            // fp32 bit patterns of non-negative values order like unsigned
            // integers, so an integer atomicMax is a float max here.
            if (km) atomicMax(p.amax_bits + 0, km << 16);
            if (vm) atomicMax(p.amax_bits + 1, vm << 16);
        }
    }
}

// Byte offset of this lane's first 8 codes in the pool entry of `slot`, or -1
// for a slot that is skipped (padding, or out of range: reported).
__device__ __forceinline__ int64_t entry512(const KvPass &p, int64_t slot, int lane) {
    if (slot < 0) return -1;
    if (slot >= p.num_slots) {
        if (lane == 0) atomicOr(&g_error_word, kErrSlot);
        return -1;
    }
    int64_t blk, off;
    if (p.block_shift >= 0) {
        blk = slot >> p.block_shift;
        off = slot & ((int64_t{1} << p.block_shift) - 1);
    } else if (p.num_slots <= 0x7FFFFFFF) {
        const uint32_t s32 = static_cast<uint32_t>(slot);
        const uint32_t b32 = s32 / static_cast<uint32_t>(p.block_size);
        blk = b32;
        off = s32 - b32 * static_cast<uint32_t>(p.block_size);
    } else {
        blk = slot / p.block_size;
        off = slot - blk * p.block_size;
    }
    return blk * p.cache_stride + off * 512 + lane * 8;
}

// This lane's 16 values of one row (chunks a and b) into the pool at `dst`.
__device__ __forceinline__ void write_half512(uint8_t *pool, int64_t dst, const uint4 &a,
                                              const uint4 &b, const TensorEncoder &enc) {
    uint2 oa, ob;
    enc.encode2(a, b, oa, ob);
    *reinterpret_cast<uint2 *>(pool + dst) = oa;
    *reinterpret_cast<uint2 *>(pool + dst + 256) = ob;
}

// The plain quantize-and-scatter of 512-element rows (4 KV heads x 128, the
// pages' shape): nothing but the write, one token per warp and a grid that
// covers every token (575 CTAs of 256 threads for a 4593-token layer, in one
// wave).  The K half is encoded and stored before the V encoder is set up,
// so only one encoder's constants are held at a time.  Same lane mapping
// and encode as the general pass, without its switches; kEarly is
// KvPass::early_loads.  Measured in chains of 16 4593-token layers on one
// box: 3.85 us per layer (general pass, then with two tokens per warp) ->
// 3.59 us; two tokens per warp on 256- or 512-thread CTAs came out at
// 3.72-3.81 us.
template <bool kEarly>
__global__ void __launch_bounds__(kKvThreads, 4) kv_write512_kernel(const KvPass p) {
    const int lane = threadIdx.x & 31;
    const int64_t t = (static_cast<int64_t>(blockIdx.x) * kKvThreads + threadIdx.x) >> 5;
    const bool have = t < p.num_tokens;
    if (!kEarly) {
        // this token's K row (lane 0) and V row (lane 1) into L2 while the
        // previous kernel finishes
        if (lane < 2 && have) prefetch_row<false>(p, t, lane);
        wait_for_previous_grid();
        allow_next_grid();
    }
    Row r;
    if (have) load_row<false, true, 64>(p, t, lane, 64, r);
    if (kEarly) {
        wait_for_previous_grid();
        allow_next_grid();
    }
    float ks = p.k_scale, vs = p.v_scale;
    if (p.scale_dev != nullptr) {
        const float2 sd = *reinterpret_cast<const float2 *>(p.scale_dev);
        ks = sd.x;
        vs = sd.y;
    }
    if (!(ks > 0.0f && vs > 0.0f) && blockIdx.x == 0 && threadIdx.x == 0)
        atomicOr(&g_error_word, kErrScale);
    if (!have) return;
    const int64_t d = entry512(p, r.slot, lane);
    if (d < 0) return;
    {
        TensorEncoder enc;
        enc.init(ks);
        if (enc.ok) write_half512(p.k_pool, d, r.ka, r.kb, enc);
    }
    TensorEncoder enc;
    enc.init(vs);
    if (enc.ok) write_half512(p.v_pool, d, r.va, r.vb, enc);
}

// The in-window pass for 512-element rows: the batch's |K| and |V| maxima
// max-accumulated into the device state, its rows copied (packed) to staging
// with their slots, and its rows written at the provisional scale 2.0, all
// from one read of K and V, one token per warp.  Same result as the general
// pass with all three jobs, without its switches.  kEarly is
// KvPass::early_loads.
template <bool kEarly>
__global__ void __launch_bounds__(kKvThreads, 4) kv_stage512_kernel(const KvPass p) {
    const int lane = threadIdx.x & 31;
    const int64_t t = (static_cast<int64_t>(blockIdx.x) * kKvThreads + threadIdx.x) >> 5;
    const bool have = t < p.num_tokens;
    if (!kEarly) {
        if (lane < 2 && have) prefetch_row<false>(p, t, lane);
        wait_for_previous_grid();
        allow_next_grid();
    }
    Row r;
    uint32_t kacc = 0, vacc = 0;
    if (have) {
        load_row<false, true, 64>(p, t, lane, 64, r);
        kacc = absmax_uint4(absmax_uint4(kacc, r.ka), r.kb);
        vacc = absmax_uint4(absmax_uint4(vacc, r.va), r.vb);
    }
    if (kEarly) {
        wait_for_previous_grid();
        allow_next_grid();
    }
    if (have) {
        const int64_t row = (p.stage_offset + t) * 512 + lane * 8;
        *reinterpret_cast<uint4 *>(p.stage_k + row) = r.ka;
        *reinterpret_cast<uint4 *>(p.stage_k + row + 256) = r.kb;
        *reinterpret_cast<uint4 *>(p.stage_v + row) = r.va;
        *reinterpret_cast<uint4 *>(p.stage_v + row + 256) = r.vb;
        if (lane == 0) p.stage_slots[p.stage_offset + t] = r.slot;
        const int64_t d = entry512(p, r.slot, lane);
        if (d >= 0) {
            TensorEncoder enc;
            enc.init_provisional();
            write_half512(p.k_pool, d, r.ka, r.kb, enc);
            write_half512(p.v_pool, d, r.va, r.vb, enc);
        }
    }
    __shared__ uint32_t red[2][kKvWarps];
    const uint32_t km = __reduce_max_sync(0xFFFFFFFFu, absmax_bits16(kacc));
    const uint32_t vm = __reduce_max_sync(0xFFFFFFFFu, absmax_bits16(vacc));
    const int w = threadIdx.x >> 5;
    if (lane == 0) {
        red[0][w] = km;
        red[1][w] = vm;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t k = red[0][0], v = red[1][0];
#pragma unroll
        for (int i = 1; i < kKvWarps; ++i) {
            k = max(k, red[0][i]);
            v = max(v, red[1][i]);
        }
        // fp32 bit patterns of non-negative values order like unsigned integers
        if (k) atomicMax(p.amax_bits + 0, k << 16);
        if (v) atomicMax(p.amax_bits + 1, v << 16);
    }
}

// The merged freeze launch for 512-element rows with the crossing set as a
// bitmap (pools of at most 2^18 slots): the last staged batch replayed and
// the crossing batch written, at the scales frozen from the device maxima,
// one token per warp.  A staged row whose slot the crossing batch also
// writes is skipped (the crossing row is the later writer).  Same result as
// the general pass's merged launch, without its switches; the K half of a row
// is written before the V encoder is set up.  kEarly is KvPass::early_loads:
// the row and this thread's first crossing slots are loaded before the
// dependency wait.  After the wait the device maxima are loaded and the
// bitmap is built while that load is in flight, so the table adds no memory
// latency of its own (measured per 4593-row launch: 3.96 -> 3.63-3.74 us;
// building the table before the wait put the slot loads and the maxima load
// one after the other).
constexpr int kFreezeThreads = 512;

template <bool kEarly>
__global__ void __launch_bounds__(kFreezeThreads, 2) kv_freeze512_kernel(const KvPass p) {
    constexpr int kWarps = kFreezeThreads / 32;
    extern __shared__ uint32_t s_bits[];   // one bit per pool slot: the crossing slots
    const int lane = threadIdx.x & 31;
    const int64_t t = (static_cast<int64_t>(blockIdx.x) * kFreezeThreads + threadIdx.x) >> 5;
    const int64_t total = p.num_tokens + p.x_tokens;
    const bool have = t < total;
    // with one token per warp, a CTA holds staged rows iff its first row is one
    const bool need_table = static_cast<int64_t>(blockIdx.x) * kWarps < p.num_tokens;
    if (!kEarly) {
        if (lane < 2 && have) prefetch_row<true>(p, t, lane);
        if (need_table && threadIdx.x == 32) {
            const int64_t bytes = p.x_tokens * 8;
            if ((reinterpret_cast<uintptr_t>(p.x_slots) & 15) == 0 && bytes % 16 == 0)
                prefetch_l2_bulk(p.x_slots, static_cast<uint32_t>(bytes));
        }
        wait_for_previous_grid();
        allow_next_grid();
    }
    Row r;
    if (have) load_row<true, true, 64>(p, t, lane, 64, r);
    // this thread's first two crossing slots, loaded with its row
    int64_t s0 = -1, s1 = -1;
    if (need_table) {
        const int64_t i0 = threadIdx.x, i1 = threadIdx.x + kFreezeThreads;
        if (i0 < p.x_tokens) s0 = __ldg(p.x_slots + i0);
        if (i1 < p.x_tokens) s1 = __ldg(p.x_slots + i1);
    }
    if (kEarly) {
        wait_for_previous_grid();
        allow_next_grid();
    }
    // the device maxima, in flight while the bitmap is built
    const uint2 a = *reinterpret_cast<const uint2 *>(p.freeze_amax);
    if (need_table) {
        const int n4 = static_cast<int>((p.num_slots + 127) >> 7);
        uint4 *bits4 = reinterpret_cast<uint4 *>(s_bits);
        for (int i = threadIdx.x; i < n4; i += kFreezeThreads) bits4[i] = make_uint4(0, 0, 0, 0);
        __syncthreads();
        auto insert = [&](int64_t sl) {
            if (sl >= 0 && sl < p.num_slots)
                atomicOr(&s_bits[static_cast<uint32_t>(sl) >> 5],
                         1u << (static_cast<uint32_t>(sl) & 31u));
        };
        insert(s0);
        insert(s1);
        for (int64_t i = threadIdx.x + 2 * kFreezeThreads; i < p.x_tokens; i += kFreezeThreads)
            insert(__ldg(p.x_slots + i));
        __syncthreads();
    }
    const float ks = freeze_scale(a.x, p.headroom);
    const float vs = freeze_scale(a.y, p.headroom);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        if (p.scale_out != nullptr) {
            p.scale_out[0] = ks;
            p.scale_out[1] = vs;
        }
        if (!(ks > 0.0f && vs > 0.0f)) atomicOr(&g_error_word, kErrScale);
    }
    if (!have) return;
    const int64_t slot = r.slot;
    if (t < p.num_tokens && slot >= 0 && slot < p.num_slots &&
        ((s_bits[static_cast<uint32_t>(slot) >> 5] >> (static_cast<uint32_t>(slot) & 31u)) & 1u))
        return;   // the crossing batch writes this slot later
    const int64_t d = entry512(p, slot, lane);
    if (d < 0) return;
    // every row written here went into the maxima the scales come from
    {
        TensorEncoder enc;
        enc.init(ks, true);
        if (enc.ok) write_half512(p.k_pool, d, r.ka, r.kb, enc);
    }
    TensorEncoder enc;
    enc.init(vs, true);
    if (enc.ok) write_half512(p.v_pool, d, r.va, r.vb, enc);
}

// Many layers' writes in one grid: blockIdx.y is the layer, blockIdx.x walks
// that layer's tokens.  Per CTA, thread 0 resolves the layer's scales; the
// rows go through the same code as a one-layer write.
template <int kChunks>
__global__ void __launch_bounds__(kKvThreads, 4) kv_write_layers_kernel(const KvLayers L) {
    const KvLayer &ly = L.layer[blockIdx.y];
    KvPass p;
    p.k = ly.k;
    p.v = ly.v;
    p.key_stride = L.key_stride;
    p.value_stride = L.value_stride;
    p.slot_mapping = ly.slot_mapping;
    p.num_tokens = L.num_tokens;
    p.elems = L.elems;
    p.k_pool = ly.k_pool;
    p.v_pool = ly.v_pool;
    p.block_size = L.block_size;
    p.block_shift = L.block_shift;
    p.cache_stride = L.cache_stride;
    p.num_slots = L.num_slots;
    p.scale_dev = ly.scale_dev;
    p.k_scale = ly.k_scale;
    p.v_scale = ly.v_scale;

    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kKvThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kKvThreads) >> 5;
    const int nchunks = kChunks > 0 ? kChunks : (p.elems >> 3);
    if (warp < p.num_tokens && lane < 2) prefetch_row<false>(p, warp, lane);
    wait_for_previous_grid();
    allow_next_grid();

    Row r;
    int64_t t = warp;
    if (t < p.num_tokens) load_row<false, true, kChunks>(p, t, lane, nchunks, r);
    TensorEncoder kenc, venc;
    resolve_layer_scales(p, kenc, venc);
    const bool small_slots = p.num_slots <= 0x7FFFFFFF;
    uint32_t kacc = 0, vacc = 0;
    if (t < p.num_tokens)
        process_row<false, false, true, false, kChunks>(p, r, t, lane, nchunks, kenc, venc,
                                                        nullptr, 0, small_slots, kacc, vacc);
    for (t += nwarps; t < p.num_tokens; t += nwarps) {
        load_row<false, true, kChunks>(p, t, lane, nchunks, r);
        process_row<false, false, true, false, kChunks>(p, r, t, lane, nchunks, kenc, venc,
                                                        nullptr, 0, small_slots, kacc, vacc);
    }
}

__global__ void calib_init_kernel(float *state) {
    wait_for_previous_grid();
    allow_next_grid();
    state[0] = 0.0f;
    state[1] = 0.0f;
    state[2] = 2.0f;
    state[3] = 2.0f;
}

__global__ void calib_set_kernel(float *state, float a, float b, float c, float d) {
    wait_for_previous_grid();
    allow_next_grid();
    state[0] = a;
    state[1] = b;
    state[2] = c;
    state[3] = d;
}

// ---------------------------------------------------------------------------
// launch geometry


struct DeviceInfo {
    int sms = 0;
};

constexpr int kMaxDevices = 64;
std::mutex g_info_mutex;
DeviceInfo g_info[kMaxDevices];

cudaError_t device_sms(int *sms) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_info_mutex);
    if (g_info[dev].sms == 0) {
        int n = 0;
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        g_info[dev].sms = n;
    }
    *sms = g_info[dev].sms;
    return cudaSuccess;
}

// Resident CTAs per SM of a kernel at a dynamic shared-memory size, cached
// per (device, kernel, size) in a fixed table: no launch path allocates, host
// or device (a full table only means the query is repeated).
struct OccEntry {
    int dev;
    const void *kernel;
    size_t smem;
    int ctas;
};
constexpr int kOccEntries = 512;
std::mutex g_occ_mutex;
OccEntry g_occ[kOccEntries];
int g_occ_used = 0;

template <typename Kernel>
cudaError_t resident_ctas(Kernel kernel, int threads, size_t smem, int *out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const void *key = reinterpret_cast<const void *>(kernel);
    std::lock_guard<std::mutex> lock(g_occ_mutex);
    for (int i = 0; i < g_occ_used; ++i) {
        if (g_occ[i].dev == dev && g_occ[i].kernel == key && g_occ[i].smem == smem) {
            *out = g_occ[i].ctas;
            return cudaSuccess;
        }
    }
    if (smem > 48 * 1024) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        if (e != cudaSuccess) return e;
    }
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem);
    if (e != cudaSuccess) return e;
    *out = n > 0 ? n : 1;
    if (g_occ_used < kOccEntries) g_occ[g_occ_used++] = OccEntry{dev, key, smem, *out};
    return cudaSuccess;
}

// Dynamic shared memory to request (and leave unused) so that at most
// `max_ctas` CTAs of `kernel` are resident per SM: the smallest size at which
// max_ctas + 1 of them no longer fit in an SM's shared memory.  0 when no more
// than max_ctas fit anyway, or when the size would pass the default per-CTA
// limit.  Cached per (device, kernel) in a fixed table like the above.
struct CapEntry {
    int dev;
    const void *kernel;
    size_t smem;
};
constexpr int kCapEntries = 64;
std::mutex g_cap_mutex;
CapEntry g_cap[kCapEntries];
int g_cap_used = 0;

template <typename Kernel>
cudaError_t cap_smem(Kernel kernel, int threads, int max_ctas, size_t *smem) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const void *key = reinterpret_cast<const void *>(kernel);
    std::lock_guard<std::mutex> lock(g_cap_mutex);
    for (int i = 0; i < g_cap_used; ++i) {
        if (g_cap[i].dev == dev && g_cap[i].kernel == key) {
            *smem = g_cap[i].smem;
            return cudaSuccess;
        }
    }
    size_t want = 0;
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0);
    if (e != cudaSuccess) return e;
    if (n > max_ctas) {
        int per_sm = 0, reserved = 0;
        cudaFuncAttributes fa;
        e = cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
        if (e == cudaSuccess)
            e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
        if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, kernel);
        if (e != cudaSuccess) return e;
        const size_t per_cta = static_cast<size_t>(per_sm) / (max_ctas + 1) + 1;
        const size_t fixed = static_cast<size_t>(reserved) + fa.sharedSizeBytes;
        const size_t x = per_cta > fixed ? (per_cta - fixed + 127) & ~size_t{127} : 0;
        if (x > 0 && x + fa.sharedSizeBytes <= 48 * 1024) {
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, x);
            if (e != cudaSuccess) return e;
            if (n == max_ctas) want = x;
        }
    }
    *smem = want;
    if (g_cap_used < kCapEntries) g_cap[g_cap_used++] = CapEntry{dev, key, want};
    return cudaSuccess;
}

template <typename Kernel>
cudaError_t grid_for(Kernel kernel, int threads, size_t smem, int64_t ctas_wanted, int *grid) {
    int sms = 0, per_sm = 0;
    cudaError_t e = device_sms(&sms);
    if (e != cudaSuccess) return e;
    e = resident_ctas(kernel, threads, smem, &per_sm);
    if (e != cudaSuccess) return e;
    const int64_t cap = static_cast<int64_t>(sms) * per_sm;
    int64_t g = ctas_wanted < cap ? ctas_wanted : cap;
    if (g < 1) g = 1;
    *grid = static_cast<int>(g);
    return cudaSuccess;
}

// Launch with programmatic stream serialization (see wait_for_previous_grid)
// and count it.
template <typename... Params, typename... Args>
cudaError_t launch(void (*kernel)(Params...), int grid, int block, size_t smem,
                   cudaStream_t stream, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(static_cast<unsigned>(block));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e == cudaSuccess) g_launch_count.fetch_add(1, std::memory_order_relaxed);
    return e;
}

template <bool A, bool S, bool W, bool X>
cudaError_t launch_kv_variant(const KvPass &p, cudaStream_t stream) {
    constexpr int kThreads = X ? 512 : kKvThreads;
    constexpr int kWarps = kThreads / 32;
    auto kernel = p.elems == 512 ? kv_pass_kernel<A, S, W, X, 64, kThreads>
                                 : kv_pass_kernel<A, S, W, X, 0, kThreads>;
    const int64_t tokens = p.num_tokens + (X ? p.x_tokens : 0);
    const int64_t wanted = (tokens + kWarps - 1) / kWarps;
    const size_t smem =
        !X ? 0
           : p.last_writer ? (size_t{8} << last_writer_log2(tokens))
                           : static_cast<size_t>(crossing_set_bytes(p.num_slots, p.x_tokens));
    int grid = 1;
    cudaError_t e = grid_for(kernel, kThreads, smem, wanted, &grid);
    if (e != cudaSuccess) return e;
    return launch(kernel, grid, kThreads, smem, stream, p);
}

}  // namespace

cudaError_t launch_group_quant(const uint16_t *x, int64_t x_row_stride, uint8_t *q,
                               float *scales, int64_t m, int64_t k, cudaStream_t stream) {
    const int64_t gpr = k / 128;
    const int64_t total = m * gpr;
    if (total == 0) return cudaSuccess;
    const int64_t warps = (total + 7) / 8;
    const int64_t wanted = (warps * 32 + kGqThreads - 1) / kGqThreads;
    int grid = 1;
    cudaError_t e;
    auto kernel = x_row_stride == k ? group_quant_kernel<true> : group_quant_kernel<false>;
    e = grid_for(kernel, kGqThreads, 0, wanted, &grid);
    if (e != cudaSuccess) return e;
    return launch(kernel, grid, kGqThreads, 0, stream, x, x_row_stride, q, scales, total,
                  static_cast<uint32_t>(gpr));
}

cudaError_t launch_group_quant_kmajor(const uint16_t *x, int64_t x_row_stride, uint8_t *q,
                                      float *scales_km, int64_t m, int64_t m_pad, int64_t k,
                                      cudaStream_t stream) {
    const int64_t gpr = k / 128;
    if (m_pad == 0) return cudaSuccess;
    const int64_t warps = ((m_pad + 7) / 8) * gpr;
    const int64_t wanted = (warps * 32 + kGqThreads - 1) / kGqThreads;
    int grid = 1;
    cudaError_t e = grid_for(group_quant_kmajor_kernel, kGqThreads, 0, wanted, &grid);
    if (e != cudaSuccess) return e;
    return launch(group_quant_kmajor_kernel, grid, kGqThreads, 0, stream, x, x_row_stride, q,
                  scales_km, m, m_pad, static_cast<uint32_t>(gpr));
}

bool can_merge_crossing(const KvPass &p) {
    return p.x_tokens > 0 && p.x_tokens <= kMaxMergedCrossing && p.num_slots <= 0x7FFFFFFF;
}

cudaError_t launch_kv_pass(const KvPass &p, cudaStream_t stream) {
    const bool publish = p.do_write && p.freeze_amax != nullptr && p.scale_out != nullptr;
    if (p.last_writer) {
        if (!p.do_write || p.do_amax || p.do_stage || p.num_slots > 0x7FFFFFFF ||
            p.num_tokens + p.x_tokens > kMaxLastWriterTokens ||
            (p.x_tokens > 0 && p.x_slots == nullptr))
            return cudaErrorInvalidValue;
        if (p.num_tokens + p.x_tokens == 0 && p.scale_out == nullptr) return cudaSuccess;
        return launch_kv_variant<false, false, true, true>(p, stream);
    }
    const bool cross = p.do_write && p.x_tokens > 0;
    if (cross) {
        if (!can_merge_crossing(p) || p.do_amax || p.do_stage) return cudaErrorInvalidValue;
        if (p.elems == 512 && p.freeze_amax != nullptr && p.num_slots <= kBitmapMaxSlots) {
            auto kernel = p.early_loads ? kv_freeze512_kernel<true> : kv_freeze512_kernel<false>;
            const int64_t grid = (p.num_tokens + p.x_tokens + kFreezeThreads / 32 - 1) /
                                 (kFreezeThreads / 32);
            const size_t smem = static_cast<size_t>((p.num_slots + 127) >> 7) * 16;
            return launch(kernel, static_cast<int>(grid), kFreezeThreads, smem, stream, p);
        }
        return launch_kv_variant<false, false, true, true>(p, stream);
    }
    if (p.num_tokens == 0 && !publish) return cudaSuccess;
    if (p.do_amax && p.do_write &&
        (p.k_scale != 2.0f || p.v_scale != 2.0f || p.scale_dev != nullptr ||
         p.freeze_amax != nullptr))
        return cudaErrorInvalidValue;   // in-window writes take the provisional scale
    if (p.do_amax && p.do_stage && p.do_write && p.elems == 512) {
        auto kernel = p.early_loads ? kv_stage512_kernel<true> : kv_stage512_kernel<false>;
        const int64_t grid = (p.num_tokens + kKvWarps - 1) / kKvWarps;   // one token per warp
        if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
        // At most four CTAs per SM.  Five fit at this kernel's register count,
        // and when it starts while the previous launch still holds some SMs,
        // the SMs freed first take five (40 tokens) and the rest three: the
        // pass ends with the loaded ones (measured in the prefill step: last
        // CTA 1.2 us after the median one; capped at four, the pass 3.81 ->
        // 3.60-3.73 us and the step 3.5% shorter).
        size_t smem = 0;
        const cudaError_t e = cap_smem(kernel, kKvThreads, 4, &smem);
        if (e != cudaSuccess) return e;
        return launch(kernel, static_cast<int>(grid), kKvThreads, smem, stream, p);
    }
    if (p.do_write && !p.do_amax && !p.do_stage && p.elems == 512 && p.freeze_amax == nullptr) {
        auto kernel = p.early_loads ? kv_write512_kernel<true> : kv_write512_kernel<false>;
        const int64_t grid = (p.num_tokens + kKvWarps - 1) / kKvWarps;   // one token per warp
        if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
        return launch(kernel, static_cast<int>(grid), kKvThreads, 0, stream, p);
    }
    if (p.do_amax && p.do_stage && p.do_write) return launch_kv_variant<true, true, true, false>(p, stream);
    if (p.do_amax && p.do_stage) return launch_kv_variant<true, true, false, false>(p, stream);
    if (p.do_amax && p.do_write) return launch_kv_variant<true, false, true, false>(p, stream);
    if (p.do_amax) return launch_kv_variant<true, false, false, false>(p, stream);
    if (p.do_write) return launch_kv_variant<false, false, true, false>(p, stream);
    return cudaErrorInvalidValue;
}

cudaError_t enqueue_freeze_replay(const KvPass &base, const uint16_t *stage_k,
                                  const uint16_t *stage_v, const int64_t *stage_slots,
                                  const int64_t *counts, int64_t num_batches,
                                  const KvPass *crossing, bool chained, cudaStream_t stream,
                                  int64_t *rewritten) {
    KvPass p = base;
    p.do_write = true;
    p.key_stride = p.elems;   // staging rows are packed
    p.value_stride = p.elems;
    p.early_loads = chained;

    int64_t used = 0, last = -1, with_rows = 0;
    for (int64_t i = 0; i < num_batches; ++i) {
        used += counts[i];
        if (counts[i] > 0) {
            last = i;
            ++with_rows;
        }
    }
    KvPass probe = p;
    if (crossing != nullptr) probe.x_tokens = crossing->num_tokens;
    const bool merge = crossing != nullptr && crossing->num_tokens > 0 &&
                       crossing->elems == p.elems && can_merge_crossing(probe);
    auto with_crossing = [&](KvPass q) {
        q.xk = crossing->k;
        q.xv = crossing->v;
        q.x_key_stride = crossing->key_stride;
        q.x_value_stride = crossing->value_stride;
        q.x_slots = crossing->slot_mapping;
        q.x_tokens = crossing->num_tokens;
        return q;
    };
    auto crossing_alone = [&]() {
        KvPass x = *crossing;
        x.early_loads = chained;
        return launch_kv_pass(x, stream);
    };
    cudaError_t e = cudaSuccess;
    *rewritten = 0;

    const int64_t whole_rows = used + (merge ? crossing->num_tokens : 0);
    if (with_rows >= 2 && whole_rows <= kMaxLastWriterTokens && p.num_slots <= 0x7FFFFFFF) {
        // the whole window in one launch, each slot from its last writer
        KvPass q = merge ? with_crossing(p) : p;
        q.k = stage_k;
        q.v = stage_v;
        q.slot_mapping = stage_slots;
        q.num_tokens = used;
        q.last_writer = true;
        if ((e = launch_kv_pass(q, stream)) != cudaSuccess) return e;
        *rewritten = used;
        if (crossing != nullptr && !merge) return crossing_alone();
        return cudaSuccess;
    }
    if (merge && last < 0) {
        // nothing staged with rows: the crossing batch alone, publishing the scales
        KvPass q = with_crossing(p);
        q.num_tokens = 0;
        return launch_kv_pass(q, stream);
    }
    bool published = false;
    int64_t off = 0;
    for (int64_t i = 0; i < num_batches; ++i) {
        const int64_t n = counts[i];
        if (n > 0 || !published) {
            p.k = stage_k + off * p.elems;
            p.v = stage_v + off * p.elems;
            p.slot_mapping = stage_slots + off;
            p.num_tokens = n;
            const KvPass q = (merge && i == last) ? with_crossing(p) : p;
            if ((e = launch_kv_pass(q, stream)) != cudaSuccess) return e;
            *rewritten += n;
            published = true;
        }
        off += n;
    }
    if (!published) {
        p.num_tokens = 0;
        if ((e = launch_kv_pass(p, stream)) != cudaSuccess) return e;
    }
    if (crossing != nullptr && !merge) return crossing_alone();
    return cudaSuccess;
}

cudaError_t launch_kv_write_layers(const KvLayers &p, cudaStream_t stream) {
    if (p.num_tokens == 0 || p.num_layers == 0) return cudaSuccess;
    auto kernel = p.elems == 512 ? kv_write_layers_kernel<64> : kv_write_layers_kernel<0>;
    const int64_t wanted = (p.num_tokens + kKvWarps - 1) / kKvWarps;
    int gx = 1;
    cudaError_t e = grid_for(kernel, kKvThreads, 0, wanted, &gx);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(gx), static_cast<unsigned>(p.num_layers));
    cfg.blockDim = dim3(kKvThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kernel, p);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e == cudaSuccess) g_launch_count.fetch_add(1, std::memory_order_relaxed);
    return e;
}

cudaError_t launch_calib_init(float *state_dev, cudaStream_t stream) {
    return launch(calib_init_kernel, 1, 1, 0, stream, state_dev);
}

cudaError_t launch_calib_set(float *state_dev, float a, float b, float c, float d,
                             cudaStream_t stream) {
    return launch(calib_set_kernel, 1, 1, 0, stream, state_dev, a, b, c, d);
}

int64_t launch_count() { return g_launch_count.load(std::memory_order_relaxed); }

cudaError_t read_device_error(uint32_t *bits, bool clear) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(bits, g_error_word, sizeof(uint32_t));
    if (e != cudaSuccess) return e;
    if (clear) {
        const uint32_t zero = 0;
        e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(uint32_t));
    }
    return e;
}

}  // namespace fp8q
