"""Pin of the oracle's E4M3 encoder against CUDA's own conversion on the GPU.

A small test-only kernel (compiled here, not part of the library) converts fp32
values with CUDA's `__nv_cvt_float2_to_fp8x2(..., __NV_SATFINITE, __NV_E4M3)`.
Its codes must equal the oracle's for:
  * every fp32 bit pattern, both signs, in the binades that can round to a
    nonzero code below saturation: |y| in [2^-11, 2^9) (about 352 M values);
  * a random sample of all other finite fp32 values (underflow to +-0,
    saturation to +-448), and the boundaries around 464.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

_SRC = r"""
#include <cuda_fp8.h>
#include <torch/extension.h>

__global__ void cvt_kernel(const float2 *y, __nv_fp8x2_storage_t *out, int64_t n) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = __nv_cvt_float2_to_fp8x2(y[i], __NV_SATFINITE, __NV_E4M3);
}

torch::Tensor cuda_e4m3(torch::Tensor y) {
    TORCH_CHECK(y.is_cuda() && y.dtype() == torch::kFloat32 && y.is_contiguous() && y.numel() % 2 == 0);
    auto out = torch::empty({y.numel()}, y.options().dtype(torch::kUInt8));
    const int64_t n = y.numel() / 2;
    if (n > 0)
        cvt_kernel<<<(unsigned)((n + 255) / 256), 256>>>(
            reinterpret_cast<const float2 *>(y.data_ptr<float>()),
            reinterpret_cast<__nv_fp8x2_storage_t *>(out.data_ptr<uint8_t>()), n);
    return out;
}
"""

_ext = None


def _cuda_e4m3(y_dev: torch.Tensor) -> np.ndarray:
    global _ext
    if _ext is None:
        from torch.utils.cpp_extension import load_inline
        _ext = load_inline(name="e4m3_hw_pin", cpp_sources="torch::Tensor cuda_e4m3(torch::Tensor y);",
                           cuda_sources=_SRC, functions=["cuda_e4m3"],
                           extra_cuda_cflags=["-gencode", "arch=compute_100a,code=sm_100a"],
                           verbose=False)
    out = _ext.cuda_e4m3(y_dev)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _check_bits(bits: np.ndarray):
    y = bits.view(np.float32)
    got = _cuda_e4m3(torch.from_numpy(y).cuda())
    want = oracle.e4m3_encode(y)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, (f"{bad.size} mismatches, first y={y[bad[0]]!r} "
                           f"(0x{bits[bad[0]]:08x}): cuda 0x{got[bad[0]]:02x} oracle 0x{want[bad[0]]:02x}")


def test_every_fp32_in_the_rounding_binades():
    lo = np.uint32(127 - 11) << np.uint32(23)     # 2^-11
    hi = np.uint32(127 + 9) << np.uint32(23)      # 2^9
    chunk = 1 << 25
    for sign in (np.uint32(0), np.uint32(0x80000000)):
        for start in range(int(lo), int(hi), chunk):
            stop = min(start + chunk, int(hi))
            bits = np.arange(start, stop, dtype=np.uint32) | sign
            _check_bits(bits)


def test_sampled_finite_fp32_and_saturation_boundaries():
    g = np.random.Generator(np.random.Philox(2026))
    bits = g.integers(0, 1 << 32, size=1 << 24, dtype=np.uint64).astype(np.uint32)
    bits = bits[(bits & 0x7F800000) != 0x7F800000]          # finite values only
    edges = np.array([448.0, 455.99, 456.0, 463.99, 464.0, 464.01, 480.0, 1e6, 3.4e38,
                      2.0 ** -10, 2.0 ** -10 * 1.0001, 3 * 2.0 ** -10, 2.0 ** -9, 2.0 ** -7,
                      0.0, 2.0 ** -149], dtype=np.float32)
    edges = np.concatenate([edges, -edges])
    _check_bits(np.concatenate([bits, edges.view(np.uint32)]))
