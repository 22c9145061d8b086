"""Helpers of the GPU parity tests: move seeded numpy inputs to the device and
bring results back as numpy bytes."""
import numpy as np
import torch


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> CUDA bfloat16 tensor of the same shape."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    torch.cuda.synchronize()
    if t.dtype == torch.float8_e4m3fn:
        t = t.view(torch.uint8)
    return t.cpu().numpy()


def f32_bits(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def first_mismatch(a: np.ndarray, b: np.ndarray) -> str:
    bad = np.flatnonzero(a.reshape(-1) != b.reshape(-1))
    if bad.size == 0:
        return "none"
    i = bad[0]
    return f"{bad.size} mismatches, first at flat {i}: got {a.reshape(-1)[i]!r} want {b.reshape(-1)[i]!r}"
