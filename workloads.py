"""Seeded synthetic inputs for the FP8 quantization workloads.

Shared by the tests, the smoke check and the benchmark, and by both the CPU
oracle and the CUDA path.  This module draws numbers and lays out buffers; it
holds none of the quantization arithmetic.

Recipe.  Values are drawn in fp32 from numpy's Philox counter-based generator,
keyed by ``(workload index, layer, purpose)`` through a SeedSequence, then
rounded to bf16 (round-to-nearest-even, via torch's CPU cast) and carried as
uint16 bit patterns.  "N(0, s)" means mean 0 and standard deviation s.  Pools
start filled with the sentinel byte 0x5A.

Workloads (index: name):
  0 tiny          quant 16 x 5120 ~ N(0,1); KV 16 tokens x 4 heads x 128 dims
                  ~ N(0,2) into 64 blocks x 16 slots at scale 2.0; 16 distinct
                  random slots in random order, two of them then set to -1.
  1 prefill       quant 4593 x 5120 ~ N(0,1); each element x30 with
                  probability 0.005; every group whose flat index m*40+j is a
                  multiple of 1000 set to +0 (184 groups).
  2 decode sweep  quant M in {1,2,4,8,16} x K in {5120,16384} ~ N(0,1).
  3 calibration   one layer, 4 heads x 128 dims ~ N(0,1.5); each element
                  replaced with probability 1e-4 by +-U(100,600); one element
                  of batch 3 set to exactly 600.  Batches of 13, then 32 tokens;
                  each batch is a new sequence whose slots come from a block
                  allocator over 128 blocks x 16 slots (a seeded shuffled free
                  stack).  After batch 5, batch 2's second block is freed and
                  batch 6 receives it again, so batches 2 and 6 share 16 slots.
  4 large KV      16 layers x 4593 tokens x 4 heads x 128 dims ~ N(0,1), each
                  element x20 with probability 0.001; 8192 blocks x 16 slots
                  per layer; 288 distinct random blocks per layer, filled in
                  order (the last block holds one token).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

SENTINEL = 0x5A

TINY, PREFILL, DECODE, CALIB, LARGE_KV = 0, 1, 2, 3, 4

PREFILL_M, PREFILL_K = 4593, 5120
DECODE_MS = (1, 2, 4, 8, 16)
DECODE_KS = (5120, 16384)
KV_HEADS, HEAD_DIM = 4, 128


def generator(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(np.random.SeedSequence(list(key))))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest-even) and return the uint16 bits."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_of(values) -> np.ndarray:
    """bf16 bits of values that are exactly representable in bf16."""
    x = np.asarray(values, dtype=np.float32)
    bits = to_bf16_bits(x)
    back = bits.astype(np.uint32) << 16
    assert np.array_equal(back, x.view(np.uint32)), "value is not representable in bf16"
    return bits


def new_pool(num_blocks: int, block_size: int, heads: int, dim: int) -> np.ndarray:
    return np.full((num_blocks, block_size, heads, dim), SENTINEL, dtype=np.uint8)


# --------------------------------------------------------------------------
# activation quantization inputs


def normal_activation(m: int, k: int, *key: int, std: float = 1.0) -> np.ndarray:
    g = generator(*key)
    x = g.standard_normal((m, k), dtype=np.float32) * np.float32(std)
    return to_bf16_bits(x)


def tiny_quant() -> np.ndarray:
    return normal_activation(16, 5120, TINY, 0, 0)


def prefill_quant(m: int = PREFILL_M, k: int = PREFILL_K) -> np.ndarray:
    g = generator(PREFILL, 0, 0)
    x = g.standard_normal((m, k), dtype=np.float32)
    outlier = g.random((m, k), dtype=np.float32) < np.float32(0.005)
    x[outlier] *= np.float32(30.0)
    groups = k // 128
    flat = np.arange(m * groups)
    zero = flat[flat % 1000 == 0]
    xv = x.reshape(m * groups, 128)
    xv[zero] = np.float32(0.0)
    return to_bf16_bits(x)


def prefill_zero_groups(m: int = PREFILL_M, k: int = PREFILL_K) -> np.ndarray:
    flat = np.arange(m * (k // 128))
    return flat[flat % 1000 == 0]


def decode_quant(m: int, k: int) -> np.ndarray:
    return normal_activation(m, k, DECODE, m, k)


# --------------------------------------------------------------------------
# KV inputs


@dataclass
class KvBatchInput:
    k: np.ndarray            # uint16 [T, row_stride]
    v: np.ndarray
    slot_mapping: np.ndarray  # int64 [T]
    key_stride: int
    value_stride: int

    @property
    def num_tokens(self) -> int:
        return int(self.slot_mapping.shape[0])


@dataclass
class PoolSpec:
    num_blocks: int
    block_size: int
    heads: int
    dim: int

    @property
    def elems(self) -> int:
        return self.heads * self.dim

    @property
    def cache_stride(self) -> int:
        return self.block_size * self.elems

    @property
    def num_slots(self) -> int:
        return self.num_blocks * self.block_size

    def new_pool(self) -> np.ndarray:
        return new_pool(self.num_blocks, self.block_size, self.heads, self.dim)


def kv_rows(t: int, heads: int, dim: int, std: float, g: np.random.Generator,
            row_pad: int = 0) -> np.ndarray:
    x = g.standard_normal((t, heads * dim), dtype=np.float32) * np.float32(std)
    if row_pad:
        pad = g.standard_normal((t, row_pad), dtype=np.float32)
        x = np.concatenate([x, pad], axis=1)
    return x


def tiny_kv(row_pad: int = 0):
    """16 tokens, 4 x 128, ~N(0,2), 64 blocks x 16, two padding slots."""
    spec = PoolSpec(64, 16, KV_HEADS, HEAD_DIM)
    g = generator(TINY, 0, 1)
    k = to_bf16_bits(kv_rows(16, KV_HEADS, HEAD_DIM, 2.0, g, row_pad))
    v = to_bf16_bits(kv_rows(16, KV_HEADS, HEAD_DIM, 2.0, g, row_pad))
    slots = g.choice(spec.num_slots, size=16, replace=False).astype(np.int64)
    pad_pos = g.choice(16, size=2, replace=False)
    slots[pad_pos] = -1
    stride = spec.elems + row_pad
    return spec, KvBatchInput(k, v, slots, stride, stride)


class BlockAllocator:
    """A stack of free blocks, shuffled once from a seed."""

    def __init__(self, num_blocks: int, g: np.random.Generator) -> None:
        self.free = list(g.permutation(num_blocks).astype(np.int64))

    def alloc(self) -> int:
        return int(self.free.pop())

    def release(self, block: int) -> None:
        self.free.append(int(block))


CALIB_WINDOW = 256
CALIB_BATCHES = (13,) + (32,) * 10   # 8 staged, batch 9 crosses, 2 after


def calib_window(batch_sizes=CALIB_BATCHES, row_pad: int = 0, recycle=None,
                 num_blocks: int = 128, heads: int = KV_HEADS, dim: int = HEAD_DIM):
    """Calibration-window workload: returns (spec, batches, blocks per batch).

    ``recycle`` maps a batch number to (earlier batch number, block index):
    before that batch, the earlier batch's block is freed and is the first
    block the batch receives.  The default reuses batch 2's second block in
    batch 6.  ``num_blocks`` sizes the pool (128 blocks of 16 slots for the
    256-token window; larger windows need a larger pool); ``heads`` x ``dim``
    is the row shape (4 x 128 in the workload)."""
    recycle = {6: (2, 1)} if recycle is None else recycle
    spec = PoolSpec(num_blocks, 16, heads, dim)
    g = generator(CALIB, 0, 0)
    alloc = BlockAllocator(spec.num_blocks, generator(CALIB, 0, 1))
    batches = []
    blocks_of = []
    for b, t in enumerate(batch_sizes, start=1):
        if b in recycle:
            src, idx = recycle[b]
            alloc.release(blocks_of[src - 1][idx])
        nblk = -(-t // spec.block_size)
        blocks = [alloc.alloc() for _ in range(nblk)]
        blocks_of.append(blocks)
        slots = np.array([blocks[i // spec.block_size] * spec.block_size
                          + i % spec.block_size for i in range(t)], dtype=np.int64)
        x = []
        for _ in range(2):
            rows = kv_rows(t, spec.heads, spec.dim, 1.5, g)
            hit = g.random(rows.shape, dtype=np.float32) < np.float32(1e-4)
            mag = g.uniform(100.0, 600.0, size=rows.shape).astype(np.float32)
            sgn = np.where(g.random(rows.shape) < 0.5, -1.0, 1.0).astype(np.float32)
            rows[hit] = (mag * sgn)[hit]
            x.append(rows)
        if b == 3 and t > 5:
            x[0][5, 77] = np.float32(600.0)
        kb, vb = (to_bf16_bits(r) for r in x)
        if row_pad:
            kb = np.concatenate([kb, np.zeros((t, row_pad), np.uint16)], axis=1)
            vb = np.concatenate([vb, np.zeros((t, row_pad), np.uint16)], axis=1)
        stride = spec.elems + row_pad
        batches.append(KvBatchInput(kb, vb, slots, stride, stride))
    return spec, batches, blocks_of


LARGE_LAYERS = 16
LARGE_TOKENS = 4593
LARGE_NUM_BLOCKS = 8192
LARGE_WINDOW_REQUEST = 8192
LARGE_CHUNKS = (4095, 498)


def large_kv_spec() -> PoolSpec:
    return PoolSpec(LARGE_NUM_BLOCKS, 16, KV_HEADS, HEAD_DIM)


def large_kv_layer(layer: int, tokens: int = LARGE_TOKENS) -> KvBatchInput:
    """One layer's prefill K, V and slot mapping."""
    spec = large_kv_spec()
    g = generator(LARGE_KV, layer, 0)
    x = []
    for _ in range(2):
        rows = kv_rows(tokens, spec.heads, spec.dim, 1.0, g)
        hit = g.random(rows.shape, dtype=np.float32) < np.float32(0.001)
        rows[hit] *= np.float32(20.0)
        x.append(rows)
    nblk = -(-tokens // spec.block_size)
    blocks = generator(LARGE_KV, layer, 1).choice(spec.num_blocks, size=nblk, replace=False)
    i = np.arange(tokens)
    slots = (blocks[i // spec.block_size] * spec.block_size + i % spec.block_size).astype(np.int64)
    kb, vb = (to_bf16_bits(r) for r in x)
    return KvBatchInput(kb, vb, slots, spec.elems, spec.elems)


def split_batch(b: KvBatchInput, sizes) -> list[KvBatchInput]:
    out, start = [], 0
    for n in sizes:
        out.append(KvBatchInput(b.k[start:start + n], b.v[start:start + n],
                                b.slot_mapping[start:start + n], b.key_stride,
                                b.value_stride))
        start += n
    assert start == b.num_tokens
    return out
