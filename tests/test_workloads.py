"""The seeded input recipe produces the stated shapes and structure (no GPU)."""
import numpy as np

import oracle
import workloads


def test_tiny_inputs():
    x = workloads.tiny_quant()
    assert x.shape == (16, 5120) and x.dtype == np.uint16
    spec, b = workloads.tiny_kv()
    assert b.k.shape == (16, 512) and spec.num_slots == 1024
    s = b.slot_mapping
    assert (s == -1).sum() == 2 and len(set(s[s >= 0].tolist())) == 14
    assert np.array_equal(workloads.tiny_quant(), x)          # seeded


def test_prefill_structure():
    x = workloads.prefill_quant()
    assert x.shape == (4593, 5120)
    zero = workloads.prefill_zero_groups()
    assert zero.size == 184
    g = oracle.bf16_to_f32(x).reshape(-1, 128)
    assert np.all(g[zero] == 0) and np.all(np.signbit(g[zero]) == False)  # noqa: E712
    nz = np.abs(g).max(axis=1) > 0
    assert nz.sum() == g.shape[0] - 184
    # about 0.5% of the elements are x30 outliers
    frac = (np.abs(g) > 8).mean()
    assert 0.003 < frac < 0.007


def test_calibration_window_structure():
    spec, batches, blocks = workloads.calib_window()
    sizes = [b.num_tokens for b in batches]
    assert sizes[0] == 13 and all(t == 32 for t in sizes[1:])
    assert sum(sizes[:8]) == 237 and sum(sizes[:9]) == 269
    shared = set(batches[1].slot_mapping) & set(batches[5].slot_mapping)
    assert len(shared) == 16
    others = [set(b.slot_mapping) for i, b in enumerate(batches) if i not in (1, 5)]
    for i, a in enumerate(others):
        for b in others[i + 1:]:
            assert not (a & b)
    k3 = oracle.bf16_to_f32(batches[2].k)
    assert k3.max() == 600.0
    kall = max(np.abs(oracle.bf16_to_f32(b.k)).max() for b in batches[:9])
    assert kall == 600.0


def test_large_layer_structure():
    b = workloads.large_kv_layer(3)
    assert b.k.shape == (4593, 512)
    s = b.slot_mapping
    assert len(set(s.tolist())) == 4593
    blocks = np.unique(s // 16)
    assert blocks.size == 288 and blocks.max() < 8192
    last_block = s[-1] // 16
    assert (s // 16 == last_block).sum() == 1
    assert sum(workloads.LARGE_CHUNKS) == 4593
