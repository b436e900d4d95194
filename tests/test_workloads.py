"""The synthetic input recipe: seeded, reproducible, and with the sizes and
structure the design states (expert counts, ragged groups, outliers, zeroed
tiles).  These are the draws every parity test and the bench start from."""
import numpy as np
import pytest
import torch

from mxfp8_grouped_gemm_quantize_b200 import workloads as wl


def test_tiny_has_an_empty_expert_and_no_multiple_of_32():
    w = wl.tiny()
    assert w.counts.tolist() == [0, 7, 21, 36] and w.M == 64
    assert w.offsets.tolist() == [0, 0, 7, 28, 64]


def test_ds_v3_16b_routing_shape():
    w = wl.ds_v3_16b()
    assert w.E == 64 and w.M == 8192 * 6
    assert w.counts.min() >= 1 and w.counts.max() < w.M
    assert int(np.ceil(w.counts / 128).sum()) == 414          # 128-row tiles of the forward pass
    assert not np.any(w.counts % 128 == 0)                     # every group has a ragged last tile
    assert [(L.name, L.N, L.K) for L in w.layers] == [("gate_up", 2816, 2048), ("down", 2048, 1408)]


def test_ds_v3_16b_counts_match_the_per_token_routing():
    """The counts of the workload and the per-token routing used by the MoE
    dispatch come from the same draws."""
    w, r = wl.ds_v3_16b(), wl.routing("ds-v3-16b")
    assert r.idx.shape == (8192, 6) and r.E == 64
    np.testing.assert_array_equal(np.bincount(r.idx.reshape(-1), minlength=64), w.counts)
    assert np.all(np.sort(r.idx, axis=1)[:, 1:] != np.sort(r.idx, axis=1)[:, :-1])   # distinct per token
    np.testing.assert_allclose(r.w.sum(axis=1), 1.0, rtol=1e-6)


def test_ds_v3_671b_is_one_gpus_balanced_share():
    w = wl.ds_v3_671b()
    assert w.E == 32 and w.M == 16384
    assert w.counts.max() > 4 * w.counts.min()                 # Zipf-skewed, not balanced per expert
    assert w.x_outlier_frac == 1e-3 and w.x_outlier_scale == 100.0


def test_llama4_scout_top1():
    w, r = wl.llama4_scout(), wl.routing("llama4-scout")
    assert w.E == 16 and w.M == 16384 and r.k == 1
    np.testing.assert_array_equal(np.bincount(r.idx.reshape(-1), minlength=16), w.counts)


@pytest.mark.parametrize("name", sorted(wl.WORKLOADS))
def test_draws_are_reproducible(name):
    a, b = wl.WORKLOADS[name](), wl.WORKLOADS[name]()
    np.testing.assert_array_equal(a.counts, b.counts)
    if name in ("tiny",):
        X1, W1, dY1 = wl.layer_tensors(a, a.layers[0])
        X2, W2, dY2 = wl.layer_tensors(b, b.layers[0])
        assert torch.equal(X1, X2) and torch.equal(W1, W2) and torch.equal(dY1, dY2)


def test_outliers_scale_the_requested_fraction():
    x = wl.normal_bf16((256, 512), 1.0, 3)
    y = wl.with_outliers(x.clone(), 1e-3, 100.0, 4)
    changed = (y != x).sum().item()
    assert 1 <= changed <= round(1e-3 * x.numel())             # positions may repeat
    ratio = (y.float()[y != x] / x.float()[y != x]).numpy()
    np.testing.assert_allclose(ratio, 100.0, rtol=1e-2)


def test_sweep_tensor_zeroes_aligned_32x32_tiles():
    x = wl.sweep_tensor(4096, 2048)
    t = x.float().reshape(128, 32, 64, 32).abs().amax(dim=(1, 3))
    zero_tiles = int((t == 0).sum())
    assert zero_tiles == round(0.01 * 128 * 64)
    assert wl.quantiser_sweep() == [(m, k) for m in (4096, 16384, 65536) for k in (2048, 5120, 7168)]
