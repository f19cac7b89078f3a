"""The seeded input recipe (CPU): the generators draw what the design states.

Shapes of every workload, the outlier structure of x and W, the bias scale,
exact 16-bit storage, determinism under a seed, and distinct draws across
workload indices.  No layer arithmetic is involved.
"""

import numpy as np
import pytest
import torch

import workloads


def test_workload_shapes():
    shapes = {k: [(l.M, l.K, l.N) for l in v] for k, v in workloads.WORKLOADS.items()}
    assert shapes["single_1024"] == [(64, 1024, 1024)]
    assert shapes["zimage_dit_block"] == [(4608, 3840, 11520), (4608, 3840, 10240),
                                          (4608, 10240, 3840)]
    assert shapes["flux1_dev_blocks"] == [(4608, 3072, 9216), (4608, 3072, 12288),
                                          (4608, 12288, 3072), (4608, 3072, 21504),
                                          (4608, 15360, 3072)]
    assert shapes["wan22_a14b_video_dit"] == [(7800, 5120, 15360), (7800, 5120, 13824),
                                              (7800, 13824, 5120)]
    assert 7800 == 104 * 60 * 5 // 4 and 4608 == 4096 + 512
    sweep = workloads.WORKLOADS["group_size_sweep"]
    assert {(l.M, l.G) for l in sweep} == {(m, g) for m in (1, 16, 128, 1024, 8192)
                                           for g in (4, 16, 64, 256)}
    assert all(l.K == l.N == 4096 for l in sweep)
    assert all(l.n_outliers == 8 for l in workloads.WORKLOADS["flux1_dev_blocks"])
    for name, lins in workloads.WORKLOADS.items():
        for l in lins:
            assert l.K % l.G == 0 and l.K % 32 == 0 and l.N % 16 == 0, (name, l)


def _outlier_cols(a: np.ndarray, ratio: float) -> np.ndarray:
    rms = np.sqrt(np.mean(a.astype(np.float64) ** 2, axis=0))
    return np.nonzero(rms > ratio * np.median(rms))[0]


def test_activation_outliers():
    x = workloads.make_activation(512, 1024, seed=1000, n_outliers=4, outlier_seed=2000)
    a = x.float().numpy()
    cols = _outlier_cols(a, 10.0)
    assert len(cols) == 4
    rms = np.sqrt(np.mean(a.astype(np.float64) ** 2, axis=0))
    normal = np.setdiff1d(np.arange(1024), cols)
    assert 0.9 < np.median(rms[normal]) < 1.1          # N(0, 1)
    assert np.all((rms[cols] > 25) & (rms[cols] < 35))  # x30
    # the outlier channels come from the outlier seed alone
    rng = np.random.default_rng(2000)
    np.testing.assert_array_equal(np.sort(rng.choice(1024, size=4, replace=False)), cols)


def test_weight_outlier_columns_and_bias():
    W = workloads.make_weight(256, 2048, seed=3000, outlier_seed=4000).float().numpy()
    cols = _outlier_cols(W, 5.0)
    assert len(cols) == round(0.01 * 2048)
    rms = np.sqrt(np.mean(W.astype(np.float64) ** 2, axis=0))
    normal = np.setdiff1d(np.arange(2048), cols)
    assert 0.018 < np.median(rms[normal]) < 0.022       # N(0, 0.02)
    assert np.all((rms[cols] > 0.16) & (rms[cols] < 0.24))  # x10
    b = workloads.make_bias(4096, seed=5000).float().numpy()
    assert 0.009 < b.std() < 0.011


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_exact_16_bit_storage_and_determinism(dtype):
    lin = workloads.WORKLOADS["single_1024"][0]
    a = workloads.make_layer_inputs(lin, 0, dtype=dtype)
    b = workloads.make_layer_inputs(lin, 0, dtype=dtype)
    c = workloads.make_layer_inputs(lin, 1, dtype=dtype)
    for t in (a.x, a.W, a.bias):
        assert t.dtype == dtype
        # the float32 draw rounded once: converting back and forth is exact
        assert torch.equal(t.float().to(dtype), t)
    assert torch.equal(a.x, b.x) and torch.equal(a.W, b.W) and torch.equal(a.bias, b.bias)
    assert not torch.equal(a.x, c.x) and not torch.equal(a.W, c.W)
    # the same draw in either format: fp16 and bf16 round the same float32 values
    other = torch.float16 if dtype == torch.bfloat16 else torch.bfloat16
    d = workloads.make_layer_inputs(lin, 0, dtype=other)
    assert torch.allclose(a.x.float(), d.x.float(), rtol=2 ** -7, atol=0)


def test_rotation_inputs():
    for G in workloads.GROUP_SIZES:
        H = workloads.sylvester_rotation(G)
        assert H.dtype == np.float32 and H.shape == (G, G)
        np.testing.assert_array_equal(H, H.T)
        Q = workloads.qr_rotation(G)
        # Haar sign convention: the QR factor's diagonal is positive
        _, r = np.linalg.qr(Q.astype(np.float64))
        assert np.all(np.abs(np.abs(np.diag(r)) - 1) < 1e-5)
        assert not np.allclose(Q, Q.T)
    with pytest.raises(ValueError):
        workloads.sylvester_rotation(12)
