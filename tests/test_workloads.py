"""The seeded input recipe (workloads/): shapes, determinism and the value
structure each configuration promises -- outlier channels (Llama-2-7B),
heavy-tailed activations and gradient scales spanning the E5M2 bias range
(Llama-2-70B), and the adversarial tensors of the amax/cast sweep.  CPU only;
biases come from the oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from workloads import LayerConfig, Linear


def test_shapes_dtypes_and_determinism():
    for cid in (0, 1):
        cfg = workloads.CONFIGS[cid]
        for li, lin in enumerate(cfg.linears):
            x, w, dy = workloads.linear_inputs(cid, li)
            assert x.shape == (cfg.tokens, lin.in_features) and x.dtype == torch.bfloat16
            assert w.shape == (lin.out_features, lin.in_features)
            if cid == 0:
                assert dy is None                      # forward only
            else:
                assert dy.shape == (cfg.tokens, lin.out_features)
            x2, w2, _ = workloads.linear_inputs(cid, li)
            assert torch.equal(x, x2) and torch.equal(w, w2)
    a, _, _ = workloads.linear_inputs(1, 0, step=0)
    b, _, _ = workloads.linear_inputs(1, 0, step=1)
    assert not torch.equal(a, b)                       # each step draws new tensors


def test_llama7b_outlier_channels():
    x, _, _ = workloads.linear_inputs(2, 0)
    chmax = x.float().abs().amax(dim=0)
    big = (chmax > 10 * chmax.median()).nonzero().flatten()
    assert big.numel() == 8                            # 8 channels scaled x50
    assert float(chmax[big].min()) > 20 * float(chmax.median())


def test_student_t_activations_are_heavy_tailed():
    cfg = LayerConfig(9, "t", 4096, (Linear("p", 1024, 16, 1.0),), "student_t")
    x = workloads._x(cfg, 1024, seed=5, device="cpu", dtype=torch.float32)
    frac = float((x.abs() > 10).float().mean())
    # P(|t_3| > 10) = 2.1e-3; a normal variable essentially never exceeds 10
    assert 1e-3 < frac < 4e-3
    assert float(x.abs().max()) > 50


def test_llama70b_gradient_scales_span_e5m2_biases():
    g = torch.Generator().manual_seed(0)
    z = torch.randn(1 << 20, generator=g)
    biases = []
    for lin in workloads.C3.linears:
        amax = float((z * lin.sigma_dy).to(torch.bfloat16).float().abs().max())
        biases.append(oracle.compute_bias(amax, oracle.E5M2, 0))
    assert biases == sorted(biases, reverse=True)     # QKV (1e-7) ... down (1e-2)
    assert biases[0] >= 34 and biases[-1] <= 22      # about 36 down to 20


def test_sweep_tensors():
    assert not workloads.sweep_tensor(1000, torch.float32, "zeros").any()
    s = workloads.sweep_tensor(1000, torch.float32, "spike_zeros", seed=3)
    assert int((s != 0).sum()) == 1 and float(s.max()) == 1e4
    for fmt_max in (448.0, 57344.0):
        v = workloads.sweep_tensor(4096, torch.float32, "exact_pow2", seed=4, fmt_max=fmt_max)
        for x in v.tolist()[:512]:
            k = math.log2(fmt_max / abs(x))
            assert k == int(k) and 0 <= k <= 20        # exactly +-fmt_max * 2^-k
        assert {float(np.sign(x)) for x in v.tolist()} == {-1.0, 1.0}


def test_seed_formula():
    assert workloads.seed_for(3, 2, 1, 0) == 3021
    assert workloads.seed_for(3, 2, 1, 4) == 403021
