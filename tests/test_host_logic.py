"""Host-side logic that needs no GPU: flop accounting, the GELU approximation
used by the bf16 tensor-core epilogue, workload definitions."""
import math

import numpy as np
from scipy.special import erf

import synthetic as syn
from video_generation_b200 import flops as FL


def gelu_as7126(v):
    """GELU with Abramowitz & Stegun 7.1.26 erf (the bf16 GEMM epilogue's method)."""
    u = np.abs(v) / math.sqrt(2.0)
    t = 1.0 / (1.0 + 0.3275911 * u)
    q = t * (0.254829592 + t * (-0.284496736 + t * (1.421413741 + t * (-1.453152027 + t * 1.061405429))))
    return 0.5 * v * (1.0 + np.sign(v) * (1.0 - q * np.exp(-u * u)))


def test_gelu_approximation_within_published_bound():
    v = np.linspace(-12, 12, 2_000_001)
    exact = 0.5 * v * (1.0 + erf(v / math.sqrt(2.0)))
    # |erf error| <= 1.5e-7 (A&S 7.1.26), so |GELU error| <= 0.5 |v| 1.5e-7
    assert (np.abs(gelu_as7126(v) - exact) <= 0.5 * np.abs(v) * 1.5e-7 + 1e-15).all()
    # and well below one bf16 ulp of the activation (2^-8 relative)
    big = np.abs(exact) > 1e-3
    assert (np.abs(gelu_as7126(v) - exact)[big] / np.abs(exact[big])).max() < 2 ** -12


def test_pass_flops_matches_the_per_token_formula():
    s = syn.WORKLOADS[3].shape
    d, C = s.d, s.C
    L = 390
    f = FL.pass_flops(d, C, s.layers, s.mlp_ratio, L, FL.causal_pairs(0, L))
    per_token = s.layers * 24 * d * d + 2 * C * d + 4 * C * d
    assert f == L * per_token + s.layers * 4 * d * (L * (L + 1) // 2)
    # forward of config 3 ~ 1.47e12 flops
    assert abs(FL.forward_flops(s, 21, 390, 3) / 1.472e12 - 1) < 0.01


def test_jacobi_flops_counts_commits_between_blocks():
    s = syn.WORKLOADS[4].shape
    one = FL.jacobi_flops(s, [[[1]]], 390, 390)
    two = FL.jacobi_flops(s, [[[1, 1]]], 780, 390)
    p0 = FL.pass_flops(s.d, s.C, s.layers, s.mlp_ratio, 390, FL.causal_pairs(0, 390))
    p1 = FL.pass_flops(s.d, s.C, s.layers, s.mlp_ratio, 390, FL.causal_pairs(390, 390))
    assert one == p0
    assert two == 2 * p0 + p1


def test_workloads_follow_the_configs():
    w = syn.WORKLOADS
    assert (w[1].shape.d, w[1].shape.heads, w[1].L, w[1].shape.C, w[1].batch) == (64, 2, 64, 16, 2)
    assert (w[2].shape.layers, w[2].batch, w[2].L) == (8, 4, 390)
    assert (w[3].T, w[3].dirs, w[3].batch) == (3, (0, 1, 0), 21)
    assert (w[4].L, w[4].shape.d, w[4].shape.layers, w[4].max_iter, w[4].warm_start) == (8190, 2048, 24, 32, 1)
    assert w[5].L == 46800 and w[5].shape.max_len >= 46800
