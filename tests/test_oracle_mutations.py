"""Plant plausible mistakes in the CPU oracle and check that a pin catches each.

Also pins the Jacobi stopping rule, the warm start and the iteration count
with a closed form: for a head-only model (every weight 0 except b_head) mu
and s are constants, so x^(1) = mu + exp(s) z exactly and x^(2) = x^(1); the
residual of the first update, ||x^(1) - x^(0)||^2 / ||x^(1)||^2, is then known
in closed form from x^(0) -- z, or with warm start the previous frame's
converged tokens -- and decides whether a block stops after 1 or 2 updates
("STARFlow-V ... paper notes", key design 3: the scale-normalised residual and
tau; a new frame starts from the previous frame's converged state).
"""
import math

import numpy as np
import pytest

import synthetic as syn
from oracle import af_oracle as O
from tests import test_oracle_pins as P


def _const_block():
    w = syn.make_weights(P.TINY, perturb=True, zero=("w", "pos", "head", "bias", "shift", "gain"))
    return O.Block(P.TINY, w), w[-1].astype(np.float64)


@pytest.mark.parametrize("warm", [False, True])
def test_jacobi_iteration_count_closed_form(warm):
    blk, bh = _const_block()
    C = P.TINY.C
    mu, sg = bh[:C], np.exp(bh[C:])
    B, nb = 4, 3
    z = np.random.default_rng(12).standard_normal((1, B * nb, C))
    x_exact = mu + sg * z[0]
    F = P.TINY.frame_len                 # 8: two blocks of 4 per frame
    r1 = []
    for b in range(nb):
        # warm start: each token starts from the same spatial token of the previous
        # frame once that frame is finished (block 2 from block 0), else from z
        x0 = np.array([x_exact[p - F] if (warm and p - F >= 0) else z[0, p] for p in range(b * B, (b + 1) * B)])
        x1 = x_exact[b * B:(b + 1) * B]
        r1.append(((x1 - x0) ** 2).sum() / (x1 ** 2).sum())
    r1 = np.array(r1)
    for tau in (r1.min() * 0.999, r1.max() * 1.001, float(np.median(r1)), 0.0):
        x, it, conv = O.af_inverse_jacobi(blk, z, O.L2R, B, tau, 5, warm)
        expect = np.where(r1 < tau, 1, 2 if tau > 0 else 5)   # r2 = 0 passes only a tau > 0
        np.testing.assert_array_equal(it[0], expect)
        np.testing.assert_allclose(x[0], x_exact, rtol=1e-14, atol=1e-14)
    x, it, conv = O.af_inverse_jacobi(blk, z, O.L2R, B, 0.0, 1, warm)
    assert (it == 1).all() and not conv.any()


# ---------------------------------------------------------------------------- mutations

def _gelu_tanh(u):
    return 0.5 * u * (1 + np.tanh(math.sqrt(2 / math.pi) * (u + 0.044715 * u ** 3)))


def _attn_bad_scale(q, K, V, p0, heads):
    return _orig_attn(q * math.sqrt(q.shape[1] // heads) ** -1, K, V, p0, heads)


_orig_attn = O.causal_attention
_orig_ln = O.layer_norm
_orig_fwd = O.af_forward_one
_orig_masked = O.masked_inputs


def _fwd_bad_sign(blk, x, direction):
    z, ld = _orig_fwd(blk, x, direction)
    return z, -ld


def _masked_no_shift(xw, p0, p1):
    return np.asarray(xw[p0:p1], dtype=np.float64)


def _ln_bad_eps(h, g, b, eps=1e-5):
    return _orig_ln(h, g, b, eps=1e-3)


def _residual_old_den(x_new, x_old):
    return float(((x_new - x_old) ** 2).sum()), float((x_old ** 2).sum())


def _warm_from_previous_block(xw, zw, P, Q, frame_len):
    # the previous block's converged x at the same offsets, whatever the frame
    B = Q - P
    return np.array([xw[p - B] if p - B >= 0 else zw[p] for p in range(P, Q)])


_orig_look = O.lookahead_attention


def _lookahead_every_layer(q, K, V, heads, frame_len, ahead):
    return _orig_look(q, K, V, heads, frame_len, 1)


def _no_lookahead(q, K, V, heads, frame_len, ahead):
    return _orig_look(q, K, V, heads, frame_len, 0)


def _positions_no_time(blk, p):
    return np.asarray(blk.pos_space, np.float64)[p % blk.frame_len]


def _positions_time_by_length(blk, p):
    # temporal row from the position divided by the sequence's whole length
    n = blk.frame_len * blk.max_frames
    return (np.asarray(blk.pos_space, np.float64)[p % blk.frame_len]
            + np.asarray(blk.pos_time, np.float64)[p // n])


MUTATIONS = {
    "gelu_tanh_approx": ("gelu", _gelu_tanh),
    "attention_scale": ("causal_attention", _attn_bad_scale),
    "layernorm_eps": ("layer_norm", _ln_bad_eps),
    "logdet_sign": ("af_forward_one", _fwd_bad_sign),
    "mask_not_self_exclusive": ("masked_inputs", _masked_no_shift),
    "residual_denominator_old_iterate": ("jacobi_residual", _residual_old_den),
    "positions_without_time_rows": ("positions", _positions_no_time),
    "warm_start_from_previous_block": ("warm_start_guess", _warm_from_previous_block),
    "denoiser_lookahead_in_every_layer": ("lookahead_attention", _lookahead_every_layer),
    "denoiser_without_lookahead": ("lookahead_attention", _no_lookahead),
    "positions_time_index_by_length": ("positions", _positions_time_by_length),
}


def _any_pin_fails():
    checks = []
    try:
        checks.append(P.pin_transformer_vs_torch() > 1e-12)
    except Exception:
        checks.append(True)
    err, sign, upper, diag = P.pin_logdet_bruteforce(O.L2R)
    checks.append(err > 1e-7 or upper > 1e-9 or diag > 1e-7)
    checks.append(P.pin_roundtrip_seq(O.R2L) > 1e-12)
    checks.append(P.pin_positions_hand_written() != 0.0)
    checks.append(P.pin_warm_start_guess() != 0.0)
    checks.append(P.pin_denoiser_vs_torch() > 1e-12)
    try:
        test_jacobi_iteration_count_closed_form(True)
        checks.append(False)
    except AssertionError:
        checks.append(True)
    return any(checks)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    assert not _any_pin_fails()          # the clean oracle passes every pin
    monkeypatch.setattr(O, attr, fn)
    assert _any_pin_fails(), f"mutation {name} slipped through every pin"
