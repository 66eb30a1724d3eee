"""Pins for the CPU oracle, checked against what the pages and mathematics fix.

Each pin is independent of the oracle's own formulas:
  * the Transformer inside the AF block against torch.nn's library layers;
  * bf16 rounding against torch's conversion;
  * the affine AF equation and the log-determinant against the exact
    change of variables (a brute-force Jacobian and its slogdet);
  * the sequential and Jacobi inverses against invertibility, the
    triangular-system guarantee (first k tokens exact after k sweeps) and
    reverse-order stack inversion ("STARFlow-V ... paper notes", key designs
    1 and 3);
  * closed forms of degenerate weights (identity head, constant head);
  * causality of later frames on earlier ones.
The pin bodies are plain functions so that ``test_oracle_mutations`` can plant
mistakes in the oracle and watch a pin fail.
"""
import numpy as np
import pytest
import torch

import synthetic as syn
from oracle import af_oracle as O

TINY = syn.ModelShape(C=4, d=16, heads=2, layers=2, mlp_ratio=4, frame_len=8, max_frames=3,
                      dtype="fp32")


def tiny_block(seed_block=0, head_std=0.3, shape=TINY, **kw):
    return O.Block(shape, syn.make_weights(shape, block=seed_block, perturb=True,
                                            head_std=head_std, **kw))


def rel(a, b):
    return float(np.linalg.norm(np.ravel(a) - np.ravel(b)) / max(np.linalg.norm(np.ravel(b)), 1e-300))


# ---------------------------------------------------------------------------- pin bodies

def pin_transformer_vs_torch(shape=TINY, n=8, p_split=3):
    """mu, s of the oracle vs a torch.nn pre-LN TransformerEncoder built from the same weights.

    Returns the max relative error over (full pass, cached second half)."""
    w = syn.make_weights(shape, block=7, perturb=True, head_std=0.3)
    blk = O.Block(shape, w)
    rng = np.random.default_rng(3)
    x_in = rng.standard_normal((n, shape.C))
    d, C = shape.d, shape.C
    torch.manual_seed(0)
    t = lambda a: torch.tensor(np.asarray(a, np.float64))
    inp = torch.nn.Linear(C, d, dtype=torch.float64)
    inp.weight.data, inp.bias.data = t(blk.w_in), t(blk.b_in)
    layers = []
    for P in blk.L_:
        L = torch.nn.TransformerEncoderLayer(d, shape.heads, shape.mlp_ratio * d, dropout=0.0,
                                             activation="gelu", layer_norm_eps=1e-5,
                                             batch_first=True, norm_first=True,
                                             dtype=torch.float64)
        L.self_attn.in_proj_weight.data, L.self_attn.in_proj_bias.data = t(P["w_qkv"]), t(P["b_qkv"])
        L.self_attn.out_proj.weight.data, L.self_attn.out_proj.bias.data = t(P["w_o"]), t(P["b_o"])
        L.linear1.weight.data, L.linear1.bias.data = t(P["w_1"]), t(P["b_1"])
        L.linear2.weight.data, L.linear2.bias.data = t(P["w_2"]), t(P["b_2"])
        L.norm1.weight.data, L.norm1.bias.data = t(P["ln1_g"]), t(P["ln1_b"])
        L.norm2.weight.data, L.norm2.bias.data = t(P["ln2_g"]), t(P["ln2_b"])
        layers.append(L.train(False))
    lnf = torch.nn.LayerNorm(d, eps=1e-5, dtype=torch.float64)
    lnf.weight.data, lnf.bias.data = t(blk.lnf_g), t(blk.lnf_b)
    head = torch.nn.Linear(d, 2 * C, dtype=torch.float64)
    head.weight.data, head.bias.data = t(blk.w_head), t(blk.b_head)
    pos = torch.arange(n)
    with torch.no_grad():
        h = inp(t(x_in)) + t(blk.pos_space)[pos % shape.frame_len] + t(blk.pos_time)[pos // shape.frame_len]
        h = h[None]
        mask = torch.nn.Transformer.generate_square_subsequent_mask(n, dtype=torch.float64)
        for L in layers:
            h = L(h, src_mask=mask, is_causal=True)
        out = head(lnf(h))[0].numpy()
    mu, s, _ = O.transformer_rows(blk, x_in, 0)
    e_full = max(rel(mu, out[:, :C]), rel(s, out[:, C:]))
    # the same rows through the KV cache: first p_split rows, then the rest
    _, _, kv = O.transformer_rows(blk, x_in[:p_split], 0)
    mu2, s2, _ = O.transformer_rows(blk, x_in[p_split:], p_split, kv)
    e_cache = max(rel(mu2, out[p_split:, :C]), rel(s2, out[p_split:, C:]))
    return max(e_full, e_cache)


def pin_logdet_bruteforce(direction, shape=TINY, L=6):
    """|logdet - slogdet(J_numeric)| and the triangular structure of J."""
    blk = tiny_block(shape=shape)
    x = np.random.default_rng(11).standard_normal((L, shape.C))
    z, ld = O.af_forward_one(blk, x, direction)
    J = O.jacobian_bruteforce(blk, x, direction)
    sign, ldJ = np.linalg.slogdet(J)
    C = shape.C
    Jb = J.reshape(L, C, L, C)
    # dependence on later tokens (L->R) / earlier tokens (R->L) must vanish
    upper = max(np.abs(Jb[i, :, j, :]).max()
                for i in range(L) for j in range(L)
                if (j > i if direction == O.L2R else j < i))
    # diagonal blocks are diag(exp(-s_i))
    xw = x[::-1] if direction == O.R2L else x
    mu, s, _ = O.transformer_rows(blk, O.masked_inputs(np.asarray(xw, float), 0, L), 0)
    s_orig = s[::-1] if direction == O.R2L else s
    diag_err = max(np.abs(Jb[i, :, i, :] - np.diag(np.exp(-s_orig[i]))).max() for i in range(L))
    return abs(ld - ldJ), sign, upper, diag_err


def pin_roundtrip_seq(direction, shape=TINY, L=12):
    blk = tiny_block(shape=shape)
    x = np.random.default_rng(5).standard_normal((2, L, shape.C))
    z, _ = O.af_forward(blk, x, direction)
    return rel(O.af_inverse_seq(blk, z, direction), x)


def pin_jacobi_prefix(direction, shape=TINY, L=8):
    """After k sweeps from an arbitrary start, tokens 0..k-1 of the block are exact."""
    blk = tiny_block(shape=shape)
    rng = np.random.default_rng(9)
    z = rng.standard_normal((L, shape.C))
    x0 = rng.standard_normal((L, shape.C)) * 3.0
    xs = O.af_inverse_seq_one(blk, z, direction)
    trace = []
    O.af_inverse_jacobi_one(blk, z, direction, L, 0.0, L, False, x0=x0, trace=trace)
    xs_w = xs[::-1] if direction == O.R2L else xs
    worst_exact, best_next = 0.0, np.inf
    for (_, k, xk) in trace:
        worst_exact = max(worst_exact, np.abs(xk[:k] - xs_w[:k]).max() / np.abs(xs_w).max())
        if k < L:
            best_next = min(best_next, np.abs(xk[k] - xs_w[k]).max())
    return worst_exact, best_next, len(trace)


def pin_stack(shape=TINY, L=8):
    dirs = (O.L2R, O.R2L, O.L2R)
    blocks = [tiny_block(seed_block=t, head_std=0.2, shape=shape) for t in range(3)]
    x = np.random.default_rng(21).standard_normal((2, L, shape.C))
    z, ld = O.stack_forward(blocks, dirs, x)
    parts = [None] * 3
    zz = x
    for t in range(3):
        zz, parts[t] = O.af_forward(blocks[t], zz, dirs[t])
    x_back, iters = O.stack_inverse(blocks, dirs, z, L, 0.0, L, False)
    # wrong order: undo block 1 first
    xw = z
    for t in range(3):
        xw, _, _ = O.af_inverse_jacobi(blocks[t], xw, dirs[t], L, 0.0, L, False)
    return rel(x_back, x), np.abs(ld - sum(parts)).max(), rel(xw, x)


# ---------------------------------------------------------------------------- tests

def test_bf16_round_matches_torch():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 3,
                        # exact ties between two bf16 values, both parities
                        (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)])
    ref = torch.tensor(a).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(O.bf16_round(a), ref)


def test_transformer_matches_torch_library_layers():
    assert pin_transformer_vs_torch() < 1e-12


@pytest.mark.parametrize("direction", [O.L2R, O.R2L])
def test_logdet_equals_bruteforce_jacobian(direction):
    err, sign, upper, diag_err = pin_logdet_bruteforce(direction)
    assert sign == 1.0
    assert err < 1e-7
    assert upper < 1e-9           # later tokens never reach earlier z (triangular)
    assert diag_err < 1e-7        # d z_i / d x_i = diag(exp(-s_i))


@pytest.mark.parametrize("direction", [O.L2R, O.R2L])
def test_sequential_inverse_roundtrip(direction):
    assert pin_roundtrip_seq(direction) < 1e-12


@pytest.mark.parametrize("direction", [O.L2R, O.R2L])
def test_jacobi_first_k_tokens_exact_after_k_sweeps(direction):
    worst_exact, best_next, n = pin_jacobi_prefix(direction)
    assert n == 8                 # tau = 0 runs all B sweeps
    assert worst_exact < 1e-13
    assert best_next > 1e-6       # token k is not yet exact: the pin is sharp


def test_jacobi_tau0_B_sweeps_equals_sequential_multiblock_warm():
    blk = tiny_block()
    rng = np.random.default_rng(4)
    z = rng.standard_normal((2, 24, TINY.C))
    xs = O.af_inverse_seq(blk, z, O.L2R)
    for warm in (False, True):
        xj, it, conv = O.af_inverse_jacobi(blk, z, O.L2R, 8, 0.0, 8, warm)
        assert rel(xj, xs) < 1e-13
        assert (it == 8).all() and not conv.any()


def test_stack_inverts_in_reverse_order_and_logdets_add():
    e_rt, e_ld, e_wrong = pin_stack()
    assert e_rt < 1e-12
    assert e_ld < 1e-12
    assert e_wrong > 1e-3


def test_head_zero_is_identity():
    blk = O.Block(TINY, syn.make_weights(TINY, perturb=True, zero=("head", "headbias")))
    x = np.random.default_rng(1).standard_normal((2, 8, TINY.C))
    z, ld = O.af_forward(blk, x, O.L2R)
    np.testing.assert_array_equal(z, x)
    assert (ld == 0).all()
    xj, it, conv = O.af_inverse_jacobi(blk, z, O.L2R, 8, 1e-3, 8, False)
    np.testing.assert_array_equal(xj, x)
    assert (it == 1).all() and conv.all()


def test_constant_head_closed_form():
    """All weights 0 except b_head: mu, s are the constant halves of b_head."""
    w = syn.make_weights(TINY, perturb=True, zero=("w", "pos", "head", "bias", "shift", "gain"))
    blk = O.Block(TINY, w)
    bh = w[-1].astype(np.float64)
    C = TINY.C
    x = np.random.default_rng(2).standard_normal((2, 8, C))
    z, ld = O.af_forward(blk, x, O.R2L)
    np.testing.assert_allclose(z, (x - bh[:C]) * np.exp(-bh[C:]), rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(ld, -8 * bh[C:].sum(), rtol=1e-13)


def test_later_frames_never_change_earlier_ones_bitwise():
    blk = tiny_block(head_std=0.1)
    L, B = 24, 8                                      # 3 "frames" of 8 tokens
    z = np.random.default_rng(6).standard_normal((1, L, TINY.C))
    x1, _, _ = O.af_inverse_jacobi(blk, z, O.L2R, B, 1e-3, 8, True)
    z2 = z.copy()
    z2[0, 16:] += 1.0                                 # perturb the last frame
    x2, _, _ = O.af_inverse_jacobi(blk, z2, O.L2R, B, 1e-3, 8, True)
    np.testing.assert_array_equal(x1[0, :16], x2[0, :16])
    assert np.abs(x1[0, 16:] - x2[0, 16:]).max() > 1e-3
    zf1, _ = O.af_forward(blk, x1, O.L2R)
    x3 = x1.copy()
    x3[0, 20] += 1.0
    zf3, _ = O.af_forward(blk, x3, O.L2R)
    np.testing.assert_array_equal(zf1[0, :20], zf3[0, :20])   # z_i depends on x_<=i only
    assert np.abs(zf1[0, 20] - zf3[0, 20]).max() > 0.1


def test_warm_start_changes_only_iterations_not_the_fixed_point():
    blk = tiny_block(head_std=0.05)
    L, B, tau = 24, 8, 1e-6
    z = np.random.default_rng(8).standard_normal((2, L, TINY.C))
    xs = O.af_inverse_seq(blk, z, O.L2R)
    xc, itc, cc = O.af_inverse_jacobi(blk, z, O.L2R, B, tau, B, False)
    xw, itw, cw = O.af_inverse_jacobi(blk, z, O.L2R, B, tau, B, True)
    assert cc.all() and cw.all()
    # both sit within the tau-level distance of the exact fixed point
    assert rel(xc, xs) < 1e-4 and rel(xw, xs) < 1e-4
    assert rel(xc, xw) < 1e-4


def test_jacobi_converges_within_B_for_any_tau():
    blk = tiny_block(head_std=0.5)
    z = np.random.default_rng(10).standard_normal((3, 8, TINY.C))
    for tau in (1e-1, 1e-3, 1e-8):
        _, it, conv = O.af_inverse_jacobi(blk, z, O.L2R, 8, tau, 8, False)
        assert (it <= 8).all()
    # a triangular system reaches its fixed point exactly by sweep B, so sweep B+1 sees r = 0
    _, it, conv = O.af_inverse_jacobi(blk, z, O.L2R, 8, 1e-30, 9, False)
    assert conv.all() and (it <= 9).all()


def test_residual_edge_cases():
    assert O.converged(0.0, 0.0, 1e-3)
    assert not O.converged(1.0, 0.0, 1e-3)
    assert not O.converged(1e-3, 1.0, 1e-3)          # strict <
    assert O.converged(0.99e-3, 1.0, 1e-3)


# ---------------------------------------------------------------------------- positions, chunked forward, known prefix

POS_SHAPE = syn.ModelShape(C=4, d=4, heads=1, layers=1, mlp_ratio=1, frame_len=2, max_frames=3, dtype="fp32")


def pin_positions_hand_written():
    """pos[p] for 3 frames of 2 tokens, written out by hand (R10: the spatial
    row is p mod frame_len, the temporal row p div frame_len).

    P_space rows are 1 and 2 in column 0; P_time rows are 10, 20, 30 in column
    1 and 100, 200, 300 in column 2; column 3 stays 0.  Returns the max abs
    error over positions 0..5."""
    w = syn.make_weights(POS_SHAPE, zero=("w", "pos", "head", "bias", "shift", "headbias"))
    w[2] = np.array([[1, 0, 0, 0], [2, 0, 0, 0]], np.float32)                            # P_space
    w[3] = np.array([[0, 10, 100, 0], [0, 20, 200, 0], [0, 30, 300, 0]], np.float32)    # P_time
    blk = O.Block(POS_SHAPE, w)
    expect = np.array([[1, 10, 100, 0],      # p = 0: frame 0, token 0
                       [2, 10, 100, 0],      # p = 1: frame 0, token 1
                       [1, 20, 200, 0],      # p = 2: frame 1, token 0
                       [2, 20, 200, 0],      # p = 3: frame 1, token 1
                       [1, 30, 300, 0],      # p = 4: frame 2, token 0
                       [2, 30, 300, 0]],     # p = 5: frame 2, token 1
                      np.float64)
    return float(np.abs(O.positions(blk, np.arange(6)) - expect).max())


def test_positions_match_hand_written_table():
    assert pin_positions_hand_written() == 0.0


def test_positions_reach_the_transformer_per_frame():
    """Two tokens with the same input but in different frames get different
    (mu, s) exactly when their temporal rows differ (and equal ones when only
    the frame's content, not its position, is shared)."""
    shape = syn.ModelShape(C=4, d=16, heads=2, layers=1, mlp_ratio=2, frame_len=2, max_frames=3, dtype="fp32")
    w = syn.make_weights(shape, perturb=True, head_std=0.3)
    blk = O.Block(shape, w)
    x_in = np.ones((6, 4))
    mu, s, _ = O.transformer_rows(blk, x_in, 0)
    w2 = [a.copy() for a in w]
    w2[3][:] = w2[3][0]                       # all temporal rows equal
    mu2, _, _ = O.transformer_rows(O.Block(shape, w2), x_in, 0)
    w3 = [a.copy() for a in w]
    w3[3][1:] += np.linspace(-1.0, 1.0, shape.d, dtype=np.float32)   # frames 1 and 2 only (not a
    #                                           constant shift, which LayerNorm would remove)
    mu3, _, _ = O.transformer_rows(O.Block(shape, w3), x_in, 0)
    np.testing.assert_array_equal(mu3[:2], mu[:2])     # frame 0 untouched (causal, row 0 of P_time)
    assert np.abs(mu3[2:] - mu[2:]).max() > 1e-3
    assert np.abs(mu2 - mu).max() > 1e-3


def test_chunked_forward_equals_plain_forward():
    blk = tiny_block()
    x = np.random.default_rng(13).standard_normal((2, 22, TINY.C))
    for direction in (O.L2R, O.R2L):
        z, ld = O.af_forward(blk, x, direction)
        for B in (5, 8, 22):
            for i in range(2):
                zc, ldc, _ = O.af_forward_chunked_one(blk, x[i], direction, B)
                zc = zc[::-1] if direction == O.R2L else zc
                assert rel(zc, z[i]) < 1e-12 and abs(ldc - ld[i]) < 1e-12 * max(1.0, abs(ld[i]))
                tail, _, _ = O.af_forward_chunked_one(blk, x[i], direction, B, keep_from=13)
                zw = z[i][::-1] if direction == O.R2L else z[i]
                assert rel(tail, zw[13:]) < 1e-12


def test_known_prefix_continues_the_same_inverse():
    """Observed leading blocks (x given) followed by Jacobi blocks: with the
    oracle's own first blocks as the observation the result is bitwise the
    full Jacobi run; with tau = 0 and B sweeps it reaches the exact inverse of
    the forward pass whatever prefix is observed."""
    blk = tiny_block(head_std=0.2)
    rng = np.random.default_rng(14)
    z = rng.standard_normal((2, 24, TINY.C))
    for warm in (False, True):
        x_full, it_full, _ = O.af_inverse_jacobi(blk, z, O.R2L, 8, 1e-6, 8, warm)
        x_tf, it_tf, conv_tf = O.af_inverse_jacobi(blk, z, O.R2L, 8, 1e-6, 8, warm, x_known=x_full, n_known=2)
        np.testing.assert_array_equal(x_tf, x_full)
        assert (it_tf[:, :2] == 0).all() and conv_tf[:, :2].all()
        np.testing.assert_array_equal(it_tf[:, 2:], it_full[:, 2:])
    x_true = rng.standard_normal((2, 24, TINY.C))
    zt, _ = O.af_forward(blk, x_true, O.L2R)
    x_tf, _, _ = O.af_inverse_jacobi(blk, zt, O.L2R, 8, 0.0, 8, True, x_known=x_true, n_known=1)
    assert rel(x_tf, x_true) < 1e-12


# ---------------------------------------------------------------------------- block-size schedules

def test_schedule_of_equal_blocks_is_the_uniform_call():
    blk = tiny_block(head_std=0.2)
    z = np.random.default_rng(15).standard_normal((2, 24, TINY.C))
    for warm in (False, True):
        a = O.af_inverse_jacobi(blk, z, O.L2R, 8, 1e-6, 8, warm)
        b = O.af_inverse_jacobi(blk, z, O.L2R, [8, 8, 8], 1e-6, 8, warm)
        for u, v in zip(a, b):
            np.testing.assert_array_equal(u, v)


@pytest.mark.parametrize("sizes", [[3, 5, 8, 8], [1, 2, 21], [10, 14], [24]])
def test_any_schedule_with_enough_sweeps_is_the_sequential_inverse(sizes):
    """The triangular guarantee per block: B_b sweeps make block b exact from
    any start, so a schedule of any sizes (tau = 0, max_iter = largest block)
    reproduces the token-by-token inverse, warm started or not."""
    blk = tiny_block(head_std=0.3)
    z = np.random.default_rng(16).standard_normal((2, 24, TINY.C))
    xs = O.af_inverse_seq(blk, z, O.R2L)
    for warm in (False, True):
        xj, it, conv = O.af_inverse_jacobi(blk, z, O.R2L, sizes, 0.0, max(sizes), warm)
        assert rel(xj, xs) < 1e-12
        assert it.shape == (2, len(sizes)) and (it == max(sizes)).all()


def pin_warm_start_guess():
    """Blocks larger than a frame: tokens of the block's second frame start
    from the last finished frame (two frames back), tokens of the first
    frame with no finished frame start from z.  Returns the max abs error
    against the hand-derived sources."""
    zw = np.arange(40, dtype=np.float64).reshape(20, 2)            # 20 tokens, frames of 4
    xw = -np.arange(40, dtype=np.float64).reshape(20, 2)
    err = 0.0
    g = O.warm_start_guess(xw, zw, 8, 18, 4)                       # block of positions 8..17
    src = [4, 5, 6, 7, 4, 5, 6, 7, 4, 5]                           # p - k*4 < 8, smallest k
    err = max(err, np.abs(g - xw[src]).max())
    g0 = O.warm_start_guess(xw, zw, 0, 6, 4)                       # first block: nothing finished
    err = max(err, np.abs(g0 - zw[0:6]).max())
    g1 = O.warm_start_guess(xw, zw, 2, 9, 4)                       # positions 2..8
    err = max(err, np.abs(g1 - np.concatenate([zw[2:4], xw[0:2], zw[6:8], xw[0:1]])).max())
    return float(err)


def test_warm_start_reaches_back_whole_frames():
    assert pin_warm_start_guess() == 0.0


# ---------------------------------------------------------------------------- the denoiser s_phi

DEN = syn.ModelShape(C=4, d=16, heads=2, layers=2, mlp_ratio=4, frame_len=2, max_frames=3, dtype="fp32")

# frames of 2 tokens, 3 frames, written out by hand: row i (query), column j
# (key); 1 = attends.  First layer: one frame of look-ahead; later layers:
# frames up to the query's own.
LOOKAHEAD_MASK_F2_N6 = np.array([[1, 1, 1, 1, 0, 0],
                                 [1, 1, 1, 1, 0, 0],
                                 [1, 1, 1, 1, 1, 1],
                                 [1, 1, 1, 1, 1, 1],
                                 [1, 1, 1, 1, 1, 1],
                                 [1, 1, 1, 1, 1, 1]], bool)
FRAME_CAUSAL_MASK_F2_N6 = np.array([[1, 1, 0, 0, 0, 0],
                                    [1, 1, 0, 0, 0, 0],
                                    [1, 1, 1, 1, 0, 0],
                                    [1, 1, 1, 1, 0, 0],
                                    [1, 1, 1, 1, 1, 1],
                                    [1, 1, 1, 1, 1, 1]], bool)


def pin_denoiser_vs_torch():
    """s_phi of the oracle vs torch.nn pre-LN TransformerEncoderLayers built
    from the same weights, with the hand-written look-ahead mask."""
    w = syn.make_denoiser_weights(DEN, perturb=True)
    blk = O.DenoiserBlock(DEN, w)
    x = np.random.default_rng(17).standard_normal((6, DEN.C))
    t = lambda a: torch.tensor(np.asarray(a, np.float64))
    d, C = DEN.d, DEN.C
    inp = torch.nn.Linear(C, d, dtype=torch.float64)
    inp.weight.data, inp.bias.data = t(blk.w_in), t(blk.b_in)
    layers = []
    for P in blk.L_:
        L = torch.nn.TransformerEncoderLayer(d, DEN.heads, DEN.mlp_ratio * d, dropout=0.0, activation="gelu",
                                             layer_norm_eps=1e-5, batch_first=True, norm_first=True,
                                             dtype=torch.float64)
        L.self_attn.in_proj_weight.data, L.self_attn.in_proj_bias.data = t(P["w_qkv"]), t(P["b_qkv"])
        L.self_attn.out_proj.weight.data, L.self_attn.out_proj.bias.data = t(P["w_o"]), t(P["b_o"])
        L.linear1.weight.data, L.linear1.bias.data = t(P["w_1"]), t(P["b_1"])
        L.linear2.weight.data, L.linear2.bias.data = t(P["w_2"]), t(P["b_2"])
        L.norm1.weight.data, L.norm1.bias.data = t(P["ln1_g"]), t(P["ln1_b"])
        L.norm2.weight.data, L.norm2.bias.data = t(P["ln2_g"]), t(P["ln2_b"])
        layers.append(L.train(False))
    lnf = torch.nn.LayerNorm(d, eps=1e-5, dtype=torch.float64)
    lnf.weight.data, lnf.bias.data = t(blk.lnf_g), t(blk.lnf_b)
    head = torch.nn.Linear(d, C, dtype=torch.float64)
    head.weight.data, head.bias.data = t(blk.w_head), t(blk.b_head)
    pos = torch.arange(6)
    masks = [torch.tensor(~LOOKAHEAD_MASK_F2_N6), torch.tensor(~FRAME_CAUSAL_MASK_F2_N6)]   # True = masked out
    with torch.no_grad():
        h = inp(t(x)) + t(blk.pos_space)[pos % DEN.frame_len] + t(blk.pos_time)[pos // DEN.frame_len]
        h = h[None]
        for l, L in enumerate(layers):
            h = L(h, src_mask=masks[0 if l == 0 else 1])
        ref = head(lnf(h))[0].numpy()
    return rel(O.denoiser_scores(blk, x), ref)


def test_denoiser_matches_torch_with_lookahead_mask():
    assert pin_denoiser_vs_torch() < 1e-12


def test_denoiser_looks_exactly_one_frame_ahead():
    """The output of frame n depends on frames <= n + 1 (the pages' s_phi(x_{<=n+1}))."""
    blk = O.DenoiserBlock(DEN, syn.make_denoiser_weights(DEN, perturb=True))
    x = np.random.default_rng(18).standard_normal((1, 6, DEN.C))
    y = O.denoise(blk, x, 0.3)
    x2 = x.copy()
    x2[0, 4:] += 1.0                                      # frame 2
    y2 = O.denoise(blk, x2, 0.3)
    np.testing.assert_array_equal(y2[0, :2], y[0, :2])    # frame 0 does not see frame 2
    assert np.abs(y2[0, 2:4] - y[0, 2:4]).max() > 1e-6    # frame 1 does
    x3 = x.copy()
    x3[0, 2:4] += 1.0                                     # frame 1
    y3 = O.denoise(blk, x3, 0.3)
    assert np.abs(y3[0, :2] - y[0, :2]).max() > 1e-6      # frame 0 sees frame 1
    np.testing.assert_array_equal(O.denoise(blk, x, 0.0), x)   # sigma = 0 leaves x unchanged


# ---------------------------------------------------------------------------- streaming window

def test_window_starts():
    assert O.window_starts(7, 4, 1) == [0, 3]            # frames 0-3, then 3-6
    assert O.window_starts(4, 4, 1) == [0]
    assert O.window_starts(5, 4, 2) == [0, 2]
    assert O.window_starts(10, 3, 0) == [0, 3, 6, 9]


def test_stream_with_one_window_is_the_plain_inverse():
    blk = tiny_block(head_std=0.2)
    z = np.random.default_rng(19).standard_normal((2, 24, TINY.C))
    x1, it1, _ = O.af_inverse_jacobi(blk, z, O.L2R, 8, 1e-6, 8, True)
    x2, it2 = O.af_inverse_jacobi_stream(blk, z, 8, 3, 1, 1e-6, 8, True)
    np.testing.assert_array_equal(x1, x2)
    np.testing.assert_array_equal(it1, it2)


def test_stream_windows_invert_their_own_forward():
    """Each window is an exact inverse problem (tau = 0, B sweeps): the stream
    reproduces x wherever z was made by the forward pass of the same window
    with the observed frames in front."""
    blk = tiny_block(head_std=0.3)                    # frames of 8 tokens, the model holds 3
    F, W, D = 8, 3, 1
    rng = np.random.default_rng(20)
    x_true = rng.standard_normal((1, 5 * F, TINY.C))   # 5 frames: windows [0,3) and [2,5)
    z = np.zeros_like(x_true)
    z[:, :3 * F], _ = O.af_forward(blk, x_true[:, :3 * F], O.L2R)
    zw, _ = O.af_forward(blk, x_true[:, 2 * F:5 * F], O.L2R)
    z[:, 3 * F:] = zw[:, F:]
    x, it = O.af_inverse_jacobi_stream(blk, z, F, W, D, 0.0, F, True)
    assert rel(x, x_true) < 1e-12
    assert it.shape == (1, 5) and (it == F).all()
