"""CPU oracle for the STARFlow-V affine autoregressive flow (AF) block.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or call
this module.  The product path (``video_generation_b200``) never does, and the
two share no code.

Plain, slow, float64 numpy.  Library primitives used as steps: matmul, exp,
sqrt and ``scipy.special.erf``.  Every function follows the pages step by step
with no blocking or fusion beyond what they state.  Sources, by page and
section:

  [N]  "STARFlow-V: End-to-End Video Generative Modeling with Autoregressive
       Normalizing Flows", CVPR 2026 paper notes (papernotes.org):
       - "Key design 1: global-local architecture" -- the affine AF equation
         z = (x - mu(x*m)) / sigma(x*m), sigma > 0, with m the self-exclusive
         causal mask; T >= 3 blocks of alternating direction; the
         deep/shallow split f = f_D o f_S; f_S inside one frame (alternating
         L->R / R->L), f_D causal across frames.
       - "Key design 3: video-aware block-wise Jacobi iteration" -- the
         fixed-point system x = mu(x*m) + sigma(x*m) * z, the update
         x^(k+1) = mu(x^(k)*m) + sigma(x^(k)*m) * z, the stopping rule
         ||x^(k+1) - x^(k)||^2 / ||x^(k+1)||^2 < tau (tau = 1e-3), blocks of
         size B run in sequence with parallel updates inside a block,
         finished blocks feeding a KV cache, and the warm start
         x^(0)_{n+1} = x^(k)_n from the previous frame's converged state.
       - "Loss / training strategy" -- L_NF = E[log p0(f(x)) + log|det J|],
         which fixes the sign of the log-determinant.
  The pages never spell out the Transformer inside the AF block beyond
  "causal Transformer".  Readings taken where they are silent (each stated
  where used):
    R1 mask m: a one-token input shift (token 0 sees a zero vector) followed
       by inclusive causal attention, so mu_i and sigma_i depend on x_{<i}.
    R2 sigma = exp(s), no clamp.
    R3 logdet = -sum_{i,c} s_{i,c} per sample (a sum, not a mean).
    R4 the residual norm runs over one block's B*C entries of one sample;
       strict '<'; 0/0 counts as converged, num>0 over 0 does not.
    R5 x^(0) = z for a block with no warm start.
    R6 the output of a block is the iterate that passed the test; ``iters``
       counts the updates computed.
    R7 the KV cache of a finished block is computed from its final x.
    R8 each sample of a batch converges on its own.
    R9 pre-LN Transformer: LayerNorm eps 1e-5, multi-head attention with
       scale 1/sqrt(head_dim), exact-erf GELU MLP of width mlp_ratio*d,
       final LayerNorm, linear head [mu | s] (mu = first C outputs).
    R10 positions: pos[p] = P_space[p mod frame_len] + P_time[p div frame_len].
    R11 direction R->L reverses the token order of each sample's sequence
       before the block and restores it after.
    R12 bf16 models: the weights are rounded to bf16 (round to nearest even)
       once; the oracle then computes in float64 with those values.
    R13 warm start per token: position p of a new block starts from the
       converged x at p - k*frame_len, the same spatial position in the most
       recent finished frame (smallest k >= 1 reaching before the block), or
       from z where no frame before it has finished.  With one-frame blocks
       this is the previous block's converged x at the same offsets.
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import numpy as np
from scipy.special import erf

L2R, R2L = 0, 1


# ----------------------------------------------------------------------------
# weights

def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); float32 out.

    bfloat16 keeps the top 16 bits of an IEEE float32.  Rounding to nearest
    even adds 0x7FFF plus the lowest kept bit before truncating.  (No NaN/Inf
    in the synthetic weights.)
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32)


class Block:
    """Weights of one AF block, indexed like ``synthetic.tensor_specs``.

    Arrays stay float32 in memory (bf16 values are exact in float32) and are
    widened to float64 at each use.
    """

    def __init__(self, shape, tensors: Sequence[np.ndarray]):
        self.C, self.d, self.heads = shape.C, shape.d, shape.heads
        self.layers, self.frame_len = shape.layers, shape.frame_len
        self.max_frames = shape.max_frames
        t = [np.asarray(a, np.float32) for a in tensors]
        if shape.dtype == "bf16":                     # R12
            t = [bf16_round(a) for a in t]
        self.w_in, self.b_in, self.pos_space, self.pos_time = t[0:4]
        self.L_ = []
        for l in range(shape.layers):
            g = t[4 + 12 * l: 4 + 12 * (l + 1)]
            self.L_.append(dict(ln1_g=g[0], ln1_b=g[1], w_qkv=g[2], b_qkv=g[3],
                                w_o=g[4], b_o=g[5], ln2_g=g[6], ln2_b=g[7],
                                w_1=g[8], b_1=g[9], w_2=g[10], b_2=g[11]))
        self.lnf_g, self.lnf_b, self.w_head, self.b_head = t[4 + 12 * shape.layers:]


def _f(a):
    return np.asarray(a, dtype=np.float64)


# ----------------------------------------------------------------------------
# the causal Transformer inside one AF block (R9)

def layer_norm(h, g, b, eps=1e-5):
    mu = h.mean(axis=-1, keepdims=True)
    var = ((h - mu) ** 2).mean(axis=-1, keepdims=True)
    return (h - mu) / np.sqrt(var + eps) * _f(g) + _f(b)


def gelu(u):
    return 0.5 * u * (1.0 + erf(u / math.sqrt(2.0)))


def linear(a, w, b):
    return a @ _f(w).T + _f(b)


def positions(blk: Block, p: np.ndarray) -> np.ndarray:
    """Learned absolute position vectors of sequence positions p (R10)."""
    return _f(blk.pos_space)[p % blk.frame_len] + _f(blk.pos_time)[p // blk.frame_len]


def causal_attention(q, K, V, p0, heads):
    """softmax(q K^T / sqrt(hd) restricted to keys j <= query position) V.

    q holds the queries of positions p0 .. p0+n-1; K, V hold keys and values
    of positions 0 .. p0+n-1 (the cache of positions < p0, then the rows
    themselves).  Plain softmax: subtract the row max, exponentiate, divide.
    """
    n, d = q.shape
    hd = d // heads
    allowed = np.arange(K.shape[0])[None, :] <= (p0 + np.arange(n))[:, None]
    out = np.empty_like(q)
    for h in range(heads):
        sl = slice(h * hd, (h + 1) * hd)
        S = (q[:, sl] @ K[:, sl].T) / math.sqrt(hd)
        S = np.where(allowed, S, -np.inf)
        S = S - S.max(axis=1, keepdims=True)
        E = np.exp(S)
        out[:, sl] = (E / E.sum(axis=1, keepdims=True)) @ V[:, sl]
    return out


def transformer_rows(blk: Block, x_in: np.ndarray, p0: int, cache=None):
    """mu, s for the rows at positions p0 .. p0+n-1 of one sample.

    ``x_in`` [n, C] are the already-masked inputs of those positions (R1: the
    input at position p is x_{p-1}, zero at p = 0).  ``cache`` is a list, per
    layer, of (K, V) of positions 0 .. p0-1 (None when p0 = 0).  Returns
    (mu [n, C], s [n, C], kv) where kv holds the rows' own (K, V) per layer.
    """
    n = x_in.shape[0]
    d, C = blk.d, blk.C
    h = linear(_f(x_in), blk.w_in, blk.b_in) + positions(blk, p0 + np.arange(n))
    kv = []
    for l, P in enumerate(blk.L_):
        a = layer_norm(h, P["ln1_g"], P["ln1_b"])
        qkv = linear(a, P["w_qkv"], P["b_qkv"])
        q, k, v = qkv[:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:]
        kv.append((k, v))
        if cache is not None and p0 > 0:
            K = np.concatenate([cache[l][0], k])
            V = np.concatenate([cache[l][1], v])
        else:
            K, V = k, v
        h = h + linear(causal_attention(q, K, V, p0, blk.heads), P["w_o"], P["b_o"])
        a = layer_norm(h, P["ln2_g"], P["ln2_b"])
        h = h + linear(gelu(linear(a, P["w_1"], P["b_1"])), P["w_2"], P["b_2"])
    out = linear(layer_norm(h, blk.lnf_g, blk.lnf_b), blk.w_head, blk.b_head)
    return out[:, :C], out[:, C:], kv


def masked_inputs(xw: np.ndarray, p0: int, p1: int) -> np.ndarray:
    """Inputs of positions p0..p1-1 under the self-exclusive mask (R1)."""
    C = xw.shape[1]
    prev = xw[p0 - 1:p1 - 1] if p0 > 0 else np.concatenate([np.zeros((1, C)), xw[:p1 - 1]])
    return _f(prev)


def _work(a, direction):            # R11
    return a[::-1] if direction == R2L else a


# ----------------------------------------------------------------------------
# forward: z and logdet ([N] key design 1, affine AF equation; loss section)

def af_forward_one(blk: Block, x: np.ndarray, direction: int, with_abs: bool = False):
    """z and logdet of one sample; with ``with_abs`` also sum |s| (the scale
    against which tests judge a logdet that is a sum of many cancelling s)."""
    xw = _f(_work(x, direction))
    L = xw.shape[0]
    mu, s, _ = transformer_rows(blk, masked_inputs(xw, 0, L), 0)
    zw = (xw - mu) * np.exp(-s)               # sigma = exp(s)   (R2)
    logdet = -s.sum()                         # log|det dz/dx| = -sum log sigma (R3)
    if with_abs:
        return _work(zw, direction).copy(), float(logdet), float(np.abs(s).sum())
    return _work(zw, direction).copy(), float(logdet)


def af_forward(blk: Block, x: np.ndarray, direction: int):
    """x [batch, L, C] -> z [batch, L, C], logdet [batch] (float64)."""
    out = [af_forward_one(blk, xb, direction) for xb in x]
    return np.stack([o[0] for o in out]), np.array([o[1] for o in out])


def af_forward_chunked_one(blk: Block, x: np.ndarray, direction: int, B: int, keep_from: int = 0):
    """The forward pass of one sample computed B positions at a time through the
    KV cache ([N] key design 3: finished blocks feed a KV cache), so that no
    score matrix is larger than B x L -- the same z as ``af_forward_one`` (it
    is the same causal computation), usable at lengths where an L x L score
    matrix does not fit in memory.  Returns (z rows of working-order positions
    >= keep_from, in working order; the logdet of the whole sequence; and its
    sum of |s|)."""
    xw = _f(_work(x, direction))
    L = xw.shape[0]
    cache = None
    zs, logdet, sabs = [], 0.0, 0.0
    for P in range(0, L, B):
        Q = min(P + B, L)
        mu, s, kv = transformer_rows(blk, masked_inputs(xw, P, Q), P, cache)
        if Q > keep_from:
            lo = max(P, keep_from) - P
            zs.append(((xw[P:Q] - mu) * np.exp(-s))[lo:])
        logdet -= s.sum()
        sabs += np.abs(s).sum()
        cache = kv if cache is None else [(np.concatenate([cache[l][0], kv[l][0]]),
                                           np.concatenate([cache[l][1], kv[l][1]]))
                                          for l in range(blk.layers)]
    return np.concatenate(zs), float(logdet), float(sabs)


# ----------------------------------------------------------------------------
# sequential inverse (textbook autoregressive inverse, token by token)

def af_inverse_seq_one(blk: Block, z: np.ndarray, direction: int):
    zw = _f(_work(z, direction))
    L, C = zw.shape
    xw = np.zeros_like(zw)
    cache = [(np.zeros((0, blk.d)), np.zeros((0, blk.d))) for _ in range(blk.layers)]
    for i in range(L):
        x_in = xw[i - 1:i] if i > 0 else np.zeros((1, C))
        mu, s, kv = transformer_rows(blk, x_in, i, cache)
        xw[i] = mu[0] + np.exp(s[0]) * zw[i]
        cache = [(np.concatenate([cache[l][0], kv[l][0]]),
                  np.concatenate([cache[l][1], kv[l][1]])) for l in range(blk.layers)]
    return _work(xw, direction).copy()


def af_inverse_seq(blk: Block, z: np.ndarray, direction: int):
    return np.stack([af_inverse_seq_one(blk, zb, direction) for zb in z])


# ----------------------------------------------------------------------------
# block-wise Jacobi inverse ([N] key design 3)

def jacobi_residual(x_new, x_old):
    """||x_new - x_old||^2 / ||x_new||^2 and the converged test (R4)."""
    num = float(((x_new - x_old) ** 2).sum())
    den = float((x_new ** 2).sum())
    return num, den


def converged(num, den, tau):
    if den == 0.0:
        return num == 0.0
    return num / den < tau


def block_starts(L: int, B) -> List[int]:
    """Start positions of the blocks of a sequence of L tokens, and L last.

    ``B`` is one block size (every block B tokens; L % B == 0), or a list of
    block sizes in sequence order summing to L ([N] "Key findings": the block
    size can change along the video, e.g. 64 for the first frame and 512
    later)."""
    sizes = [B] * (L // B) if isinstance(B, (int, np.integer)) else [int(b) for b in B]
    if isinstance(B, (int, np.integer)):
        assert L % B == 0
    assert sum(sizes) == L and all(b > 0 for b in sizes)
    return [0] + list(np.cumsum(sizes))


def warm_start_guess(xw: np.ndarray, zw: np.ndarray, P: int, Q: int, frame_len: int) -> np.ndarray:
    """x^(0) of the block of positions P..Q-1 under the video-aware warm start.

    [N] key design 3: a new frame starts from the previous frame's converged
    state.  Per token (R13): the token at position p starts from the
    converged x of the same spatial position in the most recent finished
    frame, p - k*frame_len with the smallest k >= 1 that lands before the
    block (p - k*frame_len < P); a token with no such finished position (the
    first frame) starts from z (R5).  With blocks of exactly one frame this is
    "block b starts from block b-1's x"."""
    out = np.empty((Q - P, zw.shape[1]))
    for p in range(P, Q):
        k = (p - P) // frame_len + 1
        src = p - k * frame_len
        out[p - P] = xw[src] if src >= 0 else zw[p]
    return out


def af_inverse_jacobi_one(blk: Block, z: np.ndarray, direction: int, B, tau: float,
                          max_iter: int, warm_start: bool, x0=None, trace=None,
                          x_known=None, n_known: int = 0):
    """One sample.  Returns (x, iters [n_blocks], converged [n_blocks]).

    ``B`` is the block size, or the list of block sizes (see ``block_starts``).
    ``x0`` optionally overrides the first block's starting guess (used by the
    any-start prefix-exactness pin); ``trace`` collects every iterate of every
    block when given a list.

    ``x_known`` [L, C] (original token order) with ``n_known`` > 0: the first
    ``n_known`` blocks are observed, not sampled -- their x is taken as given
    and only their K/V enter the cache ([N] "A complete example": I2V / V2V
    encode the observed frames with the flow's forward pass into the KV cache,
    then the following frames are generated autoregressively).  Those blocks
    report 0 iterations and count as converged.
    """
    zw = _f(_work(z, direction))
    L, C = zw.shape
    starts = block_starts(L, B)
    nb = len(starts) - 1
    xw = np.zeros_like(zw)
    xk_w = _f(_work(x_known, direction)) if n_known else None
    cache = None
    iters = np.zeros(nb, np.int64)
    conv = np.zeros(nb, bool)
    for b in range(nb):
        P, Q = starts[b], starts[b + 1]
        zb = zw[P:Q]
        if b < n_known:                                   # observed block: x given
            xk = xk_w[P:Q].copy()
            conv[b] = True
        elif b == 0 and x0 is not None:
            xk = _f(_work(x0, direction))[P:Q].copy()
        elif warm_start:
            xk = warm_start_guess(xw, zw, P, Q, blk.frame_len)   # previous frame's state (R13)
        else:
            xk = zb.copy()                                # R5
        for k in range(0 if b < n_known else max_iter):
            xw[P:Q] = xk
            mu, s, _ = transformer_rows(blk, masked_inputs(xw, P, Q), P, cache)
            x_new = mu + np.exp(s) * zb
            num, den = jacobi_residual(x_new, xk)
            xk = x_new
            iters[b] = k + 1
            if trace is not None:
                trace.append((b, k + 1, xk.copy()))
            if converged(num, den, tau):
                conv[b] = True
                break
        xw[P:Q] = xk                                      # R6
        if b + 1 < nb:                                    # commit K/V of the final x (R7)
            _, _, kv = transformer_rows(blk, masked_inputs(xw, P, Q), P, cache)
            if cache is None:
                cache = [(k_, v_) for (k_, v_) in kv]
            else:
                cache = [(np.concatenate([cache[l][0], kv[l][0]]),
                          np.concatenate([cache[l][1], kv[l][1]])) for l in range(blk.layers)]
    return _work(xw, direction).copy(), iters, conv


def af_inverse_jacobi(blk: Block, z: np.ndarray, direction: int, B, tau: float,
                      max_iter: int, warm_start: bool, x_known=None, n_known: int = 0):
    """z [batch, L, C] -> x [batch, L, C], iters [batch, n_blocks], converged [batch, n_blocks].

    ``B``: one block size or the list of block sizes.  ``x_known`` [batch, L,
    C] with ``n_known`` observed leading blocks: see ``af_inverse_jacobi_one``."""
    out = [af_inverse_jacobi_one(blk, zb, direction, B, tau, max_iter, warm_start,
                                 x_known=None if x_known is None else x_known[i], n_known=n_known)
           for i, zb in enumerate(z)]
    return (np.stack([o[0] for o in out]), np.stack([o[1] for o in out]),
            np.stack([o[2] for o in out]))


def window_starts(n_frames: int, window: int, overlap: int) -> List[int]:
    """First frames of the windows of a stream of n_frames frames: windows of
    `window` frames, each after the first repeating the last `overlap` frames
    of the one before ([N] "A complete example": streaming generation)."""
    assert 0 <= overlap < window
    starts = [0]
    while starts[-1] + window < n_frames:
        starts.append(starts[-1] + window - overlap)
    return starts


def af_inverse_jacobi_stream(blk: Block, z: np.ndarray, frame_len: int, window: int, overlap: int,
                             tau: float, max_iter: int, warm_start: bool):
    """Streaming block-Jacobi inverse past the model's length ([N] "A complete
    example": after a latent chunk is produced, f_D is re-run on the last
    `overlap` latents to rebuild the KV cache, and the next window_frames -
    overlap frames are generated).  z [batch, n_frames*frame_len, C], L->R,
    one frame per block.  Window w covers frames s_w .. s_w + window - 1
    (window_starts), at positions 0 .. window*frame_len - 1 of the model; its
    first `overlap` frames (after the first window) are the previous window's
    output, observed (flow-encoded into the cache), and the rest are
    generated.  Returns (x, iters [batch, n_frames]; observed frames count 0
    in the window that observes them, their own generating window's count is
    kept)."""
    batch, L, C = z.shape
    n_frames = L // frame_len
    x = np.zeros((batch, L, C))
    iters = np.zeros((batch, n_frames), np.int64)
    for i, s0 in enumerate(window_starts(n_frames, window, overlap)):
        nf = min(window, n_frames - s0)
        lo, hi = s0 * frame_len, (s0 + nf) * frame_len
        n_obs = overlap if i > 0 else 0
        xw, it, _ = af_inverse_jacobi(blk, z[:, lo:hi], L2R, frame_len, tau, max_iter, warm_start,
                                      x_known=x[:, lo:hi] if n_obs else None, n_known=n_obs)
        x[:, lo + n_obs * frame_len:hi] = xw[:, n_obs * frame_len:]
        iters[:, s0 + n_obs:s0 + nf] = it[:, n_obs:]
    return x, iters


# ----------------------------------------------------------------------------
# stacks of alternating-direction blocks ([N] key design 1: T >= 3 blocks of
# alternating direction; inversion undoes them last-to-first)

def stack_forward(blocks: List[Block], dirs: Sequence[int], x: np.ndarray):
    z = _f(x)
    total = np.zeros(x.shape[0])
    for blk, dr in zip(blocks, dirs):
        z, ld = af_forward(blk, z, dr)
        total = total + ld
    return z, total


def stack_inverse(blocks: List[Block], dirs: Sequence[int], z: np.ndarray, B: int,
                  tau: float, max_iter: int, warm_start: bool):
    x = _f(z)
    all_iters = [None] * len(blocks)
    for t in reversed(range(len(blocks))):
        x, it, _ = af_inverse_jacobi(blocks[t], x, dirs[t], B, tau, max_iter, warm_start)
        all_iters[t] = it
    return x, np.stack(all_iters)


# ----------------------------------------------------------------------------
# flow-score-matching denoiser s_phi ([N] key design 2: a light causal
# Transformer denoiser regressed on the model's score, with one frame of
# look-ahead; x is refined as x_noisy + sigma * s_phi(x_noisy), the Tweedie
# step x ~ x_noisy + sigma^2 grad log p with s_phi ~ sigma grad log p)
# Readings (D1-D3; the pages give only "8-layer Transformer, width of the
# shallow blocks", the look-ahead s_phi(x_{<=n+1}) ~ (sigma grad log p)_n and
# the loss):
#   D1 the denoiser reads x_noisy itself (no shift): h = x W_in^T + b_in + pos;
#   D2 the same pre-LN layers as the AF block; attention is by frames
#      (frame_len tokens a frame, every token of a frame sees the whole frame):
#      in the first layer a token of frame n attends frames <= n + 1, in every
#      later layer frames <= n -- so the output of frame n depends on frames
#      <= n + 1 exactly, as the pages' s_phi(x_{<=n+1}) states (a look-ahead
#      in every layer would reach one more frame per layer);
#   D3 final LayerNorm, linear head to C outputs s_phi; x = x_noisy + sigma s_phi.

class DenoiserBlock(Block):
    """Weights of the denoiser: the AF block's layout with a head of C rows."""


def lookahead_attention(q, K, V, heads, frame_len, ahead):
    """softmax(q K^T / sqrt(hd) over keys of frames <= query frame + ahead) V,
    for queries and keys at positions 0 .. n-1 of one sequence (D2)."""
    n, d = q.shape
    hd = d // heads
    pos = np.arange(n)
    allowed = (pos[None, :] // frame_len) <= (pos[:, None] // frame_len) + ahead
    out = np.empty_like(q)
    for h in range(heads):
        sl = slice(h * hd, (h + 1) * hd)
        S = (q[:, sl] @ K[:, sl].T) / math.sqrt(hd)
        S = np.where(allowed, S, -np.inf)
        S = S - S.max(axis=1, keepdims=True)
        E = np.exp(S)
        out[:, sl] = (E / E.sum(axis=1, keepdims=True)) @ V[:, sl]
    return out


def denoiser_scores(blk: DenoiserBlock, x_noisy: np.ndarray) -> np.ndarray:
    """s_phi of one sequence [n, C] (D1-D3)."""
    n = x_noisy.shape[0]
    d = blk.d
    h = linear(_f(x_noisy), blk.w_in, blk.b_in) + positions(blk, np.arange(n))
    for l, P in enumerate(blk.L_):
        a = layer_norm(h, P["ln1_g"], P["ln1_b"])
        qkv = linear(a, P["w_qkv"], P["b_qkv"])
        q, k, v = qkv[:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:]
        att = lookahead_attention(q, k, v, blk.heads, blk.frame_len, 1 if l == 0 else 0)
        h = h + linear(att, P["w_o"], P["b_o"])
        a = layer_norm(h, P["ln2_g"], P["ln2_b"])
        h = h + linear(gelu(linear(a, P["w_1"], P["b_1"])), P["w_2"], P["b_2"])
    return linear(layer_norm(h, blk.lnf_g, blk.lnf_b), blk.w_head, blk.b_head)


def denoise(blk: DenoiserBlock, x_noisy: np.ndarray, sigma: float) -> np.ndarray:
    """x_noisy [batch, L, C] -> x_noisy + sigma * s_phi(x_noisy) (float64)."""
    return np.stack([_f(xb) + sigma * denoiser_scores(blk, xb) for xb in x_noisy])


# ----------------------------------------------------------------------------
# brute-force Jacobian (pins the log-determinant on tiny inputs)

def jacobian_bruteforce(blk: Block, x: np.ndarray, direction: int, h: float = 1e-6):
    """Central-difference d z / d x of one sample, [L*C, L*C]."""
    x = _f(x)
    n = x.size
    J = np.empty((n, n))
    for j in range(n):
        e = np.zeros(n)
        e[j] = h
        zp, _ = af_forward_one(blk, (x.ravel() + e).reshape(x.shape), direction)
        zm, _ = af_forward_one(blk, (x.ravel() - e).reshape(x.shape), direction)
        J[:, j] = (zp.ravel() - zm.ravel()) / (2 * h)
    return J
