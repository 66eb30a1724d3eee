"""Algorithmic work of the AF-block path, for throughput and roofline reports.

Counts what the method computes, not what the kernels pad: per pass over n
query rows of one AF block, every dense contraction is 2*m*n*k flops and causal
attention contributes 4*d flops per (query, key) pair with key <= query.
"""


def pass_flops(d: int, C: int, layers: int, mlp_ratio: int, n_rows: int, key_pairs: int) -> float:
    per_row = (layers * (2 * d * 3 * d + 2 * d * d + 2 * 2 * mlp_ratio * d * d)
               + 2 * C * d + 2 * 2 * C * d)
    return float(n_rows) * per_row + float(layers) * 4.0 * d * key_pairs


def causal_pairs(p0: int, n: int) -> int:
    """Number of (query, key) pairs with key <= query for queries at p0..p0+n-1."""
    return n * p0 + n * (n + 1) // 2


def forward_flops(shape, batch: int, L: int, T: int = 1) -> float:
    return T * batch * pass_flops(shape.d, shape.C, shape.layers, shape.mlp_ratio, L, causal_pairs(0, L))


def jacobi_flops(shape, iters, L: int, B: int) -> float:
    """Inverse work from the updates actually run: iters[t][s][b] passes of block b's B rows
    (prefix P = b*B in the cache), plus one commit pass of every block that has a successor."""
    total = 0.0
    nb = L // B
    for per_block in iters:             # blocks of the stack
        for row in per_block:           # samples
            for b, k in enumerate(row):
                rows = B
                f = pass_flops(shape.d, shape.C, shape.layers, shape.mlp_ratio, rows, causal_pairs(b * B, B))
                total += float(k) * f
                if b + 1 < nb:
                    total += f          # the K/V commit of block b
    return total


def denoiser_flops(shape, batch: int, L: int) -> float:
    """One forward pass of the flow-score-matching denoiser: the dense
    contractions of every row, plus 4*d flops per (query, key) pair that its
    frame masks allow (one frame of look-ahead in the first layer, frames up
    to the query's own in the others)."""
    F = shape.frame_len
    d, C = shape.d, shape.C
    dense = L * (shape.layers * (2 * d * 3 * d + 2 * d * d + 2 * 2 * shape.mlp_ratio * d * d) + 2 * C * d + 2 * C * d)
    pairs_first = sum(min((p // F + 2) * F, L) for p in range(L))
    pairs_rest = sum(min((p // F + 1) * F, L) for p in range(L))
    att = 4.0 * d * (pairs_first + (shape.layers - 1) * pairs_rest)
    return float(batch) * (dense + att)
