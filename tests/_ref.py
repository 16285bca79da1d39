"""Independent references the oracle is pinned to (tests only).

Masks here are built with whole-matrix band / Kronecker operations, not with
the oracle's per-row live-key sets, and attention is torch's fp64 CPU
scaled_dot_product_attention: a library routine the oracle's special cases
must reduce to.
"""
import numpy as np
import torch


def sdpa(q, k, v, mask=None, causal=False, scale=None):
    """torch SDPA in float64 on [B, S, H, d] arrays; mask is a boolean [S, S] (True = attend)
    or a per-(b, h_q) array [B, H_q, S, S].  GQA via enable_gqa (query head h reads
    KV head h // G)."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).permute(0, 2, 1, 3)  # noqa: E731
    Q, K, V = t(q), t(k), t(v)
    m = None if mask is None else torch.from_numpy(np.asarray(mask, dtype=bool))
    o = torch.nn.functional.scaled_dot_product_attention(
        Q, K, V, attn_mask=m, is_causal=causal, scale=scale, enable_gqa=(Q.shape[1] != K.shape[1]))
    return o.permute(0, 2, 1, 3).numpy()


def causal_mask(S):
    return np.tril(np.ones((S, S), dtype=bool))


def streaming_mask(S, n_sink, window):
    """Band of the last `window` keys (diagonal included) plus the first n_sink columns, causal."""
    ones = np.ones((S, S), dtype=bool)
    band = np.tril(ones) & ~np.tril(ones, -window)
    sink = np.zeros((S, S), dtype=bool)
    sink[:, :max(0, min(n_sink, S))] = True
    return band | (sink & np.tril(ones))


def block_mask(S, block, listed_rows):
    """Kronecker expansion of a block bitmap, cut to S and made causal.
    listed_rows[qb] = iterable of listed key blocks of query block qb."""
    n = -(-S // block)
    bm = np.zeros((n, n), dtype=bool)
    for qb, cols in enumerate(listed_rows):
        bm[qb, list(cols)] = True
    full = np.kron(bm, np.ones((block, block), dtype=bool))[:S, :S]
    return full & causal_mask(S)


def csr_rows(row_ptr, cols, b, h, H_kv, n_qb):
    base = (b * H_kv + h) * n_qb
    return [cols[row_ptr[base + qb]:row_ptr[base + qb + 1]] for qb in range(n_qb)]


def random_csr(rng, B, H_kv, S, block, p_extra=0.3, full=False, diag_only=False):
    n_qb = -(-S // block)
    rows = []
    for _ in range(B * H_kv):
        for qb in range(n_qb):
            if full:
                c = np.arange(qb + 1)
            elif diag_only:
                c = np.array([qb])
            else:
                extra = np.nonzero(rng.random(qb) < p_extra)[0]
                c = np.unique(np.concatenate([extra, [qb]]))
            rows.append(c)
    rp = np.zeros(len(rows) + 1, np.int64)
    np.cumsum([len(r) for r in rows], out=rp[1:])
    return rp.astype(np.int32), np.concatenate(rows).astype(np.int32)
