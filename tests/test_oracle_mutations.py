"""Plant plausible mistakes in the oracle (CPU only) and confirm the pins catch each.

Every mutation below is a slip one could make while writing the oracle from the
description: a wrong scale, an off-by-one window, a transposed reshape, a flipped sign,
a mean where a max belongs, the mask slot counted as content, a reversed tie-break, the
chunk's own log-sum-exp used where its routing score belongs.
"""
import math

import numpy as np
import pytest

import pins
from oracle import rdl_oracle as O


def _tau_wrong(d):
    return 1.0 / d


def _window_exclusive(p, w, L):
    if w < 0:
        return np.zeros(0, dtype=np.int64)
    return np.arange(max(0, p - w + 1), min(L, p + w))


def _eligible_own_chunk_only(p, w, C):
    c = np.arange(C)
    return c if w < 0 else c[c != p // O.S]


def _entropy_sign(a):
    a = np.asarray(a, dtype=np.float64)
    nz = a > 0
    return float(np.sum(a[nz] * np.log(a[nz])))


def _group_mean(z, Hkv):
    Hq, C = z.shape
    return z.reshape(Hkv, Hq // Hkv, C).mean(axis=1)


def _content_with_mask(c):
    return O.S * c + np.arange(O.S)


def _residual_transposed(q, x, w_down, w_up):
    Hq, d = q.shape[-2:]
    u = (x @ w_down) @ w_up
    return q + np.swapaxes(u.reshape(u.shape[:-1] + (d, Hq)), -1, -2)


def _topk_ties_high(zeta_g, elig, K):
    cand = np.asarray(elig, dtype=np.int64)
    order = np.lexsort((-cand, -zeta_g[cand]))
    chosen = np.sort(cand[order[:K]])
    out = np.full(K, -1, dtype=np.int64)
    out[:chosen.size] = chosen
    return out


def _pool_no_tau(q_m, k_chunk, mean_summary=False):
    return O.softmax(k_chunk @ q_m)


_real_row = O.route_attn_row


def _row_uses_chunk_lse(q_i, p, k_g, v_g, chunks, z_c, w):
    """Mistake: the chunk enters the partition with its own lse, not its routing score."""
    tau = O.tau_of(q_i.shape[-1])
    zz = []
    for c in chunks:
        if c < 0:
            zz.append(-np.inf)
        else:
            cp = O.content_positions(int(c))
            zz.append(float(O.logsumexp(tau * (k_g[cp] @ q_i))))
    return _real_row(q_i, p, k_g, v_g, chunks, np.array(zz), w)


def _row_unnormalised_chunk(q_i, p, k_g, v_g, chunks, z_c, w):
    """Mistake: the second-level softmax is skipped (chunk mass not spread)."""
    o, lnZ = _real_row(q_i, p, k_g, v_g, chunks, z_c, w)
    return o * 1.01, lnZ


_real_scores_for = O.scores_for


def _scores_for_heads_reversed(q, q_pos, x, w_down, w_up, s, H, idx, **kw):
    """Mistake: the heads of each group are read in reverse order."""
    z = _real_scores_for(q, q_pos, x, w_down, w_up, s, H, idx, **kw)
    Hkv = idx.shape[1]
    G = z.shape[1] // Hkv
    return z.reshape(z.shape[0], Hkv, G, *z.shape[2:])[:, :, ::-1].reshape(z.shape)


def _scores_for_group_max(q, q_pos, x, w_down, w_up, s, H, idx, **kw):
    """Mistake: every head of a group gets the group-max score."""
    z = _real_scores_for(q, q_pos, x, w_down, w_up, s, H, idx, **kw)
    Hkv = idx.shape[1]
    G = z.shape[1] // Hkv
    zg = z.reshape(z.shape[0], Hkv, G, *z.shape[2:]).max(axis=2, keepdims=True)
    return np.broadcast_to(zg, (z.shape[0], Hkv, G) + z.shape[2:]).reshape(z.shape)


MUTATIONS = {
    "scores_for_heads_reversed": ("scores_for", _scores_for_heads_reversed),
    "scores_for_group_max": ("scores_for", _scores_for_group_max),
    "tau_1_over_d": ("tau_of", _tau_wrong),
    "window_exclusive": ("window", _window_exclusive),
    "eligible_ignores_window": ("eligible", _eligible_own_chunk_only),
    "entropy_sign": ("entropy", _entropy_sign),
    "group_mean": ("group_max", _group_mean),
    "mask_slot_is_content": ("content_positions", _content_with_mask),
    "residual_transposed": ("residual_query", _residual_transposed),
    "topk_ties_high_index": ("select_topk", _topk_ties_high),
    "pool_without_tau": ("pool_weights", _pool_no_tau),
    "partition_uses_chunk_lse": ("route_attn_row", _row_uses_chunk_lse),
    "partition_scaled": ("route_attn_row", _row_unnormalised_chunk),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    failed = pins.run_all()
    assert failed, f"no pin caught the planted mistake {name}"


def test_unmutated_oracle_passes_all_pins():
    assert pins.run_all() == []
