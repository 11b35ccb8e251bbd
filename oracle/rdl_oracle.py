"""Plain, slow, fp64 CPU oracle of route-layer chunk-routing sparse attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module: only the
tests, the smoke check and the benchmark's CPU-baseline leg do.  It shares no code with
the CUDA library (the seeded input generator lives in its own module and holds none of
this arithmetic).

What it computes follows the description of Prefilling-dLLM v2 ("Prefilling-dLLM v2:
Learned Chunk Routing for Long-Context Diffusion Language Models", Figure 3 caption and
Table 3; "The 172x Speedup Has an Evidence Budget", section "How learned routing controls
what the model can read"):

  * the context is cut into chunks of S = 64 positions, 63 content tokens followed by one
    routing mask in the last cell;
  * the mask's query pools its chunk's content keys with an intra-chunk softmax; the
    weighted sum is the summary key s_c, and the entropy H_c of the pooling weights is
    kept as a routing signal;
  * a content query adds a low-rank (rank r) residual and scores every summary; the score
    combines similarity to s_c and the entropy H_c;
  * scores are max-reduced across the heads of a GQA group and the top-K remote chunks are
    shared by every head of the group;
  * the selected chunk scores and the log-sum-exp of the bidirectional local window share
    one softmax partition; a second softmax spreads each chunk's mass over its 63 content
    tokens;
  * the non-route layers use bidirectional sliding-window attention.

Readings where the pages are silent (each is a keyword argument or a stated convention):
  score        z = tau * q_res . s_c - lam * H_c, tau = 1/sqrt(d), lam = 0.1
  query        the residual-adapted query scores summaries; raw q for attention logits
  summaries    per query head: each head of the mask's query pools its own KV head's keys
  radius w     window W(i) = { j : |p_i - j| <= w, 0 <= j < L } (2w+1 keys), all slots
  remote       chunk c is eligible iff none of its 64 positions lies in W(i)
  top-K order  by (group max desc, chunk index asc); fewer than K eligible: pad idx = -1
  partition    a selected chunk enters with its per-head score z_{i,h,c}
  mask rows    a mask-slot row outputs its pooled attention sum_j a_j v_j; it does not
               score or select
  storage      the selected indices are returned in ascending chunk order (a set)
Parity against the authors' trained model is unpinned: the pages print no numeric
example for v2.  Each function below is pinned by closed forms, invariants, brute force
and library reductions in tests/test_oracle_*.py.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np

S = 64                      # positions per chunk
CONTENT = S - 1             # content tokens per chunk; the last slot is the routing mask
NEG_INF = -np.inf


def tau_of(d: int) -> float:
    return 1.0 / math.sqrt(d)


def positions(Lq: int, L: int, q_pos: Optional[np.ndarray], b: int = 0) -> np.ndarray:
    """Position p_i of every query row: i itself in prefill, q_pos[b, i] in decode."""
    if q_pos is None:
        assert Lq == L
        return np.arange(L)
    return np.asarray(q_pos[b], dtype=np.int64)


def is_mask_slot(p) -> np.ndarray:
    return (np.asarray(p) % S) == S - 1


def content_positions(c: int) -> np.ndarray:
    """content(c) = {64c + j : j = 0..62}."""
    return S * c + np.arange(CONTENT)


def window(p: int, w: int, L: int) -> np.ndarray:
    """W(i): every position j with |p - j| <= w inside [0, L); empty when w < 0."""
    if w < 0:
        return np.zeros(0, dtype=np.int64)
    return np.arange(max(0, p - w), min(L, p + w + 1))


def eligible(p: int, w: int, C: int) -> np.ndarray:
    """E(i): chunks none of whose 64 positions lies within the window of p."""
    c = np.arange(C)
    if w < 0:
        return c
    first, last = S * c, S * c + S - 1
    return c[(last < p - w) | (first > p + w)]


def logsumexp(a: np.ndarray, axis=-1) -> np.ndarray:
    a = np.asarray(a, dtype=np.float64)
    m = np.max(a, axis=axis, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    with np.errstate(divide="ignore"):
        return np.squeeze(m, axis=axis) + np.log(np.sum(np.exp(a - m), axis=axis))


def softmax(a: np.ndarray, axis=-1) -> np.ndarray:
    a = np.asarray(a, dtype=np.float64)
    e = np.exp(a - np.max(a, axis=axis, keepdims=True))
    return e / np.sum(e, axis=axis, keepdims=True)


# ----------------------------------------------------------------------------- step 1

def pool_weights(q_m: np.ndarray, k_chunk: np.ndarray, mean_summary: bool = False):
    """Intra-chunk pooling weights a_j of one mask query over its chunk's 63 content keys.

    q_m [d], k_chunk [63, d].  a = softmax_j(tau * q_m . k_j); the mean-summary ablation
    (Table 6, "Mean summary") uses a_j = 1/63.
    """
    if mean_summary:
        return np.full(k_chunk.shape[0], 1.0 / k_chunk.shape[0])
    tau = tau_of(q_m.shape[-1])
    return softmax(tau * (k_chunk @ q_m))


def entropy(a: np.ndarray) -> float:
    """H = -sum_j a_j ln a_j with 0 ln 0 = 0."""
    a = np.asarray(a, dtype=np.float64)
    nz = a > 0
    return float(-np.sum(a[nz] * np.log(a[nz])))


def summary_pool(q_mask: np.ndarray, k: np.ndarray, v: Optional[np.ndarray] = None, *,
                 mean_summary: bool = False):
    """Summary keys, pooling entropies and mask-slot outputs (Figure 3 caption).

    q_mask [B, C, Hq, d]: query of the mask slot (position 64c+63) of every chunk.
    k, v   [B, Hkv, L, d].
    Returns s [B, Hq, C, d], H [B, Hq, C], o_mask [B, C, Hq, d] (None if v is None).
    For head h of KV group g = h // (Hq/Hkv):  s_{c,h} = sum_j a_j k_{64c+j},
    H_{c,h} = entropy(a), o_mask = sum_j a_j v_{64c+j}, j over the 63 content slots.
    """
    B, C, Hq, d = q_mask.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    s = np.zeros((B, Hq, C, d))
    H = np.zeros((B, Hq, C))
    o_mask = None if v is None else np.zeros((B, C, Hq, d))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for c in range(C):
                cp = content_positions(c)
                a = pool_weights(q_mask[b, c, h], k[b, g, cp], mean_summary)
                s[b, h, c] = a @ k[b, g, cp]
                H[b, h, c] = entropy(a)
                if v is not None:
                    o_mask[b, c, h] = a @ v[b, g, cp]
    return s, H, o_mask


# ----------------------------------------------------------------------------- step 2

def residual_query(q: np.ndarray, x: np.ndarray, w_down: np.ndarray, w_up: np.ndarray):
    """q_res = q + reshape((x W_down) W_up, [Hq, d]): the rank-r routing residual.

    q [..., Hq, d], x [..., D], w_down [D, r], w_up [r, Hq*d].  Only the route score uses
    q_res; the pretrained query q is left unchanged for attention.
    """
    Hq, d = q.shape[-2:]
    u = (x @ w_down) @ w_up
    return q + u.reshape(u.shape[:-1] + (Hq, d))


# ----------------------------------------------------------------------------- steps 3-4

def route_scores(q_res_i: np.ndarray, s_b: np.ndarray, H_b: np.ndarray, p: int, w: int,
                 lam: float) -> np.ndarray:
    """Per-head route scores of one query row.

    q_res_i [Hq, d]; s_b [Hq, C, d]; H_b [Hq, C].
    z[h, c] = tau * q_res_{h} . s_{c,h} - lam * H_{c,h} for c in E(i), -inf otherwise.
    """
    Hq, C, d = s_b.shape
    tau = tau_of(d)
    z = np.full((Hq, C), NEG_INF)
    E = eligible(p, w, C)
    for h in range(Hq):
        z[h, E] = tau * (s_b[h, E] @ q_res_i[h]) - lam * H_b[h, E]
    return z


def group_max(z: np.ndarray, Hkv: int) -> np.ndarray:
    """zeta[g, c] = max over the heads h of group g of z[h, c]."""
    Hq, C = z.shape
    return z.reshape(Hkv, Hq // Hkv, C).max(axis=1)


def select_topk(zeta_g: np.ndarray, elig: np.ndarray, K: int) -> np.ndarray:
    """Top-K eligible chunks of one (query, group), ordered by (zeta desc, chunk asc).

    A full stable sort (brute force), then the first K; padded with -1 when fewer than
    K chunks are eligible.  Returned in ascending chunk order.
    """
    cand = np.asarray(elig, dtype=np.int64)
    order = np.lexsort((cand, -zeta_g[cand]))          # primary: -zeta, then chunk index
    chosen = np.sort(cand[order[:K]])
    out = np.full(K, -1, dtype=np.int64)
    out[:chosen.size] = chosen
    return out


def kth_gap(zeta_g: np.ndarray, elig: np.ndarray, K: int) -> float:
    """zeta_(K) - zeta_(K+1) over eligible chunks (inf if at most K are eligible)."""
    vals = np.sort(zeta_g[np.asarray(elig, dtype=np.int64)])[::-1]
    if vals.size <= K:
        return math.inf
    return float(vals[K - 1] - vals[K])


def route_score_topk(q: np.ndarray, q_pos: Optional[np.ndarray], x: np.ndarray,
                     w_down: np.ndarray, w_up: np.ndarray, s: np.ndarray, H: np.ndarray, *,
                     Hkv: int, K: int, w: int, lam: float = 0.1, L: Optional[int] = None,
                     rows: Optional[np.ndarray] = None, with_zeta: bool = False):
    """Selected chunks and their per-head scores for query rows.

    q [B, Lq, Hq, d], x [B, Lq, D], s [B, Hq, C, d], H [B, Hq, C].
    rows: optional subset of query rows (the rest are not computed: idx = -2 marks them).
    Returns idx [B, Hkv, Lq, K] int64 (-1: no chunk; mask-slot rows are all -1),
            z_sel [B, Hq, Lq, K] (-inf where idx = -1), and, with with_zeta, the group
            max scores zeta [B, Hkv, Lq, C] and the K-th gaps [B, Hkv, Lq].
    """
    B, Lq, Hq, d = q.shape
    C = s.shape[2]
    L = L if L is not None else C * S
    G = Hq // Hkv
    rows = np.arange(Lq) if rows is None else np.asarray(rows)
    idx = np.full((B, Hkv, Lq, K), -2, dtype=np.int64)
    z_sel = np.full((B, Hq, Lq, K), np.nan)
    zeta_all = np.full((B, Hkv, Lq, C), np.nan) if with_zeta else None
    gaps = np.full((B, Hkv, Lq), np.nan) if with_zeta else None
    for b in range(B):
        pos = positions(Lq, L, q_pos, b)
        for i in rows:
            p = int(pos[i])
            if is_mask_slot(p):
                idx[b, :, i] = -1
                z_sel[b, :, i] = NEG_INF
                continue
            q_res = residual_query(q[b, i], x[b, i], w_down, w_up)
            z = route_scores(q_res, s[b], H[b], p, w, lam)
            zeta = group_max(z, Hkv)
            E = eligible(p, w, C)
            for g in range(Hkv):
                t = select_topk(zeta[g], E, K)
                idx[b, g, i] = t
                for hh in range(G):
                    h = g * G + hh
                    z_sel[b, h, i] = np.where(t >= 0, z[h, np.maximum(t, 0)], NEG_INF)
                if with_zeta:
                    zeta_all[b, g, i] = zeta[g]
                    gaps[b, g, i] = kth_gap(zeta[g], E, K)
    if with_zeta:
        return idx, z_sel, zeta_all, gaps
    return idx, z_sel


def scores_for(q: np.ndarray, q_pos, x, w_down, w_up, s, H, idx, *, w: int, lam: float = 0.1,
               L: Optional[int] = None, rows=None) -> np.ndarray:
    """Per-head scores z_{i,h,c} of given chunk lists idx [B, Hkv, Lq, K] (e.g. chosen by
    another implementation), so outputs can be compared on the same selection."""
    B, Lq, Hq, d = q.shape
    Hkv, K = idx.shape[1], idx.shape[3]
    C = s.shape[2]
    L = L if L is not None else C * S
    G = Hq // Hkv
    rows = np.arange(Lq) if rows is None else np.asarray(rows)
    z_sel = np.full((B, Hq, Lq, K), NEG_INF)
    for b in range(B):
        pos = positions(Lq, L, q_pos, b)
        for i in rows:
            p = int(pos[i])
            if is_mask_slot(p):
                continue
            z = route_scores(residual_query(q[b, i], x[b, i], w_down, w_up), s[b], H[b], p,
                             w, lam)
            for g in range(Hkv):
                t = idx[b, g, i]
                for hh in range(G):
                    h = g * G + hh
                    z_sel[b, h, i] = np.where(t >= 0, z[h, np.maximum(t, 0)], NEG_INF)
    return z_sel


# ----------------------------------------------------------------------------- steps 5-7

def attend(qv: np.ndarray, keys: np.ndarray, vals: np.ndarray):
    """Softmax attention of one query over a key list: (lse, normalised output)."""
    tau = tau_of(qv.shape[-1])
    logits = tau * (keys @ qv)
    if logits.size == 0:
        return NEG_INF, np.zeros(vals.shape[-1])
    return float(logsumexp(logits)), softmax(logits) @ vals


def route_attn_row(q_i: np.ndarray, p: int, k_g: np.ndarray, v_g: np.ndarray,
                   chunks: np.ndarray, z_c: np.ndarray, w: int):
    """Two-level partition for one (query row, head).

    q_i [d]; k_g, v_g [L, d] of the head's KV group; chunks: selected chunk ids (-1 =
    none); z_c: their scores for this head.
    lambda_loc = LSE of the window logits, o_loc its softmax output;
    for each selected c: lse_c, o_c over content(c) only;
    Z = e^lambda_loc + sum_c e^{z_c};  o = (e^lambda_loc o_loc + sum_c e^{z_c} o_c) / Z.
    Returns (o [d], ln Z).
    """
    L = k_g.shape[0]
    W = window(p, w, L)
    lam_loc, o_loc = attend(q_i, k_g[W], v_g[W])
    parts_logit = [lam_loc]
    parts_out = [o_loc]
    for c, zc in zip(chunks, z_c):
        if c < 0:
            continue
        cp = content_positions(int(c))
        _, o_c = attend(q_i, k_g[cp], v_g[cp])
        parts_logit.append(float(zc))
        parts_out.append(o_c)
    logits = np.array(parts_logit)
    lnZ = float(logsumexp(logits))
    mass = np.exp(logits - lnZ)                        # partition masses, sum to 1
    o = np.zeros_like(o_loc)
    for m, oc in zip(mass, parts_out):
        if m > 0:
            o = o + m * oc
    return o, lnZ


def route_attn(q: np.ndarray, q_pos: Optional[np.ndarray], k: np.ndarray, v: np.ndarray,
               idx: np.ndarray, z_sel: np.ndarray, *, w: int, rows=None):
    """Route-layer attention output for content query rows.

    q [B, Lq, Hq, d]; k, v [B, Hkv, L, d]; idx [B, Hkv, Lq, K]; z_sel [B, Hq, Lq, K].
    Returns o [B, Lq, Hq, d] and lse [B, Hq, Lq]; rows not computed (mask slots, rows
    outside `rows`) are NaN.
    """
    B, Lq, Hq, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    G = Hq // Hkv
    rows = np.arange(Lq) if rows is None else np.asarray(rows)
    o = np.full((B, Lq, Hq, d), np.nan)
    lse = np.full((B, Hq, Lq), np.nan)
    for b in range(B):
        pos = positions(Lq, L, q_pos, b)
        for i in rows:
            p = int(pos[i])
            if is_mask_slot(p):
                continue
            for h in range(Hq):
                g = h // G
                o[b, i, h], lse[b, h, i] = route_attn_row(q[b, i, h], p, k[b, g], v[b, g],
                                                          idx[b, g, i], z_sel[b, h, i], w)
    return o, lse


# ----------------------------------------------------------------------------- companion

def swa_attn(q: np.ndarray, q_pos: Optional[np.ndarray], k: np.ndarray, v: np.ndarray, *,
             w: int, rows=None):
    """Bidirectional sliding-window attention (the non-route layers): every row, mask
    slots included, attends to W(i) = {j : |p_i - j| <= w}.
    Returns o [B, Lq, Hq, d], lse [B, Hq, Lq] (NaN outside `rows`)."""
    B, Lq, Hq, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    G = Hq // Hkv
    rows = np.arange(Lq) if rows is None else np.asarray(rows)
    o = np.full((B, Lq, Hq, d), np.nan)
    lse = np.full((B, Hq, Lq), np.nan)
    for b in range(B):
        pos = positions(Lq, L, q_pos, b)
        for i in rows:
            W = window(int(pos[i]), w, L)
            for h in range(Hq):
                g = h // G
                lse[b, h, i], o[b, i, h] = attend(q[b, i, h], k[b, g, W], v[b, g, W])
    return o, lse


# ----------------------------------------------------------------------------- whole layer

def route_layer(q, q_pos, k, v, x, w_down, w_up, *, Hkv: int, K: int, w: int,
                lam: float = 0.1, q_mask=None, mean_summary: bool = False, rows=None):
    """Steps 1-7 for one route layer (prefill when q_pos is None)."""
    B, Lq, Hq, d = q.shape
    L = k.shape[2]
    if q_mask is None:
        q_mask = q[:, S - 1::S]
    s, H, o_mask = summary_pool(q_mask, k, v, mean_summary=mean_summary)
    idx, z_sel = route_score_topk(q, q_pos, x, w_down, w_up, s, H, Hkv=Hkv, K=K, w=w,
                                  lam=lam, L=L, rows=rows)
    o, lse = route_attn(q, q_pos, k, v, idx, z_sel, w=w, rows=rows)
    return dict(s=s, H=H, o_mask=o_mask, idx=idx, z_sel=z_sel, o=o, lse=lse)
