"""Checks that pin the fp64 oracle to facts outside itself.

Each check raises AssertionError when the oracle disagrees with a closed form, an
invariant, a brute-force result or an independent library routine (torch CPU SDPA in
fp64).  test_oracle.py runs them on the oracle as it is; test_oracle_mutations.py plants
plausible mistakes in the oracle and confirms that at least one check catches each.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

from oracle import rdl_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
LN63 = math.log(63.0)


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rng(seed):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------------------- layout

def check_layout_facts():
    """Chunk layout and key budget against the pages' printed figures."""
    gl = golden("pages_layout.json")
    L = gl["training_positions"]
    content = [p for p in range(L) if not O.is_mask_slot(p)]
    assert len(content) == gl["text_tokens_per_sequence"]
    assert O.content_positions(0).size == gl["content_tokens_per_chunk"]
    assert O.S == gl["chunk_positions"]
    # window of an interior query: 2*radius + 1 positions
    r = gl["route_layer"]["local_radius"]
    W = O.window(8000, r, L)
    route_budget = W.size + gl["route_layer"]["remote_chunks"] * gl["route_layer"]["chunk"]
    swa_budget = O.window(8000, gl["other_layers"]["local_radius"], L).size
    assert abs(route_budget - gl["total_budget_approx"]) <= 1, route_budget
    assert abs(swa_budget - gl["total_budget_approx"]) <= 1, swa_budget
    assert route_budget == swa_budget == 2561


def check_window_eligibility(L=1024, seed=0):
    """Eligible chunks never touch the window; every non-eligible chunk touches it."""
    C = L // O.S
    rng = _rng(seed)
    for _ in range(200):
        p = int(rng.integers(0, L))
        w = int(rng.integers(-1, 300))
        W = set(O.window(p, w, L).tolist())
        if w >= 0:
            assert W == {j for j in range(L) if abs(p - j) <= w}
            assert len(W) == min(L, p + w + 1) - max(0, p - w)
        E = set(O.eligible(p, w, C).tolist())
        for c in range(C):
            touches = any((O.S * c + j) in W for j in range(O.S))
            assert (c in E) == (not touches), (p, w, c)
        if w >= 0:
            assert p // O.S not in E


# ----------------------------------------------------------------------------- pooling

def check_pool_invariants(seed=1):
    rng = _rng(seed)
    B, C, Hq, Hkv, d = 1, 3, 4, 2, 16
    qm = rng.standard_normal((B, C, Hq, d)) * 2.0
    k = rng.standard_normal((B, Hkv, C * O.S, d))
    v = rng.standard_normal((B, Hkv, C * O.S, d))
    s, H, om = O.summary_pool(qm, k, v)
    for h in range(Hq):
        g = h // (Hq // Hkv)
        for c in range(C):
            cp = O.content_positions(c)
            a = O.pool_weights(qm[0, c, h], k[0, g, cp])
            assert abs(a.sum() - 1.0) < 1e-12 and (a >= 0).all()
            assert -1e-12 <= H[0, h, c] <= LN63 + 1e-12
            # the summary is a convex combination of the chunk's content keys
            lo, hi = k[0, g, cp].min(0), k[0, g, cp].max(0)
            assert (s[0, h, c] >= lo - 1e-12).all() and (s[0, h, c] <= hi + 1e-12).all()
            # the mask slot's own key (position 64c+63) takes no part
            k2 = k.copy()
            k2[0, g, O.S * c + O.S - 1] += 100.0
            s2, H2, _ = O.summary_pool(qm[:, c:c + 1], k2[:, :, O.S * c:O.S * (c + 1)])
            assert np.allclose(s2[0, h, 0], s[0, h, c]) and np.isclose(H2[0, h, 0], H[0, h, c])
    # pooling with v = k reproduces the summary in the mask-row output
    _, _, om_k = O.summary_pool(qm, k, k)
    assert np.allclose(np.transpose(om_k, (0, 2, 1, 3)), s, atol=1e-12)


def check_pool_closed_forms():
    d = 2
    # (a) all 63 content keys equal: s = that key, H = ln 63, for any mask query
    kbar = np.array([0.7, -1.3])
    k = np.zeros((1, 1, O.S, d))
    k[0, 0, :O.CONTENT] = kbar
    k[0, 0, O.CONTENT] = [50.0, 50.0]           # mask-slot key: must be ignored
    qm = np.array([[[[3.0, -2.0]]]])
    s, H, _ = O.summary_pool(qm, k)
    assert np.allclose(s[0, 0, 0], kbar, atol=1e-14)
    assert abs(H[0, 0, 0] - LN63) < 1e-12
    # (b) one logit raised by t, the other 62 equal (zero): with q_m = (sqrt(2), 0) and
    #     tau = 1/sqrt(2) the logit of key (t, y) is t.
    for t in (0.0, 0.5, 2.0, 7.0):
        k = np.zeros((1, 1, O.S, d))
        ys = np.linspace(-1.0, 1.0, O.CONTENT)
        k[0, 0, :O.CONTENT, 1] = ys
        jstar = 17
        k[0, 0, jstar, 0] = t
        qm = np.array([[[[math.sqrt(2.0), 0.0]]]])
        s, H, _ = O.summary_pool(qm, k)
        e = math.exp(t)
        astar = e / (e + 62.0)
        Hexp = math.log(e + 62.0) - t * e / (e + 62.0)
        sexp = np.array([astar * t,
                         astar * ys[jstar] + (1 - astar) / 62.0 * (ys.sum() - ys[jstar])])
        assert abs(H[0, 0, 0] - Hexp) < 1e-12, (t, H[0, 0, 0], Hexp)
        assert np.allclose(s[0, 0, 0], sexp, atol=1e-12)


def check_pool_shift_invariance(seed=2):
    rng = _rng(seed)
    d = 8
    qm = rng.standard_normal((1, 2, 1, d))
    k = rng.standard_normal((1, 1, 2 * O.S, d))
    s, H, _ = O.summary_pool(qm, k)
    # shifting every content key of a chunk by delta changes logits by a constant only if
    # q.delta is constant -- true for any delta: tau*q.(k+delta) = tau*q.k + tau*q.delta
    delta = rng.standard_normal(d)
    k2 = k.copy()
    k2[0, 0, :O.CONTENT] += delta
    s2, H2, _ = O.summary_pool(qm, k2)
    assert np.allclose(s2[0, 0, 0], s[0, 0, 0] + delta, atol=1e-12)
    assert abs(H2[0, 0, 0] - H[0, 0, 0]) < 1e-12
    assert np.allclose(s2[0, 0, 1], s[0, 0, 1]) and H2[0, 0, 1] == H[0, 0, 1]


def check_pool_gqa_and_mean():
    d, Hq, Hkv = 4, 4, 2
    rng = _rng(3)
    k = rng.standard_normal((1, Hkv, O.S, d))
    k[0, 0] = 0.0                                    # group 0 keys are zero
    qm = rng.standard_normal((1, 1, Hq, d))
    s, H, _ = O.summary_pool(qm, k)
    assert np.all(s[0, :2] == 0.0) and np.all(np.abs(s[0, 2:]) > 0)
    assert np.allclose(H[0, :2], LN63)
    sm, Hm, _ = O.summary_pool(qm, k, mean_summary=True)
    assert np.allclose(sm[0, 2, 0], k[0, 1, :O.CONTENT].mean(0))
    assert np.allclose(Hm, LN63)


def check_pool_peaked_cosine():
    """A very peaked pooling makes the summary the peaked key (cosine -> 1), the Figure 4
    diagnostic in miniature."""
    d = 16
    rng = _rng(4)
    k = rng.standard_normal((1, 1, O.S, d))
    j = 40
    qm = (60.0 * math.sqrt(d) * k[0, 0, j] / np.linalg.norm(k[0, 0, j]) ** 2)[None, None, None]
    s, H, _ = O.summary_pool(qm, k)
    cos = s[0, 0, 0] @ k[0, 0, j] / np.linalg.norm(s[0, 0, 0]) / np.linalg.norm(k[0, 0, j])
    assert cos > 0.999 and H[0, 0, 0] < 0.05


# ----------------------------------------------------------------------------- routing

def check_residual_layout():
    """The rank-r residual lands on head h, element e through column h*d + e of W_up."""
    Hq, d, D, r = 3, 4, 5, 5
    q = np.zeros((Hq, d))
    x = np.arange(1.0, D + 1)
    w_down = np.eye(D, r)
    w_up = np.zeros((r, Hq * d))
    w_up[2, 1 * d + 3] = 10.0                       # t_2 = x_2 = 3  ->  q_res[1, 3] = 30
    w_up[4, 2 * d + 0] = -1.0                       # t_4 = x_4 = 5  ->  q_res[2, 0] = -5
    qr = O.residual_query(q, x, w_down, w_up)
    exp = np.zeros((Hq, d))
    exp[1, 3] = 30.0
    exp[2, 0] = -5.0
    assert np.array_equal(qr, exp), qr
    # rank structure: the residual of every query lies in the row space of W_up
    rng = _rng(5)
    X = rng.standard_normal((50, D))
    U = O.residual_query(np.zeros((50, Hq, d)), X, rng.standard_normal((D, 2)),
                         rng.standard_normal((2, Hq * d)))
    assert np.linalg.matrix_rank(U.reshape(50, -1), tol=1e-9) == 2


def check_score_hand_example():
    """d = 2, one head, two chunks, x = 0 (no residual): z = q.s/sqrt(2) - lam*H."""
    d, lam = 2, 0.1
    q = np.array([[[[1.0, 2.0]]]])                  # [B, Lq, Hq, d] one row at position 5
    s = np.array([[[[0.5, 0.25], [-1.0, 3.0]]]])     # [B, Hq, C, d]
    H = np.array([[[1.0, 2.0]]])
    x = np.zeros((1, 1, 3))
    qp = np.array([[5]])
    idx, z, zeta, gaps = O.route_score_topk(q, qp, x, np.zeros((3, 2)), np.zeros((2, 2)), s, H,
                                            Hkv=1, K=1, w=-1, lam=lam, L=128, with_zeta=True)
    z0 = (1.0 * 0.5 + 2.0 * 0.25) / math.sqrt(2) - 0.1 * 1.0
    z1 = (-1.0 + 6.0) / math.sqrt(2) - 0.1 * 2.0
    assert np.allclose(zeta[0, 0, 0], [z0, z1], atol=1e-14)
    assert idx[0, 0, 0, 0] == 1 and abs(z[0, 0, 0, 0] - z1) < 1e-14
    assert abs(gaps[0, 0, 0] - (z1 - z0)) < 1e-14
    # entropy: equal summaries, lower entropy wins
    s2 = np.array([[[[1.0, 1.0], [1.0, 1.0]]]])
    H2 = np.array([[[3.0, 0.5]]])
    idx2, _ = O.route_score_topk(q, qp, x, np.zeros((3, 2)), np.zeros((2, 2)), s2, H2,
                                 Hkv=1, K=1, w=-1, lam=lam, L=128)
    assert idx2[0, 0, 0, 0] == 1


def _brute_topk(zeta_g, elig, K):
    cand = sorted(((-float(zeta_g[c]), int(c)) for c in elig))
    chosen = sorted(c for _, c in cand[:K])
    return chosen + [-1] * (K - len(chosen))


def check_topk_bruteforce(seed=6):
    rng = _rng(seed)
    for trial in range(300):
        C = int(rng.integers(1, 40))
        K = int(rng.integers(1, 12))
        zeta = np.round(rng.standard_normal(C), 1)      # rounding creates exact ties
        elig = np.sort(rng.choice(C, size=int(rng.integers(0, C + 1)), replace=False))
        got = O.select_topk(zeta, elig, K).tolist()
        assert got == _brute_topk(zeta, elig, K), (zeta, elig, K, got)


def _route_case(seed, *, L=512, Hq=6, Hkv=2, d=8, D=12, r=3, K=3, w=40, lam=0.1):
    rng = _rng(seed)
    C = L // O.S
    q = rng.standard_normal((1, L, Hq, d))
    k = rng.standard_normal((1, Hkv, L, d))
    v = rng.standard_normal((1, Hkv, L, d))
    x = rng.standard_normal((1, L, D))
    wd = rng.standard_normal((D, r)) * 0.3
    wu = rng.standard_normal((r, Hq * d)) * 0.3
    return dict(q=q, k=k, v=v, x=x, wd=wd, wu=wu, Hkv=Hkv, K=K, w=w, lam=lam, C=C, L=L)


def check_selection_properties(seed=7):
    cs = _route_case(seed)
    q, k, v, x, wd, wu = cs["q"], cs["k"], cs["v"], cs["x"], cs["wd"], cs["wu"]
    s, H, _ = O.summary_pool(q[:, O.S - 1::O.S], k, v)
    rows = np.arange(0, cs["L"], 7)
    idx, z, zeta, gaps = O.route_score_topk(q, None, x, wd, wu, s, H, Hkv=cs["Hkv"], K=cs["K"],
                                            w=cs["w"], lam=cs["lam"], rows=rows, with_zeta=True)
    G = q.shape[2] // cs["Hkv"]
    for i in rows:
        if O.is_mask_slot(i):
            assert np.all(idx[0, :, i] == -1)
            continue
        E = O.eligible(i, cs["w"], cs["C"])
        W = set(O.window(i, cs["w"], cs["L"]).tolist())
        for g in range(cs["Hkv"]):
            t = idx[0, g, i]
            assert list(t) == _brute_topk(zeta[0, g, i], E, cs["K"])
            for c in t[t >= 0]:
                assert not (set(range(O.S * c, O.S * c + O.S)) & W)
            # the group max is the max of per-head scores recomputed from the definition
            qr = q[0, i] + ((x[0, i] @ wd) @ wu).reshape(q.shape[2], -1)
            for c in E:
                heads = [qr[g * G + hh] @ s[0, g * G + hh, c] / math.sqrt(q.shape[3])
                         - cs["lam"] * H[0, g * G + hh, c] for hh in range(G)]
                assert abs(zeta[0, g, i, c] - max(heads)) < 1e-12
            for kk, c in enumerate(t):
                for hh in range(G):
                    h = g * G + hh
                    if c < 0:
                        assert z[0, h, i, kk] == -np.inf
                    else:
                        assert abs(z[0, h, i, kk] - (qr[h] @ s[0, h, c] / math.sqrt(q.shape[3])
                                                     - cs["lam"] * H[0, h, c])) < 1e-12
    # permuting the heads inside a group leaves every selection unchanged
    perm = np.arange(q.shape[2])
    perm[:G] = perm[:G][::-1]
    wu3 = wu.reshape(wu.shape[0], q.shape[2], -1)[:, perm].reshape(wu.shape)
    idx_p, _ = O.route_score_topk(q[:, :, perm], None, x, wd, wu3, s[:, perm], H[:, perm],
                                  Hkv=cs["Hkv"], K=cs["K"], w=cs["w"], lam=cs["lam"], rows=rows)
    assert np.array_equal(idx_p[:, :, rows], idx[:, :, rows])


def check_shortage_and_group_max():
    # one head of the group votes a chunk very high: the whole group selects it
    d = 4
    q = np.zeros((1, 1, 2, d))
    q[0, 0, 1, 0] = 1.0
    s = np.zeros((1, 2, 4, d))
    s[0, 1, 2, 0] = 50.0
    H = np.zeros((1, 2, 4))
    x = np.zeros((1, 1, 1))
    idx, z = O.route_score_topk(q, np.array([[100]]), x, np.zeros((1, 1)), np.zeros((1, 2 * d)),
                                s, H, Hkv=1, K=1, w=-1, lam=0.1, L=256)
    assert idx[0, 0, 0, 0] == 2
    assert z[0, 0, 0, 0] == 0.0 and z[0, 1, 0, 0] == 50.0 / 2.0
    # only chunk 0 is eligible for a query at position 200 with w = 100 (C = 4)
    idx, z = O.route_score_topk(q, np.array([[200]]), x, np.zeros((1, 1)), np.zeros((1, 2 * d)),
                                s, H, Hkv=1, K=3, w=100, lam=0.1, L=256)
    assert idx[0, 0, 0].tolist() == [0, -1, -1]
    assert np.all(np.isneginf(z[0, :, 0, 1:]))


def check_scores_for():
    """Per-head scores of a given selection (the parity check scores the GPU's own choice).

    (a) Hand-worked, d = 2, one group of two heads, C = 3, query at position 10, no window,
        rank-1 residual that adds (0, 1) to head 1 only:
          head 0: q_res = (1, 0); head 1: q_res = (0, 2) + (0, 1) = (0, 3)
          s[h0] = (1, 1), (2, 0), (0, 3);  H[h0] = 0.5, 1.0, 1.5
          s[h1] = (0, 1), (1, 1), (-1, 0); H[h1] = 2.0, 0.0, 1.0
        z = tau q_res.s - 0.1 H with tau = 1/sqrt(2); forced idx (2, 0, -1):
          head 0: (-0.15, tau - 0.05, -inf);  head 1: (-0.1, 3 tau - 0.2, -inf).
        With a window of radius 10 around position 10, chunk 0 touches the window: its
        score is -inf for both heads whatever was forced.
    (b) On the selection route_score_topk makes itself, the same scores it returned.
    """
    tau = 1.0 / math.sqrt(2.0)
    q = np.zeros((1, 1, 2, 2))
    q[0, 0, 0] = [1.0, 0.0]
    q[0, 0, 1] = [0.0, 2.0]
    x = np.ones((1, 1, 1))
    wd = np.ones((1, 1))
    wu = np.array([[0.0, 0.0, 0.0, 1.0]])
    s = np.zeros((1, 2, 3, 2))
    s[0, 0] = [[1, 1], [2, 0], [0, 3]]
    s[0, 1] = [[0, 1], [1, 1], [-1, 0]]
    H = np.array([[[0.5, 1.0, 1.5], [2.0, 0.0, 1.0]]])
    idx = np.array([[[[2, 0, -1]]]])
    z = O.scores_for(q, np.array([[10]]), x, wd, wu, s, H, idx, w=-1, lam=0.1, L=192)
    exp = np.array([[-0.15, tau - 0.05, -np.inf], [-0.1, 3 * tau - 0.2, -np.inf]])
    assert np.allclose(z[0, :, 0], exp, atol=1e-14), z[0, :, 0]
    assert np.array_equal(np.isneginf(z[0, :, 0]), np.isneginf(exp))
    zw = O.scores_for(q, np.array([[10]]), x, wd, wu, s, H, idx, w=10, lam=0.1, L=192)
    assert np.isneginf(zw[0, :, 0, 1]).all()
    assert np.allclose(zw[0, :, 0, 0], exp[:, 0], atol=1e-14)
    # (b) agreement with the scores the selection step attaches to its own choice
    cs = _route_case(13, L=448, w=30, K=3)
    q, k, v = cs["q"], cs["k"], cs["v"]
    s, H, _ = O.summary_pool(q[:, O.S - 1::O.S], k, v)
    rows = np.arange(0, cs["L"], 5)
    idx, z_sel = O.route_score_topk(q, None, cs["x"], cs["wd"], cs["wu"], s, H, Hkv=cs["Hkv"],
                                    K=cs["K"], w=cs["w"], lam=cs["lam"], rows=rows)
    z2 = O.scores_for(q, None, cs["x"], cs["wd"], cs["wu"], s, H, idx, w=cs["w"], lam=cs["lam"],
                      rows=rows)
    content = [i for i in rows if not O.is_mask_slot(i)]
    assert np.array_equal(z2[:, :, content], z_sel[:, :, content])


# ----------------------------------------------------------------------------- attention

def _sdpa(qv, keys, vals, bias=None):
    """torch CPU fp64 scaled_dot_product_attention of one query: (output, lse)."""
    qt = torch.from_numpy(np.ascontiguousarray(qv)).view(1, 1, 1, -1)
    kt = torch.from_numpy(np.ascontiguousarray(keys)).view(1, 1, keys.shape[0], -1)
    vt = torch.from_numpy(np.ascontiguousarray(vals)).view(1, 1, vals.shape[0], -1)
    mask = None if bias is None else torch.from_numpy(np.asarray(bias, dtype=np.float64)).view(1, 1, 1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)
    logits = (kt[0, 0] @ qt[0, 0, 0]) / math.sqrt(qv.shape[-1])
    if bias is not None:
        logits = logits + mask[0, 0, 0]
    return o[0, 0, 0].numpy(), float(torch.logsumexp(logits, 0))


def check_partition_identity(seed=8):
    """The two-level partition equals one softmax over the window keys plus the selected
    chunks' content keys with logit offsets z_c - lse_c (torch SDPA, fp64)."""
    cs = _route_case(seed, L=640, w=70, K=4)
    q, k, v = cs["q"], cs["k"], cs["v"]
    s, H, _ = O.summary_pool(q[:, O.S - 1::O.S], k, v)
    rows = np.array([0, 1, 62, 64, 100, 300, 447, 500, 638])
    idx, z = O.route_score_topk(q, None, cs["x"], cs["wd"], cs["wu"], s, H, Hkv=cs["Hkv"],
                                K=cs["K"], w=cs["w"], lam=cs["lam"], rows=rows)
    o, lse = O.route_attn(q, None, k, v, idx, z, w=cs["w"], rows=rows)
    G = q.shape[2] // cs["Hkv"]
    d = q.shape[3]
    for i in rows:
        if O.is_mask_slot(i):                      # mask rows are not route-layer queries
            assert np.all(np.isnan(o[0, i])) and np.all(idx[0, :, i] == -1)
            continue
        for h in range(q.shape[2]):
            g = h // G
            W = O.window(i, cs["w"], cs["L"])
            keys, vals, bias = [k[0, g, W]], [v[0, g, W]], [np.zeros(W.size)]
            for kk, c in enumerate(idx[0, g, i]):
                if c < 0:
                    continue
                cp = O.content_positions(c)
                lc = k[0, g, cp] @ q[0, i, h] / math.sqrt(d)
                lse_c = float(torch.logsumexp(torch.from_numpy(lc), 0))
                keys.append(k[0, g, cp])
                vals.append(v[0, g, cp])
                bias.append(np.full(cp.size, z[0, h, i, kk] - lse_c))
            oe, lse_e = _sdpa(q[0, i, h], np.concatenate(keys), np.concatenate(vals),
                              np.concatenate(bias))
            assert np.allclose(o[0, i, h], oe, atol=1e-12), (i, h)
            assert abs(lse[0, h, i] - lse_e) < 1e-11
            # masses sum to 1 and o is inside the hull of attended values
            allv = np.concatenate(vals)
            assert (o[0, i, h] >= allv.min(0) - 1e-12).all()
            assert (o[0, i, h] <= allv.max(0) + 1e-12).all()


def check_masses_sum_to_one(seed=9):
    rng = _rng(seed)
    d, L = 8, 256
    kg = rng.standard_normal((L, d))
    vg = np.ones((L, d))                          # every value row equal to 1 ...
    qi = rng.standard_normal(d)
    o, lnZ = O.route_attn_row(qi, 10, kg, vg, np.array([2, 3, -1]), np.array([0.3, -1.0, -np.inf]), 20)
    assert np.allclose(o, 1.0, atol=1e-13)        # ... so o = sum of masses = 1
    lam_loc = float(torch.logsumexp(torch.from_numpy(kg[0:31] @ qi / math.sqrt(d)), 0))
    assert abs(lnZ - math.log(math.exp(lam_loc) + math.exp(0.3) + math.exp(-1.0))) < 1e-12


def check_special_cases(seed=10):
    cs = _route_case(seed, L=384, K=1, w=-1)
    q, k, v = cs["q"], cs["k"], cs["v"]
    s, H, _ = O.summary_pool(q[:, O.S - 1::O.S], k, v)
    rows = np.array([3, 70, 200, 383 - 1])
    idx, z = O.route_score_topk(q, None, cs["x"], cs["wd"], cs["wu"], s, H, Hkv=cs["Hkv"], K=1,
                                w=-1, lam=cs["lam"], rows=rows)
    o, lse = O.route_attn(q, None, k, v, idx, z, w=-1, rows=rows)
    G = q.shape[2] // cs["Hkv"]
    for i in rows:
        for h in range(q.shape[2]):
            c = idx[0, h // G, i, 0]
            assert c >= 0
            cp = O.content_positions(c)
            oe, _ = _sdpa(q[0, i, h], k[0, h // G, cp], v[0, h // G, cp])
            assert np.allclose(o[0, i, h], oe, atol=1e-12)      # intra-chunk softmax attention
            assert abs(lse[0, h, i] - z[0, h, i, 0]) < 1e-12     # Z = e^{z_c}
    # window covering the whole sequence: nothing eligible, full bidirectional attention
    L = cs["L"]
    idx, z = O.route_score_topk(q, None, cs["x"], cs["wd"], cs["wu"], s, H, Hkv=cs["Hkv"], K=2,
                                w=L, lam=cs["lam"], rows=rows)
    assert np.all(idx[0][:, rows] == -1)
    o, lse = O.route_attn(q, None, k, v, idx, z, w=L, rows=rows)
    for i in rows:
        for h in range(q.shape[2]):
            oe, le = _sdpa(q[0, i, h], k[0, h // G], v[0, h // G])
            assert np.allclose(o[0, i, h], oe, atol=1e-12) and abs(lse[0, h, i] - le) < 1e-11


def check_swa_band(seed=11):
    rng = _rng(seed)
    B, L, Hq, Hkv, d, w = 1, 200, 4, 2, 8, 17
    q = rng.standard_normal((B, L, Hq, d))
    k = rng.standard_normal((B, Hkv, L, d))
    v = rng.standard_normal((B, Hkv, L, d))
    o, lse = O.swa_attn(q, None, k, v, w=w)
    G = Hq // Hkv
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)                      # [B, Hq, L, d]
    kt = torch.from_numpy(k).repeat_interleave(G, dim=1)
    vt = torch.from_numpy(v).repeat_interleave(G, dim=1)
    pos = torch.arange(L)
    band = (pos[:, None] - pos[None, :]).abs() <= w
    oe = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=band)
    assert np.allclose(o, oe.permute(0, 2, 1, 3).numpy(), atol=1e-12)
    logits = (qt @ kt.transpose(-1, -2)) / math.sqrt(d)
    le = torch.logsumexp(logits.masked_fill(~band, -math.inf), -1)
    assert np.allclose(lse, le.numpy(), atol=1e-11)
    # decode rows given by position
    qp = np.array([[0, 199, 57]])
    o2, _ = O.swa_attn(q[:, [0, 199, 57]], qp, k, v, w=w)
    assert np.allclose(o2[0], o[0, [0, 199, 57]], atol=1e-14)


def check_locality(seed=12):
    cs = _route_case(seed, L=768, K=2, w=60)
    q, k, v = cs["q"], cs["k"], cs["v"]
    out = O.route_layer(q, None, k, v, cs["x"], cs["wd"], cs["wu"], Hkv=cs["Hkv"], K=2, w=60,
                        rows=np.array([300]))
    idx, z = out["idx"], out["z_sel"]
    touched = set(O.window(300, 60, cs["L"]).tolist())
    used = set()
    for g in range(cs["Hkv"]):
        for c in idx[0, g, 300]:
            used.update(range(O.S * c, O.S * c + O.S))
    far = np.array([j for j in range(cs["L"]) if j not in touched and j not in used])
    # (a) new V outside the attended set: output bit-identical (selection unchanged)
    v2 = v.copy()
    v2[:, :, far] = _rng(99).standard_normal(v2[:, :, far].shape)
    out2 = O.route_layer(q, None, k, v2, cs["x"], cs["wd"], cs["wu"], Hkv=cs["Hkv"], K=2, w=60,
                         rows=np.array([300]))
    assert np.array_equal(out2["idx"][:, :, 300], idx[:, :, 300])
    assert np.array_equal(out2["o"][0, 300], out["o"][0, 300])
    # (b) new K there too, with the selection held fixed: output identical
    k2 = k.copy()
    k2[:, :, far] = _rng(98).standard_normal(k2[:, :, far].shape)
    o3, _ = O.route_attn(q, None, k2, v2, idx, z, w=60, rows=np.array([300]))
    assert np.array_equal(o3[0, 300], out["o"][0, 300])


def check_two_chunk_hand_examples():
    """L = 128, d = 2, Hq = Hkv = 1, worked by hand.

    Chunk 0 content keys all (0, 0); chunk 1 content keys all (2, 0) except none; every
    pooling is uniform (equal keys), so s_0 = (0,0), s_1 = (2,0), H = ln 63 for both.
    V: content slot j of chunk c holds (j, c).
    """
    L, d, lam = 128, 2, 0.1
    tau = 1 / math.sqrt(2)
    k = np.zeros((1, 1, L, d))
    k[0, 0, 64:127] = [2.0, 0.0]
    k[0, 0, 63] = [9.0, 9.0]                    # mask-slot keys (only the window sees them)
    k[0, 0, 127] = [-9.0, 9.0]
    v = np.zeros((1, 1, L, d))
    for c in range(2):
        for j in range(64):
            v[0, 0, 64 * c + j] = [j, c]
    q = np.zeros((1, L, 1, d))
    q[0, :, 0] = [1.0, 0.0]
    x = np.zeros((1, L, 1))
    wd, wu = np.zeros((1, 1)), np.zeros((1, 2))
    # (i) no window, K = 1: chunk 1 wins (z_1 = tau*2 - lam ln63 > z_0 = -lam ln63);
    #     output = uniform average of chunk-1 content values = (31, 1); lse = z_1
    out = O.route_layer(q, None, k, v, x, wd, wu, Hkv=1, K=1, w=-1, rows=np.array([5]))
    assert np.allclose(out["s"][0, 0], [[0, 0], [2, 0]]) and np.allclose(out["H"], math.log(63))
    assert out["idx"][0, 0, 5, 0] == 1
    z1 = tau * 2.0 - lam * math.log(63)
    assert abs(out["z_sel"][0, 0, 5, 0] - z1) < 1e-14
    assert np.allclose(out["o"][0, 5, 0], [31.0, 1.0], atol=1e-12)
    assert abs(out["lse"][0, 0, 5] - z1) < 1e-14
    # (ii) w = 0, K = 1, query at position 5 (chunk 0): chunk 0 is not eligible, T = {1};
    #      Z = e^{tau q.k_5} + e^{z_1} = e^0 + e^{z_1};  o = (v_5 + e^{z_1} (31, 1)) / Z
    out = O.route_layer(q, None, k, v, x, wd, wu, Hkv=1, K=1, w=0, rows=np.array([5]))
    assert out["idx"][0, 0, 5, 0] == 1
    Z = 1.0 + math.exp(z1)
    oe = (np.array([5.0, 0.0]) + math.exp(z1) * np.array([31.0, 1.0])) / Z
    assert np.allclose(out["o"][0, 5, 0], oe, atol=1e-12)
    assert abs(out["lse"][0, 0, 5] - math.log(Z)) < 1e-13
    # (iii) the mask slot 63 of chunk 0 with w = 0: its row is skipped by the route path;
    #       its pooled output is the uniform average of chunk-0 content values = (31, 0)
    assert np.all(np.isnan(O.route_layer(q, None, k, v, x, wd, wu, Hkv=1, K=1, w=0,
                                         rows=np.array([63]))["o"][0, 63]))
    assert np.allclose(out["o_mask"][0, 0, 0], [31.0, 0.0])
    # (iv) w = 70 around position 100 covers positions 30..170 -> both chunks touched:
    #      no eligible chunk, the route layer reduces to window attention
    out = O.route_layer(q, None, k, v, x, wd, wu, Hkv=1, K=1, w=70, rows=np.array([100]))
    assert out["idx"][0, 0, 100, 0] == -1
    W = np.arange(30, 128)
    oe, le = _sdpa(q[0, 100, 0], k[0, 0, W], v[0, 0, W])
    assert np.allclose(out["o"][0, 100, 0], oe, atol=1e-12)


ALL_CHECKS = [
    check_layout_facts, check_window_eligibility, check_pool_invariants,
    check_pool_closed_forms, check_pool_shift_invariance, check_pool_gqa_and_mean,
    check_pool_peaked_cosine, check_residual_layout, check_score_hand_example,
    check_topk_bruteforce, check_selection_properties, check_shortage_and_group_max,
    check_scores_for,
    check_partition_identity, check_masses_sum_to_one, check_special_cases, check_swa_band,
    check_locality, check_two_chunk_hand_examples,
]


def run_all():
    """Names of the checks that fail (empty list: the oracle passes every pin)."""
    failed = []
    for chk in ALL_CHECKS:
        try:
            chk()
        except Exception:           # noqa: BLE001 - any failure counts as a caught mistake
            failed.append(chk.__name__)
    return failed
