"""GPU-vs-oracle comparison under the acceptance rule of the route-layer study.

Indices: for each (query row, group), with gap = zeta_(K) - zeta_(K+1) from the oracle's
fp64 group-max scores: if gap > GAP the GPU's set must equal the oracle's; otherwise
every GPU-chosen chunk must have zeta >= zeta_(K) - GAP and every chunk with
zeta > zeta_(K) + GAP must be chosen (near ties admit several correct sets).
Outputs: compared with the oracle run on the GPU's own selection (so a legal near-tie
swap is not an output error), element by element.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

from diffusion_lms_b200 import api, rdl
from diffusion_lms_b200.workloads import Workload, as_f64
from oracle import rdl_oracle as O

GAP = 1e-3


@dataclass
class Tol:
    o: float        # max-abs on outputs
    lse: float      # max-abs on log-partitions
    s: float        # summaries/entropy, relative to max(1, |ref|)
    z: float        # per-head route scores of the selected chunks


TOL = {"bf16": Tol(o=2e-2, lse=1e-3, s=1e-5, z=1e-4), "f32": Tol(o=1e-5, lse=1e-5, s=1e-5, z=1e-5)}


def f64(wl: Workload):
    return {n: as_f64(getattr(wl, n)) for n in ("q", "q_mask", "k", "v", "x", "w_down", "w_up")}


def run_gpu(wl: Workload, *, flags=0, with_residual=True, route=True, swa=False):
    inp = api.to_device(wl)
    inp.dims.flags = flags
    if not with_residual:
        inp.dims.r = 0
        inp.x = None
    out = api.alloc_outputs(inp.dims, inp.dtype)
    api.summary_pool(inp, out)
    res = {}
    if route:
        api.score_topk(inp, out)
        api.route_attn(inp, out)
    torch.cuda.synchronize()
    st = rdl.rdl_last_device_status()
    assert st == rdl.OK, rdl.status_string(st)
    s_out = out.s
    if flags & rdl.FLAG_SPLIT_SUMMARY:     # rows of [hi d | lo d] bf16: s = hi + lo
        sp = out.s.view(torch.bfloat16).reshape(*out.s.shape[:-1], 2, out.s.shape[-1])
        s_out = sp[..., 0, :].double() + sp[..., 1, :].double()
    res.update(s=s_out.double().cpu().numpy(), H=out.H.double().cpu().numpy(),
               idx=out.idx.cpu().numpy().astype(np.int64), z=out.z_sel.double().cpu().numpy(),
               o=out.o.double().cpu().numpy(), lse=out.lse.double().cpu().numpy())
    if swa:
        out2 = api.alloc_outputs(inp.dims, inp.dtype)
        api.swa_attn(inp, out2)
        torch.cuda.synchronize()
        res.update(swa_o=out2.o.double().cpu().numpy(), swa_lse=out2.lse.double().cpu().numpy())
    return res


def check_summaries(gpu, ref_s, ref_H, tol: Tol):
    es = np.abs(gpu["s"] - ref_s) / np.maximum(1.0, np.abs(ref_s))
    eH = np.abs(gpu["H"] - ref_H) / np.maximum(1.0, np.abs(ref_H))
    assert es.max() <= tol.s, f"summary error {es.max():.3e}"
    assert eH.max() <= tol.s, f"entropy error {eH.max():.3e}"
    assert (gpu["H"] >= -1e-6).all() and (gpu["H"] <= math.log(63) + 1e-5).all()


def check_selection(gpu_idx, ora_idx, zeta, gaps, rows, q_pos, L, w, K):
    """Index rule over the sampled rows; returns (#exact-compared, #near-tie)."""
    B, Hkv = gpu_idx.shape[:2]
    C = L // O.S
    n_exact = n_tie = 0
    for b in range(B):
        pos = O.positions(gpu_idx.shape[2], L, q_pos, b)
        for i in rows:
            p = int(pos[i])
            for g in range(Hkv):
                gi = gpu_idx[b, g, i]
                if O.is_mask_slot(p):
                    assert np.all(gi == -1), (i, g, gi)
                    continue
                E = O.eligible(p, w, C)
                nv = min(K, E.size)
                valid = gi[gi >= 0]
                assert valid.size == nv and np.all(gi[nv:] == -1), (i, g, gi)
                assert np.all(np.diff(valid) > 0), ("not ascending", i, g, gi)
                assert set(valid.tolist()) <= set(E.tolist()), ("ineligible", i, g)
                ref = set(ora_idx[b, g, i][ora_idx[b, g, i] >= 0].tolist())
                if gaps[b, g, i] > GAP:
                    assert set(valid.tolist()) == ref, (i, g, sorted(valid), sorted(ref), gaps[b, g, i])
                    n_exact += 1
                else:
                    z = zeta[b, g, i]
                    zk = np.sort(z[E])[::-1][K - 1]
                    assert np.all(z[valid] >= zk - GAP), (i, g)
                    must = E[z[E] > zk + GAP]
                    assert set(must.tolist()) <= set(valid.tolist()), (i, g)
                    n_tie += 1
    return n_exact, n_tie


def check_route_layer(wl: Workload, gpu, rows, *, lam=None, w=None, K=None, mean_summary=False,
                      with_residual=True):
    """Summaries (all chunks), selection and outputs (sampled rows) against the oracle."""
    dm = wl.dims
    tol = TOL[dm.dtype]
    w = dm.w if w is None else w
    K = dm.K if K is None else K
    lam = dm.lam if lam is None else lam
    f = f64(wl)
    if not with_residual:
        f["x"] = np.zeros_like(f["x"])
    s, H, o_mask = O.summary_pool(f["q_mask"], f["k"], f["v"], mean_summary=mean_summary)
    check_summaries(gpu, s, H, tol)
    idx, z, zeta, gaps = O.route_score_topk(f["q"], wl.q_pos, f["x"], f["w_down"], f["w_up"], s,
                                            H, Hkv=dm.Hkv, K=K, w=w, lam=lam, L=dm.L,
                                            rows=rows, with_zeta=True)
    n_exact, n_tie = check_selection(gpu["idx"], idx, zeta, gaps, rows, wl.q_pos, dm.L, w, K)
    # outputs on the GPU's own selection
    z_g = O.scores_for(f["q"], wl.q_pos, f["x"], f["w_down"], f["w_up"], s, H, gpu["idx"], w=w,
                       lam=lam, L=dm.L, rows=rows)
    o_ref, lse_ref = O.route_attn(f["q"], wl.q_pos, f["k"], f["v"], gpu["idx"], z_g, w=w, rows=rows)
    content = [i for i in rows if not O.is_mask_slot(int(O.positions(dm.Lq, dm.L, wl.q_pos)[i]))]
    fin = np.isfinite(z_g[:, :, content])
    ez = np.abs(np.where(fin, gpu["z"][:, :, content] - np.where(fin, z_g[:, :, content], 0), 0))
    assert np.all(np.isfinite(gpu["z"][:, :, content]) == np.isfinite(z_g[:, :, content]))
    assert ez.max() <= tol.z, f"z_sel error {ez.max():.3e}"
    eo = np.abs(gpu["o"][:, content] - o_ref[:, content]).max()
    el = np.abs(gpu["lse"][:, :, content] - lse_ref[:, :, content]).max()
    assert eo <= tol.o, f"route output error {eo:.3e}"
    assert el <= tol.lse, f"route lse error {el:.3e}"
    if wl.q_pos is None:      # prefill: mask-slot rows hold the pooled output
        mrows = np.arange(O.S - 1, dm.L, O.S)
        em = np.abs(gpu["o"][:, mrows] - o_mask).max()
        assert em <= tol.o, f"mask-row output error {em:.3e}"
    return dict(n_exact=n_exact, n_tie=n_tie, err_o=float(eo), err_lse=float(el),
                err_z=float(ez.max()))


def check_swa(wl: Workload, gpu, rows, w=None):
    dm = wl.dims
    tol = TOL[dm.dtype]
    f = f64(wl)
    o_ref, lse_ref = O.swa_attn(f["q"], wl.q_pos, f["k"], f["v"], w=dm.w if w is None else w,
                                rows=rows)
    eo = np.abs(gpu["swa_o"][:, rows] - o_ref[:, rows]).max()
    el = np.abs(gpu["swa_lse"][:, :, rows] - lse_ref[:, :, rows]).max()
    assert eo <= tol.o, f"swa output error {eo:.3e}"
    assert el <= tol.lse, f"swa lse error {el:.3e}"
    return dict(err_o=float(eo), err_lse=float(el))


def sample_rows(wl: Workload, n=512, seed=0):
    """Content-query sample: first/last chunks, window edges, rows next to needles, random."""
    dm = wl.dims
    if wl.q_pos is not None:
        return np.arange(dm.Lq)
    rng = np.random.default_rng(seed)
    L = dm.L
    pick = set(range(0, 70)) | set(range(L - 70, L))
    for c in wl.needles.reshape(-1):
        for dlt in (-dm.w - 65, -dm.w - 1, -dm.w, 0, 30, dm.w, dm.w + 1, dm.w + 64):
            p = int(c) * O.S + dlt
            if 0 <= p < L:
                pick.add(p)
    while len(pick) < n:
        pick.add(int(rng.integers(0, L)))
    return np.array(sorted(pick))
