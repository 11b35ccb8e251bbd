"""The seeded input generator: bf16 rounding, determinism and the intended structure."""
import numpy as np
import torch

from diffusion_lms_b200 import workloads as W
from oracle import rdl_oracle as O


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([0.0, -0.0, 1.0, 3.0e38, 1e-40, 1.00390625, 1.01171875],
                                 dtype=np.float32)])
    ours = W.bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(W.bf16_to_f32(ours), torch.from_numpy(ours.view(np.int16))
                          .view(torch.bfloat16).float().numpy())


def test_deterministic_and_shapes():
    a = W.tiny_f32()
    b = W.tiny_f32()
    for name in ("q", "q_mask", "k", "v", "x", "w_down", "w_up"):
        assert np.array_equal(getattr(a, name), getattr(b, name))
    d = a.dims
    assert a.q.shape == (1, 1024, 4, 64) and a.k.shape == (1, 1, 1024, 64)
    assert a.q_mask.shape == (1, 16, 4, 64) and np.array_equal(a.q_mask[0], a.q[0, 63::64])
    assert a.x.shape == (1, 1024, 256) and a.w_down.shape == (256, 16)
    assert a.w_up.shape == (16, 256) and a.needles.shape == (1, 2)
    assert a.q.dtype == np.float32 and d.C == 16


def test_decode_block_positions():
    dims = W.scaled(W.DECODE_128K, L=4096, Lq=32)
    wl = W.make_inputs(dims, seed=3, n_needles=4, decode_block=32)
    assert wl.q_pos.tolist() == [list(range(4096 - 64, 4096 - 32))]
    assert wl.q.dtype == np.uint16 and wl.q_mask.shape == (1, 64, 28, 128)


def test_needles_steer_the_tiny_selection():
    """The planted needle chunks are chosen by most content queries (non-trivial top-K)."""
    wl = W.tiny_f32()
    f = {n: W.as_f64(getattr(wl, n)) for n in ("q", "k", "v", "x", "w_down", "w_up")}
    s, H, _ = O.summary_pool(f["q"][:, 63::64], f["k"], f["v"])
    rows = np.arange(0, 1024, 3)
    idx, _ = O.route_score_topk(f["q"], None, f["x"], f["w_down"], f["w_up"], s, H,
                                Hkv=1, K=4, w=64, lam=0.1, rows=rows)
    sel = idx[0, 0, rows]
    content = [r for r in range(len(rows)) if not O.is_mask_slot(rows[r])]
    for c in wl.needles[0]:
        eligible_rows = [r for r in content if c in O.eligible(rows[r], 64, 16)]
        hit = np.mean([c in sel[r] for r in eligible_rows])
        assert hit > 0.5, (c, hit)


def test_mixture_summaries_cluster():
    dims = W.scaled(W.PREFILL_64K, L=2048, Lq=2048, Hq=8, Hkv=2)
    wl = W.make_inputs(dims, seed=4, mixture=8)
    k = W.as_f64(wl.k)
    comp = wl.meta["components"]
    s, _, _ = O.summary_pool(W.as_f64(wl.q_mask), k)
    sn = s[0, 0] / np.linalg.norm(s[0, 0], axis=-1, keepdims=True)
    cos = sn @ sn.T
    same = comp[0, 0][:, None] == comp[0, 0][None, :]
    assert cos[same].min() > 0.9 and cos[~same].mean() < 0.3
