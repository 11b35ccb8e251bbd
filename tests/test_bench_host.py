"""Host logic of the measurement (no GPU): the algorithmic work counts behind the roofline
fractions, and the DRAM-traffic record, which is reported only while the library sources
it was captured on are unchanged."""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from diffusion_lms_b200 import workloads as W  # noqa: E402


def _dims(**kw):
    base = dict(B=1, L=256, Lq=256, Hq=4, Hkv=2, d=8, D=16, r=4, K=2, w=10, lam=0.1, dtype="bf16")
    base.update(kw)
    return W.Dims(**base)


def test_attn_flops_counts_window_and_selected_content_keys():
    """4 d flops per attended key per (row, head): |W(p)| window keys (clipped at the ends)
    plus 63 per selected chunk, content rows only, by brute force over rows."""
    dm = _dims()
    rng = np.random.default_rng(0)
    idx = rng.integers(-1, 4, size=(1, dm.Hkv, dm.Lq, dm.K)).astype(np.int32)
    want = 0
    G = dm.Hq // dm.Hkv
    for g in range(dm.Hkv):
        for p in range(dm.L):
            if p % 64 == 63:
                continue
            win = sum(1 for j in range(dm.L) if abs(p - j) <= dm.w)
            nsel = int((idx[0, g, p] >= 0).sum())
            want += 4 * dm.d * G * (win + 63 * nsel)
    assert bench.attn_flops(dm, None, idx) == float(want)


def test_decode_bytes_count_distinct_group_chunk_pairs():
    dm = _dims(L=4096, Lq=4, K=3, w=8)
    idx = np.full((1, dm.Hkv, dm.Lq, dm.K), -1, dtype=np.int32)
    idx[0, 0, :, 0] = 5                    # one chunk shared by every row of group 0
    idx[0, 0, 1, 1] = 7
    idx[0, 1, 2, :] = [5, 9, -1]          # chunk 5 again, but in group 1: a distinct slab
    r = bench.decode_bytes(dm, idx)
    assert r["unique_pairs"] == 4          # (0, 5), (0, 7), (1, 5), (1, 9)
    assert r["chunks"] == 4 * 2 * 64 * dm.d * 2
    assert r["summary"] == 4 * dm.Hq * (dm.L // 64) * (dm.d + 1)


def test_recorded_traffic_only_for_current_sources(tmp_path, monkeypatch):
    path = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    assert bench.recorded_traffic("k")[0] is None              # nothing recorded
    sha = bench.kernel_sources_sha()
    path.write_text(json.dumps({"k": {"sources_sha": sha, "bytes": 123.0, "what": "capture"}}))
    assert bench.recorded_traffic("k") == (123.0, "capture")
    assert bench.recorded_traffic("other")[0] is None
    path.write_text(json.dumps({"k": {"sources_sha": "0" * 16, "bytes": 123.0, "what": "capture"}}))
    val, note = bench.recorded_traffic("k")
    assert val is None and "changed" in note


def test_sources_hash_follows_the_library_sources(tmp_path, monkeypatch):
    """The hash covers every csrc file and the header: a changed byte changes it."""
    csrc = tmp_path / "diffusion_lms_b200" / "csrc"
    inc = tmp_path / "include"
    csrc.mkdir(parents=True)
    inc.mkdir()
    (csrc / "a.cu").write_text("x")
    (csrc / "b.cuh").write_text("y")
    (inc / "rdl.h").write_text("z")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h1 = bench.kernel_sources_sha()
    (csrc / "b.cuh").write_text("y2")
    h2 = bench.kernel_sources_sha()
    (inc / "rdl.h").write_text("z2")
    h3 = bench.kernel_sources_sha()
    assert len({h1, h2, h3}) == 3


def test_committed_traffic_record_is_well_formed():
    path = os.path.join(ROOT, "profiles", "traffic.json")
    with open(path) as f:
        rec = json.load(f)
    for key in ("route_prefill_16k.rdl_route_attn", "route_decode_128k.step"):
        assert set(rec[key]) == {"sources_sha", "bytes", "what"}
        assert rec[key]["bytes"] > 0 and len(rec[key]["sources_sha"]) == 16
