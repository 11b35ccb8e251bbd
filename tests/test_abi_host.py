"""The C-ABI library on the host: it builds, loads, exports every declared symbol, and
rejects invalid arguments before launching anything (no GPU needed for any of this)."""
import ctypes

import pytest

from diffusion_lms_b200 import build as rdl_build

rdl_build.build()
from diffusion_lms_b200 import rdl  # noqa: E402

FAKE = 0x7F0000000000          # 256-byte aligned fake device address (never dereferenced)


def dims(**kw):
    base = dict(B=1, L=1024, Lq=1024, Hq=4, Hkv=1, d=64, D=256, r=16, K=4, w=64, lam=0.1)
    base.update(kw)
    return rdl.Dims(**base)


def test_every_declared_symbol_is_exported():
    names = rdl.declared_functions()
    assert {"rdl_summary_pool", "rdl_route_score_topk", "rdl_route_attn", "rdl_swa_attn",
            "rdl_workspace_bytes", "rdl_last_device_status", "rdl_status_string",
            "rdl_version"} <= set(names)
    for n in names:
        assert rdl.exported(n), n


def test_status_strings_and_version():
    assert rdl.status_string(rdl.OK) == "ok"
    assert "invalid" in rdl.status_string(rdl.ERR_INVALID_ARG)
    assert "workspace" in rdl.status_string(rdl.ERR_WORKSPACE)
    assert rdl.status_string(12345) == "unknown status"
    assert rdl.version().count(".") == 2


def _score(dm, **ptrs):
    p = dict(q=FAKE, q_pos=None, x=FAKE, w_down=FAKE, w_up=FAKE, s=FAKE, H=FAKE, idx=FAKE,
             z=FAKE, ws=FAKE, ws_bytes=1 << 40)
    p.update(ptrs)
    return rdl.rdl_route_score_topk(p["q"], p["q_pos"], p["x"], p["w_down"], p["w_up"], p["s"],
                                    p["H"], dm, rdl.F32, p["idx"], p["z"], p["ws"],
                                    ws_bytes=p["ws_bytes"], stream=0, raise_on_error=False)


@pytest.mark.parametrize("bad", [
    dict(L=1000), dict(L=0), dict(Lq=0), dict(Hq=6, Hkv=4), dict(d=96), dict(K=0),
    dict(K=17), dict(K=65, L=64 * 80, Lq=64 * 80), dict(r=-1), dict(r=129), dict(B=0),
    dict(Lq=512),   # q_pos NULL requires Lq == L
])
def test_score_rejects_invalid_dims(bad):
    assert _score(dims(**bad)) == rdl.ERR_INVALID_ARG


@pytest.mark.parametrize("ptr", ["q", "s", "H", "idx", "z", "ws"])
def test_score_rejects_null_and_misaligned(ptr):
    assert _score(dims(), **{ptr: None}) == rdl.ERR_INVALID_ARG
    assert _score(dims(), **{ptr: FAKE + 8}) == rdl.ERR_INVALID_ARG


def test_score_workspace_too_small():
    dm = dims()
    need = rdl.workspace_bytes(rdl.WS_SCORE, dm, "f32")
    assert need > 0
    assert _score(dm, ws_bytes=need - 1) == rdl.ERR_WORKSPACE


def test_workspace_sizes():
    a = rdl.workspace_bytes(rdl.WS_SCORE, dims(), "f32")
    b = rdl.workspace_bytes(rdl.WS_SCORE, dims(L=2048, Lq=2048), "f32")
    assert b > a > 0
    assert rdl.workspace_bytes(rdl.WS_SCORE, dims(L=1000), "f32") == 0
    # the fp32 / d=64 attention runs in one kernel: no attention workspace
    assert rdl.workspace_bytes(rdl.WS_ATTN, dims(), "f32") == 0
    big = dims(L=16384, Lq=16384, Hq=28, Hkv=4, d=128, D=3584, r=64, K=32, w=256)
    assert rdl.workspace_bytes(rdl.WS_ATTN, big, "bf16") >= 16384 * 28 * 128 * 4
    assert rdl.workspace_bytes(7, big, "bf16") == 0


def test_summary_pool_rejects():
    dm = dims()
    f = lambda *a, **k: rdl.rdl_summary_pool(*a, **k, stream=0, raise_on_error=False)  # noqa
    row = dm.Hq * dm.d
    assert f(FAKE, 64 * row, 0, FAKE, None, dims(L=100), rdl.F32, FAKE, FAKE) == rdl.ERR_INVALID_ARG
    assert f(None, 64 * row, 0, FAKE, None, dm, rdl.F32, FAKE, FAKE) == rdl.ERR_INVALID_ARG
    assert f(FAKE, row - 1, 0, FAKE, None, dm, rdl.F32, FAKE, FAKE) == rdl.ERR_INVALID_ARG
    # o_mask without v
    assert f(FAKE, 64 * row, 0, FAKE, None, dm, rdl.F32, FAKE, FAKE, FAKE) == rdl.ERR_INVALID_ARG
    assert f(FAKE, 64 * row, 0, FAKE + 4, None, dm, rdl.F32, FAKE, FAKE) == rdl.ERR_INVALID_ARG
    assert f(FAKE, 64 * row, 0, FAKE, None, dm, 7, FAKE, FAKE) == rdl.ERR_INVALID_ARG


def test_attn_rejects():
    f = lambda dm, **k: rdl.rdl_route_attn(  # noqa: E731
        k.get("q", FAKE), None, FAKE, FAKE, k.get("idx", FAKE), FAKE, dm, k.get("dt", rdl.BF16),
        FAKE, None, k.get("ws", FAKE), ws_bytes=k.get("wsb", 1 << 40), stream=0,
        raise_on_error=False)
    big = dims(L=4096, Lq=4096, Hq=28, Hkv=4, d=128, D=3584, r=64, K=8, w=256)
    assert f(dims(Hq=5, Hkv=2)) == rdl.ERR_INVALID_ARG
    assert f(big, q=None) == rdl.ERR_INVALID_ARG
    assert f(big, idx=FAKE + 2) == rdl.ERR_INVALID_ARG
    assert f(big, ws=None) == rdl.ERR_INVALID_ARG
    assert f(big, ws=FAKE + 16) == rdl.ERR_INVALID_ARG           # workspace must be 256-aligned
    assert f(big, wsb=16) == rdl.ERR_WORKSPACE
    g = lambda dm, **k: rdl.rdl_swa_attn(FAKE, None, FAKE, FAKE, dm, rdl.BF16, FAKE, None,  # noqa
                                         stream=0, raise_on_error=False)
    assert g(dims(w=-1)) == rdl.ERR_INVALID_ARG
    assert g(dims(Lq=10)) == rdl.ERR_INVALID_ARG


def test_raise_on_error():
    with pytest.raises(rdl.RdlError) as e:
        _ = rdl.rdl_swa_attn(FAKE, None, FAKE, FAKE, dims(w=-1), rdl.BF16, FAKE, None, stream=0)
    assert e.value.status == rdl.ERR_INVALID_ARG


def test_dims_struct_layout():
    assert ctypes.sizeof(rdl.rdl_dims) == 12 * 4


def test_split_summary_layout_only_on_decode_blocks():
    """The split summary layout is read by the decode-block scorer only; other shapes refuse
    it before launching anything."""
    dm = dims(flags=rdl.FLAG_SPLIT_SUMMARY)          # fp32, d = 64, prefill-shaped
    assert _score(dm) == rdl.ERR_UNSUPPORTED


def test_decode_block_workspaces():
    """A 32-query decode block over 128K: the attention keeps one fp32 output per chunk task
    plus the window part per (row, head); the scorer the 8 hidden-slice partials of t and the
    per-head scores.  The attention workspace fits the no-allocation scratch."""
    dm = dims(L=131072, Lq=32, Hq=28, Hkv=4, d=128, D=3584, r=64, K=32, w=256)
    rows = 32 * 28
    want_attn = rows * 32 * 128 * 4 + rows * 128 * 4 + rows * 8
    got_attn = rdl.workspace_bytes(rdl.WS_ATTN, dm, "bf16")
    assert want_attn <= got_attn <= want_attn + 3 * 256            # three 256-byte aligned parts
    assert got_attn < rdl.NOALLOC_SCRATCH_BYTES
    want_score = 28 * 32 * 2048 * 4 + 8 * 32 * 64 * 4
    got_score = rdl.workspace_bytes(rdl.WS_SCORE, dm, "bf16")
    assert want_score <= got_score <= want_score + 2 * 256
