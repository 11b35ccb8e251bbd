"""rdl_route_attn_noalloc against rdl_route_attn, through the C ABI.

The no-allocation entry point serves hosts that cannot give the library device memory at
call time (engines that plan every buffer before serving, plugin interfaces without an
allocator); it runs the same attention with a scratch array the library holds itself.
Two calls in a row on different inputs must both match the workspace-taking call within
the parity tolerances, so nothing left in the shared scratch leaks into the next call.
This file is collected last and also passes when run alone in a fresh process (its first
call looks the scratch address up).
"""
import numpy as np
import pytest
import torch

from diffusion_lms_b200 import api, rdl
from diffusion_lms_b200 import workloads as W
import parity as P

pytestmark = pytest.mark.gpu


def _inputs(seed, decode):
    base = dict(B=1, L=8192, Lq=32, Hq=28, Hkv=4, d=128, D=512, r=64, K=32, w=256, lam=0.1,
                dtype="bf16")
    if not decode:
        base.update(L=1024, Lq=1024, K=2)    # about 28 MB of scratch: within the limit
    wl = W.make_inputs(W.Dims(**base), seed=seed, n_needles=4, decode_block=32 if decode else 0)
    inp = api.to_device(wl)
    out = api.alloc_outputs(inp.dims, inp.dtype)
    api.summary_pool(inp, out)
    api.score_topk(inp, out)
    return inp, out


@pytest.mark.parametrize("decode", [True, False])
def test_noalloc_matches_workspace_entry_on_two_calls(decode):
    tol = P.TOL["bf16"]
    for seed in (41, 42):                      # two calls in a row, different inputs
        inp, out = _inputs(seed, decode)
        api.route_attn(inp, out)               # existing entry point, caller workspace
        o2 = torch.zeros_like(out.o)
        lse2 = torch.full_like(out.lse, float("nan"))
        rdl.rdl_route_attn_noalloc(inp.q, inp.q_pos, inp.k, inp.v, out.idx, out.z_sel,
                                   inp.dims, inp.dtype, o2, lse2)
        torch.cuda.synchronize()
        assert rdl.rdl_last_device_status() == rdl.OK
        pos = np.arange(inp.dims.L) if inp.q_pos is None else inp.q_pos[0].cpu().numpy()
        content = torch.from_numpy((pos % 64) != 63).to(o2.device)
        a, b = out.o[:, content].float(), o2[:, content].float()
        assert torch.isfinite(b).all()
        assert (a - b).abs().max().item() <= tol.o
        la, lb = out.lse[:, :, content], lse2[:, :, content]
        assert (la - lb).abs().max().item() <= tol.lse


def _compare(inp, ref_o, ref_lse, o2, lse2, tol):
    pos = np.arange(inp.dims.L) if inp.q_pos is None else inp.q_pos[0].cpu().numpy()
    content = torch.from_numpy((pos % 64) != 63).to(o2.device)
    a, b = ref_o[:, content].float(), o2[:, content].float()
    assert torch.isfinite(b).all()
    assert (a - b).abs().max().item() <= tol.o
    assert (ref_lse[:, :, content] - lse2[:, :, content]).abs().max().item() <= tol.lse


@pytest.mark.parametrize("decode", [True, False])
def test_noalloc_back_to_back_on_one_stream(decode):
    """Calls issued one right after another on one stream, with no synchronisation and no
    other kernel between them, alternating two different inputs: each call's kernels must
    not overwrite the shared scratch while the previous call still reads it."""
    tol = P.TOL["bf16"]
    cases = [_inputs(seed, decode) for seed in (43, 44)]
    refs = []
    for inp, out in cases:
        api.route_attn(inp, out)
        refs.append((out.o.clone(), out.lse.clone()))
    torch.cuda.synchronize()
    got = []
    for rep in range(6):                       # 43, 44, 43, 44, ... back to back
        inp, out = cases[rep % 2]
        o2 = torch.zeros_like(out.o)
        lse2 = torch.full_like(out.lse, float("nan"))
        got.append((o2, lse2))
    torch.cuda.synchronize()                   # buffers ready; no sync between the calls
    for rep, (o2, lse2) in enumerate(got):
        inp, out = cases[rep % 2]
        rdl.rdl_route_attn_noalloc(inp.q, inp.q_pos, inp.k, inp.v, out.idx, out.z_sel,
                                   inp.dims, inp.dtype, o2, lse2)
    torch.cuda.synchronize()
    assert rdl.rdl_last_device_status() == rdl.OK
    for rep, (o2, lse2) in enumerate(got):
        inp, _ = cases[rep % 2]
        _compare(inp, *refs[rep % 2], o2, lse2, tol)


def test_noalloc_rejects_sizes_beyond_the_scratch():
    big = rdl.Dims(B=1, L=16384, Lq=16384, Hq=28, Hkv=4, d=128, D=3584, r=64, K=32, w=256)
    assert rdl.workspace_bytes(rdl.WS_ATTN, big, "bf16") > rdl.NOALLOC_SCRATCH_BYTES
    st = rdl.rdl_route_attn_noalloc(0x7F0000000000, None, 0x7F0000000000, 0x7F0000000000,
                                    0x7F0000000000, 0x7F0000000000, big, rdl.BF16,
                                    0x7F0000000000, None, raise_on_error=False)
    assert st == rdl.ERR_SCRATCH_LIMIT
    assert "scratch" in rdl.status_string(st)
