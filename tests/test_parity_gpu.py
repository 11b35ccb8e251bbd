"""CUDA path (through the C ABI) against the fp64 oracle, element by element.

Small cases cover every row and span several tiles with ragged tails (C not a multiple
of the 64-chunk score tile, Lq not a multiple of the 16-row window tile); the full-size
workloads (16K / 64K prefill, 128K decode, 28-layer stack) are checked on sampled rows.
"""
import dataclasses

import numpy as np
import pytest
import torch

from diffusion_lms_b200 import api, rdl
from diffusion_lms_b200 import workloads as W
from oracle import rdl_oracle as O
import parity as P

pytestmark = pytest.mark.gpu


def small(**kw):
    base = dict(B=1, L=2368, Lq=2368, Hq=28, Hkv=4, d=128, D=512, r=64, K=8, w=100, lam=0.1,
                dtype="bf16")
    base.update(kw)
    return W.Dims(**base)


def test_tiny_f32_every_row():
    wl = W.tiny_f32()
    gpu = P.run_gpu(wl, swa=True)
    rows = np.arange(wl.dims.L)
    r = P.check_route_layer(wl, gpu, rows)
    assert r["n_exact"] > 0
    P.check_swa(wl, gpu, rows)


def test_bf16_prefill_ragged_every_row():
    wl = W.make_inputs(small(), seed=11, n_needles=4)
    gpu = P.run_gpu(wl, swa=True)
    rows = np.arange(wl.dims.L)
    r = P.check_route_layer(wl, gpu, rows)
    assert r["n_exact"] > 1000
    P.check_swa(wl, gpu, rows)


@pytest.mark.parametrize("split", [False, True])
def test_bf16_decode_block(split):
    """32-query decode block; with the split summary layout the pooled summaries are stored
    as bf16 hi/lo rows and the scorer reads them directly."""
    dm = small(L=8192, Lq=32, K=32, w=256)
    wl = W.make_inputs(dm, seed=12, n_needles=8, decode_block=32)
    gpu = P.run_gpu(wl, swa=True, flags=rdl.FLAG_SPLIT_SUMMARY if split else 0)
    rows = np.arange(32)
    P.check_route_layer(wl, gpu, rows)
    P.check_swa(wl, gpu, rows)


def test_bf16_scattered_positions_ragged_rows():
    """37 rows at arbitrary positions (mask slots, both ends), not a multiple of 16."""
    dm = small(L=4096, Lq=37, K=8, w=100)
    wl = W.make_inputs(dm, seed=13, n_needles=4, decode_block=37)
    rng = np.random.default_rng(5)
    pos = np.concatenate([[0, 1, 63, 64, 127, 4095, 4094, 4032], rng.integers(0, 4096, 29)])
    wl.q_pos = pos.astype(np.int32)[None, :]
    gpu = P.run_gpu(wl, swa=True)
    rows = np.arange(37)
    P.check_route_layer(wl, gpu, rows)
    P.check_swa(wl, gpu, rows)


def test_bf16_many_scattered_rows_partial_tiles():
    """600 rows at scattered positions: enough tiles for the single-pass tensor-core window
    and scorer kernels, with a partial 16-token window tile and partial 128-row score tiles."""
    full = W.make_inputs(small(L=4096, Lq=4096, K=8, w=100), seed=21, n_needles=4)
    rng = np.random.default_rng(7)
    pos = np.sort(rng.choice(4096, size=600, replace=False))
    wl = dataclasses.replace(full, dims=dataclasses.replace(full.dims, Lq=600),
                             q=full.q[:, pos].copy(), x=full.x[:, pos].copy(),
                             q_pos=pos.astype(np.int32)[None, :])
    gpu = P.run_gpu(wl, swa=True)
    rows = np.arange(600)
    P.check_route_layer(wl, gpu, rows)
    P.check_swa(wl, gpu, rows)


def test_bf16_prefill_batch_2_every_row():
    """Two independently drawn sequences (B = 2) through the tensor-core prefill kernels at
    head dim 128 (scorer, window and chunk attention index across the batch), every row."""
    wl = W.make_inputs(small(B=2), seed=31, n_needles=4)
    assert not np.array_equal(wl.k[0], wl.k[1]) and not np.array_equal(wl.q[0], wl.q[1])
    assert not np.array_equal(wl.needles[0], wl.needles[1])
    gpu = P.run_gpu(wl, swa=True)
    rows = np.arange(wl.dims.L)
    r = P.check_route_layer(wl, gpu, rows)
    assert r["n_exact"] > 2000
    P.check_swa(wl, gpu, rows)
    assert not np.array_equal(gpu["idx"][0], gpu["idx"][1])


@pytest.mark.parametrize("dtype,r,D", [("f32", 64, 512), ("bf16", 16, 512), ("bf16", 64, 520)])
def test_decode_block_general_scorer(dtype, r, D):
    """Decode blocks outside the chained tensor-core scorer's shapes (fp32 storage, a rank
    other than 0/64/128, a hidden size not a multiple of 64) take the general decode
    scorer: sliced residual, split-bf16 summary contraction, group max, top-K."""
    dm = small(L=8192, Lq=32, K=16, w=256, r=r, D=D, dtype=dtype)
    wl = W.make_inputs(dm, seed=32, n_needles=6, decode_block=32, unit_scale=(dtype == "f32"))
    gpu = P.run_gpu(wl, swa=True)
    rows = np.arange(32)
    P.check_route_layer(wl, gpu, rows)
    P.check_swa(wl, gpu, rows)


def test_window_radius_1280_prefill_sampled():
    """The window radius of the pages' Table 3 layout for the non-route layers (1280), on a
    prefill: route layer and sliding window, sampled rows including both ends."""
    dm = small(L=4096, Lq=4096, K=8, w=1280)
    wl = W.make_inputs(dm, seed=33, n_needles=4)
    gpu = P.run_gpu(wl, swa=True)
    rows = P.sample_rows(wl, 400, seed=3)
    P.check_route_layer(wl, gpu, rows)
    P.check_swa(wl, gpu, rows)


def test_window_radius_1280_decode_stack_layers():
    """A route layer and a sliding-window layer of the 128K stack with radius 1280."""
    for layer in (2, 3):
        wl = W.stack_layer(layer)
        wl = dataclasses.replace(wl, dims=dataclasses.replace(wl.dims, w=1280))
        route = W.is_route_layer(layer)
        gpu = P.run_gpu(wl, route=route, swa=not route)
        rows = np.arange(32)
        if route:
            P.check_route_layer(wl, gpu, rows)
        else:
            P.check_swa(wl, gpu, rows)


@pytest.mark.parametrize("Hq,Hkv", [(16, 2), (2, 2), (6, 1)])
def test_group_sizes(Hq, Hkv):
    wl = W.make_inputs(small(L=1024, Lq=1024, Hq=Hq, Hkv=Hkv, K=6, w=70), seed=14, n_needles=2)
    gpu = P.run_gpu(wl, swa=True)
    rows = np.arange(1024)
    P.check_route_layer(wl, gpu, rows)
    P.check_swa(wl, gpu, rows)


def test_bf16_head_dim_64_batch_2():
    wl = W.make_inputs(small(B=2, L=1024, Lq=1024, Hq=8, Hkv=2, d=64, K=4, w=64), seed=15,
                       n_needles=2)
    gpu = P.run_gpu(wl, swa=True)
    rows = np.arange(0, 1024, 3)
    P.check_route_layer(wl, gpu, rows)
    P.check_swa(wl, gpu, rows)


@pytest.mark.parametrize("case", ["no_window", "window_covers_all", "lambda0_no_residual",
                                  "lambda0_with_residual", "no_residual", "mean_summary",
                                  "K_equals_C"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_edge_cases(case, dtype):
    kw = dict(L=1024, Lq=1024, Hq=8, Hkv=2, K=4, w=64, dtype=dtype)
    flags, with_res, mean = 0, True, False
    if case == "no_window":
        kw["w"] = -1
    elif case == "window_covers_all":
        kw["w"] = 5000
    elif case == "lambda0_no_residual":
        kw["lam"] = 0.0
        with_res = False
    elif case == "lambda0_with_residual":        # Table 6 "No entropy"
        kw["lam"] = 0.0
    elif case == "no_residual":                  # Table 6 "No residual"
        with_res = False
    elif case == "mean_summary":
        flags, mean = rdl.FLAG_MEAN_SUMMARY, True
    elif case == "K_equals_C":
        kw.update(K=16, w=10)
    wl = W.make_inputs(small(**kw), seed=16, n_needles=2, unit_scale=(dtype == "f32"))
    gpu = P.run_gpu(wl, flags=flags, with_residual=with_res, swa=kw["w"] >= 0)
    rows = np.arange(1024)
    P.check_route_layer(wl, gpu, rows, mean_summary=mean, with_residual=with_res)
    if kw["w"] >= 0:
        P.check_swa(wl, gpu, rows)


def test_device_checks_record_without_fault():
    """Out-of-range and in-window chunk ids are recorded in the status word and skipped."""
    wl = W.make_inputs(small(L=1024, Lq=1024, Hq=8, Hkv=2, K=4, w=64), seed=17)
    inp = api.to_device(wl)
    inp.dims.flags = rdl.FLAG_CHECKS
    out = api.alloc_outputs(inp.dims, inp.dtype)
    api.summary_pool(inp, out)
    api.score_topk(inp, out)
    torch.cuda.synchronize()
    assert rdl.rdl_last_device_status() == rdl.OK          # valid selection: no record
    out.idx[0, 0, 500, 0] = 10_000                          # beyond C
    out.idx[0, 1, 500, 1] = 500 // 64                       # the query's own chunk
    api.route_attn(inp, out)
    assert rdl.rdl_last_device_status() == rdl.ERR_DEVICE_CHECK
    assert rdl.rdl_last_device_status() == rdl.OK          # cleared on read


def test_decode_device_checks_record_without_fault():
    """Decode-block kernels: a chunk id beyond C and one inside the row's window are recorded
    in the status word and skipped; every output stays finite."""
    wl = W.make_inputs(small(L=8192, Lq=32, K=32, w=256), seed=17, n_needles=4, decode_block=32)
    inp = api.to_device(wl)
    inp.dims.flags = rdl.FLAG_CHECKS
    out = api.alloc_outputs(inp.dims, inp.dtype)
    api.summary_pool(inp, out)
    api.score_topk(inp, out)
    api.route_attn(inp, out)
    torch.cuda.synchronize()
    assert rdl.rdl_last_device_status() == rdl.OK
    own = int(inp.q_pos[0, 6].item()) // 64
    out.idx[0, 0, 5, 0] = 10_000
    out.idx[0, 1, 6, 1] = own
    api.route_attn(inp, out)
    assert rdl.rdl_last_device_status() == rdl.ERR_DEVICE_CHECK
    assert rdl.rdl_last_device_status() == rdl.OK
    assert torch.isfinite(out.o.float()).all()


@pytest.mark.parametrize("L,K", [(2048, 4), (4096, 2)])
def test_wait_timeout_returns_and_the_next_call_computes(L, K):
    """Failure detection without a fault: with RDL_FLAG_WAIT_TEST the prefill selected-chunk
    kernel waits, with a short limit, on a barrier nothing arrives on, once its first K/V slab
    and query loads are in flight (row-tile form for L = 2048 with K = 4; chunk-major form for
    L = 4096 with K = 2).  The call returns, the status word reads RDL_ERR_TIMEOUT (then
    clears), and the next calls in the same process match the oracle."""
    wl = W.make_inputs(small(L=L, Lq=L, Hq=8, Hkv=2, K=K, w=64), seed=35, n_needles=2)
    inp = api.to_device(wl)
    out = api.alloc_outputs(inp.dims, inp.dtype)
    api.summary_pool(inp, out)
    api.score_topk(inp, out)
    torch.cuda.synchronize()
    assert rdl.rdl_last_device_status() == rdl.OK
    inp.dims.flags = rdl.FLAG_WAIT_TEST
    api.route_attn(inp, out)
    assert rdl.rdl_last_device_status() == rdl.ERR_TIMEOUT
    assert rdl.rdl_last_device_status() == rdl.OK           # cleared on read
    gpu = P.run_gpu(wl)
    P.check_route_layer(wl, gpu, np.arange(0, L, 3))


def test_chunk_major_prefill_rows():
    """The chunk-major form of the selected-chunk attention (each chunk's rows gathered over
    the whole sequence, fp16 chunk outputs, a separate combine) on a prefill whose chunk
    buckets per 45-row tile would be small (8K rows, K = 2 of 128 chunks), every third row,
    with a second batch element."""
    wl = W.make_inputs(small(B=2, L=8192, Lq=8192, Hq=8, Hkv=2, K=2, w=64), seed=36, n_needles=4)
    gpu = P.run_gpu(wl)
    rows = np.unique(np.concatenate([np.arange(0, 8192, 3), np.arange(8100, 8192)]))
    P.check_route_layer(wl, gpu, rows)


def test_bitwise_repeatable():
    for dm, dec in ((small(), 0), (small(L=8192, Lq=32, K=32, w=256), 32)):
        wl = W.make_inputs(dm, seed=18, n_needles=4, decode_block=dec)
        a = P.run_gpu(wl, swa=True)
        b = P.run_gpu(wl, swa=True)
        for key in ("s", "H", "idx", "z", "o", "lse", "swa_o", "swa_lse"):
            assert np.array_equal(a[key], b[key], equal_nan=True), key


def test_head_permutation_and_locality():
    wl = W.make_inputs(small(L=1024, Lq=1024, Hq=8, Hkv=2, K=3, w=64), seed=19, n_needles=2)
    base = P.run_gpu(wl)
    # permute the heads inside group 0 (queries, mask queries, residual columns)
    perm = np.arange(8)
    perm[:4] = perm[:4][::-1]
    wl2 = dataclasses.replace(wl, q=wl.q[:, :, perm].copy(), q_mask=wl.q_mask[:, :, perm].copy(),
                              w_up=wl.w_up.reshape(wl.w_up.shape[0], 8, -1)[:, perm]
                              .reshape(wl.w_up.shape).copy())
    per = P.run_gpu(wl2)
    assert np.array_equal(per["idx"], base["idx"])
    assert np.array_equal(per["o"][:, :, perm], base["o"])
    # new values in chunks no row of group 0 selects or sees: group 0 outputs unchanged
    i = 600
    used = set(range(max(0, i - 64), i + 65))
    for c in base["idx"][0, 0, i]:
        used.update(range(64 * c, 64 * c + 64))
    far = np.array([j for j in range(1024) if j not in used])
    v2 = wl.v.copy()
    v2[:, 0, far] = W.bf16_bits(np.random.default_rng(3).standard_normal(v2[:, 0, far].shape)
                                .astype(np.float32))
    mod = P.run_gpu(dataclasses.replace(wl, v=v2))
    assert np.array_equal(mod["idx"], base["idx"])
    assert np.array_equal(mod["o"][0, i, :4], base["o"][0, i, :4])


# ----------------------------------------------------------------------------- full size

@pytest.fixture(scope="module")
def prefill16k():
    return W.prefill_16k()


def test_prefill_16k_sampled(prefill16k):
    wl = prefill16k
    gpu = P.run_gpu(wl, swa=True)
    rows = P.sample_rows(wl, 512)
    r = P.check_route_layer(wl, gpu, rows)
    assert r["n_exact"] > 1000
    P.check_swa(wl, gpu, rows)
    # properties that hold at any size, on every row
    idx = gpu["idx"][0]
    assert idx.shape == (4, 16384, 32) and idx.max() < 256
    content = (np.arange(16384) % 64) != 63
    assert np.all(idx[:, ~content] == -1) and np.all(idx[:, content] >= 0)
    assert np.all(np.isfinite(gpu["o"])) and np.all(np.isfinite(gpu["lse"][:, :, content]))


def test_decode_128k():
    wl = W.decode_128k()
    gpu = P.run_gpu(wl, swa=True)
    rows = np.arange(32)
    P.check_route_layer(wl, gpu, rows)
    P.check_swa(wl, gpu, rows)


def test_prefill_64k_mixture_sampled():
    wl = W.prefill_64k()
    gpu = P.run_gpu(wl)
    rows = P.sample_rows(wl, 512, seed=1)
    r = P.check_route_layer(wl, gpu, rows)
    assert r["n_tie"] > 0          # the mixture keys create near ties


def test_prefill_exact_ties_long_rows():
    """Every eligible chunk of every row ties: zero content queries and hidden states, and the
    content keys of each chunk all equal (uniform pooling, the same entropy everywhere), so
    z = -lambda ln 63 for every remote chunk.  512 chunks per row (the prefill top-K's
    candidate filter path); the selection must be the K lowest eligible chunks (ties to the
    smaller chunk index) and the outputs must match the oracle on sampled rows."""
    dm = small(L=32768, Lq=32768, Hq=8, Hkv=2, K=32, w=64)
    wl = W.make_inputs(dm, seed=37, n_needles=0)
    wl.q[:] = 0
    wl.x[:] = 0
    B, Hkv, L, d = wl.k.shape
    kc = wl.k.reshape(B, Hkv, L // 64, 64, d)
    kc[:, :, :, 1:63, :] = kc[:, :, :, 0:1, :]
    gpu = P.run_gpu(wl)
    rows = np.unique(np.concatenate([np.arange(0, 200, 7), np.arange(16000, 16200, 9), np.arange(32600, 32768, 5)]))
    r = P.check_route_layer(wl, gpu, rows)
    assert r["n_tie"] > 0
    idx = gpu["idx"][0]
    for i in (5, 1000, 20000, 32700):
        if i % 64 == 63:
            continue
        wl_lo, wl_hi = max(0, i - 64) // 64, min(L - 1, i + 64) // 64
        want = [c for c in range(L // 64) if c < wl_lo or c > wl_hi][:32]
        assert idx[0, i].tolist() == want and idx[1, i].tolist() == want


def test_prefill_128k_sampled():
    """Route-layer prefill at 128K: summaries of all 2048 chunks, 512 sampled rows (first
    and last chunks, window edges, rows next to needles), properties on every row."""
    wl = W.prefill_128k()
    gpu = P.run_gpu(wl)
    rows = P.sample_rows(wl, 512, seed=2)
    r = P.check_route_layer(wl, gpu, rows)
    assert r["n_exact"] > 1000
    idx = gpu["idx"][0]
    assert idx.shape == (4, 131072, 32) and idx.max() < 2048
    content = (np.arange(131072) % 64) != 63
    assert np.all(idx[:, ~content] == -1) and np.all(idx[:, content] >= 0)
    assert np.all(np.isfinite(gpu["o"])) and np.all(np.isfinite(gpu["lse"][:, :, content]))


def test_stack_128k_all_layers():
    for layer in range(W.STACK_LAYERS):
        wl = W.stack_layer(layer)
        route = W.is_route_layer(layer)
        gpu = P.run_gpu(wl, route=route, swa=not route)
        rows = np.arange(32)
        if route:
            P.check_route_layer(wl, gpu, rows)
        else:
            P.check_swa(wl, gpu, rows)
