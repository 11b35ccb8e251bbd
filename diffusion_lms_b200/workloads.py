"""Seeded synthetic inputs for the route-layer and sliding-window attention workloads.

This module only draws inputs. It holds none of the attention method's arithmetic, so
both the fp64 CPU oracle (tests) and the CUDA path consume exactly the same bits from it.

Layouts (element order, row-major):
    q      [B, Lq, Hq, d]   queries of the rows being computed (post-RoPE)
    q_mask [B, C,  Hq, d]   queries of the routing-mask slots (position 64c+63 of chunk c)
    k, v   [B, Hkv, L, d]   key/value cache; one 64-position chunk of one KV head is contiguous
    x      [B, Lq, D]       hidden states feeding the low-rank routing residual
    w_down [D, r], w_up [r, Hq*d]
    q_pos  [B, Lq] int32 or None (None: row i sits at position i and Lq == L)

Storage: "bf16" workloads hold uint16 bit patterns (round-to-nearest-even from fp32);
"f32" workloads hold float32.  `as_f64` turns either into float64 for the oracle.

Recipes follow the workloads described for the Prefilling-dLLM v2 latency study
("The 172x Speedup Has an Evidence Budget", section on the 172x result: one synthetic
sequence per length; the attention shapes of Dream-v0-Base-7B: 28 query heads, 4 KV
heads, head_dim 128, hidden 3584).  Draw order per workload is fixed:
    Q (decode block first, then mask-slot queries when they are separate), K, V, x,
    W_down, W_up, then needle chunks / mixture parameters.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np

CHUNK = 64          # positions per chunk: 63 content tokens + 1 routing mask (last slot)
_BLOCK = 1 << 22    # elements per draw call; fixed so the stream is reproducible


@dataclass(frozen=True)
class Dims:
    B: int
    L: int            # cache / sequence length (multiple of 64)
    Lq: int           # query rows
    Hq: int
    Hkv: int
    d: int
    D: int            # hidden size feeding the residual
    r: int            # residual rank
    K: int            # selected chunks per query
    w: int            # local-window radius (|p - j| <= w); w < 0: no window
    lam: float = 0.1  # entropy weight in the route score
    dtype: str = "bf16"
    flags: int = 0

    @property
    def C(self) -> int:
        return self.L // CHUNK

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


@dataclass
class Workload:
    name: str
    dims: Dims
    q: np.ndarray
    q_mask: np.ndarray
    k: np.ndarray
    v: np.ndarray
    x: np.ndarray
    w_down: np.ndarray
    w_up: np.ndarray
    q_pos: Optional[np.ndarray]
    needles: np.ndarray                  # [B, n] chunk indices (may be empty)
    meta: dict = field(default_factory=dict)


# ----------------------------------------------------------------------------- bf16 bits

def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest, ties to even); returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    flat = x.reshape(-1).view(np.uint32)
    out = np.empty(flat.size, dtype=np.uint16)
    t = np.empty(min(flat.size, _BLOCK), dtype=np.uint32)
    for s in range(0, flat.size, _BLOCK):
        e = min(flat.size, s + _BLOCK)
        b, tt = flat[s:e], t[:e - s]
        np.right_shift(b, 16, out=tt)
        np.bitwise_and(tt, 1, out=tt)
        tt += np.uint32(0x7FFF)
        tt += b
        tt >>= np.uint32(16)
        out[s:e] = tt
    return out.reshape(x.shape)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def as_f64(a: np.ndarray) -> np.ndarray:
    """Exact float64 value of a stored workload tensor (uint16 bf16 bits or float32)."""
    if a.dtype == np.uint16:
        return bf16_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def _store(a32: np.ndarray, dtype: str) -> np.ndarray:
    return bf16_bits(a32) if dtype == "bf16" else np.ascontiguousarray(a32, dtype=np.float32)


def _normal(rng: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    """float32 N(0, scale^2), drawn in fixed-size blocks (same stream for any memory budget)."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    for s in range(0, n, _BLOCK):
        e = min(n, s + _BLOCK)
        out[s:e] = rng.standard_normal(e - s, dtype=np.float32)
    if scale != 1.0:
        out *= np.float32(scale)
    return out.reshape(shape)


# ----------------------------------------------------------------------------- generator

def make_inputs(dims: Dims, *, seed: int, n_needles: int = 0, unit_scale: bool = False,
                decode_block: int = 0, mixture: int = 0, mixture_sigma: float = 0.3,
                name: str = "custom") -> Workload:
    """Draw one workload.

    unit_scale:   Q, K, V ~ N(0,1)/sqrt(d) instead of N(0,1).
    decode_block: if > 0, Lq = decode_block queries at the first content slots of the
                  final chunk (positions L-64 ... L-64+decode_block-1); their K/V are part
                  of the cache.  The mask-slot queries are then drawn separately.
    n_needles:    chunks whose 63 content keys are shifted by 0.5*E|k|*u_g, u_g the unit
                  mean raw query of KV group g over content rows (E|k| = 1 at unit scale,
                  sqrt(d) otherwise).
    mixture:      if > 0, keys come from a per-group mixture of `mixture` unit centroids:
                  every key of chunk c is sqrt(d)*(mu_m(c) + sigma*eps/sqrt(d)).
    """
    B, L, Hq, Hkv, d, D, r = dims.B, dims.L, dims.Hq, dims.Hkv, dims.d, dims.D, dims.r
    assert L % CHUNK == 0 and Hq % Hkv == 0
    C = L // CHUNK
    G = Hq // Hkv
    rng = np.random.default_rng(seed)
    qk_scale = 1.0 / np.sqrt(d) if unit_scale else 1.0

    if decode_block:
        Lq = decode_block
        assert dims.Lq == Lq and decode_block <= CHUNK - 1
        q32 = _normal(rng, (B, Lq, Hq, d), qk_scale)
        qm32 = _normal(rng, (B, C, Hq, d), qk_scale)
        pos = np.arange(L - CHUNK, L - CHUNK + Lq, dtype=np.int32)
        q_pos = np.broadcast_to(pos, (B, Lq)).copy()
    else:
        assert dims.Lq == L
        q32 = _normal(rng, (B, L, Hq, d), qk_scale)
        qm32 = None
        q_pos = None
    q = _store(q32, dims.dtype)
    q_mask = (_store(qm32, dims.dtype) if qm32 is not None
              else np.ascontiguousarray(q[:, CHUNK - 1::CHUNK]))

    k32 = None if mixture else _normal(rng, (B, Hkv, L, d), qk_scale)
    v = _store(_normal(rng, (B, Hkv, L, d), qk_scale), dims.dtype)
    x = _store(_normal(rng, (B, dims.Lq, D)), dims.dtype)
    w_down = _store(_normal(rng, (D, r), 0.02), dims.dtype)
    w_up = _store(_normal(rng, (r, Hq * d), 0.02), dims.dtype)

    meta = {}
    if mixture:
        mu = _normal(rng, (B, Hkv, mixture, d)).astype(np.float64)
        mu /= np.linalg.norm(mu, axis=-1, keepdims=True)
        comp = rng.integers(0, mixture, size=(B, Hkv, C))
        eps = _normal(rng, (B, Hkv, L, d)).astype(np.float64)
        centre = np.take_along_axis(mu, comp[..., None], axis=2)          # [B,Hkv,C,d]
        centre = np.repeat(centre, CHUNK, axis=2)                          # [B,Hkv,L,d]
        k32 = (np.sqrt(d) * (centre + mixture_sigma * eps / np.sqrt(d))).astype(np.float32)
        meta["components"] = comp

    needles = np.zeros((B, 0), dtype=np.int64)
    if n_needles:
        needles = np.stack([np.sort(rng.choice(C, size=n_needles, replace=False))
                            for _ in range(B)])
        knorm = 1.0 if unit_scale else float(np.sqrt(d))
        for b in range(B):
            qb = bf16_to_f32(q[b]) if q.dtype == np.uint16 else q[b]        # [Lq,Hq,d] exact
            for g in range(Hkv):
                # mean raw query of the group over content rows (mask-slot rows excluded)
                tot = qb[:, g * G:(g + 1) * G, :].sum(axis=(0, 1), dtype=np.float64)
                n = qb.shape[0] * G
                if q_pos is None:
                    tot -= qb[CHUNK - 1::CHUNK, g * G:(g + 1) * G, :].sum(axis=(0, 1),
                                                                           dtype=np.float64)
                    n -= (qb.shape[0] // CHUNK) * G
                u = tot / n
                u /= np.linalg.norm(u)
                shift = (0.5 * knorm * u).astype(np.float32)
                for c in needles[b]:
                    k32[b, g, c * CHUNK:c * CHUNK + CHUNK - 1, :] += shift
    k = _store(k32, dims.dtype)
    return Workload(name, dims, q, q_mask, k, v, x, w_down, w_up, q_pos, needles, meta)


# ----------------------------------------------------------------------------- named workloads
#
# The five workloads of the route-layer study, named by what they are.

TINY_F32 = Dims(B=1, L=1024, Lq=1024, Hq=4, Hkv=1, d=64, D=256, r=16, K=4, w=64,
                lam=0.1, dtype="f32")
PREFILL_16K = Dims(B=1, L=16384, Lq=16384, Hq=28, Hkv=4, d=128, D=3584, r=64, K=32,
                   w=256, lam=0.1, dtype="bf16")
DECODE_128K = Dims(B=1, L=131072, Lq=32, Hq=28, Hkv=4, d=128, D=3584, r=64, K=32,
                   w=256, lam=0.1, dtype="bf16")
PREFILL_64K = Dims(B=1, L=65536, Lq=65536, Hq=28, Hkv=4, d=128, D=3584, r=64, K=32,
                   w=256, lam=0.1, dtype="bf16")
PREFILL_128K = Dims(B=1, L=131072, Lq=131072, Hq=28, Hkv=4, d=128, D=3584, r=64, K=32,
                    w=256, lam=0.1, dtype="bf16")
PREFILL_16K_K8 = Dims(B=1, L=16384, Lq=16384, Hq=28, Hkv=4, d=128, D=3584, r=64, K=8,
                      w=256, lam=0.1, dtype="bf16")
STACK_LAYERS = 28
STACK_ROUTE_EVERY = 4          # route layer when layer % 4 == 3


def tiny_f32(seed: int = 1) -> Workload:
    """fp32 route layer at L=1024: 16 chunks, Hq=4, Hkv=1, d=64, rank 16, K=4, w=64, 2 needles."""
    return make_inputs(TINY_F32, seed=seed, n_needles=2, unit_scale=True, name="tiny_f32_1k")


def prefill_16k(seed: int = 2) -> Workload:
    """Dream-7B-shaped route layer, full prefill at 16K, bf16, 8 needles."""
    return make_inputs(PREFILL_16K, seed=seed, n_needles=8, name="route_prefill_16k")


def decode_128k(seed: int = 3) -> Workload:
    """32-query decode block over a 128K bf16 cache, 16 needles."""
    return make_inputs(DECODE_128K, seed=seed, n_needles=16, decode_block=32,
                       name="route_decode_128k")


def prefill_64k(seed: int = 4) -> Workload:
    """Route layer prefill at 64K with keys from a 32-component mixture (near-tie top-K)."""
    return make_inputs(PREFILL_64K, seed=seed, mixture=32, name="route_prefill_64k_mixture")


def prefill_16k_k8(seed: int = 7) -> Workload:
    """The 16K prefill shapes with K = 8 chunks per query: sparse chunk buckets per row tile,
    so the selected-chunk attention takes its chunk-major form on a case a few GB in size."""
    return make_inputs(PREFILL_16K_K8, seed=seed, n_needles=8, name="route_prefill_16k_k8")


def prefill_128k(seed: int = 6) -> Workload:
    """Route-layer prefill at 128K (the top of the 16K-128K range), bf16, 16 needles."""
    return make_inputs(PREFILL_128K, seed=seed, n_needles=16, name="route_prefill_128k")


def stack_layer(layer: int, seed: int = 5) -> Workload:
    """One layer of the 28-layer attention-only stack at 128K (decode block of 32 queries).

    Every layer draws its own K/V (and queries, residual weights) from seed [5, layer].
    """
    return make_inputs(replace(DECODE_128K), seed=np.random.SeedSequence([seed, layer])
                       .generate_state(1)[0].item(), decode_block=32,
                       name=f"stack_128k_layer{layer}")


def is_route_layer(layer: int) -> bool:
    return layer % STACK_ROUTE_EVERY == STACK_ROUTE_EVERY - 1


def scaled(dims: Dims, **kw) -> Dims:
    """Same workload family at other sizes (parity cases)."""
    return replace(dims, **kw)
