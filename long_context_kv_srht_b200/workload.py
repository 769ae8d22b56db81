"""Seeded synthetic workloads for the ParisKV retrieval path.

This module only draws inputs: keys, values, queries, planted positions and the SRHT sign
vector. It holds none of the method's arithmetic, and both the CUDA path and the CPU oracle
consume what it produces.

Recipe (one draw per (sequence, KV head) unit, in this order):
  * mean vector mu ~ N(0, 0.5^2) per dim (0.5 is read as a standard deviation);
  * 8 distinct outlier channels chosen uniformly among the d dims;
  * keys  k = (z + mu) * o,  z ~ N(0, 1), o = 8 on outlier channels and 1 elsewhere;
  * values v ~ N(0, 1);
  * one query per query head of the group, q = (z' + mu) * o, a fresh draw of the same law;
  * planted keys: per query head, P positions (distinct over the whole group) whose keys are
    replaced by q + N(0, 0.3^2) noise;
  * keys/values/queries are rounded to bf16 (round-to-nearest-even) unless the workload is f32.
The SRHT sign vector (d entries of +-1) is drawn first from the same seed.

Two backends follow the recipe: numpy's PCG64 on the host (exact and reproducible, used by
the tests) and torch's generator on a CUDA device (used for the million-token workloads,
where host generation would take minutes). The two backends give different numbers for the
same seed; each is deterministic.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np


@dataclass(frozen=True)
class Spec:
    name: str
    batch: int
    num_kv_heads: int
    group: int            # query heads per KV head (GQA group size)
    n: int                # cached keys per (sequence, KV head)
    d: int = 128
    dtype: str = "bf16"   # "bf16" or "f32"
    planted: int = 32     # planted keys per query head (0 = none)
    planted_sigma: float = 0.3
    mean_sigma: float = 0.5
    outliers: int = 8
    outlier_scale: float = 8.0
    B: int = 16
    m: int = 8
    rho: int = 4
    cand_bp: int = 500    # candidate fraction in basis points
    k: int = 2048
    seed: int = 0
    decode_steps: int = 0  # long-generation workload: keys appended one per step
    description: str = ""

    @property
    def num_q_heads(self) -> int:
        return self.num_kv_heads * self.group


# The five synthetic workloads the retrieval path is measured and tested on.
SPECS = {
    "tiny": Spec("tiny", batch=1, num_kv_heads=1, group=1, n=4096, dtype="f32", planted=32,
                 cand_bp=1000, k=64, seed=0,
                 description="single head, d=128, N=4096 f32, 32 planted keys, 10% cand, k=64"),
    "llama3_8b_128k": Spec("llama3_8b_128k", batch=1, num_kv_heads=8, group=4, n=131072,
                           k=2048, seed=1,
                           description="Llama-3-8B-shaped decode: 32q/8kv, N=131072 bf16, 5%, k=2048"),
    "drift_32k": Spec("drift_32k", batch=1, num_kv_heads=8, group=1, n=32768, planted=0,
                      k=1024, seed=2, decode_steps=32768,
                      description="8 kv heads, 32768 prefill + 32768 drifting appends, k=1024"),
    "batched_64k": Spec("batched_64k", batch=16, num_kv_heads=8, group=4, n=65536, k=2048,
                        seed=3,
                        description="batch 16, 32q/8kv, N=65536 bf16 per sequence, 5%, k=2048"),
    "million_offload": Spec("million_offload", batch=1, num_kv_heads=8, group=4, n=1 << 20,
                            k=4096, seed=4,
                            description="1M tokens, 32q/8kv, index in HBM, K/V in pinned host"),
}


def spec(name: str, **overrides) -> Spec:
    return replace(SPECS[name], **overrides)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp32 -> nearest bf16 (ties to even), returned as fp32 values (exactly representable)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    # finite inputs never wrap: the largest finite pattern plus 0x8000 rounds up to infinity
    r = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    r &= np.uint32(0xFFFF0000)
    return r.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 values that are exact bf16 numbers -> their 16-bit patterns (uint16)."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


@dataclass
class Workload:
    """Host-side (numpy) workload. Arrays hold exact fp32 values (bf16-representable when
    spec.dtype == 'bf16')."""
    spec: Spec
    signs: np.ndarray     # int8  [d]
    keys: np.ndarray      # f32   [batch, Hkv, n, d]
    values: np.ndarray    # f32   [batch, Hkv, n, d]
    queries: np.ndarray   # f32   [batch, Hq, d]
    planted: np.ndarray   # int32 [batch, Hq, P]
    mu: np.ndarray = field(default=None)        # f32 [batch, Hkv, d]
    outlier_mask: np.ndarray = field(default=None)  # f32 [batch, Hkv, d]


def _round(x: np.ndarray, dtype: str) -> np.ndarray:
    return bf16_round(x) if dtype == "bf16" else x.astype(np.float32)


def generate(sp: Spec, n: Optional[int] = None) -> Workload:
    """numpy backend. ``n`` overrides the number of keys (smaller test sizes)."""
    n = sp.n if n is None else n
    d, G = sp.d, sp.group
    rng = np.random.Generator(np.random.PCG64(sp.seed))
    signs = np.where(rng.integers(0, 2, size=d) == 1, -1, 1).astype(np.int8)
    keys = np.empty((sp.batch, sp.num_kv_heads, n, d), np.float32)
    vals = np.empty_like(keys)
    qs = np.empty((sp.batch, sp.num_q_heads, d), np.float32)
    P = min(sp.planted, n // max(G, 1))
    planted = np.zeros((sp.batch, sp.num_q_heads, P), np.int32)
    mus = np.empty((sp.batch, sp.num_kv_heads, d), np.float32)
    masks = np.empty_like(mus)
    for b in range(sp.batch):
        for h in range(sp.num_kv_heads):
            mu = (rng.standard_normal(d) * sp.mean_sigma).astype(np.float32)
            ch = rng.choice(d, size=sp.outliers, replace=False)
            o = np.ones(d, np.float32)
            o[ch] = sp.outlier_scale
            z = rng.standard_normal((n, d), dtype=np.float32)
            k = (z + mu) * o
            v = rng.standard_normal((n, d), dtype=np.float32)
            pos = rng.choice(n, size=G * P, replace=False).astype(np.int32) if P else None
            for g in range(G):
                q = (rng.standard_normal(d).astype(np.float32) + mu) * o
                qs[b, h * G + g] = _round(q, sp.dtype)
                if P:
                    p = pos[g * P:(g + 1) * P]
                    planted[b, h * G + g] = p
                    noise = (rng.standard_normal((P, d)) * sp.planted_sigma).astype(np.float32)
                    k[p] = qs[b, h * G + g][None, :] + noise
            keys[b, h] = _round(k, sp.dtype)
            vals[b, h] = _round(v, sp.dtype)
            mus[b, h] = mu
            masks[b, h] = o
    return Workload(sp, signs, keys, vals, qs, planted, mus, masks)


@dataclass
class DriftWorkload:
    """Long-generation workload: prefill keys, then one appended key and one query per step
    per KV head; the mean vector moves linearly from mu0 to a fresh draw mu1."""
    spec: Spec
    signs: np.ndarray     # int8 [d]
    prefill: np.ndarray   # f32 [Hkv, n, d]
    appended: np.ndarray  # f32 [steps, Hkv, d]
    queries: np.ndarray   # f32 [steps, Hkv, d]  (one query head per KV head)


def generate_drift(sp: Spec, n: Optional[int] = None, steps: Optional[int] = None) -> DriftWorkload:
    n = sp.n if n is None else n
    T = sp.decode_steps if steps is None else steps
    d, H = sp.d, sp.num_kv_heads
    rng = np.random.Generator(np.random.PCG64(sp.seed))
    signs = np.where(rng.integers(0, 2, size=d) == 1, -1, 1).astype(np.int8)
    pre = np.empty((H, n, d), np.float32)
    app = np.empty((T, H, d), np.float32)
    qs = np.empty((T, H, d), np.float32)
    for h in range(H):
        mu0 = (rng.standard_normal(d) * sp.mean_sigma).astype(np.float32)
        mu1 = (rng.standard_normal(d) * sp.mean_sigma).astype(np.float32)
        ch = rng.choice(d, size=sp.outliers, replace=False)
        o = np.ones(d, np.float32)
        o[ch] = sp.outlier_scale
        pre[h] = _round((rng.standard_normal((n, d), dtype=np.float32) + mu0) * o, sp.dtype)
        t = (np.arange(1, T + 1, dtype=np.float32) / max(T, 1))[:, None]
        mut = mu0[None, :] + t * (mu1 - mu0)[None, :]
        app[:, h] = _round((rng.standard_normal((T, d), dtype=np.float32) + mut) * o, sp.dtype)
        qs[:, h] = _round((rng.standard_normal((T, d), dtype=np.float32) + mut) * o, sp.dtype)
    return DriftWorkload(sp, signs, pre, app, qs)


def generate_torch(sp: Spec, device, n: Optional[int] = None, kv_on_host: bool = False):
    """torch backend on ``device`` (the same recipe, torch's generator). Returns a dict of
    tensors: signs int8 [d] (host), keys/values bf16|f32 [batch, Hkv, n, d] (on ``device``,
    or in pinned host memory when ``kv_on_host``), queries [batch, Hq, d] and planted int32
    [batch, Hq, P] on ``device``."""
    import torch

    n = sp.n if n is None else n
    d, G = sp.d, sp.group
    dt = torch.bfloat16 if sp.dtype == "bf16" else torch.float32
    g = torch.Generator(device=device)
    g.manual_seed(sp.seed)
    signs = torch.where(torch.randint(0, 2, (d,), generator=g, device=device) == 1, -1, 1)
    signs = signs.to(torch.int8).cpu()
    shape = (sp.batch, sp.num_kv_heads, n, d)
    if kv_on_host:
        keys = torch.empty(shape, dtype=dt, pin_memory=True)
        vals = torch.empty(shape, dtype=dt, pin_memory=True)
    else:
        keys = torch.empty(shape, dtype=dt, device=device)
        vals = torch.empty(shape, dtype=dt, device=device)
    qs = torch.empty((sp.batch, sp.num_q_heads, d), dtype=dt, device=device)
    P = min(sp.planted, n // max(G, 1))
    planted = torch.zeros((sp.batch, sp.num_q_heads, P), dtype=torch.int32, device=device)
    for b in range(sp.batch):
        for h in range(sp.num_kv_heads):
            mu = torch.randn(d, generator=g, device=device) * sp.mean_sigma
            ch = torch.randperm(d, generator=g, device=device)[: sp.outliers]
            o = torch.ones(d, device=device)
            o[ch] = sp.outlier_scale
            k = (torch.randn((n, d), generator=g, device=device) + mu) * o
            v = torch.randn((n, d), generator=g, device=device)
            pos = torch.randperm(n, generator=g, device=device)[: G * P].to(torch.int32)
            for gi in range(G):
                q = ((torch.randn(d, generator=g, device=device) + mu) * o).to(dt)
                qs[b, h * G + gi] = q
                if P:
                    p = pos[gi * P:(gi + 1) * P]
                    planted[b, h * G + gi] = p
                    noise = torch.randn((P, d), generator=g, device=device) * sp.planted_sigma
                    k[p.long()] = q.float()[None, :] + noise
            keys[b, h].copy_(k.to(dt))
            vals[b, h].copy_(v.to(dt))
            del k, v
    return {"signs": signs, "keys": keys, "values": vals, "queries": qs, "planted": planted}
