"""Seeded synthetic inputs for Skip Softmax attention (prefill and decode).

This module holds no attention arithmetic: it only draws Gaussian tensors and
places the "attention sink" rows, so that the CUDA path, the tests and the
bench all see bit-identical bf16 inputs.  Draws happen on the CPU with
``torch.Generator`` (deterministic for a given torch build).  With
``device="cuda"`` the same recipe is drawn by the GPU's generator instead
(same distribution, different bits): the bench uses that only to time very
large workloads whose CPU draw would take minutes.

Recipe (one line per knob):
  * every (tensor, batch, head) gets its own seed ``derive(seed, tag, b, h)``;
    tensors are drawn as fp32 ``randn`` of shape [rows, d];
  * queries:  q = q_sigma * z + q_u * u, rounded to bf16 (round-to-nearest-even);
  * keys, values: z ~ N(0, 1) rounded to bf16;
  * u is one unit vector per workload, drawn from its own seed (fp32 randn,
    normalised in fp64, stored as fp32) and shared by every batch and head;
  * sinks: key rows 0..n_sinks-1 of every (b, kv head) are replaced by
    bf16(sink_scale * sqrt(d) * u), which gives every query a large logit on
    the first keys (the attention-sink structure of long-context LLMs).
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor

import torch

_TAGS = {"u": 1, "q": 2, "k": 3, "v": 4, "dq": 5}
_MASK64 = (1 << 64) - 1


def derive(seed: int, tag: str, b: int = 0, h: int = 0) -> int:
    """splitmix64 of the packed (seed, tag, b, h) -> a 63-bit generator seed."""
    x = (seed * 0x9E3779B97F4A7C15 + _TAGS[tag] * 0xBF58476D1CE4E5B9
         + b * 0x94D049BB133111EB + h * 0x2545F4914F6CDD1D) & _MASK64
    x = (x + 0x9E3779B97F4A7C15) & _MASK64
    x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & _MASK64
    x ^= x >> 31
    return x & ((1 << 63) - 1)


def _randn(rows: int, d: int, seed: int, device: str = "cpu") -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(rows, d, generator=g, dtype=torch.float32, device=device)


def unit_vector(d: int, seed: int) -> torch.Tensor:
    z = _randn(1, d, derive(seed, "u"))[0].double()
    return (z / z.norm()).float()


def _par_map(fn, items, workers: int = 0):
    items = list(items)
    if len(items) <= 1 or workers == 1:
        return [fn(i) for i in items]
    import os

    w = workers or min(len(items), max(1, len(os.sched_getaffinity(0))))
    with ThreadPoolExecutor(w) as ex:
        return list(ex.map(fn, items))


def prefill_inputs(B: int, Hq: int, Hkv: int, N: int, d: int, *, seed: int = 0,
                   q_sigma: float = 1.0, q_u: float = 0.0, sink_scale: float | None = None,
                   n_sinks: int = 4, q_heads=None, device: str = "cpu"):
    """Q [B,Hq,N,d], K, V [B,Hkv,N,d] bf16 on the CPU.

    ``q_heads``: optional iterable of (b, h) pairs; only those query heads are
    drawn (the others stay zero), which lets very long workloads be checked on
    a sample of heads without drawing all of Q.
    """
    u = unit_vector(d, seed).to(device)
    Q = torch.zeros(B, Hq, N, d, dtype=torch.bfloat16, device=device)
    K = torch.empty(B, Hkv, N, d, dtype=torch.bfloat16, device=device)
    V = torch.empty(B, Hkv, N, d, dtype=torch.bfloat16, device=device)
    qh = [(b, h) for b in range(B) for h in range(Hq)] if q_heads is None else list(q_heads)

    def make_q(bh):
        b, h = bh
        z = _randn(N, d, derive(seed, "q", b, h), device)
        x = z * q_sigma
        if q_u:
            x = x + q_u * u
        Q[b, h] = x.to(torch.bfloat16)

    def make_kv(bh):
        b, h = bh
        k = _randn(N, d, derive(seed, "k", b, h), device)
        if sink_scale is not None and n_sinks > 0:
            k[: min(n_sinks, N)] = sink_scale * math.sqrt(d) * u
        K[b, h] = k.to(torch.bfloat16)
        V[b, h] = _randn(N, d, derive(seed, "v", b, h), device).to(torch.bfloat16)

    workers = 1 if device != "cpu" else 0
    _par_map(make_q, qh, workers)
    _par_map(make_kv, [(b, h) for b in range(B) for h in range(Hkv)], workers)
    return Q, K, V


def prefill_head_inputs(Hq: int, Hkv: int, N: int, d: int, b: int, h: int, *, seed: int = 0,
                        q_sigma: float = 1.0, q_u: float = 0.0, sink_scale: float | None = None,
                        n_sinks: int = 4):
    """Query head (b, h) and its KV head, as [1, 1, N, d] bf16 CPU tensors.

    Bit for bit the slices Q[b, h], K[b, h // (Hq/Hkv)], V[b, h // (Hq/Hkv)]
    of ``prefill_inputs(...)`` with the same seed and knobs, without drawing
    the other heads (a very long workload can be sampled one head at a time).
    """
    kv = h // (Hq // Hkv)
    u = unit_vector(d, seed)
    x = _randn(N, d, derive(seed, "q", b, h)) * q_sigma
    if q_u:
        x = x + q_u * u
    k = _randn(N, d, derive(seed, "k", b, kv))
    if sink_scale is not None and n_sinks > 0:
        k[: min(n_sinks, N)] = sink_scale * math.sqrt(d) * u
    v = _randn(N, d, derive(seed, "v", b, kv))
    return tuple(t.to(torch.bfloat16).view(1, 1, N, d) for t in (x, k, v))


def decode_inputs(B: int, Hq: int, Hkv: int, L: int, d: int, *, seed: int = 0,
                  q_sigma: float = 1.0, q_u: float = 0.0, sink_scale: float | None = None,
                  n_sinks: int = 4):
    """q [B,Hq,d], K, V [B,Hkv,L,d] bf16 on the CPU (one new token per sequence)."""
    u = unit_vector(d, seed)
    q = torch.empty(B, Hq, d, dtype=torch.bfloat16)
    K = torch.empty(B, Hkv, L, d, dtype=torch.bfloat16)
    V = torch.empty(B, Hkv, L, d, dtype=torch.bfloat16)
    for b in range(B):
        for h in range(Hq):
            x = _randn(1, d, derive(seed, "dq", b, h))[0] * q_sigma
            if q_u:
                x = x + q_u * u
            q[b, h] = x.to(torch.bfloat16)

    def make_kv(bh):
        b, h = bh
        k = _randn(L, d, derive(seed, "k", b, h))
        if sink_scale is not None and n_sinks > 0:
            k[: min(n_sinks, L)] = sink_scale * math.sqrt(d) * u
        K[b, h] = k.to(torch.bfloat16)
        V[b, h] = _randn(L, d, derive(seed, "v", b, h)).to(torch.bfloat16)

    _par_map(make_kv, [(b, h) for b in range(B) for h in range(Hkv)])
    return q, K, V


# The five workloads: shapes, distributions and tile sizes.  "taus" are the
# thresholds each one is run at (inf = exact attention).
WORKLOADS = {
    "causal_1x1x256_d64": dict(kind="prefill", B=1, Hq=1, Hkv=1, N=256, d=64, causal=True,
                               Br=64, Bc=64, taus=[math.inf], gen=dict(q_sigma=1.0)),
    "encoder_64x32x512_d128": dict(kind="prefill", B=64, Hq=32, Hkv=32, N=512, d=128, causal=False,
                                   Br=128, Bc=64, taus=[math.inf, 4.0], gen=dict(q_sigma=1.5)),
    "gqa_decode_16x32q8kv_L32768": dict(kind="decode", B=16, Hq=32, Hkv=8, L=32768, d=128,
                                        taus=[math.inf, 4.0],
                                        gen=dict(q_sigma=2.0, q_u=1.0, sink_scale=3.0)),
    "llama3_8b_causal_N8192": dict(kind="prefill", B=1, Hq=32, Hkv=8, N=8192, d=128, causal=True,
                                   Br=128, Bc=128, taus=[math.inf, 2.0, 4.0, 8.0],
                                   gen=dict(q_sigma=2.0, q_u=1.0, sink_scale=3.0)),
    "llama33_70b_causal_N131072": dict(kind="prefill", B=1, Hq=64, Hkv=8, N=131072, d=128,
                                       causal=True, Br=128, Bc=128, taus=[math.inf, 4.0],
                                       gen=dict(q_sigma=2.0, q_u=1.0, sink_scale=3.0)),
}
