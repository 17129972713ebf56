"""Pins for the fp64 CPU oracle: what the mathematics and the pages fix.

The oracle is only trusted after it is pinned to something other than
itself.  Each pin below is written against the definition of attention
(brute force on tiny inputs), a closed form, an invariant, or the hand-built
two-tile example in ``tests/golden/two_tile_example.txt``.  The rule pinned
is the one of "Accelerating Long-Context Inference with Skip Softmax in NVIDIA
TensorRT-LLM" (Key Points; Detailed Analysis).

Every pin takes ``lib`` (None for the real oracle, or the path of a variant
built by ``test_oracle_mutants.py``) so that the same pins can be shown to
catch planted mistakes.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from block_skipping_softmax_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "two_tile_example.txt")
PINS = []


def pin(fn):
    PINS.append(fn)
    return fn


# ----------------------------------------------------------------------------
# independent numpy helpers (fp64, whole score matrix, no tiling)
# ----------------------------------------------------------------------------

def f64(x):
    return x.float().double().numpy() if isinstance(x, torch.Tensor) else np.asarray(x, np.float64)


def scores(Q, K, causal):
    """S[b,h,i,k] = q_i . k_k / sqrt(d), -inf above the diagonal when causal."""
    q, k = f64(Q), f64(K)
    g = q.shape[1] // k.shape[1]
    k = np.repeat(k, g, axis=1)                       # head h reads KV head h // g
    s = np.einsum("bhid,bhkd->bhik", q, k) / math.sqrt(q.shape[-1])
    if causal:
        n = s.shape[-1]
        s = np.where(np.triu(np.ones((n, n), bool), 1), -np.inf, s)
    return s


def softmax_av(s, V, keep=None):
    """softmax over the last axis (optionally restricted by a boolean keep) times V."""
    g = s.shape[1] // V.shape[1]
    v = np.repeat(f64(V), g, axis=1)
    if keep is not None:
        s = np.where(keep, s, -np.inf)
    mx = s.max(-1, keepdims=True)
    w = np.exp(s - mx)
    return np.einsum("bhik,bhkd->bhid", w, v) / w.sum(-1, keepdims=True)


def brute_decisions(s, Br, Bc, tau):
    """Skip decisions from the definition: the running max before tile j is the
    max of all visible scores in tiles < j (skipped tiles never exceed it)."""
    B, H, N, _ = s.shape
    n_rb, n_t = -(-N // Br), -(-N // Bc)
    mask = np.full((B, H, n_rb, n_t), 2, np.uint8)
    margin = np.full((B, H, n_rb, n_t), np.nan)
    for b in range(B):
        for h in range(H):
            for rb in range(n_rb):
                r0, r1 = rb * Br, min(N, rb * Br + Br)
                for j in range(n_t):
                    c0, c1 = j * Bc, min(N, j * Bc + Bc)
                    if np.all(np.isneginf(s[b, h, r0:r1, c0:c1])) and c0 > r1 - 1:
                        continue                               # never visited (causal)
                    rows = []
                    for r in range(r0, r1):
                        prev = s[b, h, r, :c0]
                        m = prev.max() if prev.size else -np.inf
                        mt = s[b, h, r, c0:c1].max()
                        if m == -np.inf:
                            rows.append(np.inf)
                        elif mt == -np.inf:
                            rows.append(-np.inf)
                        else:
                            rows.append(mt - m + tau)
                    mg = max(rows)
                    margin[b, h, rb, j] = mg
                    mask[b, h, rb, j] = 1 if mg < 0 else 0
    return mask, margin


def kept_keys(mask, N, Br, Bc):
    """Boolean [B,H,N,N]: key k is used by row i (its tile was kept for i's row block)."""
    B, H, n_rb, n_t = mask.shape
    keep = np.zeros((B, H, N, N), bool)
    for rb in range(n_rb):
        for j in range(n_t):
            sel = mask[:, :, rb, j] == 0
            keep[:, :, rb * Br:(rb + 1) * Br, j * Bc:(j + 1) * Bc] |= sel[:, :, None, None]
    return keep


def skippy(B=1, Hq=2, Hkv=1, N=200, d=64, seed=3, q_u=8.0, sink=6.0, q_sigma=2.0):
    """Inputs on which many tiles skip: a strong shared direction u in every
    query and a few sink keys along u."""
    return inputs.prefill_inputs(B, Hq, Hkv, N, d, seed=seed, q_sigma=q_sigma, q_u=q_u,
                                 sink_scale=sink, n_sinks=4)


SHAPES = [  # B, Hq, Hkv, N, d, causal, Br, Bc
    (1, 1, 1, 1, 64, True, 64, 64),
    (1, 1, 1, 7, 64, False, 64, 64),
    (1, 2, 2, 64, 64, True, 64, 64),
    (2, 2, 1, 65, 64, True, 64, 64),
    (1, 4, 2, 200, 128, True, 128, 64),
    (1, 2, 1, 256, 128, False, 128, 128),
    (1, 1, 1, 200, 64, True, 64, 128),
]


# ----------------------------------------------------------------------------
# pins
# ----------------------------------------------------------------------------

@pin
def pin_exact_equals_bruteforce(lib):
    """tau = inf is exact softmax(QK^T/sqrt d)V: brute force on tiny inputs."""
    for i, (B, Hq, Hkv, N, d, causal, Br, Bc) in enumerate(SHAPES):
        Q, K, V = inputs.prefill_inputs(B, Hq, Hkv, N, d, seed=10 + i, q_sigma=1.5)
        ref = softmax_av(scores(Q, K, causal), V)
        r = oracle.prefill(Q, K, V, causal, math.inf, Br, Bc, lib_path=lib)
        np.testing.assert_allclose(r["O"], ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["O_exact"], ref, rtol=0, atol=1e-12)
        assert np.all(r["mask"][r["mask"] != 2] == 0)


@pin
def pin_uniform_logits_give_mean_of_v(lib):
    """Q = 0 makes every logit equal: O is the mean of the visible V rows
    (the prefix mean under causal attention)."""
    for causal in (False, True):
        _, K, V = inputs.prefill_inputs(1, 2, 1, 130, 64, seed=4)
        Q = torch.zeros(1, 2, 130, 64, dtype=torch.bfloat16)
        r = oracle.prefill(Q, K, V, causal, 3.0, 64, 64, lib_path=lib)
        v = f64(V)[0, 0]
        if causal:
            mean = np.cumsum(v, 0) / np.arange(1, 131)[:, None]
        else:
            mean = np.broadcast_to(v.mean(0), v.shape)
        for h in range(2):
            np.testing.assert_allclose(r["O"][0, h], mean, rtol=0, atol=1e-12)


@pin
def pin_one_logit_closed_form(lib):
    """Logits {a at key j*, 0 elsewhere}: O = (e^a V[j*] + sum_{k!=j*} V[k]) / (e^a + N - 1).
    Pins the exponential base and the 1/sqrt(d) scale."""
    N, d = 96, 64
    _, _, V = inputs.prefill_inputs(1, 1, 1, N, d, seed=5)
    Q = torch.zeros(1, 1, N, d, dtype=torch.bfloat16)
    Q[..., 0] = 8.0                                     # q . k / sqrt(64) = K[k, 0]
    K = torch.zeros(1, 1, N, d, dtype=torch.bfloat16)
    for a, js in ((3.0, 70), (40.0, 17)):
        K.zero_()
        K[0, 0, js, 0] = a
        v = f64(V)[0, 0]
        expect = (math.exp(a) * v[js] + v.sum(0) - v[js]) / (math.exp(a) + N - 1)
        r = oracle.prefill(Q, K, V, False, math.inf, 64, 64, lib_path=lib)
        np.testing.assert_allclose(r["O"][0, 0], np.broadcast_to(expect, (N, d)), rtol=1e-13, atol=1e-14)
        if a == 40.0:                                   # one dominant logit -> that V row
            bound = 2 * np.abs(v).max() * (N - 1) * math.exp(-a)
            assert np.abs(r["O"][0, 0] - v[js]).max() <= bound


@pin
def pin_rows_sum_to_one(lib):
    """With V = 1 every output is the row sum of the (kept) probabilities: 1."""
    Q, K, _ = skippy(N=200)
    V = torch.ones(1, 1, 200, 64, dtype=torch.bfloat16)
    for tau in (0.0, 2.0, 8.0, math.inf):
        for causal in (False, True):
            r = oracle.prefill(Q, K, V, causal, tau, 64, 64, lib_path=lib)
            np.testing.assert_allclose(r["O"], 1.0, rtol=0, atol=1e-13)


@pin
def pin_skip_error_bound(lib):
    """|O_skip - O_exact| <= 2 max|V| p_r, with p_r the skipped softmax mass."""
    Q, K, V = skippy(N=256)
    vmax = np.abs(f64(V)).max()
    saw_skip = False
    for tau in (0.5, 4.0, 16.0):
        for causal in (False, True):
            r = oracle.prefill(Q, K, V, causal, tau, 64, 64, lib_path=lib)
            saw_skip |= bool((r["mask"] == 1).any())
            dev = np.abs(r["O"] - r["O_exact"]).max(-1)
            assert np.all(dev <= 2 * vmax * r["pskip"] + 1e-12)
            # the skipped mass is exactly the mass of the keys in skipped tiles
            s = scores(Q, K, causal)
            w = np.exp(s - s.max(-1, keepdims=True))
            skipped = ~kept_keys(r["mask"], 256, 64, 64) & np.isfinite(s)
            np.testing.assert_allclose(r["pskip"], (w * skipped).sum(-1) / w.sum(-1), rtol=0, atol=1e-12)
    assert saw_skip


@pin
def pin_output_is_softmax_over_kept_tiles(lib):
    """Given the skip set, O is plain softmax restricted to the kept tiles (two-pass form)."""
    for (Br, Bc) in ((64, 64), (128, 64), (64, 128)):
        Q, K, V = skippy(N=200, Hq=2, Hkv=1)
        for causal in (False, True):
            r = oracle.prefill(Q, K, V, causal, 3.0, Br, Bc, lib_path=lib)
            keep = kept_keys(r["mask"], 200, Br, Bc)
            ref = softmax_av(scores(Q, K, causal), V, keep)
            np.testing.assert_allclose(r["O"], ref, rtol=0, atol=1e-12)


@pin
def pin_decisions_from_prefix_max(lib):
    """Mask and margin equal those derived from the exact prefix row max."""
    for (Br, Bc, N) in ((64, 64, 200), (128, 64, 256), (64, 128, 190)):
        Q, K, V = skippy(N=N, Hq=2, Hkv=1, seed=Br + Bc + N)
        for causal in (False, True):
            s = scores(Q, K, causal)
            for tau in (0.0, 1.5, 6.0):
                r = oracle.prefill(Q, K, V, causal, tau, Br, Bc, lib_path=lib)
                mask, margin = brute_decisions(s, Br, Bc, tau)
                np.testing.assert_array_equal(r["mask"], mask)
                np.testing.assert_allclose(r["margin"], margin, rtol=0, atol=1e-10)


def read_golden():
    rows = []
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if line:
            t, m0, m1, mg = line.split()
            rows.append((float(t), int(m0), int(m1), float(mg)))
    return rows


@pin
def pin_golden_two_tile_example(lib):
    """The hand-built example: tile 1 is skipped iff tau < 5 (strict)."""
    N, d = 128, 64
    Q = torch.zeros(1, 1, N, d, dtype=torch.bfloat16)
    Q[..., 0] = 8.0
    K = torch.zeros(1, 1, N, d, dtype=torch.bfloat16)
    K[0, 0, 0, 0], K[0, 0, 64, 0] = 10.0, 5.0
    V = torch.zeros(1, 1, N, d, dtype=torch.bfloat16)
    V[0, 0, 0, 0], V[0, 0, 64, 1], V[0, 0, :, 2] = 1.0, 1.0, 1.0
    z_skip, z_keep = math.exp(10) + 63, math.exp(10) + 63 + math.exp(5) + 63
    rows = read_golden()
    assert len(rows) == 5
    for tau, m0, m1, mg in rows:
        r = oracle.prefill(Q, K, V, False, tau, 64, 64, lib_path=lib)
        for rb in range(2):
            assert r["mask"][0, 0, rb, 0] == m0 and r["mask"][0, 0, rb, 1] == m1
            assert r["margin"][0, 0, rb, 0] == math.inf
            if math.isinf(mg):
                assert r["margin"][0, 0, rb, 1] == math.inf
            else:
                assert abs(r["margin"][0, 0, rb, 1] - mg) < 1e-12
        o = r["O"][0, 0]
        if m1:
            expect = (math.exp(10) / z_skip, 0.0, 1.0)
            np.testing.assert_allclose(r["pskip"][0, 0], (math.exp(5) + 63) / z_keep, rtol=1e-13)
        else:
            expect = (math.exp(10) / z_keep, math.exp(5) / z_keep, 1.0)
            np.testing.assert_allclose(r["pskip"][0, 0], 0.0, atol=0)
        for c in range(3):
            np.testing.assert_allclose(o[:, c], expect[c], rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(o[:, 3:], 0.0, atol=0)


@pin
def pin_tau_monotone_and_limits(lib):
    """Skip sets shrink as tau grows; tile 0 is never skipped; tau=inf skips nothing."""
    Q, K, V = skippy(N=256, Hq=2, Hkv=2)
    prev = None
    for tau in (0.0, 0.5, 2.0, 8.0, 32.0, math.inf):
        r = oracle.prefill(Q, K, V, True, tau, 64, 64, lib_path=lib)
        sk = r["mask"] == 1
        assert not sk[..., 0].any()
        if prev is not None:
            assert np.all(sk <= prev)           # skipped at larger tau => skipped at smaller
        prev = sk
    assert not prev.any()


@pin
def pin_gqa_equals_repeated_heads(lib):
    """Hkv < Hq gives the same result as Hkv = Hq with each KV head repeated g times."""
    Q, K, V = skippy(N=130, Hq=4, Hkv=2, seed=7)
    Kr, Vr = K.repeat_interleave(2, dim=1), V.repeat_interleave(2, dim=1)
    for tau in (1.0, math.inf):
        a = oracle.prefill(Q, K, V, True, tau, 64, 64, lib_path=lib)
        b = oracle.prefill(Q, Kr, Vr, True, tau, 64, 64, lib_path=lib)
        np.testing.assert_array_equal(a["O"], b["O"])
        np.testing.assert_array_equal(a["mask"], b["mask"])


@pin
def pin_causal_first_row_is_v0(lib):
    """Under causal attention query 0 sees only key 0: O[0] = V[0] exactly."""
    Q, K, V = inputs.prefill_inputs(1, 2, 2, 70, 64, seed=8)
    r = oracle.prefill(Q, K, V, True, 1.0, 64, 64, lib_path=lib)
    np.testing.assert_array_equal(r["O"][0, :, 0], f64(V)[0, :, 0])


@pin
def pin_row_block_subset_is_exact(lib):
    """Computing a subset of row blocks gives bit-identical results for them."""
    Q, K, V = skippy(N=256, Hq=2, Hkv=1, seed=9)
    full = oracle.prefill(Q, K, V, True, 2.0, 64, 64, lib_path=lib)
    units = [(0, 1, 3), (0, 0, 0), (0, 1, 1)]
    sub = oracle.prefill(Q, K, V, True, 2.0, 64, 64, units=units, lib_path=lib)
    for b, h, rb in units:
        np.testing.assert_array_equal(sub["O"][b, h, rb * 64:(rb + 1) * 64], full["O"][b, h, rb * 64:(rb + 1) * 64])
        np.testing.assert_array_equal(sub["mask"][b, h, rb], full["mask"][b, h, rb])
    assert np.isnan(sub["O"][0, 0, 64:128]).all()


# ---------------------------------------------------------------- decode pins

def dec_inputs(B=2, Hq=4, Hkv=2, L=300, d=64, seed=11, q_u=8.0, sink=6.0):
    return inputs.decode_inputs(B, Hq, Hkv, L, d, seed=seed, q_sigma=2.0, q_u=q_u,
                                sink_scale=sink, n_sinks=4)


def dec_scores(q, K):
    qq, k = f64(q), f64(K)
    g = qq.shape[1] // k.shape[1]
    k = np.repeat(k, g, axis=1)
    return np.einsum("bhd,bhkd->bhk", qq, k) / math.sqrt(qq.shape[-1])


@pin
def pin_decode_exact_equals_bruteforce(lib):
    q, K, V = dec_inputs()
    s = dec_scores(q, K)
    v = np.repeat(f64(V), 2, axis=1)
    w = np.exp(s - s.max(-1, keepdims=True))
    ref = np.einsum("bhk,bhkd->bhd", w, v) / w.sum(-1, keepdims=True)
    for Ls in (64, 128, 320):                    # split layout does not change exact results
        r = oracle.decode(q, K, V, math.inf, Ls, 64, lib_path=lib)
        np.testing.assert_allclose(r["o"], ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["o_exact"], ref, rtol=0, atol=1e-12)
        assert not (r["mask"] == 1).any()


@pin
def pin_decode_decisions_split_local(lib):
    """Decode rows are the g heads of a KV group; the running max restarts at
    each split; output = softmax over kept tiles; bound holds; V=1 gives 1."""
    q, K, V = dec_inputs(L=640)
    s = dec_scores(q, K)                          # [B,Hq,L]
    B, Hq, L = s.shape
    g, Bt = 2, 64
    saw = False
    for Ls in (128, 320, 640):
        for tau in (0.0, 2.0, 6.0):
            r = oracle.decode(q, K, V, tau, Ls, Bt, lib_path=lib)
            keep = np.zeros_like(s, bool)
            for b in range(B):
                for kv in range(Hq // g):
                    rows = s[b, kv * g:(kv + 1) * g]
                    for j in range(-(-L // Bt)):
                        c0, c1 = j * Bt, min(L, j * Bt + Bt)
                        split0 = (c0 // Ls) * Ls
                        m = rows[:, split0:c0].max(-1) if c0 > split0 else np.full(g, -np.inf)
                        mt = rows[:, c0:c1].max(-1)
                        mg = max(np.inf if mm == -np.inf else t - mm + tau for t, mm in zip(mt, m))
                        assert r["mask"][b, kv, j] == (1 if mg < 0 else 0)
                        if np.isfinite(mg):
                            assert abs(r["margin"][b, kv, j] - mg) < 1e-10
                        if mg >= 0:
                            keep[b, kv * g:(kv + 1) * g, c0:c1] = True
            saw |= bool((r["mask"] == 1).any())
            w = np.where(keep, np.exp(s - s.max(-1, keepdims=True)), 0.0)
            v = np.repeat(f64(V), g, axis=1)
            ref = np.einsum("bhk,bhkd->bhd", w, v) / w.sum(-1, keepdims=True)
            np.testing.assert_allclose(r["o"], ref, rtol=0, atol=1e-12)
            dev = np.abs(r["o"] - r["o_exact"]).max(-1)
            assert np.all(dev <= 2 * np.abs(f64(V)).max() * r["pskip"] + 1e-12)
    assert saw
    ones = torch.ones_like(V)
    np.testing.assert_allclose(oracle.decode(q, K, ones, 1.0, 128, 64, lib_path=lib)["o"], 1.0, atol=1e-13)


@pin
def pin_decode_matches_prefill_single_row(lib):
    """g = 1 and one split: decode of q equals prefill row 0 of a non-causal
    problem whose first query is q, with one-row row blocks and 64-key tiles."""
    q, K, V = dec_inputs(B=1, Hq=1, Hkv=1, L=256, seed=12)
    Q = torch.zeros(1, 1, 256, 64, dtype=torch.bfloat16)
    Q[0, 0, 0] = q[0, 0]
    for tau in (0.0, 3.0, math.inf):
        d_ = oracle.decode(q, K, V, tau, 256, 64, lib_path=lib)
        p_ = oracle.prefill(Q, K, V, False, tau, 1, 64, units=[(0, 0, 0)], lib_path=lib)
        np.testing.assert_allclose(d_["o"][0, 0], p_["O"][0, 0, 0], rtol=0, atol=1e-13)
        np.testing.assert_array_equal(d_["mask"][0, 0], p_["mask"][0, 0, 0])


def dec_brute(s, V, g, Ls, Bt, tau, per_head, seeded):
    """Decode decisions and output from the definition of each rule variant.

    Per head: row r of a KV group skips tile j iff its running max m_r (the
    max over the split's earlier tiles, and with seeding also over keys
    [0, Bt)) exists and the tile max is below m_r - tau.  Group rule: the tile
    is skipped iff every row of the group would skip it.  Returns the mask
    ([B,Hq,T] per head, [B,Hkv,T] group) and softmax over each row's kept keys."""
    B, Hq, L = s.shape
    T = -(-L // Bt)
    mask = np.zeros((B, Hq if per_head else Hq // g, T), np.uint8)
    keep = np.zeros_like(s, bool)
    for b in range(B):
        for kv in range(Hq // g):
            rows = s[b, kv * g:(kv + 1) * g]
            seed = rows[:, :min(Bt, L)].max(-1)
            for j in range(T):
                c0, c1 = j * Bt, min(L, j * Bt + Bt)
                split0 = (c0 // Ls) * Ls
                m = rows[:, split0:c0].max(-1) if c0 > split0 else np.full(g, -np.inf)
                if seeded:
                    m = np.maximum(m, seed)
                mt = rows[:, c0:c1].max(-1)
                row_skip = np.array([mm != -np.inf and t < mm - tau for t, mm in zip(mt, m)])
                if per_head:
                    mask[b, kv * g:(kv + 1) * g, j] = row_skip
                    for r in range(g):
                        keep[b, kv * g + r, c0:c1] = not row_skip[r]
                else:
                    mask[b, kv, j] = row_skip.all()
                    keep[b, kv * g:(kv + 1) * g, c0:c1] = not row_skip.all()
    w = np.where(keep, np.exp(s - s.max(-1, keepdims=True)), 0.0)
    v = np.repeat(f64(V), g, axis=1)
    return mask, np.einsum("bhk,bhkd->bhd", w, v) / w.sum(-1, keepdims=True)


@pin
def pin_decode_rule_variants_from_definition(lib):
    """Per-head and sink-seeded decode rules equal their definitions; the
    error bound holds per row; per-head skips a superset (per row) of the
    group rule, seeding a superset of the unseeded rule; per-head with g = 1
    and seeding with a single split change nothing."""
    q, K, V = dec_inputs(L=700)
    s = dec_scores(q, K)
    g, Bt = 2, 64
    vmax = np.abs(f64(V)).max()
    saw = {1: False, 2: False, 3: False}
    for Ls in (128, 320, 704):
        for tau in (0.0, 2.0, 6.0):
            base = oracle.decode(q, K, V, tau, Ls, Bt, lib_path=lib)
            for rule in (1, 2, 3):
                r = oracle.decode(q, K, V, tau, Ls, Bt, lib_path=lib, rule=rule)
                mask, ref = dec_brute(s, V, g, Ls, Bt, tau, rule & 1, rule & 2)
                np.testing.assert_array_equal(r["mask"], mask)
                np.testing.assert_allclose(r["o"], ref, rtol=0, atol=1e-12)
                dev = np.abs(r["o"] - r["o_exact"]).max(-1)
                assert np.all(dev <= 2 * vmax * r["pskip"] + 1e-12)
                saw[rule] |= bool((r["mask"] == 1).any())
                gm = np.repeat(base["mask"], g, axis=1) if rule & 1 else base["mask"]
                if rule in (1, 2):  # a superset of the base rule's skips
                    assert np.all(r["mask"][gm == 1] == 1)
            if Ls >= 700:  # one split: seeding changes nothing
                seeded = oracle.decode(q, K, V, tau, Ls, Bt, lib_path=lib, rule=2)
                np.testing.assert_array_equal(seeded["mask"], base["mask"])
                np.testing.assert_allclose(seeded["o"], base["o"], rtol=0, atol=1e-13)
    assert all(saw.values())
    q1, K1, V1 = dec_inputs(Hq=2, Hkv=2, L=500, seed=21)  # g = 1: per head is the group rule
    for tau in (1.0, 4.0):
        a = oracle.decode(q1, K1, V1, tau, 192, Bt, lib_path=lib)
        b_ = oracle.decode(q1, K1, V1, tau, 192, Bt, lib_path=lib, rule=1)
        np.testing.assert_array_equal(a["mask"], b_["mask"])
        np.testing.assert_allclose(a["o"], b_["o"], rtol=0, atol=1e-13)


# ----------------------------------------------------------------------------
# e4m3 quantisation (FP8 Q K^T path)
# ----------------------------------------------------------------------------

def bf16_bits(vals):
    t = torch.tensor(np.asarray(vals, np.float64)).to(torch.bfloat16)
    assert np.array_equal(t.double().numpy(), np.asarray(vals, np.float64)), "value not exact in bf16"
    return t.view(torch.int16).numpy().view(np.uint16)


@pin
def pin_e4m3_code_values(lib):
    """The 256 code values equal the library's float8_e4m3fn decoding and the
    format's fixed points: 448 the largest, 2^-9 the smallest subnormal,
    2^-6 the smallest normal, 1 and -1, the two NaNs."""
    v = oracle.e4m3_values(lib_path=lib)
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(v, ref)
    assert v[0x7E] == 448.0 and v[0x01] == 2.0 ** -9 and v[0x08] == 2.0 ** -6
    assert v[0x38] == 1.0 and v[0xB8] == -1.0 and v[0x80] == 0.0 and np.signbit(v[0x80])
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF]) and np.isfinite(np.delete(v, [0x7F, 0xFF])).all()


@pin
def pin_e4m3_rounding_and_ties(lib):
    """Codes are round-to-nearest, ties to the even mantissa, with the sign
    kept: midpoints between neighbours (normal and subnormal) go to the even
    code; random data equals the library's RNE cast of x / s."""
    # one group with max 448 (scale 1): exact midpoints and their images
    mids = [448.0, 1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, -1.0625, -(2.0 ** -10), 432.0, 13 * 2.0 ** -10]
    want = [0x7E, 0x38, 0x3A, 0x00, 0x02, 0xB8, 0x80, 0x7E, 0x06]
    codes, scales = oracle.quantize_e4m3(bf16_bits(mids), 1, lib_path=lib)
    assert scales[0] == 1.0
    assert list(codes) == want, [hex(c) for c in codes]
    g = torch.Generator().manual_seed(3)
    x = (torch.randn(12, 2048, generator=g, dtype=torch.float64)
         * torch.logspace(-6, 6, 12, base=2.0, dtype=torch.float64)[:, None]).to(torch.bfloat16)
    x[3, :100] = 0.0
    x[4, 7] = -0.0
    codes, scales = oracle.quantize_e4m3(x, 12, lib_path=lib)
    cast = (x.double() / torch.tensor(scales)[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(codes, cast)
    deq = oracle.dequantize_e4m3(codes, scales, lib_path=lib)
    v = oracle.e4m3_values(lib_path=lib)
    step = np.diff(v[:127])  # spacing above each non-negative code
    for r in range(12):  # |error| <= half the local spacing
        a = np.abs(x[r].double().numpy()) / scales[r]
        c = np.searchsorted(v[:127], a, side="right") - 1
        half = step[np.minimum(c, 125)] / 2
        assert np.all(np.abs(deq[r] - x[r].double().numpy()) <= half * scales[r] + 0.0)


@pin
def pin_e4m3_scale_rule(lib):
    """Scale = smallest power of two 2^k (k >= -126) with max|x| <= 448 * 2^k:
    exact boundaries, one bf16 step above them, zeros, tiny and non-finite
    groups; the largest code of a normal group lies in (224, 448]."""
    for k in (-20, -3, 0, 1, 7, 40):
        at = 448.0 * 2.0 ** k
        above = float(torch.tensor(at, dtype=torch.bfloat16).view(torch.int16).add(1).view(torch.bfloat16))
        c, s = oracle.quantize_e4m3(bf16_bits([at, -1.0 * 2.0 ** k, 0.0, 0.0]), 1, lib_path=lib)
        assert s[0] == 2.0 ** k and c[0] == 0x7E
        c, s = oracle.quantize_e4m3(bf16_bits([0.5 * 2.0 ** k, -above, 0.0, 0.0]), 1, lib_path=lib)
        assert above == 450.0 * 2.0 ** k
        assert s[0] == 2.0 ** (k + 1) and c[1] == 0xF6  # -225 rounds to -224 = -1.75 * 2^7 (code 0xF6)
    _, s = oracle.quantize_e4m3(bf16_bits([0.0] * 16), 2, lib_path=lib)
    assert list(s) == [1.0, 1.0]
    _, s = oracle.quantize_e4m3(bf16_bits([2.0 ** -130, 0.0, 0.0, 0.0]), 1, lib_path=lib)
    assert s[0] == 2.0 ** -126
    inf16 = torch.tensor([1.0, float("inf"), 2.0, 3.0], dtype=torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    _, s = oracle.quantize_e4m3(inf16, 2, lib_path=lib)
    assert np.isnan(s[0]) and s[1] == 2.0 ** -7
    g = torch.Generator().manual_seed(5)
    x = (torch.rand(8, 512, generator=g, dtype=torch.float64) * 1000 - 500).to(torch.bfloat16)
    codes, s = oracle.quantize_e4m3(x, 8, lib_path=lib)
    top = np.abs(oracle.e4m3_values(lib_path=lib)[codes]).max(-1)
    assert np.all((top > 224) & (top <= 448))
    assert np.all(np.abs(x.double().numpy()).max(-1) <= 448 * s)
    assert np.all(np.abs(x.double().numpy()).max(-1) > 224 * s)


@pin
def pin_i8_rounding_and_ties(lib):
    """int8 codes are the nearest integer, ties to even, sign kept; random
    data equals numpy's round-half-to-even of x / s."""
    mids = [127.0, 2.5, 3.5, -2.5, -3.5, 0.5, 1.5, -0.5, 126.5, -126.5, -127.0, 0.25]
    want = [127, 2, 4, -2, -4, 0, 2, 0, 126, -126, -127, 0]
    codes, scales = oracle.quantize_i8(bf16_bits(mids), 1, lib_path=lib)
    assert scales[0] == 1.0
    assert list(codes) == want, list(codes)
    g = torch.Generator().manual_seed(4)
    x = (torch.randn(12, 2048, generator=g, dtype=torch.float64)
         * torch.logspace(-6, 6, 12, base=2.0, dtype=torch.float64)[:, None]).to(torch.bfloat16)
    x[2, :50] = 0.0
    codes, scales = oracle.quantize_i8(x, 12, lib_path=lib)
    ref = np.rint(x.double().numpy() / scales[:, None])
    np.testing.assert_array_equal(codes.astype(np.float64), ref)
    deq = oracle.dequantize_i8(codes, scales)
    assert np.all(np.abs(deq - x.double().numpy()) <= 0.5 * scales[:, None])


@pin
def pin_i8_scale_rule(lib):
    """Scale = smallest power of two 2^k (k >= -126) with max|x| <= 127 * 2^k:
    exact boundaries and one bf16 step above them, zeros, tiny and non-finite
    groups; the largest |code| of a normal group lies in (63, 127]."""
    for k in (-20, -3, 0, 1, 7, 40):
        at = 127.0 * 2.0 ** k
        c, s = oracle.quantize_i8(bf16_bits([at, -1.0 * 2.0 ** k, 0.0, 0.0]), 1, lib_path=lib)
        assert s[0] == 2.0 ** k and c[0] == 127 and c[1] == -1
        c, s = oracle.quantize_i8(bf16_bits([0.5 * 2.0 ** k, -128.0 * 2.0 ** k, 0.0, 0.0]), 1, lib_path=lib)
        assert s[0] == 2.0 ** (k + 1) and c[1] == -64
    _, s = oracle.quantize_i8(bf16_bits([0.0] * 16), 2, lib_path=lib)
    assert list(s) == [1.0, 1.0]
    _, s = oracle.quantize_i8(bf16_bits([2.0 ** -130, 0.0, 0.0, 0.0]), 1, lib_path=lib)
    assert s[0] == 2.0 ** -126
    inf16 = torch.tensor([1.0, float("nan"), 2.0, 3.0], dtype=torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    _, s = oracle.quantize_i8(inf16, 2, lib_path=lib)
    assert np.isnan(s[0]) and s[1] == 2.0 ** -5
    g = torch.Generator().manual_seed(6)
    x = (torch.rand(8, 512, generator=g, dtype=torch.float64) * 1000 - 500).to(torch.bfloat16)
    codes, s = oracle.quantize_i8(x, 8, lib_path=lib)
    top = np.abs(codes.astype(int)).max(-1)
    assert np.all((top > 63) & (top <= 127))


@pytest.mark.parametrize("fn", PINS, ids=[f.__name__ for f in PINS])
def test_pin(fn):
    fn(None)
