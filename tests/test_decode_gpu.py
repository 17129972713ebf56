"""GPU parity of the split-KV decode kernels against the fp64 oracle, called
through the C ABI.  The split length is part of the op's definition (the
running max restarts at every split) and is read from the library's host
function attn_decode_split_len, a pure function of (B, Hkv, L)."""
import math

import numpy as np
import pytest
import torch

import block_skipping_softmax_b200 as bss
import oracle
from block_skipping_softmax_b200 import build as bss_build
from block_skipping_softmax_b200 import inputs
from parity import compare_masks, compare_outputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    bss_build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bss.lib()


def check(q, K, V, tau, batches=None):
    B, Hq, d = q.shape
    Hkv, L = K.shape[1], K.shape[2]
    o, mask = bss.decode(q.cuda(), K.cuda(), V.cuda(), tau, skip_mask=True)
    assert bss.attn_sync_status() == 0
    o, mask = o.cpu(), mask.cpu().numpy()
    Ls = bss.attn_decode_split_len(B, Hkv, L)
    sel = list(range(B)) if batches is None else list(batches)
    r = oracle.decode(q[sel], K[sel], V[sel], tau, Ls, 64, want_exact=False)
    flips = compare_masks(mask[sel], r["mask"], r["margin"])
    g = Hq // Hkv
    rows = np.ones((len(sel), Hq, 1), bool)
    for b, kv in zip(*np.nonzero(flips.any(-1))):
        rows[b, kv * g:(kv + 1) * g] = False
    compare_outputs(o[sel], r["o"], np.broadcast_to(rows, r["o"].shape))
    return float((mask[sel] == 1).mean())


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("g", [1, 2, 4, 8])
@pytest.mark.parametrize("L", [1, 63, 64, 65, 1000, 5000])
def test_grid_exact(d, g, L):
    q, K, V = inputs.decode_inputs(2, 2 * g, 2, L, d, seed=L + g + d, q_sigma=2.0, q_u=1.0,
                                   sink_scale=3.0)
    assert check(q, K, V, math.inf) == 0.0


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("g", [1, 4, 8])
@pytest.mark.parametrize("tau", [0.0, 2.0, 6.0])
def test_grid_skipping(d, g, tau):
    q, K, V = inputs.decode_inputs(3, 2 * g, 2, 4000, d, seed=5 + g, q_sigma=2.0, q_u=8.0,
                                   sink_scale=6.0)
    frac = check(q, K, V, tau)
    assert frac > 0.0


def test_gqa_decode_full_size_sampled_batches():
    """B=16, Hq=32, Hkv=8, L=32768, d=128 in the launch configuration the
    bench times; batches 0 and 15 checked against the oracle."""
    w = inputs.WORKLOADS["gqa_decode_16x32q8kv_L32768"]
    q, K, V = inputs.decode_inputs(w["B"], w["Hq"], w["Hkv"], w["L"], w["d"], seed=0, **w["gen"])
    for tau in w["taus"]:
        check(q, K, V, tau, batches=[0, 15])


def test_caller_workspace_matches_library_workspace():
    q, K, V = inputs.decode_inputs(2, 8, 2, 3000, 128, seed=9, q_sigma=2.0, q_u=8.0, sink_scale=6.0)
    qd, Kd, Vd = q.cuda(), K.cuda(), V.cuda()
    n = bss.attn_decode_workspace_bytes(2, 8, 2, 3000, 128)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    a = bss.decode(qd, Kd, Vd, 2.0)
    b = bss.decode(qd, Kd, Vd, 2.0, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# ---------------------------------------------------------------- rule variants

def check_rule(q, K, V, tau, rule, batches=None):
    """GPU decode with a rule variant against the oracle with the same rule."""
    B, Hq, d = q.shape
    Hkv, L = K.shape[1], K.shape[2]
    g = Hq // Hkv
    o, mask = bss.decode(q.cuda(), K.cuda(), V.cuda(), tau, skip_mask=True, rule=rule)
    assert bss.attn_sync_status() == 0
    o, mask = o.cpu(), mask.cpu().numpy()
    Ls = bss.attn_decode_split_len(B, Hkv, L)
    sel = list(range(B)) if batches is None else list(batches)
    r = oracle.decode(q[sel], K[sel], V[sel], tau, Ls, 64, want_exact=False, rule=rule)
    assert mask[sel].shape == r["mask"].shape
    flips = compare_masks(mask[sel], r["mask"], r["margin"])
    rows = np.ones((len(sel), Hq, 1), bool)
    for b, x in zip(*np.nonzero(flips.any(-1))):  # a borderline flip only moves its own rows
        if rule & bss.RULE_PER_HEAD:
            rows[b, x] = False
        else:
            rows[b, x * g:(x + 1) * g] = False
    compare_outputs(o[sel], r["o"], np.broadcast_to(rows, r["o"].shape))
    return float((mask[sel] == 1).mean())


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("g", [1, 4, 8])
@pytest.mark.parametrize("tau", [0.0, 2.0, 6.0])
def test_rule_variants_skipping(d, g, tau):
    # 4000 keys in splits of 512: seeding matters for every split but the first
    q, K, V = inputs.decode_inputs(3, 2 * g, 2, 4000, d, seed=5 + g, q_sigma=2.0, q_u=8.0,
                                   sink_scale=6.0)
    base = check_rule(q, K, V, tau, bss.RULE_GROUP)
    per_head = check_rule(q, K, V, tau, bss.RULE_PER_HEAD)
    seeded = check_rule(q, K, V, tau, bss.RULE_SINK_SEED)
    both = check_rule(q, K, V, tau, bss.RULE_PER_HEAD | bss.RULE_SINK_SEED)
    assert seeded >= base and both >= per_head >= base - 1e-9


def test_rule_variants_exact_and_invalid():
    q, K, V = inputs.decode_inputs(2, 8, 2, 3000, 128, seed=3, q_sigma=2.0, q_u=1.0, sink_scale=3.0)
    for rule in (1, 2, 3):
        assert check_rule(q, K, V, math.inf, rule) == 0.0
    qd, Kd, Vd = q.cuda(), K.cuda(), V.cuda()
    o = torch.empty_like(qd)
    assert bss.attn_decode_rule(qd.data_ptr(), Kd.data_ptr(), Vd.data_ptr(), o.data_ptr(), 2, 8, 2,
                                3000, 128, 2.0, 4) == 1  # unknown rule bit


def test_rule_variants_full_size_sampled_batches():
    """The GQA decode workload with each rule variant at tau = 4 and 2."""
    w = inputs.WORKLOADS["gqa_decode_16x32q8kv_L32768"]
    q, K, V = inputs.decode_inputs(w["B"], w["Hq"], w["Hkv"], w["L"], w["d"], seed=0, **w["gen"])
    for tau in (2.0, 4.0):
        for rule in (1, 2, 3):
            check_rule(q, K, V, tau, rule, batches=[0, 15])
