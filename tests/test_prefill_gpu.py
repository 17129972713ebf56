"""GPU parity of the sm_100a prefill kernel against the fp64 oracle, called
through the C ABI (via the binding).  Rule: "Accelerating Long-Context
Inference with Skip Softmax in NVIDIA TensorRT-LLM" (Key Points; Detailed
Analysis)."""
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


def run_gpu(Q, K, V, causal, tau, Br, Bc):
    O, mask = bss.prefill(Q.cuda(), K.cuda(), V.cuda(), causal, tau, Br, Bc, skip_mask=True)
    assert bss.attn_sync_status() == 0
    return O.cpu(), mask.cpu().numpy()


def check(Q, K, V, causal, tau, Br, Bc, units=None):
    O, mask = run_gpu(Q, K, V, causal, tau, Br, Bc)
    r = oracle.prefill(Q, K, V, causal, tau, Br, Bc, units=units, want_exact=False)
    flips = compare_masks(mask, r["mask"], r["margin"])
    B, H, N, d = Q.shape
    rows = np.ones((B, H, N, 1), bool)
    fl = flips.any(-1)
    for b, h, rb in zip(*np.nonzero(fl)):     # a borderline flip changes that block's output
        rows[b, h, rb * Br:(rb + 1) * Br] = False
    compare_outputs(O, r["O"], np.broadcast_to(rows, O.shape))
    computed = r["mask"] != 255
    return float((mask[computed] == 1).mean())


# ---------------------------------------------------------------- workloads
def test_causal_1x1x256_d64_exact():
    """The smallest workload: causal, N=256, d=64, Br=Bc=64, tau=inf."""
    w = inputs.WORKLOADS["causal_1x1x256_d64"]
    Q, K, V = inputs.prefill_inputs(w["B"], w["Hq"], w["Hkv"], w["N"], w["d"], seed=0, **w["gen"])
    assert check(Q, K, V, True, math.inf, 64, 64) == 0.0


TILES = [(64, 64), (128, 64), (128, 128)]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Br,Bc", TILES)
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [300, 512])
def test_grid_exact(d, Br, Bc, causal, N):
    Q, K, V = inputs.prefill_inputs(2, 4, 2, N, d, seed=N + d + Br + Bc, q_sigma=1.5)
    assert check(Q, K, V, causal, math.inf, Br, Bc) == 0.0


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Br,Bc", TILES)
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("tau", [0.0, 2.0, 8.0])
def test_grid_skipping(d, Br, Bc, causal, tau):
    """Inputs with a strong shared direction and sink keys, so many tiles skip."""
    Q, K, V = inputs.prefill_inputs(1, 4, 2, 700, d, seed=7 + d + Br, q_sigma=2.0, q_u=8.0,
                                    sink_scale=6.0)
    frac = check(Q, K, V, causal, tau, Br, Bc)
    if tau <= 8.0:
        assert frac > 0.05


@pytest.mark.parametrize("N", [1, 7, 64, 65, 129])
def test_tiny_and_ragged(N):
    for causal in (False, True):
        Q, K, V = inputs.prefill_inputs(1, 2, 1, N, 128, seed=N, q_sigma=2.0, q_u=8.0, sink_scale=6.0)
        check(Q, K, V, causal, 1.0, 128, 64)
        check(Q, K, V, causal, math.inf, 64, 64)


def test_equal_logits_tau_zero_keeps_everything():
    """Q = 0: every tile max equals the running max, and the comparison is strict."""
    _, K, V = inputs.prefill_inputs(1, 2, 2, 512, 128, seed=3)
    Q = torch.zeros(1, 2, 512, 128, dtype=torch.bfloat16)
    for causal in (False, True):
        O, mask = run_gpu(Q, K, V, causal, 0.0, 128, 128)
        assert not (mask == 1).any()
        r = oracle.prefill(Q, K, V, causal, 0.0, 128, 128, want_exact=False)
        compare_outputs(O, r["O"])


def test_skip_mask_unvisited_tiles_marked():
    Q, K, V = inputs.prefill_inputs(1, 1, 1, 512, 64, seed=1)
    _, mask = run_gpu(Q, K, V, True, math.inf, 64, 64)
    for rb in range(8):
        assert (mask[0, 0, rb, :rb + 1] == 0).all() and (mask[0, 0, rb, rb + 1:] == 2).all()


def sampled_units(B, Hq, N, Br, n, seed):
    rng = np.random.default_rng(seed)
    n_rb = -(-N // Br)
    units = {(0, 0, 0), (B - 1, Hq - 1, n_rb - 1), (0, Hq - 1, n_rb // 2)}
    while len(units) < n:
        units.add((int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(n_rb))))
    return sorted(units)


@pytest.mark.parametrize("name", ["encoder_64x32x512_d128", "llama3_8b_causal_N8192"])
def test_full_size_workloads_sampled(name):
    """Full-size workloads, checked on a sample of row blocks (row blocks are
    independent, so each sampled block is exact)."""
    w = inputs.WORKLOADS[name]
    Q, K, V = inputs.prefill_inputs(w["B"], w["Hq"], w["Hkv"], w["N"], w["d"], seed=0, **w["gen"])
    units = sampled_units(w["B"], w["Hq"], w["N"], w["Br"], 12, seed=1)
    for tau in w["taus"]:
        check(Q, K, V, w["causal"], tau, w["Br"], w["Bc"], units=units)


def test_long_context_70b_layer_sampled():
    """N = 131072, Hq = 64, Hkv = 8 causal; Q drawn only for the sampled heads."""
    w = inputs.WORKLOADS["llama33_70b_causal_N131072"]
    B, Hq, Hkv, N, d = w["B"], w["Hq"], w["Hkv"], w["N"], w["d"]
    units = [(0, 0, 0), (0, 63, 1023), (0, 9, 517), (0, 40, 1022)]
    heads = sorted({(b, h) for b, h, _ in units})
    Q, K, V = inputs.prefill_inputs(B, Hq, Hkv, N, d, seed=0, q_heads=heads, **w["gen"])
    for tau in w["taus"]:
        check(Q, K, V, True, tau, 128, 128, units=units)
