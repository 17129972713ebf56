"""GPU parity of the prefill path whose exponentials are partly computed by
the FMA-pipe polynomial (attn_prefill_poly), against the fp64 oracle at the
same bar as the MUFU path.  The polynomial follows the SAS idea of
"TurboAttention: Efficient Attention Approximation for High-Throughput LLM
Serving" (Technical Deep Dive: SAS); the skip rule is the one of
"Accelerating Long-Context Inference with Skip Softmax in NVIDIA
TensorRT-LLM" (Key Points; Detailed Analysis)."""
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


def check(Q, K, V, causal, tau, poly_pairs):
    O, mask = bss.prefill_poly(Q.cuda(), K.cuda(), V.cuda(), causal, tau, poly_pairs, skip_mask=True)
    assert bss.attn_sync_status() == 0
    O, mask = O.cpu(), mask.cpu().numpy()
    r = oracle.prefill(Q, K, V, causal, tau, 128, 128, want_exact=False)
    flips = compare_masks(mask, r["mask"], r["margin"])
    B, H, N, d = Q.shape
    rows = np.ones((B, H, N, 1), bool)
    for b, h, rb in zip(*np.nonzero(flips.any(-1))):  # a borderline flip changes that block's output
        rows[b, h, rb * 128:(rb + 1) * 128] = False
    compare_outputs(O, r["O"], np.broadcast_to(rows, O.shape), what=f"O (poly {poly_pairs}/16)")
    return float((mask[r["mask"] != 255] == 1).mean())


@pytest.mark.parametrize("poly_pairs", [4, 8])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [128, 300, 517])
def test_poly_grid_exact(poly_pairs, causal, N):
    """tau = inf over several tiles with a ragged last tile, GQA, d = 128."""
    Q, K, V = inputs.prefill_inputs(2, 4, 2, N, 128, seed=N + poly_pairs, q_sigma=2.0, q_u=1.0,
                                    sink_scale=3.0)
    assert check(Q, K, V, causal, math.inf, poly_pairs) == 0.0


@pytest.mark.parametrize("poly_pairs", [4, 8])
@pytest.mark.parametrize("tau", [2.0, 4.0])
def test_poly_with_skipping(poly_pairs, tau):
    """Strong sinks make the every-row rule skip tiles; masks and outputs
    match the oracle with the polynomial exponentials as well."""
    Q, K, V = inputs.prefill_inputs(1, 4, 1, 1000, 128, seed=41, q_sigma=2.0, q_u=8.0, sink_scale=6.0)
    assert check(Q, K, V, True, tau, poly_pairs) > 0.0


def test_poly_zero_equals_mufu_path_bit_for_bit():
    """poly_pairs = 0 computes every exponential on MUFU: the same kernel as
    attn_prefill_ex at d = Bc = 128."""
    Q, K, V = (t.cuda() for t in inputs.prefill_inputs(1, 4, 2, 700, 128, seed=5, q_sigma=2.0, q_u=1.0,
                                                         sink_scale=3.0))
    a = bss.prefill(Q, K, V, True, 4.0, 128, 128)
    b = bss.prefill_poly(Q, K, V, True, 4.0, 0)
    assert bss.attn_sync_status() == 0
    assert torch.equal(a, b)


def test_poly_rejects_other_shapes():
    Q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16, device="cuda")
    st = bss.attn_prefill_poly(Q.data_ptr(), Q.data_ptr(), Q.data_ptr(), Q.data_ptr(), 1, 1, 1, 128, 64,
                               0, math.inf, 128, 128, 4)
    assert st == 1
    Q = torch.zeros(1, 1, 128, 128, dtype=torch.bfloat16, device="cuda")
    for pairs in (3, 16, -4):
        st = bss.attn_prefill_poly(Q.data_ptr(), Q.data_ptr(), Q.data_ptr(), Q.data_ptr(), 1, 1, 1, 128,
                                   128, 0, math.inf, 128, 128, pairs)
        assert st == 1
    st = bss.attn_prefill_poly(Q.data_ptr(), Q.data_ptr(), Q.data_ptr(), Q.data_ptr(), 1, 1, 1, 128, 128,
                               0, math.inf, 128, 64, 4)
    assert st == 1
