"""GPU parity of the 8-bit quantisers and of the 8-bit Q K^T prefill paths
(e4m3 on kind::f8f6f4 MMAs, signed int8 on kind::i8 MMAs).

The quantisers must match the oracle's bit for bit (codes and scales).  The
prefill with 8-bit Q and K is attention over the dequantised tensors, which
are exact in bf16 (power-of-two scales, three-bit mantissas or 7-bit
integers): the oracle's
own quantisation of the seeded inputs, dequantised, is fed to the fp64
prefill oracle and the GPU result must meet the usual bar (tolerances and
skip-mask agreement as in the bf16 prefill tests).  Rule: "Accelerating
Long-Context Inference with Skip Softmax in NVIDIA TensorRT-LLM" (Key Points;
Detailed Analysis)."""
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


# format -> (GPU quantiser, GPU prefill, oracle quantiser, oracle dequantiser)
FORMATS = {
    "e4m3": (lambda x: bss.quantize_e4m3(x), bss.prefill_qk8, oracle.quantize_e4m3,
             lambda c, s: oracle.dequantize_e4m3(c, s)),
    "i8": (lambda x: bss.quantize_i8(x), bss.prefill_qki8, oracle.quantize_i8, oracle.dequantize_i8),
}


def oracle_dequant_bf16(x, heads=None, fmt="e4m3"):
    """The oracle's quantisation of x [B,H,N,d] (optionally of some (b, h)
    slabs only, the rest left as they are), dequantised; exact in bf16."""
    _, _, oq, odq = FORMATS[fmt]
    B, H, N, d = x.shape
    out = x.clone()
    codes = {}
    for b, h in (heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]):
        c, s = oq(x[b, h], 1)
        deq = odq(c, s)
        t = torch.from_numpy(deq).to(torch.bfloat16)
        assert np.array_equal(t.double().numpy(), deq), "dequantised value not exact in bf16"
        out[b, h] = t
        codes[(b, h)] = (c, s[0])
    return out, codes


def gpu_quant(x, fmt="e4m3"):
    q, s = FORMATS[fmt][0](x.cuda())
    torch.cuda.synchronize()
    return q.cpu().numpy(), s.cpu().double().numpy()


def assert_codes_equal(gq, gs, codes):
    for (b, h), (c, s) in codes.items():
        assert gs[b, h] == s, f"scale of head ({b}, {h}): {gs[b, h]} vs {s}"
        np.testing.assert_array_equal(gq[b, h], c)


def check(Q, K, V, causal, tau, Bc, units=None, q_heads=None, fmt="e4m3"):
    gq, gp, _, _ = FORMATS[fmt]
    Q8, qs = gq(Q.cuda())
    K8, ks = gq(K.cuda())
    O, mask = gp(Q8, K8, qs, ks, V.cuda(), causal, tau, 128, Bc, skip_mask=True)
    assert bss.attn_sync_status() == 0
    O, mask = O.cpu(), mask.cpu().numpy()
    Qd, qc = oracle_dequant_bf16(Q, q_heads, fmt)
    Kd, kc = oracle_dequant_bf16(K, None, fmt)
    assert_codes_equal(Q8.cpu().numpy(), qs.cpu().double().numpy(), qc)
    assert_codes_equal(K8.cpu().numpy(), ks.cpu().double().numpy(), kc)
    r = oracle.prefill(Qd, Kd, V, causal, tau, 128, Bc, units=units, want_exact=False)
    flips = compare_masks(mask, r["mask"], r["margin"])
    B, H, N, d = Q.shape
    rows = np.ones((B, H, N, 1), bool)
    for b, h, rb in zip(*np.nonzero(flips.any(-1))):
        rows[b, h, rb * 128:(rb + 1) * 128] = False
    compare_outputs(O, r["O"], np.broadcast_to(rows, O.shape))
    computed = r["mask"] != 255
    return float((mask[computed] == 1).mean())


# ------------------------------------------------------------- quantiser
@pytest.mark.parametrize("fmt", sorted(FORMATS))
@pytest.mark.parametrize("shape", [(2, 4, 333, 128), (1, 3, 1, 16), (3, 2, 4096, 64)])
def test_quantize_matches_oracle_bitwise(shape, fmt):
    B, H, N, d = shape
    g = torch.Generator().manual_seed(N + d)
    x = torch.randn(shape, generator=g, dtype=torch.float64)
    x *= torch.logspace(-20, 20, B * H, base=2.0, dtype=torch.float64).view(B, H, 1, 1)
    x = x.to(torch.bfloat16)
    gq, gs = gpu_quant(x, fmt)
    _, codes = oracle_dequant_bf16(x, None, fmt)
    assert_codes_equal(gq, gs, codes)


def test_quantize_i8_special_groups():
    """int8: a zero head, a head at an exact 127 * 2^k boundary, tiny values,
    exact ties (2.5 -> 2, 3.5 -> 4, -2.5 -> -2)."""
    x = torch.zeros(1, 4, 64, 16, dtype=torch.float64)
    x[0, 1] = torch.linspace(-3, 3, 1024).view(64, 16) * 2.0 ** -4
    x[0, 1, 0, 0] = 127 * 2.0 ** -4
    x[0, 2] = torch.linspace(-1, 1, 1024).view(64, 16) * 2.0 ** -125
    x[0, 3, :, :4] = 2.5
    x[0, 3, :, 4:8] = 3.5
    x[0, 3, :, 8:] = -2.5
    x[0, 3, 0, 0] = 127.0
    x = x.to(torch.bfloat16)
    gq, gs = gpu_quant(x, "i8")
    _, codes = oracle_dequant_bf16(x, None, "i8")
    assert_codes_equal(gq, gs, codes)
    assert gs[0, 0] == 1.0 and gs[0, 1] == 2.0 ** -4 and gs[0, 2] == 2.0 ** -126
    assert (gq[0, 3, 1:, :4] == 2).all() and (gq[0, 3, :, 4:8] == 4).all() and (gq[0, 3, :, 8:] == -2).all()


def test_quantize_special_groups():
    """A zero head (scale 1), a head at an exact 448 * 2^k boundary, a head of
    tiny values (scale held at 2^-126), negative zeros and exact midpoints."""
    x = torch.zeros(1, 4, 64, 16, dtype=torch.float64)
    x[0, 1] = torch.linspace(-3, 3, 1024).view(64, 16) * 2.0 ** -4
    x[0, 1, 0, 0] = 448 * 2.0 ** -4
    x[0, 2] = torch.linspace(-1, 1, 1024).view(64, 16) * 2.0 ** -125
    x[0, 3, :, :8] = 1.0625  # ties between 1 and 1.125
    x[0, 3, :, 8:] = -0.0
    x[0, 3, 0, 0] = 448.0
    x = x.to(torch.bfloat16)
    gq, gs = gpu_quant(x)
    _, codes = oracle_dequant_bf16(x)
    assert_codes_equal(gq, gs, codes)
    assert gs[0, 0] == 1.0 and gs[0, 1] == 2.0 ** -4 and gs[0, 2] == 2.0 ** -126
    assert (gq[0, 3, 1:, :8] == 0x38).all() and (gq[0, 3, :, 8:] == 0x80).all()


def test_quantize_rejects_bad_arguments():
    x = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    q = torch.empty(64, dtype=torch.uint8, device="cuda")
    s = torch.empty(4, dtype=torch.float32, device="cuda")
    assert bss.attn_quantize_e4m3(x.data_ptr(), q.data_ptr(), s.data_ptr(), 4, 15) == 1  # not x16
    assert bss.attn_quantize_e4m3(x.data_ptr(), q.data_ptr(), s.data_ptr(), 0, 16) == 1
    assert bss.attn_quantize_e4m3(x.data_ptr() + 2, q.data_ptr(), s.data_ptr(), 2, 16) == 1
    assert bss.attn_quantize_e4m3(None, q.data_ptr(), s.data_ptr(), 4, 16) == 1


# ------------------------------------------------------------- prefill
@pytest.mark.parametrize("fmt", sorted(FORMATS))
@pytest.mark.parametrize("Bc", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [300, 512])
def test_qk8_grid_exact(Bc, causal, N, fmt):
    Q, K, V = inputs.prefill_inputs(2, 4, 2, N, 128, seed=N + Bc + 5, q_sigma=1.5)
    assert check(Q, K, V, causal, math.inf, Bc, fmt=fmt) == 0.0


@pytest.mark.parametrize("fmt", sorted(FORMATS))
@pytest.mark.parametrize("Bc", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("tau", [0.0, 2.0, 8.0])
def test_qk8_grid_skipping(Bc, causal, tau, fmt):
    """Inputs with a strong shared direction and sink keys, so many tiles skip."""
    Q, K, V = inputs.prefill_inputs(1, 4, 2, 700, 128, seed=17 + Bc, q_sigma=2.0, q_u=8.0,
                                    sink_scale=6.0)
    assert check(Q, K, V, causal, tau, Bc, fmt=fmt) > 0.05


@pytest.mark.parametrize("fmt", sorted(FORMATS))
@pytest.mark.parametrize("N", [1, 7, 129])
def test_qk8_tiny_and_ragged(N, fmt):
    Q, K, V = inputs.prefill_inputs(1, 2, 1, N, 128, seed=N)
    for causal in (False, True):
        check(Q, K, V, causal, 4.0, 128, fmt=fmt)


def test_qk8_rejects_unsupported():
    Q8 = torch.zeros(1, 1, 128, 64, dtype=torch.uint8, device="cuda")
    s = torch.ones(1, 1, dtype=torch.float32, device="cuda")
    V = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16, device="cuda")
    O = torch.empty_like(V)
    st = bss.attn_prefill_qk8(Q8.data_ptr(), Q8.data_ptr(), s.data_ptr(), s.data_ptr(), V.data_ptr(),
                              O.data_ptr(), 1, 1, 1, 128, 64, 0, math.inf, 128, 128)  # d = 64
    assert st == 1
    st = bss.attn_prefill_qk8(Q8.data_ptr(), Q8.data_ptr(), None, s.data_ptr(), V.data_ptr(),
                              O.data_ptr(), 1, 1, 1, 128, 128, 0, math.inf, 128, 128)
    assert st == 1


@pytest.mark.parametrize("fmt", sorted(FORMATS))
def test_qk8_llama3_8b_layer_sampled(fmt):
    """The 8B causal layer (N = 8192, 32 query / 8 KV heads) at full size,
    checked on sampled row blocks; codes checked on the sampled Q heads and
    every K head."""
    w = inputs.WORKLOADS["llama3_8b_causal_N8192"]
    Q, K, V = inputs.prefill_inputs(w["B"], w["Hq"], w["Hkv"], w["N"], w["d"], seed=0, **w["gen"])
    rng = np.random.default_rng(2)
    n_rb = w["N"] // 128
    units = sorted({(0, 0, 0), (0, 31, n_rb - 1)} |
                   {(0, int(rng.integers(32)), int(rng.integers(n_rb))) for _ in range(6)})
    heads = sorted({(b, h) for b, h, _ in units})
    for tau in (math.inf, 4.0):
        check(Q, K, V, True, tau, 128, units=units, q_heads=heads, fmt=fmt)
