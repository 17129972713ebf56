"""Guard bands around every output: the kernels write exactly their outputs.

O and the skip masks are placed inside larger device buffers whose margins
hold a fixed byte pattern.  After each call the margins must be unchanged,
and the guarded outputs must equal those of an ordinary call bit for bit.
Shapes are ragged (N and L not multiples of the tiles), so the last row
block, the last key tile and the TMA-store epilogue's clipping are all at the
edge of their buffers."""
import math

import numpy as np
import pytest
import torch

import block_skipping_softmax_b200 as bss
from block_skipping_softmax_b200 import build as bss_build
from block_skipping_softmax_b200 import inputs

pytestmark = pytest.mark.gpu
GUARD = 4096  # bytes on each side (a multiple of 16 keeps the outputs aligned)
PATTERN = 0xA5


@pytest.fixture(scope="module", autouse=True)
def lib():
    bss_build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bss.lib()


class Guarded:
    """A device byte buffer with guard bands; .inner is the usable region."""

    def __init__(self, nbytes):
        self.n = nbytes
        self.buf = torch.full((nbytes + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.inner = self.buf[GUARD:GUARD + nbytes]

    def ptr(self):
        return self.inner.data_ptr()

    def intact(self):
        b = self.buf.cpu().numpy()
        return bool((b[:GUARD] == PATTERN).all() and (b[GUARD + self.n:] == PATTERN).all())


@pytest.mark.parametrize("Br,Bc", [(128, 64), (128, 128), (64, 64)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("tau", [math.inf, 2.0])
def test_prefill_writes_only_its_outputs(Br, Bc, causal, tau):
    B, Hq, Hkv, N, d = 2, 4, 2, 333, 128
    Q, K, V = inputs.prefill_inputs(B, Hq, Hkv, N, d, seed=41, q_sigma=2.0, q_u=8.0, sink_scale=6.0)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    ref_o, ref_m = bss.prefill(Qd, Kd, Vd, causal, tau, Br, Bc, skip_mask=True)
    n_rb, n_t = -(-N // Br), -(-N // Bc)
    go = Guarded(B * Hq * N * d * 2)
    gm = Guarded(B * Hq * n_rb * n_t)
    st = bss.attn_prefill_ex(Qd.data_ptr(), Kd.data_ptr(), Vd.data_ptr(), go.ptr(), B, Hq, Hkv, N, d,
                             causal, tau, Br, Bc, torch.cuda.current_stream().cuda_stream, gm.ptr())
    assert st == 0
    assert bss.attn_sync_status() == 0
    assert go.intact() and gm.intact()
    assert torch.equal(go.inner.view(torch.bfloat16).view(B, Hq, N, d), ref_o)
    assert torch.equal(gm.inner.view(B, Hq, n_rb, n_t), ref_m)


@pytest.mark.parametrize("int8", [False, True])
@pytest.mark.parametrize("Bc", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_prefill_qk8_writes_only_its_outputs(Bc, causal, int8):
    B, Hq, Hkv, N, d = 2, 4, 2, 333, 128
    Q, K, V = inputs.prefill_inputs(B, Hq, Hkv, N, d, seed=53, q_sigma=2.0, q_u=8.0, sink_scale=6.0)
    quant = bss.quantize_i8 if int8 else bss.quantize_e4m3
    Q8, qs = quant(Q.cuda())
    K8, ks = quant(K.cuda())
    Vd = V.cuda()
    run = bss.prefill_qki8 if int8 else bss.prefill_qk8
    ref_o, ref_m = run(Q8, K8, qs, ks, Vd, causal, 2.0, 128, Bc, skip_mask=True)
    n_rb, n_t = -(-N // 128), -(-N // Bc)
    go = Guarded(B * Hq * N * d * 2)
    gm = Guarded(B * Hq * n_rb * n_t)
    raw = bss.attn_prefill_qki8 if int8 else bss.attn_prefill_qk8
    st = raw(Q8.data_ptr(), K8.data_ptr(), qs.data_ptr(), ks.data_ptr(), Vd.data_ptr(),
             go.ptr(), B, Hq, Hkv, N, d, causal, 2.0, 128, Bc,
             torch.cuda.current_stream().cuda_stream, gm.ptr())
    assert st == 0
    assert bss.attn_sync_status() == 0
    assert go.intact() and gm.intact()
    assert torch.equal(go.inner.view(torch.bfloat16).view(B, Hq, N, d), ref_o)
    assert torch.equal(gm.inner.view(B, Hq, n_rb, n_t), ref_m)


def test_quantize_writes_only_its_outputs():
    x = torch.randn(2, 3, 333, 128, dtype=torch.float32).to(torch.bfloat16).cuda()
    ref_q, ref_s = bss.quantize_e4m3(x)
    gq = Guarded(x.numel())
    gs = Guarded(2 * 3 * 4)
    st = bss.attn_quantize_e4m3(x.data_ptr(), gq.ptr(), gs.ptr(), 6, 333 * 128,
                                torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    assert gq.intact() and gs.intact()
    assert torch.equal(gq.inner.view(2, 3, 333, 128), ref_q)
    assert torch.equal(gs.inner.view(torch.float32).view(2, 3), ref_s)


@pytest.mark.parametrize("rule", [0, 1, 2, 3])
def test_decode_writes_only_its_outputs(rule):
    B, Hq, Hkv, L, d = 3, 8, 2, 1999, 128
    q, K, V = inputs.decode_inputs(B, Hq, Hkv, L, d, seed=43, q_sigma=2.0, q_u=8.0, sink_scale=6.0)
    qd, Kd, Vd = q.cuda(), K.cuda(), V.cuda()
    ref_o, ref_m = bss.decode(qd, Kd, Vd, 2.0, skip_mask=True, rule=rule)
    rows = Hq if rule & bss.RULE_PER_HEAD else Hkv
    n_t = -(-L // 64)
    go = Guarded(B * Hq * d * 2)
    gm = Guarded(B * rows * n_t)
    st = bss.attn_decode_rule(qd.data_ptr(), Kd.data_ptr(), Vd.data_ptr(), go.ptr(), B, Hq, Hkv, L, d,
                              2.0, rule, torch.cuda.current_stream().cuda_stream, gm.ptr())
    assert st == 0
    assert bss.attn_sync_status() == 0
    assert go.intact() and gm.intact()
    assert torch.equal(go.inner.view(torch.bfloat16).view(B, Hq, d), ref_o)
    assert torch.equal(gm.inner.view(B, rows, n_t), ref_m)


def test_paged_decode_writes_only_its_outputs():
    B, Hq, Hkv, d = 3, 8, 2, 128
    lens = [1, 700, 1999]
    L = max(lens)
    q, K, V = inputs.decode_inputs(B, Hq, Hkv, L, d, seed=47, q_sigma=2.0, q_u=8.0, sink_scale=6.0)
    npg = -(-L // 64)
    Kp = torch.zeros(B * npg, Hkv, 64, d, dtype=torch.bfloat16)
    Vp = torch.zeros(B * npg, Hkv, 64, d, dtype=torch.bfloat16)
    for b in range(B):
        for t in range(npg):
            k0, k1 = t * 64, min(L, t * 64 + 64)
            Kp[b * npg + t, :, :k1 - k0] = K[b, :, k0:k1]
            Vp[b * npg + t, :, :k1 - k0] = V[b, :, k0:k1]
    table = torch.arange(B * npg, dtype=torch.int32).view(B, npg).cuda()
    sl = torch.tensor(lens, dtype=torch.int32).cuda()
    qd, Kpd, Vpd = q.cuda(), Kp.cuda(), Vp.cuda()
    ref_o, ref_m = bss.decode_paged(qd, Kpd, Vpd, table, sl, L, 2.0, skip_mask=True)
    go = Guarded(B * Hq * d * 2)
    gm = Guarded(B * Hkv * npg)
    st = bss.attn_decode_paged(qd.data_ptr(), Kpd.data_ptr(), Vpd.data_ptr(), table.data_ptr(), sl.data_ptr(),
                               go.ptr(), B, Hq, Hkv, B * npg, npg, L, d, 2.0, 0,
                               torch.cuda.current_stream().cuda_stream, gm.ptr())
    assert st == 0
    assert bss.attn_sync_status() == 0
    assert go.intact() and gm.intact()
    assert torch.equal(go.inner.view(torch.bfloat16).view(B, Hq, d), ref_o)
    assert torch.equal(gm.inner.view(B, Hkv, npg), ref_m)
    assert (ref_m[0, :, 1:] == 2).all().item()
