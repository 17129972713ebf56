"""Variable-length (packed) prefill against the fp64 oracle, sequence by
sequence: every sequence attends only to itself, O rows outside every
sequence stay untouched, and skip masks match the oracle's (2 past each
sequence's end)."""
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
SENTINEL = 0x7E7E  # bf16 bit pattern of a large finite value


@pytest.fixture(scope="module", autouse=True)
def lib():
    bss_build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bss.lib()


def packed(lens, Hq, Hkv, d, seed, gap=0):
    """Per-sequence inputs (BHND, for the oracle) and their packed THD form,
    sequences back to back after `gap` unowned tokens, with `gap` more after
    the last one."""
    seqs = [inputs.prefill_inputs(1, Hq, Hkv, n, d, seed=seed + i, q_sigma=2.0, q_u=8.0, sink_scale=6.0)
            for i, n in enumerate(lens)]
    starts = [gap + sum(lens[:i]) for i in range(len(lens))]
    total = gap + sum(lens) + gap
    Q = torch.zeros(total, Hq, d, dtype=torch.bfloat16)
    K = torch.zeros(total, Hkv, d, dtype=torch.bfloat16)
    V = torch.zeros(total, Hkv, d, dtype=torch.bfloat16)
    for (q, k, v), s0, n in zip(seqs, starts, lens):
        Q[s0:s0 + n] = q[0].transpose(0, 1)
        K[s0:s0 + n] = k[0].transpose(0, 1)
        V[s0:s0 + n] = v[0].transpose(0, 1)
    cu_t = torch.tensor(starts + [starts[-1] + lens[-1]], dtype=torch.int32)
    return seqs, Q, K, V, cu_t, starts


@pytest.mark.parametrize("Bc", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("tau", [math.inf, 2.0])
def test_varlen_matches_per_sequence_oracle(Bc, causal, tau):
    lens = [1, 100, 128, 129, 300, 513, 1000]
    Hq, Hkv, d = 4, 2, 128
    seqs, Q, K, V, cu, starts = packed(lens, Hq, Hkv, d, seed=3, gap=7)
    O = torch.empty_like(Q).view(torch.int16).fill_(SENTINEL).view(torch.bfloat16).cuda()
    O, mask = bss.prefill_varlen(Q.cuda(), K.cuda(), V.cuda(), cu.cuda(), max(lens), causal, tau, 128, Bc,
                                 out=O, skip_mask=True)
    assert bss.attn_sync_status() == 0
    O, mask = O.cpu(), mask.cpu().numpy()
    owned = np.zeros(O.shape[0], bool)
    for i, ((q, k, v), s0, n) in enumerate(zip(seqs, starts, lens)):
        owned[s0:s0 + n] = True
        r = oracle.prefill(q, k, v, causal, tau, 128, Bc, want_exact=False)
        n_rb, n_t = r["mask"].shape[2], r["mask"].shape[3]
        flips = compare_masks(mask[i:i + 1, :, :n_rb, :n_t], r["mask"], r["margin"])
        assert (mask[i, :, n_rb:] == 2).all() and (mask[i, :, :, n_t:] == 2).all()
        rows = np.ones((1, Hq, n, 1), bool)
        for h, rb in zip(*np.nonzero(flips[0].any(-1))):
            rows[0, h, rb * 128:(rb + 1) * 128] = False
        got = O[s0:s0 + n].transpose(0, 1).unsqueeze(0)
        compare_outputs(got, r["O"], np.broadcast_to(rows, r["O"].shape))
    untouched = O[~torch.from_numpy(owned)].view(torch.int16)
    assert (untouched == SENTINEL).all(), "rows outside every sequence were written"


def test_varlen_d64_gqa8_and_bad_arguments():
    lens = [64, 200, 77]
    seqs, Q, K, V, cu, starts = packed(lens, 8, 1, 64, seed=9)
    O = bss.prefill_varlen(Q.cuda(), K.cuda(), V.cuda(), cu.cuda(), max(lens), True, math.inf, 128, 64)
    assert bss.attn_sync_status() == 0
    for (q, k, v), s0, n in zip(seqs, starts, lens):
        r = oracle.prefill(q, k, v, True, math.inf, 128, 64, want_exact=False)
        compare_outputs(O[s0:s0 + n].cpu().transpose(0, 1).unsqueeze(0), r["O"])
    Qd = Q.cuda()
    args = (Qd.data_ptr(), K.cuda().data_ptr(), V.cuda().data_ptr(), Qd.data_ptr(), cu.cuda().data_ptr(),
            3, 200, Q.shape[0], 8, 1, 64, 1, 1.0)
    assert bss.attn_prefill_varlen(*args, 64, 64) == 1       # Br must be 128
    assert bss.attn_prefill_varlen(*args[:4], None, *args[5:], 128, 64) == 1
