"""The decode entry point that allocates nothing, checked against the
regular one.

Callers such as a serving engine that has reserved all of HBM for its own
pools, or a loop that must not meet cudaMalloc's implicit synchronisation,
cannot let the library allocate; attn_decode_noalloc serves them from a fixed
scratch array.  This file is collected last, so a run that stops at the first
failure has already run every other test; it also passes alone."""
import math

import numpy as np
import pytest
import torch

import block_skipping_softmax_b200 as bss
from block_skipping_softmax_b200 import build as bss_build
from block_skipping_softmax_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    bss_build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bss.lib()


def regular(q, K, V, tau):
    B, Hq, d = q.shape
    Hkv, L = K.shape[1], K.shape[2]
    o = torch.empty_like(q)
    mask = torch.empty(B, Hkv, -(-L // 64), dtype=torch.uint8, device=q.device)
    st = bss.attn_decode_ex(q.data_ptr(), K.data_ptr(), V.data_ptr(), o.data_ptr(), B, Hq, Hkv, L, d,
                            tau, torch.cuda.current_stream().cuda_stream, mask.data_ptr(), None, 0)
    assert st == 0
    return o, mask


def no_alloc(q, K, V, tau):
    B, Hq, d = q.shape
    Hkv, L = K.shape[1], K.shape[2]
    o = torch.full_like(q, float("nan"))
    mask = torch.full((B, Hkv, -(-L // 64)), 255, dtype=torch.uint8, device=q.device)
    st = bss.attn_decode_noalloc(q.data_ptr(), K.data_ptr(), V.data_ptr(), o.data_ptr(), B, Hq, Hkv, L,
                                 d, tau, torch.cuda.current_stream().cuda_stream, mask.data_ptr())
    assert st == 0, bss.attn_status_string(st)
    return o, mask


def test_no_alloc_matches_regular_entry_point_twice():
    cases = [
        (inputs.decode_inputs(4, 32, 8, 9000, 128, seed=21, q_sigma=2.0, q_u=8.0, sink_scale=6.0), 2.0),
        (inputs.decode_inputs(2, 8, 8, 3001, 64, seed=22, q_sigma=2.0, q_u=1.0, sink_scale=3.0), math.inf),
    ]
    for (q, K, V), tau in cases:  # two calls in a row, different shapes: no stale state
        q, K, V = q.cuda(), K.cuda(), V.cuda()
        o_ref, m_ref = regular(q, K, V, tau)
        o_new, m_new = no_alloc(q, K, V, tau)
        torch.cuda.synchronize()
        assert bss.attn_sync_status() == 0
        np.testing.assert_array_equal(m_new.cpu().numpy(), m_ref.cpu().numpy())
        # the same kernels over the same split layout: bit-identical outputs
        assert torch.equal(o_new, o_ref), "no-alloc decode differs from attn_decode_ex"
