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
from parity import compare_masks, compare_outputs

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
        compare_outputs(o_new.cpu(), o_ref.float().cpu().double().numpy(), what="o (no-alloc)")


def test_no_alloc_rejects_problems_beyond_its_array():
    """A problem whose split scratch exceeds the fixed 16 MiB array is refused.

    The buffers are real and sized for the problem, and the test first checks
    from the split layout that the scratch really exceeds the array, so the
    call cannot reach a kernel with memory it does not own."""
    B, Hq, Hkv, L, d = 512, 64, 8, 64, 128
    ls = bss.attn_decode_split_len(B, Hkv, L)
    n_splits = -(-L // ls)
    r256 = lambda x: (x + 255) // 256 * 256
    need = r256(B * Hq * n_splits * d * 4) + r256(B * Hq * n_splits * 4)
    assert need > 16 << 20, "shape must exceed the no-alloc scratch array"
    q = torch.zeros(B, Hq, d, dtype=torch.bfloat16, device="cuda")
    K = torch.zeros(B, Hkv, L, d, dtype=torch.bfloat16, device="cuda")
    V = torch.zeros_like(K)
    o = torch.empty_like(q)
    st = bss.attn_decode_noalloc(q.data_ptr(), K.data_ptr(), V.data_ptr(), o.data_ptr(), B, Hq, Hkv, L,
                                 d, 1.0, torch.cuda.current_stream().cuda_stream, None)
    assert st == 2, bss.attn_status_string(st)
    torch.cuda.synchronize()
    assert bss.attn_sync_status() == 0
