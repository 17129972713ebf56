"""The timeout path of the bounded waits, exercised without any GPU fault.

Every wait inside the kernels gives up after the limit set by
attn_set_wait_limit_ms, records a status code and unwinds.  Here the library
withholds one copy on purpose (attn_test_withhold_copy), so the waits for it
run out: nothing traps, faults or hangs, the call reports ATTN_ERR_TIMEOUT
through attn_sync_status(), and the context stays usable for the next call,
whose result is checked against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import block_skipping_softmax_b200 as bss
import oracle
from block_skipping_softmax_b200 import build as bss_build
from block_skipping_softmax_b200 import inputs
from parity import compare_outputs

pytestmark = pytest.mark.gpu

ATTN_ERR_TIMEOUT = 4
DECODE_V_WAIT_SITE = 20


@pytest.fixture(scope="module", autouse=True)
def lib():
    bss_build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bss.lib()


def test_withheld_copy_times_out_and_context_recovers():
    B, Hq, Hkv, L, d = 1, 4, 1, 1024, 128
    q, K, V = inputs.decode_inputs(B, Hq, Hkv, L, d, seed=77, q_sigma=2.0, q_u=1.0,
                                   sink_scale=3.0)
    qd, Kd, Vd = q.cuda(), K.cuda(), V.cuda()
    assert bss.attn_sync_status() == 0  # nothing pending from earlier tests
    assert bss.attn_test_withhold_copy(2) == 1  # only 0 and 1 are valid
    assert bss.attn_set_wait_limit_ms(100) == 0
    try:
        assert bss.attn_test_withhold_copy(1) == 0
        o = torch.empty_like(qd)
        st = bss.attn_decode(qd.data_ptr(), Kd.data_ptr(), Vd.data_ptr(), o.data_ptr(),
                             B, Hq, Hkv, L, d, math.inf)
        assert st == 0  # launching succeeds; the wait gives up on the device
        assert bss.attn_sync_status() == ATTN_ERR_TIMEOUT
        assert bss.attn_last_timeout_site() == DECODE_V_WAIT_SITE
        assert bss.attn_sync_status() == 0  # reading the status cleared it
    finally:
        bss.attn_test_withhold_copy(0)
        bss.attn_set_wait_limit_ms(2000)
    # the same context still computes correct results
    o = bss.decode(qd, Kd, Vd, math.inf)
    assert bss.attn_sync_status() == 0
    Ls = bss.attn_decode_split_len(B, Hkv, L)
    r = oracle.decode(q, K, V, math.inf, Ls, 64, want_exact=False)
    compare_outputs(o.cpu(), r["o"], np.ones(r["o"].shape, bool))
