"""Prefill from host memory (attn_prefill_host): the chunked copy pipeline
gives exactly the device path's output, for whole and partial last chunks of
KV-head groups, including a single sequence cut by KV heads."""
import math

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


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal,Br,Bc,chunk", [
    (5, 4, 2, 300, 128, True, 128, 128, 3),     # 10 groups: chunks of 3, 3, 3, 1
    (8, 4, 4, 512, 128, False, 128, 64, 0),     # default chunking
    (3, 2, 1, 200, 64, True, 64, 64, 1),
    (4, 8, 2, 640, 128, True, 128, 128, 8),     # one chunk
    (1, 16, 4, 1000, 128, True, 128, 128, 0),   # one sequence, one KV head per chunk
    (1, 8, 8, 700, 128, False, 128, 64, 3),     # one sequence, chunks of 3, 3, 2 heads
])
def test_host_pipeline_matches_device_path(B, Hq, Hkv, N, d, causal, Br, Bc, chunk):
    Q, K, V = inputs.prefill_inputs(B, Hq, Hkv, N, d, seed=B + N, q_sigma=2.0, q_u=1.0, sink_scale=3.0)
    ref = bss.prefill(Q.cuda(), K.cuda(), V.cuda(), causal, 4.0, Br, Bc)
    Qp, Kp, Vp = Q.pin_memory(), K.pin_memory(), V.pin_memory()
    Oh = bss.prefill_host(Qp, Kp, Vp, causal, 4.0, Br, Bc, chunk=chunk)
    torch.cuda.synchronize()
    assert bss.attn_sync_status() == 0
    assert torch.equal(Oh, ref.cpu())


def test_host_pipeline_argument_errors():
    Q = torch.zeros(1, 1, 64, 128, dtype=torch.bfloat16)
    assert bss.attn_prefill_host(None, Q.data_ptr(), Q.data_ptr(), Q.data_ptr(), 1, 1, 1, 64, 128, 0,
                                 math.inf, 128, 128) == 1
    assert bss.attn_prefill_host(Q.data_ptr(), Q.data_ptr(), Q.data_ptr(), Q.data_ptr(), 1, 1, 1, 64, 128,
                                 0, math.inf, 128, 128, chunk=-1) == 1
    assert bss.attn_prefill_host(Q.data_ptr(), Q.data_ptr(), Q.data_ptr(), Q.data_ptr(), 1, 1, 1, 64, 96,
                                 0, math.inf, 128, 128) == 1
