"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point declared in include/attn.h, and rejects bad arguments
before touching the device."""
import math
import os
import re
import subprocess

import pytest

import block_skipping_softmax_b200 as bss
from block_skipping_softmax_b200 import build as bss_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    bss_build.build()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^ATTN_API\s+[\w\s\*]*?\b(attn_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("attn_prefill", "attn_decode", "attn_prefill_ex", "attn_decode_ex",
              "attn_decode_split_len", "attn_decode_workspace_bytes", "attn_status_string",
              "attn_sync_status", "attn_shutdown"):
        assert n in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", bss.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    lib = bss.lib()
    for n in declared_functions():
        assert hasattr(lib, n)


def test_status_strings():
    assert bss.attn_status_string(0) == "ATTN_OK"
    assert bss.attn_status_string(4) == "ATTN_ERR_TIMEOUT"
    assert bss.attn_status_string(99) == "ATTN_ERR_UNKNOWN"


P = 1 << 20  # a 16-byte aligned fake address: validation fails before it is ever used


def _cuda_present():
    import torch

    return torch.cuda.is_available()


# Tests that pass fake addresses run only where no GPU can be reached, so a
# validation gap could never turn into a kernel launch on them.
no_gpu = pytest.mark.skipif(_cuda_present(), reason="fake device addresses are passed only without a GPU")


@no_gpu
@pytest.mark.parametrize("args", [
    dict(Q=0), dict(O=0), dict(B=0), dict(N=-1), dict(Hq=3, Hkv=2), dict(d=96),
    dict(Br=64, Bc=128), dict(Br=32, Bc=32), dict(tau=float("nan")), dict(tau=-1.0),
    dict(Q=P + 8),
])
def test_prefill_rejects_bad_arguments(args):
    a = dict(Q=P, K=P, V=P, O=P, B=1, Hq=2, Hkv=1, N=128, d=64, causal=1, tau=1.0, Br=64, Bc=64)
    a.update(args)
    st = bss.attn_prefill(a["Q"], a["K"], a["V"], a["O"], a["B"], a["Hq"], a["Hkv"], a["N"], a["d"],
                          a["causal"], a["tau"], a["Br"], a["Bc"])
    assert st == 1


@no_gpu
@pytest.mark.parametrize("args", [
    dict(Q=0), dict(d=64), dict(Bc=64), dict(Br=64, Bc=64), dict(pairs=3), dict(pairs=16),
    dict(tau=float("nan")), dict(Hq=3, Hkv=2), dict(Q=P + 8),
])
def test_prefill_poly_rejects_bad_arguments(args):
    a = dict(Q=P, K=P, V=P, O=P, B=1, Hq=2, Hkv=1, N=256, d=128, causal=1, tau=1.0, Br=128, Bc=128, pairs=4)
    a.update(args)
    st = bss.attn_prefill_poly(a["Q"], a["K"], a["V"], a["O"], a["B"], a["Hq"], a["Hkv"], a["N"], a["d"],
                               a["causal"], a["tau"], a["Br"], a["Bc"], a["pairs"])
    assert st == 1


@no_gpu
@pytest.mark.parametrize("args", [
    dict(q=0), dict(L=0), dict(Hq=4, Hkv=3), dict(d=32), dict(tau=float("nan")), dict(tau=-0.5),
    dict(K=P + 4),
])
@pytest.mark.parametrize("entry", ["attn_decode", "attn_decode_noalloc"])
def test_decode_rejects_bad_arguments(args, entry):
    a = dict(q=P, K=P, V=P, o=P, B=1, Hq=4, Hkv=1, L=1000, d=128, tau=2.0)
    a.update(args)
    pos = (a["q"], a["K"], a["V"], a["o"], a["B"], a["Hq"], a["Hkv"], a["L"], a["d"], a["tau"])
    if entry == "attn_decode":
        st = bss.attn_decode(*pos)
    else:
        st = bss.attn_decode_noalloc(*pos, None, None)
    assert st == 1


@no_gpu
def test_decode_noalloc_rejects_problems_beyond_its_array():
    """The no-alloc decode refuses a problem whose split scratch exceeds its
    fixed 16 MiB array, before any CUDA call (so no GPU is needed to test it)."""
    B, Hq, Hkv, L, d = 512, 64, 8, 64, 128
    ls = bss.attn_decode_split_len(B, Hkv, L)
    n_splits = -(-L // ls)
    r256 = lambda x: (x + 255) // 256 * 256
    need = r256(B * Hq * n_splits * d * 4) + r256(B * Hq * n_splits * 4)
    assert need > 16 << 20, "shape must exceed the no-alloc scratch array"
    st = bss.attn_decode_noalloc(P, P, P, P, B, Hq, Hkv, L, d, 1.0, None, None)
    assert st == 2, bss.attn_status_string(st)


@no_gpu
def test_decode_rejects_bad_workspace():
    st = bss.attn_decode_ex(P, P, P, P, 1, 4, 1, 1000, 128, 1.0, None, None, None, 64)
    assert st == 1
    st = bss.attn_decode_ex(P, P, P, P, 1, 4, 1, 1000, 128, 1.0, None, None, P + 16, 1 << 20)
    assert st == 1


def test_split_len_is_deterministic_and_tiles_the_keys():
    assert bss.attn_decode_tile() == 64
    for (B, Hkv, L) in [(16, 8, 32768), (1, 1, 1), (1, 8, 131072), (3, 2, 1000), (64, 8, 4096)]:
        ls = bss.attn_decode_split_len(B, Hkv, L)
        assert ls == bss.attn_decode_split_len(B, Hkv, L)
        assert ls > 0 and ls % 64 == 0
        n_splits = -(-L // ls)
        assert (n_splits - 1) * ls < L <= n_splits * ls
        ws = bss.attn_decode_workspace_bytes(B, 4 * Hkv, Hkv, L, 128)
        assert ws >= B * 4 * Hkv * n_splits * (128 + 1) * 4
    assert bss.attn_decode_split_len(0, 1, 1) == -1
    assert bss.attn_decode_workspace_bytes(1, 4, 1, 100, 96) == 0


def test_wait_limit_validation():
    assert bss.attn_set_wait_limit_ms(0) == 1
    assert bss.attn_set_wait_limit_ms(2000) == 0


@no_gpu
@pytest.mark.parametrize("fn", ["attn_quantize_e4m3", "attn_quantize_i8"])
@pytest.mark.parametrize("args", [
    dict(x=0), dict(q=0), dict(scales=0), dict(groups=0), dict(group_elems=0), dict(group_elems=24),
    dict(x=P + 8), dict(q=P + 4), dict(scales=P + 2),
])
def test_quantize_rejects_bad_arguments(fn, args):
    a = dict(x=P, q=P, scales=P, groups=4, group_elems=1024)
    a.update(args)
    st = getattr(bss, fn)(a["x"], a["q"], a["scales"], a["groups"], a["group_elems"])
    assert st == 1


@no_gpu
@pytest.mark.parametrize("fn", ["attn_prefill_qk8", "attn_prefill_qki8"])
@pytest.mark.parametrize("args", [
    dict(qs=0), dict(ks=0), dict(qs=P + 2), dict(d=64), dict(Br=64, Bc=64), dict(Q8=0), dict(V=P + 8),
    dict(tau=float("nan")), dict(Hq=3, Hkv=2),
])
def test_prefill_8bit_rejects_bad_arguments(fn, args):
    a = dict(Q8=P, K8=P, qs=P, ks=P, V=P, O=P, B=1, Hq=2, Hkv=1, N=256, d=128, causal=1, tau=1.0,
             Br=128, Bc=128)
    a.update(args)
    st = getattr(bss, fn)(a["Q8"], a["K8"], a["qs"], a["ks"], a["V"], a["O"], a["B"], a["Hq"], a["Hkv"],
                          a["N"], a["d"], a["causal"], a["tau"], a["Br"], a["Bc"])
    assert st == 1


@no_gpu
@pytest.mark.parametrize("args", [
    dict(cu=0), dict(cu=P + 2), dict(total=0), dict(maxlen=0), dict(Br=64, Bc=64), dict(d=96),
])
def test_prefill_varlen_rejects_bad_arguments(args):
    a = dict(Q=P, K=P, V=P, O=P, cu=P, B=2, maxlen=300, total=500, Hq=2, Hkv=1, d=128, causal=1,
             tau=1.0, Br=128, Bc=64)
    a.update(args)
    st = bss.attn_prefill_varlen(a["Q"], a["K"], a["V"], a["O"], a["cu"], a["B"], a["maxlen"], a["total"],
                                 a["Hq"], a["Hkv"], a["d"], a["causal"], a["tau"], a["Br"], a["Bc"])
    assert st == 1


def test_python_wrappers_reject_host_tensors():
    """The marshalling layer refuses tensors that are not CUDA tensors of the
    expected type before it reaches the library (there is no CPU path)."""
    import torch

    x = torch.zeros(1, 1, 128, 128, dtype=torch.bfloat16)
    with pytest.raises(bss.AttnError):
        bss.quantize_e4m3(x)
    with pytest.raises(bss.AttnError):
        bss.quantize_i8(x)
    q8 = torch.zeros(1, 1, 128, 128, dtype=torch.uint8)
    s = torch.ones(1, 1)
    with pytest.raises(bss.AttnError):
        bss.prefill_qk8(q8, q8, s, s, x, True)
    with pytest.raises(bss.AttnError):
        bss.prefill(x, x, x, True)
