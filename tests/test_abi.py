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


@pytest.mark.parametrize("args", [
    dict(q=0), dict(L=0), dict(Hq=4, Hkv=3), dict(d=32), dict(tau=float("nan")), dict(tau=-0.5),
    dict(K=P + 4),
])
def test_decode_rejects_bad_arguments(args):
    a = dict(q=P, K=P, V=P, o=P, B=1, Hq=4, Hkv=1, L=1000, d=128, tau=2.0)
    a.update(args)
    st = bss.attn_decode(a["q"], a["K"], a["V"], a["o"], a["B"], a["Hq"], a["Hkv"], a["L"], a["d"], a["tau"])
    assert st == 1


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
