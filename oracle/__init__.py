"""Plain fp64 CPU oracle for Skip Softmax attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference arm of ``bench.py`` may import this package.  The
product library never routes through it, and it shares no code with the CUDA
path: the arithmetic lives in ``skipsoftmax_oracle.c`` (plain C, fp64,
OpenMP over independent row blocks), this module only marshals numpy arrays.

Method source: "Accelerating Long-Context Inference with Skip Softmax in
NVIDIA TensorRT-LLM" (Key Points; Detailed Analysis): a key tile is skipped
when every query row's local tile maximum lies more than tau below that row's
running maximum.  The exact conventions are stated at the top of the C file.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
(brute force, closed forms, invariants, and the hand-built example in
``tests/golden/``); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "skipsoftmax_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False, src: str | None = None, out: str | None = None) -> str:
    """Compile the C oracle into a shared library with gcc (fp64, OpenMP).

    ``src``/``out`` let tests build variants (for instance a copy with a
    planted mistake) without touching the real library.
    """
    src = src or _SRC
    out = out or _LIB
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    # -ffp-contract=off keeps every multiply and add a separate fp64 rounding,
    # exactly as written in the C source.
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
           "-std=c11", src, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


def _load(path: str | None = None):
    global _lib
    if path is None and _lib is not None:
        return _lib
    lib = ctypes.CDLL(path or build())
    u16p = ctypes.POINTER(ctypes.c_uint16)
    f64p = ctypes.POINTER(ctypes.c_double)
    u8p = ctypes.POINTER(ctypes.c_uint8)
    i32p = ctypes.POINTER(ctypes.c_int32)
    ci = ctypes.c_int
    lib.oracle_prefill.restype = ci
    lib.oracle_prefill.argtypes = [u16p, u16p, u16p, ci, ci, ci, ci, ci, ci, ctypes.c_double,
                                   ci, ci, i32p, ctypes.c_int64, f64p, f64p, u8p, f64p, f64p, ci]
    lib.oracle_decode.restype = ci
    lib.oracle_decode.argtypes = [u16p, u16p, u16p, ci, ci, ci, ci, ci, ctypes.c_double, ci, ci,
                                  ci, f64p, f64p, u8p, f64p, f64p, ci]
    lib.oracle_e4m3_value.restype = ctypes.c_double
    lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
    lib.oracle_quantize_e4m3.restype = ci
    lib.oracle_quantize_e4m3.argtypes = [u16p, ctypes.c_int64, ctypes.c_int64, u8p, f64p]
    lib.oracle_quantize_i8.restype = ci
    lib.oracle_quantize_i8.argtypes = [u16p, ctypes.c_int64, ctypes.c_int64,
                                       ctypes.POINTER(ctypes.c_int8), f64p]
    if path is None:
        _lib = lib
    return lib


def _bits(x) -> np.ndarray:
    """bf16 input (torch bf16 tensor or uint16 bit array) -> contiguous uint16 bits."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch  # bf16 tensors come from torch; the oracle only reads their bits

    assert x.dtype == torch.bfloat16
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _p(a, t):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(t))


def prefill(Q, K, V, causal: bool, tau: float, Br: int, Bc: int, units=None,
            want_exact: bool = True, nthreads: int = 0, lib_path: str | None = None) -> dict:
    """fp64 Skip Softmax prefill.  Q [B,Hq,N,d], K/V [B,Hkv,N,d] (bf16).

    Returns a dict with ``O`` [B,Hq,N,d] fp64, ``mask`` uint8 [B,Hq,nRB,nT]
    (0 kept, 1 skipped, 2 not visited), ``margin`` fp64 (same shape; skip iff
    margin < 0), and when ``want_exact`` ``O_exact`` and ``pskip`` [B,Hq,N].
    ``units`` optionally restricts the work to (b, h, rb) triples; entries of
    other row blocks are left as NaN (O) / 255 (mask).
    """
    q, k, v = _bits(Q), _bits(K), _bits(V)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    n_rb, n_t = -(-N // Br), -(-N // Bc)
    O = np.full((B, Hq, N, d), np.nan)
    O_exact = np.full((B, Hq, N, d), np.nan) if want_exact else None
    pskip = np.full((B, Hq, N), np.nan) if want_exact else None
    mask = np.full((B, Hq, n_rb, n_t), 255, dtype=np.uint8)
    margin = np.full((B, Hq, n_rb, n_t), np.nan)
    u = None
    n_units = 0
    if units is not None:
        u = np.ascontiguousarray(np.asarray(units, dtype=np.int32).reshape(-1, 3))
        n_units = u.shape[0]
    lib = _load(lib_path)
    st = lib.oracle_prefill(_p(q, ctypes.c_uint16), _p(k, ctypes.c_uint16), _p(v, ctypes.c_uint16),
                            B, Hq, Hkv, N, d, int(bool(causal)), float(tau), Br, Bc,
                            _p(u, ctypes.c_int32), n_units, _p(O, ctypes.c_double),
                            _p(O_exact, ctypes.c_double), _p(mask, ctypes.c_uint8),
                            _p(margin, ctypes.c_double), _p(pskip, ctypes.c_double), int(nthreads))
    if st != 0:
        raise ValueError(f"oracle_prefill failed with status {st}")
    out = {"O": O, "mask": mask, "margin": margin}
    if want_exact:
        out["O_exact"], out["pskip"] = O_exact, pskip
    return out


RULE_PER_HEAD = 1   # each query head takes the test on its own row
RULE_SINK_SEED = 2  # each split's running max starts at the first key tile's max


def decode(q, K, V, tau: float, Ls: int, Bt: int = 64, want_exact: bool = True,
           nthreads: int = 0, lib_path: str | None = None, rule: int = 0) -> dict:
    """fp64 Skip Softmax decode.  q [B,Hq,d], K/V [B,Hkv,L,d] (bf16).

    Returns ``o`` [B,Hq,d], ``mask``/``margin`` [B,Hkv,ceil(L/Bt)] ([B,Hq,...]
    with RULE_PER_HEAD), and when ``want_exact`` ``o_exact`` and ``pskip`` [B,Hq].
    ``rule`` selects the decode rule variant (bits RULE_PER_HEAD, RULE_SINK_SEED).
    """
    qb, k, v = _bits(q), _bits(K), _bits(V)
    B, Hq, d = qb.shape
    Hkv, L = k.shape[1], k.shape[2]
    n_t = -(-L // Bt)
    o = np.full((B, Hq, d), np.nan)
    o_exact = np.full((B, Hq, d), np.nan) if want_exact else None
    pskip = np.full((B, Hq), np.nan) if want_exact else None
    rows = Hq if rule & RULE_PER_HEAD else Hkv
    mask = np.full((B, rows, n_t), 255, dtype=np.uint8)
    margin = np.full((B, rows, n_t), np.nan)
    lib = _load(lib_path)
    st = lib.oracle_decode(_p(qb, ctypes.c_uint16), _p(k, ctypes.c_uint16), _p(v, ctypes.c_uint16),
                           B, Hq, Hkv, L, d, float(tau), int(Ls), int(Bt), int(rule),
                           _p(o, ctypes.c_double),
                           _p(o_exact, ctypes.c_double), _p(mask, ctypes.c_uint8),
                           _p(margin, ctypes.c_double), _p(pskip, ctypes.c_double), int(nthreads))
    if st != 0:
        raise ValueError(f"oracle_decode failed with status {st}")
    out = {"o": o, "mask": mask, "margin": margin}
    if want_exact:
        out["o_exact"], out["pskip"] = o_exact, pskip
    return out


INF = math.inf


def e4m3_values(lib_path: str | None = None) -> np.ndarray:
    """fp64 value of each of the 256 e4m3 codes (NaN for the two NaN codes)."""
    lib = _load(lib_path)
    return np.array([lib.oracle_e4m3_value(c) for c in range(256)])


def quantize_e4m3(x, groups: int, lib_path: str | None = None):
    """e4m3 codes (uint8, x's shape) and fp64 power-of-two scales [groups] of a
    bf16 tensor cut into ``groups`` equal contiguous groups."""
    xb = _bits(x)
    n = xb.size
    if groups <= 0 or n % groups:
        raise ValueError("quantize_e4m3: the element count must split into equal groups")
    codes = np.empty(xb.shape, dtype=np.uint8)
    scales = np.empty(groups)
    st = _load(lib_path).oracle_quantize_e4m3(_p(xb, ctypes.c_uint16), groups, n // groups,
                                              _p(codes, ctypes.c_uint8), _p(scales, ctypes.c_double))
    if st != 0:
        raise ValueError(f"oracle_quantize_e4m3 failed with status {st}")
    return codes, scales


def dequantize_e4m3(codes: np.ndarray, scales: np.ndarray, lib_path: str | None = None) -> np.ndarray:
    """fp64 values code * scale, one scale per equal contiguous group."""
    vals = e4m3_values(lib_path)[codes.reshape(scales.size, -1)]
    return (vals * scales[:, None]).reshape(codes.shape)


def quantize_i8(x, groups: int, lib_path: str | None = None):
    """int8 codes (x's shape) and fp64 power-of-two scales [groups] of a bf16
    tensor cut into ``groups`` equal contiguous groups."""
    xb = _bits(x)
    n = xb.size
    if groups <= 0 or n % groups:
        raise ValueError("quantize_i8: the element count must split into equal groups")
    codes = np.empty(xb.shape, dtype=np.int8)
    scales = np.empty(groups)
    st = _load(lib_path).oracle_quantize_i8(_p(xb, ctypes.c_uint16), groups, n // groups,
                                            _p(codes, ctypes.c_int8), _p(scales, ctypes.c_double))
    if st != 0:
        raise ValueError(f"oracle_quantize_i8 failed with status {st}")
    return codes, scales


def dequantize_i8(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """fp64 values code * scale, one scale per equal contiguous group."""
    return (codes.reshape(scales.size, -1).astype(np.float64) * scales[:, None]).reshape(codes.shape)
