"""Skip Softmax attention for NVIDIA B200 (sm_100a): Python binding of libattn.so.

The functions named like the C ABI (``attn_prefill``, ``attn_decode`` ...)
take raw device pointers and sizes and only marshal arguments; the torch
helpers ``prefill`` and ``decode`` take tensors and pass their pointers.
Every step of the computation runs in the library's CUDA kernels.  There is
no CPU fallback: if the library cannot be loaded, or no sm_100 device is
present, calls raise ``AttnError``.

Method: "Accelerating Long-Context Inference with Skip Softmax in NVIDIA
TensorRT-LLM" (Key Points; Detailed Analysis) -- a key tile is skipped when
every query row's tile maximum is below its running maximum minus tau.
"""
from __future__ import annotations

import ctypes
import math
import os

__all__ = [
    "AttnError", "lib", "attn_prefill", "attn_prefill_ex", "attn_prefill_host", "prefill_host",
    "attn_prefill_varlen", "prefill_varlen", "attn_quantize_e4m3", "quantize_e4m3",
    "attn_prefill_qk8", "prefill_qk8", "attn_quantize_i8", "quantize_i8", "attn_prefill_qki8",
    "prefill_qki8", "attn_prefill_poly", "prefill_poly", "attn_decode", "attn_decode_ex",
    "attn_decode_noalloc", "attn_decode_rule", "attn_decode_paged", "decode_paged", "RULE_GROUP", "RULE_PER_HEAD", "RULE_SINK_SEED",
    "attn_decode_split_len", "attn_decode_tile", "attn_decode_workspace_bytes",
    "attn_set_stream", "attn_sync_status", "attn_last_timeout_site", "attn_set_wait_limit_ms",
    "attn_test_withhold_copy", "attn_status_string", "attn_shutdown", "prefill", "decode", "STATUS",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libattn.so")
STATUS = {0: "ATTN_OK", 1: "ATTN_ERR_INVALID_ARG", 2: "ATTN_ERR_UNSUPPORTED", 3: "ATTN_ERR_CUDA",
          4: "ATTN_ERR_TIMEOUT"}


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what} failed: {STATUS.get(status, status)}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libattn.so (built in-tree by ``block_skipping_softmax_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise AttnError(-1, f"loading {LIB_PATH} (not built; run python -m block_skipping_softmax_b200.build)")
    L = ctypes.CDLL(LIB_PATH)
    vp, ci, cf, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sig = {
        "attn_prefill": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, ci, ci]),
        "attn_prefill_ex": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, ci, ci, vp, vp]),
        "attn_prefill_host": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, ci, ci, ci, vp]),
        "attn_prefill_poly": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, ci, ci, ci, vp, vp]),
        "attn_prefill_varlen": (ci, [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, cf, ci, ci, vp, vp]),
        "attn_quantize_e4m3": (ci, [vp, vp, vp, ctypes.c_longlong, ctypes.c_longlong, vp]),
        "attn_prefill_qk8": (ci, [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, ci, ci, vp, vp]),
        "attn_quantize_i8": (ci, [vp, vp, vp, ctypes.c_longlong, ctypes.c_longlong, vp]),
        "attn_prefill_qki8": (ci, [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, ci, ci, vp, vp]),
        "attn_decode": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, cf]),
        "attn_decode_ex": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, vp, vp, vp, sz]),
        "attn_decode_noalloc": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, vp, vp]),
        "attn_decode_rule": (ci, [vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, vp, vp, vp, sz]),
        "attn_decode_paged": (ci, [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, cf, ci, vp, vp,
                                   vp, sz]),
        "attn_decode_split_len": (ci, [ci, ci, ci]),
        "attn_decode_tile": (ci, []),
        "attn_decode_workspace_bytes": (sz, [ci, ci, ci, ci, ci]),
        "attn_set_stream": (ci, [vp]),
        "attn_sync_status": (ci, []),
        "attn_last_timeout_site": (ci, []),
        "attn_set_wait_limit_ms": (ci, [ci]),
        "attn_test_withhold_copy": (ci, [ci]),
        "attn_status_string": (ctypes.c_char_p, [ci]),
        "attn_shutdown": (None, []),
    }
    for name, (res, args) in sig.items():
        try:
            f = getattr(L, name)
        except AttributeError:  # an older build: the entry point raises when called
            continue
        f.restype, f.argtypes = res, args
    _lib = L
    return L


# ---- C-ABI names: argument marshalling only ---------------------------------

def attn_prefill(Q, K, V, O, B, Hq, Hkv, N, d, causal, tau, Br, Bc) -> int:
    return lib().attn_prefill(Q, K, V, O, B, Hq, Hkv, N, d, int(causal), float(tau), Br, Bc)


def attn_prefill_ex(Q, K, V, O, B, Hq, Hkv, N, d, causal, tau, Br, Bc, stream=None, skip_mask=None) -> int:
    return lib().attn_prefill_ex(Q, K, V, O, B, Hq, Hkv, N, d, int(causal), float(tau), Br, Bc,
                                 stream, skip_mask)


def attn_prefill_poly(Q, K, V, O, B, Hq, Hkv, N, d, causal, tau, Br, Bc, poly_pairs, stream=None,
                      skip_mask=None) -> int:
    return lib().attn_prefill_poly(Q, K, V, O, B, Hq, Hkv, N, d, int(causal), float(tau), Br, Bc,
                                   int(poly_pairs), stream, skip_mask)


def attn_prefill_host(Qh, Kh, Vh, Oh, B, Hq, Hkv, N, d, causal, tau, Br, Bc, chunk=0, stream=None) -> int:
    return lib().attn_prefill_host(Qh, Kh, Vh, Oh, B, Hq, Hkv, N, d, int(causal), float(tau), Br, Bc,
                                   int(chunk), stream)


def attn_prefill_varlen(Q, K, V, O, cu_seqlens, B, max_seqlen, total_tokens, Hq, Hkv, d, causal, tau,
                        Br, Bc, stream=None, skip_mask=None) -> int:
    return lib().attn_prefill_varlen(Q, K, V, O, cu_seqlens, B, max_seqlen, total_tokens, Hq, Hkv, d,
                                     int(causal), float(tau), Br, Bc, stream, skip_mask)


def attn_quantize_e4m3(x, q, scales, groups, group_elems, stream=None) -> int:
    return lib().attn_quantize_e4m3(x, q, scales, int(groups), int(group_elems), stream)


def attn_prefill_qk8(Q8, K8, q_scales, k_scales, V, O, B, Hq, Hkv, N, d, causal, tau, Br, Bc, stream=None,
                     skip_mask=None) -> int:
    return lib().attn_prefill_qk8(Q8, K8, q_scales, k_scales, V, O, B, Hq, Hkv, N, d, int(causal),
                                  float(tau), Br, Bc, stream, skip_mask)


def attn_quantize_i8(x, q, scales, groups, group_elems, stream=None) -> int:
    return lib().attn_quantize_i8(x, q, scales, int(groups), int(group_elems), stream)


def attn_prefill_qki8(Q8, K8, q_scales, k_scales, V, O, B, Hq, Hkv, N, d, causal, tau, Br, Bc, stream=None,
                      skip_mask=None) -> int:
    return lib().attn_prefill_qki8(Q8, K8, q_scales, k_scales, V, O, B, Hq, Hkv, N, d, int(causal),
                                   float(tau), Br, Bc, stream, skip_mask)


def attn_decode(q, K, V, o, B, Hq, Hkv, L, d, tau) -> int:
    return lib().attn_decode(q, K, V, o, B, Hq, Hkv, L, d, float(tau))


def attn_decode_ex(q, K, V, o, B, Hq, Hkv, L, d, tau, stream=None, skip_mask=None, ws=None, ws_bytes=0) -> int:
    return lib().attn_decode_ex(q, K, V, o, B, Hq, Hkv, L, d, float(tau), stream, skip_mask, ws, ws_bytes)


RULE_GROUP, RULE_PER_HEAD, RULE_SINK_SEED = 0, 1, 2


def attn_decode_rule(q, K, V, o, B, Hq, Hkv, L, d, tau, rule, stream=None, skip_mask=None, ws=None,
                     ws_bytes=0) -> int:
    return lib().attn_decode_rule(q, K, V, o, B, Hq, Hkv, L, d, float(tau), int(rule), stream,
                                  skip_mask, ws, ws_bytes)


def attn_decode_paged(q, K_pages, V_pages, block_table, seq_lens, o, B, Hq, Hkv, num_pages,
                      max_pages_per_seq, max_seq_len, d, tau, rule=0, stream=None, skip_mask=None,
                      ws=None, ws_bytes=0) -> int:
    return lib().attn_decode_paged(q, K_pages, V_pages, block_table, seq_lens, o, B, Hq, Hkv,
                                   num_pages, max_pages_per_seq, max_seq_len, d, float(tau),
                                   int(rule), stream, skip_mask, ws, ws_bytes)


def attn_decode_noalloc(q, K, V, o, B, Hq, Hkv, L, d, tau, stream=None, skip_mask=None) -> int:
    """Decode with the library's fixed scratch array: no device allocation."""
    return lib().attn_decode_noalloc(q, K, V, o, B, Hq, Hkv, L, d, float(tau), stream, skip_mask)


def attn_decode_split_len(B, Hkv, L) -> int:
    return lib().attn_decode_split_len(B, Hkv, L)


def attn_decode_tile() -> int:
    return lib().attn_decode_tile()


def attn_decode_workspace_bytes(B, Hq, Hkv, L, d) -> int:
    return lib().attn_decode_workspace_bytes(B, Hq, Hkv, L, d)


def attn_set_stream(stream) -> int:
    return lib().attn_set_stream(stream)


def attn_sync_status() -> int:
    return lib().attn_sync_status()


def attn_last_timeout_site() -> int:
    return lib().attn_last_timeout_site()


def attn_set_wait_limit_ms(ms) -> int:
    return lib().attn_set_wait_limit_ms(int(ms))


def attn_test_withhold_copy(which) -> int:
    """Test support: 1 = decode CTAs withhold their first V copy (the waits run out)."""
    return lib().attn_test_withhold_copy(int(which))


def attn_status_string(status) -> str:
    return lib().attn_status_string(int(status)).decode()


def attn_shutdown() -> None:
    lib().attn_shutdown()


# ---- torch helpers: pass tensor pointers, no compute -------------------------

def _check(st: int, what: str):
    if st != 0:
        raise AttnError(st, what)


def _stream_ptr(stream):
    import torch

    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def prefill(Q, K, V, causal: bool, tau: float = math.inf, Br: int = 128, Bc: int = 128,
            out=None, skip_mask: bool = False, stream=None):
    """O = Skip Softmax attention of bf16 CUDA tensors Q [B,Hq,N,d], K/V [B,Hkv,N,d].

    Returns O (and the uint8 skip mask [B,Hq,ceil(N/Br),ceil(N/Bc)] when asked).
    """
    import torch

    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    for t in (Q, K, V):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise AttnError(1, "prefill (tensors must be contiguous bf16 CUDA tensors)")
    O = out if out is not None else torch.empty_like(Q)
    mask = None
    if skip_mask:
        mask = torch.empty(B, Hq, -(-N // Br), -(-N // Bc), dtype=torch.uint8, device=Q.device)
    st = attn_prefill_ex(Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(), B, Hq, Hkv, N, d,
                         causal, tau, Br, Bc, _stream_ptr(stream),
                         mask.data_ptr() if mask is not None else None)
    _check(st, "attn_prefill_ex")
    return (O, mask) if skip_mask else O


def prefill_poly(Q, K, V, causal: bool, tau: float = math.inf, poly_pairs: int = 4, out=None,
                 skip_mask: bool = False, stream=None):
    """attn_prefill_poly on bf16 CUDA tensors (d = 128, Br = Bc = 128):
    poly_pairs of every 16 exponential pairs on the FMA-pipe polynomial."""
    import torch

    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    for t in (Q, K, V):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise AttnError(1, "prefill_poly (tensors must be contiguous bf16 CUDA tensors)")
    O = out if out is not None else torch.empty_like(Q)
    mask = None
    if skip_mask:
        mask = torch.empty(B, Hq, -(-N // 128), -(-N // 128), dtype=torch.uint8, device=Q.device)
    st = attn_prefill_poly(Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(), B, Hq, Hkv, N, d,
                           causal, tau, 128, 128, poly_pairs, _stream_ptr(stream),
                           mask.data_ptr() if mask is not None else None)
    _check(st, "attn_prefill_poly")
    return (O, mask) if skip_mask else O


def prefill_varlen(Q, K, V, cu_seqlens, max_seqlen: int, causal: bool, tau: float = math.inf,
                   Br: int = 128, Bc: int = 128, out=None, skip_mask: bool = False, stream=None):
    """Packed variable-length prefill: Q [total, Hq, d], K/V [total, Hkv, d]
    bf16 CUDA tensors; cu_seqlens int32 CUDA tensor [B + 1]."""
    import torch

    total, Hq, d = Q.shape
    Hkv = K.shape[1]
    B = cu_seqlens.numel() - 1
    for t in (Q, K, V):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise AttnError(1, "prefill_varlen (tensors must be contiguous bf16 CUDA tensors)")
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda:
        raise AttnError(1, "prefill_varlen (cu_seqlens must be an int32 CUDA tensor)")
    O = out if out is not None else torch.empty_like(Q)
    mask = None
    if skip_mask:
        mask = torch.empty(B, Hq, -(-max_seqlen // Br), -(-max_seqlen // Bc), dtype=torch.uint8,
                           device=Q.device)
    st = attn_prefill_varlen(Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(), cu_seqlens.data_ptr(),
                             B, max_seqlen, total, Hq, Hkv, d, causal, tau, Br, Bc, _stream_ptr(stream),
                             mask.data_ptr() if mask is not None else None)
    _check(st, "attn_prefill_varlen")
    return (O, mask) if skip_mask else O


def quantize_e4m3(x, out=None, stream=None):
    """e4m3 codes (uint8, x's shape) and one power-of-two scale per head slab
    (float32 [B, H]) of a contiguous bf16 CUDA tensor x [B, H, N, d].
    ``out`` = (codes, scales) writes into existing tensors."""
    return _quantize(x, out, stream, int8=False)


def quantize_i8(x, out=None, stream=None):
    """int8 codes (int8, x's shape) and one power-of-two scale per head slab
    (float32 [B, H]) of a contiguous bf16 CUDA tensor x [B, H, N, d]."""
    return _quantize(x, out, stream, int8=True)


def _quantize(x, out, stream, int8):
    import torch

    code_dtype = torch.int8 if int8 else torch.uint8
    what = "quantize_i8" if int8 else "quantize_e4m3"

    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous() or x.dim() != 4:
        raise AttnError(1, f"{what} (x must be a contiguous 4-d bf16 CUDA tensor)")
    B, H, N, d = x.shape
    if out is not None:
        q, scales = out
        if (q.dtype != code_dtype or q.shape != x.shape or not q.is_contiguous() or
                scales.dtype != torch.float32 or scales.numel() != B * H or not scales.is_contiguous()):
            raise AttnError(1, f"{what} (out must be {code_dtype} codes of x's shape and float32 [B, H])")
    else:
        q = torch.empty(x.shape, dtype=code_dtype, device=x.device)
        scales = torch.empty(B, H, dtype=torch.float32, device=x.device)
    fn = attn_quantize_i8 if int8 else attn_quantize_e4m3
    _check(fn(x.data_ptr(), q.data_ptr(), scales.data_ptr(), B * H, N * d, _stream_ptr(stream)),
           "attn_" + what)
    return q, scales


def prefill_qk8(Q8, K8, q_scales, k_scales, V, causal: bool, tau: float = math.inf, Br: int = 128,
                Bc: int = 128, out=None, skip_mask: bool = False, stream=None):
    """Prefill with e4m3 Q8 [B,Hq,N,d], K8 [B,Hkv,N,d] (uint8 codes from
    quantize_e4m3), float32 scales [B,Hq] / [B,Hkv], and bf16 V."""
    return _prefill_8bit(Q8, K8, q_scales, k_scales, V, causal, tau, Br, Bc, out, skip_mask, stream, False)


def prefill_qki8(Q8, K8, q_scales, k_scales, V, causal: bool, tau: float = math.inf, Br: int = 128,
                 Bc: int = 128, out=None, skip_mask: bool = False, stream=None):
    """Prefill with int8 Q8 [B,Hq,N,d], K8 [B,Hkv,N,d] (codes from
    quantize_i8), float32 scales [B,Hq] / [B,Hkv], and bf16 V."""
    return _prefill_8bit(Q8, K8, q_scales, k_scales, V, causal, tau, Br, Bc, out, skip_mask, stream, True)


def _prefill_8bit(Q8, K8, q_scales, k_scales, V, causal, tau, Br, Bc, out, skip_mask, stream, int8):
    import torch

    what = "prefill_qki8" if int8 else "prefill_qk8"
    code_dtype = torch.int8 if int8 else torch.uint8
    B, Hq, N, d = Q8.shape
    Hkv = K8.shape[1]
    for t in (Q8, K8):
        if t.dtype != code_dtype or not t.is_cuda or not t.is_contiguous():
            raise AttnError(1, f"{what} (Q8, K8 must be contiguous {code_dtype} CUDA tensors)")
    for t in (q_scales, k_scales):
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
            raise AttnError(1, f"{what} (scales must be contiguous float32 CUDA tensors)")
    if V.dtype != torch.bfloat16 or not V.is_cuda or not V.is_contiguous():
        raise AttnError(1, f"{what} (V must be a contiguous bf16 CUDA tensor)")
    O = out if out is not None else torch.empty(Q8.shape, dtype=torch.bfloat16, device=Q8.device)
    mask = None
    if skip_mask:
        mask = torch.empty(B, Hq, -(-N // Br), -(-N // Bc), dtype=torch.uint8, device=Q8.device)
    fn = attn_prefill_qki8 if int8 else attn_prefill_qk8
    st = fn(Q8.data_ptr(), K8.data_ptr(), q_scales.data_ptr(), k_scales.data_ptr(),
            V.data_ptr(), O.data_ptr(), B, Hq, Hkv, N, d, causal, tau, Br, Bc,
            _stream_ptr(stream), mask.data_ptr() if mask is not None else None)
    _check(st, "attn_" + what)
    return (O, mask) if skip_mask else O


def prefill_host(Qh, Kh, Vh, causal: bool, tau: float = math.inf, Br: int = 128, Bc: int = 128,
                 out=None, chunk: int = 0, stream=None):
    """attn_prefill_host on host (CPU) bf16 tensors; pinned memory lets the
    copies overlap.  Asynchronous on ``stream``: synchronise it before reading
    the returned tensor."""
    import torch

    B, Hq, N, d = Qh.shape
    Hkv = Kh.shape[1]
    for t in (Qh, Kh, Vh):
        if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous():
            raise AttnError(1, "prefill_host (tensors must be contiguous bf16 host tensors)")
    Oh = out if out is not None else torch.empty_like(Qh, pin_memory=Qh.is_pinned())
    st = attn_prefill_host(Qh.data_ptr(), Kh.data_ptr(), Vh.data_ptr(), Oh.data_ptr(), B, Hq, Hkv, N, d,
                           causal, tau, Br, Bc, chunk, _stream_ptr(stream))
    _check(st, "attn_prefill_host")
    return Oh


def decode(q, K, V, tau: float = math.inf, out=None, skip_mask: bool = False, stream=None,
           workspace=None, rule: int = RULE_GROUP):
    """o = Skip Softmax decode attention: q [B,Hq,d], K/V [B,Hkv,L,d] bf16 CUDA tensors.

    ``workspace``: optional uint8 CUDA tensor of at least
    attn_decode_workspace_bytes(...) bytes; otherwise the library's own is used.
    """
    import torch

    B, Hq, d = q.shape
    Hkv, L = K.shape[1], K.shape[2]
    for t in (q, K, V):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise AttnError(1, "decode (tensors must be contiguous bf16 CUDA tensors)")
    o = out if out is not None else torch.empty_like(q)
    mask = None
    if skip_mask:
        rows = Hq if rule & RULE_PER_HEAD else Hkv
        mask = torch.empty(B, rows, -(-L // attn_decode_tile()), dtype=torch.uint8, device=q.device)
    ws, wsb = (None, 0) if workspace is None else (workspace.data_ptr(), workspace.numel())
    st = attn_decode_rule(q.data_ptr(), K.data_ptr(), V.data_ptr(), o.data_ptr(), B, Hq, Hkv, L, d,
                          tau, rule, _stream_ptr(stream),
                          mask.data_ptr() if mask is not None else None, ws, wsb)
    _check(st, "attn_decode_rule")
    return (o, mask) if skip_mask else o


def decode_paged(q, K_pages, V_pages, block_table, seq_lens, max_seq_len: int, tau: float = math.inf,
                 out=None, skip_mask: bool = False, stream=None, rule: int = RULE_GROUP):
    """o = Skip Softmax decode from a paged KV cache.

    q [B,Hq,d]; K_pages/V_pages [num_pages,Hkv,64,d] bf16; block_table int32
    [B,max_pages]; seq_lens int32 [B]; all CUDA tensors.
    """
    import torch

    B, Hq, d = q.shape
    num_pages, Hkv = K_pages.shape[0], K_pages.shape[1]
    for t in (q, K_pages, V_pages):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise AttnError(1, "decode_paged (tensors must be contiguous bf16 CUDA tensors)")
    for t in (block_table, seq_lens):
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
            raise AttnError(1, "decode_paged (block_table/seq_lens must be contiguous int32 CUDA tensors)")
    o = out if out is not None else torch.empty_like(q)
    mask = None
    if skip_mask:
        rows = Hq if rule & RULE_PER_HEAD else Hkv
        mask = torch.empty(B, rows, -(-max_seq_len // attn_decode_tile()), dtype=torch.uint8,
                           device=q.device)
    st = attn_decode_paged(q.data_ptr(), K_pages.data_ptr(), V_pages.data_ptr(), block_table.data_ptr(),
                           seq_lens.data_ptr(), o.data_ptr(), B, Hq, Hkv, num_pages,
                           block_table.shape[1], max_seq_len, d, tau, rule, _stream_ptr(stream),
                           mask.data_ptr() if mask is not None else None)
    _check(st, "attn_decode_paged")
    return (o, mask) if skip_mask else o
