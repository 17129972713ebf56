"""Decode from a paged KV cache (attn_decode_paged) against the fp64 oracle.

Sequences of ragged lengths are scattered over a shuffled page pool; every
key slot that no sequence owns (unused pages, the tail of each last page)
holds NaN, so a kernel that reads past a sequence's end cannot pass.  The
oracle sees each sequence as a contiguous cache of its own length, with the
split length the library uses for the longest sequence."""
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
PAGE = 64


@pytest.fixture(scope="module", autouse=True)
def lib():
    bss_build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bss.lib()


def paginate(K, V, lens, extra_pages, seed):
    """Contiguous [B,Hkv,L,d] -> NaN-padded page pools and a shuffled block table."""
    B, Hkv, L, d = K.shape
    n_pages = [-(-n // PAGE) for n in lens]
    max_pages = max(n_pages)
    pool = sum(n_pages) + extra_pages
    perm = np.random.default_rng(seed).permutation(pool)
    Kp = torch.full((pool, Hkv, PAGE, d), float("nan"), dtype=torch.bfloat16)
    Vp = torch.full((pool, Hkv, PAGE, d), float("nan"), dtype=torch.bfloat16)
    table = np.full((B, max_pages), -1, np.int32)  # unread entries stay invalid
    nxt = 0
    for b in range(B):
        for t in range(n_pages[b]):
            p = int(perm[nxt])
            nxt += 1
            table[b, t] = p
            k0, k1 = t * PAGE, min(lens[b], (t + 1) * PAGE)
            Kp[p, :, : k1 - k0] = K[b, :, k0:k1]
            Vp[p, :, : k1 - k0] = V[b, :, k0:k1]
    return Kp, Vp, torch.from_numpy(table), torch.tensor(lens, dtype=torch.int32)


def check_paged(q, K, V, lens, tau, rule, extra_pages=5, seed=0):
    B, Hq, d = q.shape
    Hkv = K.shape[1]
    g = Hq // Hkv
    max_len = max(lens)
    Kp, Vp, table, sl = paginate(K, V, lens, extra_pages, seed)
    o, mask = bss.decode_paged(q.cuda(), Kp.cuda(), Vp.cuda(), table.cuda(), sl.cuda(), max_len, tau,
                               skip_mask=True, rule=rule)
    assert bss.attn_sync_status() == 0
    o, mask = o.cpu(), mask.cpu().numpy()
    Ls = bss.attn_decode_split_len(B, Hkv, max_len)
    for b in range(B):
        n = lens[b]
        r = oracle.decode(q[b:b + 1], K[b:b + 1, :, :n].contiguous(), V[b:b + 1, :, :n].contiguous(), tau,
                          Ls, PAGE, want_exact=False, rule=rule)
        nt = -(-n // PAGE)
        assert (mask[b, :, nt:] == 2).all(), "tiles past the end must be marked not visited"
        flips = compare_masks(mask[b:b + 1, :, :nt], r["mask"], r["margin"])
        rows = np.ones((1, Hq, 1), bool)
        for x in np.nonzero(flips[0].any(-1))[0]:
            if rule & bss.RULE_PER_HEAD:
                rows[0, x] = False
            else:
                rows[0, x * g:(x + 1) * g] = False
        compare_outputs(o[b:b + 1], r["o"], np.broadcast_to(rows, r["o"].shape))


LENS = [1, 63, 64, 65, 700, 2500, 4096]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("g", [1, 4])
@pytest.mark.parametrize("rule", [0, 1, 2, 3])
def test_paged_ragged_exact_and_skipping(d, g, rule):
    B = len(LENS)
    q, K, V = inputs.decode_inputs(B, 2 * g, 2, max(LENS), d, seed=31 + g + d, q_sigma=2.0, q_u=8.0,
                                   sink_scale=6.0)
    check_paged(q, K, V, LENS, math.inf, rule, seed=rule)
    check_paged(q, K, V, LENS, 2.0, rule, seed=rule + 7)


def test_paged_identity_table_equals_contiguous_bitwise():
    """Full lengths and pages in order: the same tiles in the same order as the
    contiguous kernel, so the outputs agree bit for bit (GQA decode workload)."""
    w = inputs.WORKLOADS["gqa_decode_16x32q8kv_L32768"]
    B, Hq, Hkv, L, d = w["B"], w["Hq"], w["Hkv"], w["L"], w["d"]
    q, K, V = inputs.decode_inputs(B, Hq, Hkv, L, d, seed=0, **w["gen"])
    qd, Kd, Vd = q.cuda(), K.cuda(), V.cuda()
    npg = L // PAGE
    # page (b, t) = b * npg + t; pool layout [pages, Hkv, 64, d]
    Kp = Kd.view(B, Hkv, npg, PAGE, d).permute(0, 2, 1, 3, 4).reshape(B * npg, Hkv, PAGE, d).contiguous()
    Vp = Vd.view(B, Hkv, npg, PAGE, d).permute(0, 2, 1, 3, 4).reshape(B * npg, Hkv, PAGE, d).contiguous()
    table = torch.arange(B * npg, dtype=torch.int32, device="cuda").view(B, npg)
    sl = torch.full((B,), L, dtype=torch.int32, device="cuda")
    for tau in (math.inf, 4.0):
        a = bss.decode(qd, Kd, Vd, tau)
        p = bss.decode_paged(qd, Kp, Vp, table, sl, L, tau)
        assert bss.attn_sync_status() == 0
        assert torch.equal(a, p)


def test_paged_long_splits_refill_staged_pages():
    """One split per sequence (37 x 8 KV heads fill the 296 resident CTAs)
    of 1032 tiles: the kernel stages a split's pages 512 at a time, so this
    split refills them inside its tile loop.  Full lengths in a shuffled pool
    agree bit for bit with the contiguous cache; ragged sequences, whose
    unowned key slots hold NaN, agree with the oracle."""
    B, Hkv, Hq, d = 37, 8, 8, 64
    npg = 1032
    L = npg * PAGE - 17
    Ls = bss.attn_decode_split_len(B, Hkv, L)
    assert Ls >= L, "one split per sequence"
    gen = torch.Generator(device="cuda").manual_seed(3)
    q = torch.randn(B, Hq, d, generator=gen, device="cuda").to(torch.bfloat16)
    K = torch.randn(B, Hkv, npg * PAGE, d, generator=gen, device="cuda").to(torch.bfloat16)
    V = torch.randn(B, Hkv, npg * PAGE, d, generator=gen, device="cuda").to(torch.bfloat16)
    K[:, :, L:] = 0  # the contiguous cache is L long: rows past L read as zeros there
    V[:, :, L:] = 0
    perm = torch.randperm(B * npg, generator=torch.Generator().manual_seed(5)).cuda()
    Kp = torch.empty(B * npg, Hkv, PAGE, d, dtype=torch.bfloat16, device="cuda")
    Vp = torch.empty_like(Kp)
    Kp[perm] = K.view(B, Hkv, npg, PAGE, d).permute(0, 2, 1, 3, 4).reshape(B * npg, Hkv, PAGE, d)
    Vp[perm] = V.view(B, Hkv, npg, PAGE, d).permute(0, 2, 1, 3, 4).reshape(B * npg, Hkv, PAGE, d)
    table = perm.view(B, npg).to(torch.int32).contiguous()
    full = torch.full((B,), L, dtype=torch.int32, device="cuda")
    a = bss.decode(q, K[:, :, :L].contiguous(), V[:, :, :L].contiguous(), math.inf)
    p = bss.decode_paged(q, Kp, Vp, table, full, L, math.inf)
    assert bss.attn_sync_status() == 0
    assert torch.equal(a, p)
    # ragged: sequence 1 ends inside the second staged chunk, sequence 2
    # inside the first; their unowned slots hold NaN and their table rows end
    # in invalid entries
    lens = [L, 700 * PAGE + 5, 600] + [L] * (B - 3)
    for b in (1, 2):
        n = lens[b]
        used = -(-n // PAGE)
        pages = table[b, :used].long()
        Kp[pages[-1], :, n - (used - 1) * PAGE:] = float("nan")
        Vp[pages[-1], :, n - (used - 1) * PAGE:] = float("nan")
        Kp[table[b, used:].long()] = float("nan")
        Vp[table[b, used:].long()] = float("nan")
        table[b, used:] = -1
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o = bss.decode_paged(q, Kp, Vp, table, sl, L, math.inf)
    assert bss.attn_sync_status() == 0
    assert torch.equal(o[0], a[0])
    for b in (1, 2):
        n = lens[b]
        r = oracle.decode(q[b:b + 1].cpu(), K[b:b + 1, :, :n].cpu().contiguous(),
                          V[b:b + 1, :, :n].cpu().contiguous(), math.inf, Ls, PAGE, want_exact=False)
        compare_outputs(o[b:b + 1].cpu(), r["o"], np.ones(r["o"].shape, bool))


def test_paged_argument_errors():
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device="cuda")
    Kp = torch.zeros(2, 1, PAGE, 128, dtype=torch.bfloat16, device="cuda")
    table = torch.zeros(1, 2, dtype=torch.int32, device="cuda")
    sl = torch.ones(1, dtype=torch.int32, device="cuda")
    o = torch.empty_like(q)
    args = dict(q=q.data_ptr(), K_pages=Kp.data_ptr(), V_pages=Kp.data_ptr(), block_table=table.data_ptr(),
                seq_lens=sl.data_ptr(), o=o.data_ptr(), B=1, Hq=4, Hkv=1, num_pages=2, max_pages_per_seq=2,
                max_seq_len=100, d=128, tau=1.0)
    assert bss.attn_decode_paged(**args) == 0
    assert bss.attn_sync_status() == 0
    assert bss.attn_decode_paged(**{**args, "max_seq_len": 129}) == 1  # more than 2 pages hold
    assert bss.attn_decode_paged(**{**args, "block_table": None}) == 1
    assert bss.attn_decode_paged(**{**args, "num_pages": 0}) == 1
    assert bss.attn_decode_paged(**args, rule=4) == 1
