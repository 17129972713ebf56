"""Run one named workload's kernel a few times, for a profiler to capture.

    python -m block_skipping_softmax_b200.profile_run --workload llama3_8b_causal_N8192 \
        --tau inf --launches 3 [--qk e4m3|i8]

Inputs follow the workload's recipe (drawn on the GPU, as in bench.py); no
timing is printed, since numbers taken under a profiler are not
measurements.  The process exits non-zero if a kernel reports a status.
"""
from __future__ import annotations

import argparse
import math
import sys


def main(argv=None) -> int:
    import torch

    import block_skipping_softmax_b200 as bss
    from block_skipping_softmax_b200 import inputs

    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", required=True, choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--tau", default="inf")
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--qk", default="bf16", choices=["bf16", "e4m3", "i8"],
                    help="operand format of Q K^T (prefill; 8-bit inputs are quantised first)")
    ap.add_argument("--paged", action="store_true",
                    help="decode: read the cache as a pool of 64-key pages in seeded random order")
    args = ap.parse_args(argv)
    tau = math.inf if args.tau == "inf" else float(args.tau)
    w = inputs.WORKLOADS[args.workload]
    dev = torch.device("cuda", 0)
    if w["kind"] == "prefill":
        Q, K, V = inputs.prefill_inputs(w["B"], w["Hq"], w["Hkv"], w["N"], w["d"], seed=0,
                                        device=str(dev), **w["gen"])
        O = torch.empty_like(Q)
        if args.qk == "bf16":
            for _ in range(args.launches):
                bss.prefill(Q, K, V, w["causal"], tau, w["Br"], w["Bc"], out=O)
        else:
            quant = bss.quantize_i8 if args.qk == "i8" else bss.quantize_e4m3
            run = bss.prefill_qki8 if args.qk == "i8" else bss.prefill_qk8
            Q8, qs = quant(Q)
            K8, ks = quant(K)
            for _ in range(args.launches):
                run(Q8, K8, qs, ks, V, w["causal"], tau, w["Br"], w["Bc"], out=O)
    else:
        q, K, V = inputs.decode_inputs(w["B"], w["Hq"], w["Hkv"], w["L"], w["d"], seed=0, **w["gen"])
        q, K, V = q.to(dev), K.to(dev), V.to(dev)
        o = torch.empty_like(q)
        if args.paged:
            B, Hkv, L, d = w["B"], w["Hkv"], w["L"], w["d"]
            npg = -(-L // 64)
            assert L % 64 == 0, "the page pool here holds whole pages"
            perm = torch.randperm(B * npg, generator=torch.Generator().manual_seed(7)).to(dev)
            Kp = torch.empty(B * npg, Hkv, 64, d, dtype=torch.bfloat16, device=dev)
            Vp = torch.empty_like(Kp)
            Kp[perm] = K.view(B, Hkv, npg, 64, d).permute(0, 2, 1, 3, 4).reshape(B * npg, Hkv, 64, d)
            Vp[perm] = V.view(B, Hkv, npg, 64, d).permute(0, 2, 1, 3, 4).reshape(B * npg, Hkv, 64, d)
            table = perm.view(B, npg).to(torch.int32).contiguous()
            lens = torch.full((B,), L, dtype=torch.int32, device=dev)
            del K, V
            for _ in range(args.launches):
                bss.decode_paged(q, Kp, Vp, table, lens, L, tau, out=o)
        else:
            for _ in range(args.launches):
                bss.decode(q, K, V, tau, out=o)
    st = bss.attn_sync_status()
    if st != 0:
        print(f"kernel status {bss.attn_status_string(st)}", file=sys.stderr)
        return 1
    return 0


if __name__ == "__main__":
    sys.exit(main())
