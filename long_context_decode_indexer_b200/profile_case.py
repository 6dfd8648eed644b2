"""One DSA decode step on a resized workload, for profiler captures.

    python -m long_context_decode_indexer_b200.profile_case \\
        [--workload long_decode_16x128k] [--nseq 16] [--L 98304] [--warmup 1] [--iters 1]

Runs `warmup + iters` dsa_forward calls (fused indexer + TopK, sparse MLA,
split combine) and checks the device status word.  Sizes are chosen by the
caller so that a capture holds a few GB at most while the index-K stream
stays larger than L2.
"""
from __future__ import annotations

import argparse
import sys

import torch

from . import dsa
from .batch import upload, workspace
from .synth import CONFIGS, make_inputs


def main(argv=None) -> int:
    names = {c["name"]: cid for cid, c in CONFIGS.items()}
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", choices=sorted(names), default=CONFIGS[3]["name"])
    ap.add_argument("--nseq", type=int, default=None)
    ap.add_argument("--L", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=1)
    ap.add_argument("--iters", type=int, default=1)
    args = ap.parse_args(argv)
    inp = make_inputs(names[args.workload], nseq=args.nseq, L=args.L)
    db = upload(inp)
    p, kv = db.params(), db.kvdesc()
    ws = workspace(dsa.workspace_size(p, kv, dsa.OP_FORWARD))
    out = torch.empty((inp.nq, inp.h, inp.d_v), dtype=torch.int16, device="cuda")
    lse = torch.empty((inp.nq, inp.h), dtype=torch.float32, device="cuda")
    idx = torch.empty((inp.nq, inp.topk), dtype=torch.int32, device="cuda")
    for _ in range(args.warmup + args.iters):
        dsa.forward(p, kv, db.q_idx, db.w, db.kidx, db.k_scale, db.q, db.kv, db.kv_row_stride,
                    out, lse, idx, ws, paged=db.page_table is not None)
    st = dsa.check_status(ws)
    print("workload %s nq=%d max_n=%d status=%d" % (inp.name, inp.nq, inp.max_n, st))
    return 0 if st == dsa.DSA_OK else 1


if __name__ == "__main__":
    sys.exit(main())
