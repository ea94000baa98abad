"""Run the hot path on a named synthetic workload (for profilers and smoke runs).

    python -m block_sparse_attention_32_b200.run_workload --workload profile_8k_r8 --passes 2
    python -m block_sparse_attention_32_b200.run_workload --workload prefill_32k --select-only
    python -m block_sparse_attention_32_b200.run_workload --workload profile_bwd_4k_r8 --backward

Each pass enqueues the five C-ABI calls (or only index scoring + selection
with --select-only; or, after one forward, the attention's backward for a
seeded upstream gradient with --backward) on the current stream; the process
exits non-zero if a kernel reports a device-side error.
"""
from __future__ import annotations

import argparse
import sys

import torch

from . import capi, pipeline, workloads


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default=workloads.PROFILE_8K.name,
                    choices=sorted(workloads.ALL))
    ap.add_argument("--passes", type=int, default=2)
    ap.add_argument("--select-only", action="store_true")
    ap.add_argument("--backward", action="store_true")
    args = ap.parse_args(argv)
    w = workloads.ALL[args.workload]
    d = pipeline.dims_for(w)
    inp = workloads.make_inputs(w, "cuda", with_qkv=not args.select_only)
    if args.select_only:
        nblk = capi.msa_num_blocks(d)
        stride = (nblk + 3) // 4 * 4
        pooled = torch.empty((w.batch, w.h_kv, w.n_q, stride), device="cuda")
        sel = torch.empty((w.batch, w.h_kv, w.n_q, capi.TOPK), dtype=torch.int32, device="cuda")
        err = torch.zeros((4,), dtype=torch.int32, device="cuda")
        for _ in range(args.passes):
            capi.msa_index_score_maxpool(d, inp["q_idx"], inp["k_idx"], pooled, stride, err)
            capi.msa_topk_blocks(d, pooled, stride, sel, err)
    elif args.backward:
        buf = pipeline.Buffers.allocate(d)
        grads = pipeline.Grads.allocate(d)
        err = buf.dev_err
        d_out = workloads.upstream_grad(w, "cuda")
        pipeline.forward(buf, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"])
        for _ in range(args.passes):
            pipeline.backward(buf, grads, inp["q"], inp["k"], inp["v"], d_out)
    else:
        buf = pipeline.Buffers.allocate(d)
        err = buf.dev_err
        for _ in range(args.passes):
            pipeline.forward(buf, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"])
    torch.cuda.synchronize()
    code = int(err[0].item())
    print(f"{w.name}: {args.passes} pass(es), device error {code}")
    return 1 if code else 0


if __name__ == "__main__":
    sys.exit(main())
