"""Run one operation of the layer on a named workload, for profilers.

    python -m bit_nf4_quantized_qlora_b200.profile_ops --op fwd --workload mlp_gate --m 4096 --iters 3

Sets the seeded inputs up on cuda:0, runs the operation `--warmup` times and
then `--iters` more times, and prints the mean device time per call.  Under
``ncu -k <kernel> -s <skip> -c <count>`` it gives captures of a single
kernel on the real shapes.
"""
import argparse
import json

import torch

from . import binding as B
from . import workloads as WL

WORKLOADS = {
    "mlp_gate": lambda m: WL.mlp_7b("gate", m),
    "mlp_down": lambda m: WL.mlp_7b("down", m),
    "attn_proj": lambda m: WL.attn_proj_7b(m),
    "up_proj_70b": lambda m: WL.up_proj_70b(m),
    "single": lambda m: WL.single_linear().with_m(m),
}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", choices=("quantize", "quantize_fp8", "dequant", "fwd", "fwd_nolora", "bwd_dx", "lora_bwd",
                                     "merge", "dropout", "fwd_dropout", "bwd_dx_dropout"), required=True)
    ap.add_argument("--workload", choices=sorted(WORKLOADS), required=True)
    ap.add_argument("--m", type=int, default=4096)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=2)
    a = ap.parse_args(argv)

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    case = WORKLOADS[a.workload](a.m)
    W = case.W().to(dev)
    w = B.qlora_quantize_nf4_dq(W)
    w8 = B.qlora_quantize_4bit_dq(W, B.QLORA_CODEBOOK_NF4, dq_format=B.QLORA_DQ_FP8_MEAN) if a.op == "quantize_fp8" else None
    if a.op not in ("quantize", "quantize_fp8"):
        del W
    r = case.r
    X = A = Bm = dY = Y = None
    if a.op in ("fwd", "fwd_nolora", "lora_bwd", "dropout", "fwd_dropout"):
        X = case.X().to(dev)
    if a.op in ("bwd_dx", "lora_bwd", "bwd_dx_dropout"):
        dY = case.dY().to(dev)
    A, Bm = case.A().to(dev), case.B().to(dev)
    out_w = torch.empty(case.n, case.k, dtype=torch.bfloat16, device=dev) if a.op in ("dequant", "merge") else None
    if a.op in ("fwd", "fwd_nolora", "fwd_dropout"):
        Y = torch.empty(case.m, case.n, dtype=torch.bfloat16, device=dev)
    Xd = torch.empty_like(X) if a.op in ("dropout", "fwd_dropout") else None
    if a.op in ("bwd_dx", "bwd_dx_dropout"):
        Y = torch.empty(case.m, case.k, dtype=torch.bfloat16, device=dev)

    def run():
        if a.op == "quantize":
            B.qlora_quantize_nf4_dq(W, out=w)
        elif a.op == "quantize_fp8":
            B.qlora_quantize_4bit_dq(W, B.QLORA_CODEBOOK_NF4, out=w8, dq_format=B.QLORA_DQ_FP8_MEAN)
        elif a.op == "dequant":
            B.qlora_dequant(w, out=out_w)
        elif a.op == "merge":
            B.qlora_merge_adapter(w, A, Bm, r, case.scale, out_bf16=out_w)
        elif a.op == "fwd":
            B.qlora_linear_fwd(X, w, A, Bm, r, case.scale, out=Y)
        elif a.op == "fwd_nolora":
            B.qlora_linear_fwd(X, w, None, None, 0, 0.0, out=Y)
        elif a.op == "bwd_dx":
            B.qlora_linear_bwd_dx(dY, w, A, Bm, r, case.scale, out=Y)
        elif a.op == "dropout":
            B.qlora_lora_dropout(X, 0.05, 1234, 7, out=Xd)
        elif a.op == "fwd_dropout":
            B.qlora_linear_fwd_dropout(X, w, A, Bm, r, case.scale, 0.05, 1234, 7, out=Y, Xd=Xd)
        elif a.op == "bwd_dx_dropout":
            B.qlora_linear_bwd_dx_dropout(dY, w, A, Bm, r, case.scale, 0.05, 1234, 7, out=Y)
        else:
            B.qlora_lora_bwd(X, dY, A, Bm, r, case.scale)

    for _ in range(a.warmup):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.iters):
        run()
    e1.record()
    torch.cuda.synchronize()
    print(json.dumps({"op": a.op, "workload": case.name, "m": case.m, "n": case.n, "k": case.k, "r": r,
                      "us_per_call": e0.elapsed_time(e1) * 1e3 / a.iters,
                      "device_error": B.qlora_poll_device_error()}))


if __name__ == "__main__":
    main()
