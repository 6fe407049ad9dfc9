"""Run one forward call of the library a few times on seeded device inputs.

A driver for profilers (``ncu`` and the like), which want a short program
that launches the kernel of interest a known number of times:

    python -m kernelized_feature_map_b200.run_case --path mg --B 8 --H 16 --T 2048 --d 64 --groups 2 --layout bthd

Inputs are drawn on the device (q, k L2-normalised N(0, 1) per token, v
N(0, 1), bf16); the program prints the call's status and nothing is timed.
Paths: ``quadratic`` (kata_fwd_quadratic, q/k width d), ``chunked``
(kata_fwd_chunked), ``mg`` (kata_fwd_mg_quadratic with --groups),
``decode`` (kata_decode_step_mg on a zero state, T ignored) and ``train``
(kata_fwd_quadratic_train then kata_bwd_quadratic for a random dO).
"""
from __future__ import annotations

import argparse


def main(argv=None):
    import torch

    import kernelized_feature_map_b200 as K

    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--path", choices=["quadratic", "chunked", "mg", "decode", "train"], required=True)
    ap.add_argument("--B", type=int, default=8)
    ap.add_argument("--H", type=int, default=16)
    ap.add_argument("--T", type=int, default=2048)
    ap.add_argument("--d", type=int, default=16, help="q/k width (p for the single-factor paths)")
    ap.add_argument("--dv", type=int, default=64)
    ap.add_argument("--groups", type=int, default=1)
    ap.add_argument("--layout", choices=["bhtd", "bthd"], default="bhtd")
    ap.add_argument("--C", type=int, default=64)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--seed", type=int, default=0)
    a = ap.parse_args(argv)

    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    gen.manual_seed(a.seed)
    bf = torch.bfloat16

    def unit(shape):
        x = torch.randn(shape, generator=gen, device=dev)
        return (x / x.norm(dim=-1, keepdim=True)).to(bf)

    if a.path == "decode":
        p = a.d // a.groups
        q, k = unit((a.B, a.H, a.d)), unit((a.B, a.H, a.d))
        v = torch.randn((a.B, a.H, a.dv), generator=gen, device=dev).to(bf)
        S = torch.zeros((a.B, a.H, a.groups * p * p, a.dv), dtype=torch.float32, device=dev)
        z = torch.zeros((a.B, a.H, a.groups * p * p), dtype=torch.float32, device=dev)
        call = lambda: K.kata_decode_step_mg(q, k, v, S, z, a.groups)  # noqa: E731
    else:
        lead = (a.B, a.T, a.H) if a.layout == "bthd" else (a.B, a.H, a.T)
        q, k = unit(lead + (a.d,)), unit(lead + (a.d,))
        v = torch.randn(lead + (a.dv,), generator=gen, device=dev).to(bf)
        o = torch.empty_like(v)
        if a.path == "mg":
            call = lambda: K.kata_fwd_mg_quadratic(q, k, v, a.groups, layout=a.layout, o=o)  # noqa: E731
        elif a.layout != "bhtd":
            ap.error("--layout bthd is for --path mg")
        elif a.path == "quadratic":
            call = lambda: K.kata_fwd_quadratic(q, k, v, o=o)  # noqa: E731
        elif a.path == "train":
            dO = torch.randn(v.shape, generator=gen, device=dev).to(bf)
            D = torch.empty((a.B, a.H, a.T), dtype=torch.float32, device=dev)

            def call():
                K.kata_fwd_quadratic_train(q, k, v, o=o, D=D)
                K.kata_bwd_quadratic(q, k, v, o, D, dO)
        else:
            ws = torch.empty(max(256, K.kata_fwd_chunked_workspace_size(a.B, a.H, a.T, a.d, a.dv, a.C, bf)),
                             dtype=torch.uint8, device=dev)
            call = lambda: K.kata_fwd_chunked(q, k, v, C=a.C, o=o, workspace=ws)  # noqa: E731
    for _ in range(a.reps):
        call()
    torch.cuda.synchronize()
    status = K.kata_get_status()
    print("%s reps=%d status=%d (%s)" % (a.path, a.reps, status, K.status_string(status)))
    return 0 if status == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())
