"""Run one RMM entry point a few times on a named synthetic workload (for profilers).

    python -m input_adaptive_reduced_colnorm_b200.profile_cases decode --n 32 --rho 0.5 --iters 3
    python -m input_adaptive_reduced_colnorm_b200.profile_cases prefill --proj gate_proj --rho 0.5
    python -m input_adaptive_reduced_colnorm_b200.profile_cases qk --rho 0.5 --heads 8
    python -m input_adaptive_reduced_colnorm_b200.profile_cases pv --rho 0.5 --heads 2 --seq 16384
    python -m input_adaptive_reduced_colnorm_b200.profile_cases decode_attn --rho 0.5 --seq 32768
    python -m input_adaptive_reduced_colnorm_b200.profile_cases attention --rho 0.5 --heads 32

Each case draws its inputs with the seeded generators in ``synthetic`` (the same
recipes the tests and the benchmark use), then calls the library ``--iters``
times through the public binding and synchronises.  Head counts can be reduced
so that a profiler capture holds only a few GB on the device.
"""
from __future__ import annotations

import argparse
import os
import sys


def main(argv=None) -> int:
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    import torch

    import input_adaptive_reduced_colnorm_b200 as rmm
    import synthetic
    from input_adaptive_reduced_colnorm_b200 import build

    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["prefill", "decode", "qk", "pv", "linear", "decode_attn", "attention"])
    ap.add_argument("--rho", type=float, default=0.5)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--n", type=int, default=32, help="decode rows")
    ap.add_argument("--proj", default="gate_proj", choices=list(synthetic.PREFILL_SHAPES))
    ap.add_argument("--heads", type=int, default=32)
    ap.add_argument("--seq", type=int, default=None)
    a = ap.parse_args(argv)

    build.build()
    dev = torch.device("cuda", 0)
    if a.case == "linear":
        A, B = synthetic.linear_small()
        A, B = A.to(dev), B.to(dev)
        fn = lambda: rmm.linear(A, B, a.rho)
    elif a.case == "prefill":
        A, B = synthetic.prefill_projection(a.proj)
        A, B = A.to(dev), B.to(dev)
        fn = lambda: rmm.linear(A, B, a.rho)
    elif a.case == "decode":
        A, B = synthetic.decode_gemv(a.n)
        A, B = A.to(dev), B.to(dev)
        fn = lambda: rmm.linear(A, B, a.rho)
    elif a.case == "qk":
        hkv = max(1, a.heads // 4)
        Q, K = synthetic.qk_inputs(hq=a.heads, hkv=hkv, n=a.seq or 4096)
        Q, K = Q.to(dev), K.to(dev)
        fn = lambda: rmm.qk(Q, K, a.rho, causal=True)
    elif a.case == "attention":
        hkv = max(1, a.heads // 4)
        Q, K = synthetic.qk_inputs(hq=a.heads, hkv=hkv, n=a.seq or 4096)
        V = synthetic.to_bf16(synthetic.rng(7).standard_normal(tuple(K.shape), dtype="float32"))
        Q, K, V = Q.to(dev), K.to(dev), V.to(dev)
        fn = lambda: rmm.attention(Q, K, V, a.rho, causal=True, scale=0.088)
    elif a.case == "decode_attn":
        Q, Kt, P, V = synthetic.decode_attention_inputs_device(dev, nk=a.seq or 32768)
        fn = lambda: (rmm.decode_qk(Q, Kt, a.rho, scale=0.088), rmm.decode_pv(P, V, a.rho))
    else:
        P, V = synthetic.pv_inputs_device(dev, heads=a.heads, n=a.seq or 16384)
        fn = lambda: rmm.pv(P, V, a.rho, causal=True)
    for _ in range(a.iters):
        fn()
    torch.cuda.synchronize(dev)
    err = rmm.device_error()
    print(f"{a.case}: {a.iters} calls done, device error word {err}")
    return 0 if err == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
