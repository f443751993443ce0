"""Writes large_layer_T262144_seed0_reduced.txt: the reduced gradients of the
large-layer workload (262,144 tokens, 8 heads x 128, causal, seed 0) from the
fp64 oracle, so that the GPU parity test can compare them at full size without
re-running a whole-batch oracle backward on the GPU machine.

Two columns per value:
  exact    the oracle's layer backward in fp64 (d_rab_pos, d_rab_time, d_gamma, d_beta);
  model    the same backward in the oracle's bf16 error model: the tensor-core
           operands rounded to bf16 (A = SiLU(z) and dz before the matrix
           products) and the saved Y and the LayerNorm backward's dY stored in
           bf16, the roundings any bf16 tensor-core implementation has.

Only the oracle and the seeded generator are called.  Run from the repository
root:  python tests/golden/make_large_layer_reduced.py
"""
import os
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from hstu_jagged_pointwise_b200 import workloads as W  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "large_layer_T262144_seed0_reduced.txt")
KEYS = ("d_rab_pos", "d_rab_time", "dgamma", "dbeta")


def bf16(a):
    return torch.as_tensor(np.asarray(a, np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def main():
    w = W.large_layer(seed=0)
    t0 = time.time()
    y = oracle.attn_fwd(w)
    dy, du, dg, db = oracle.norm_bwd(w, y, w.grad)
    del du
    _, _, _, drp, drt = oracle.attn_bwd(w, dy)
    exact = dict(d_rab_pos=drp, d_rab_time=drt, dgamma=dg, dbeta=db)
    print(f"exact backward {time.time() - t0:.0f} s", flush=True)
    del y, dy
    with oracle.bf16_operands():
        yb = bf16(oracle.attn_fwd(w))
        dy_s, _, dg_s, db_s = oracle.norm_bwd(w, yb, w.grad)
        _, _, _, drp_s, drt_s = oracle.attn_bwd(w, bf16(dy_s))
    storage = dict(d_rab_pos=drp_s, d_rab_time=drt_s, dgamma=dg_s, dbeta=db_s)
    print(f"both backwards {time.time() - t0:.0f} s", flush=True)
    with open(OUT, "w") as f:
        f.write("# Reduced gradients of the large-layer workload (T=262144, H=8, d=128, causal, seed 0)\n")
        f.write("# from the fp64 oracle; written by make_large_layer_reduced.py.  Columns: name index exact model\n")
        for k in KEYS:
            for i, (a, b) in enumerate(zip(exact[k], storage[k])):
                f.write(f"{k} {i} {float(a)!r} {float(b)!r}\n")
    print("wrote", OUT)


if __name__ == "__main__":
    main()
