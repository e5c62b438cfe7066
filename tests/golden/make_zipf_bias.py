"""Writes tests/golden/zipf_bias_skewed.txt: the selection bias of the skewed
workload (Mixtral shape, T=16384, top-2 of 8, capacity factor 1.25).

The notes do not say how their Zipf-skewed loads were produced. Reading
taken: start from the seed-0 router inputs of the workload and run the
per-expert bias update of "Week 2 Day 2: Mixture of Experts" §4.2 / "Lecture
21" §2.4 (raise the bias of under-loaded experts, lower it for over-loaded
ones), but toward Zipf(s=1.2) target loads instead of uniform ones, with a
log-ratio step b_e += eta * (log target_e - log load_e), for a fixed number
of iterations. The bias acts on the logits (selection on z + b), gates stay
on the raw logits. The result is frozen and used as data.

Only the oracle computes here (router logits, top-k, permutation counts).
Run: python tests/golden/make_zipf_bias.py
"""

import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from oracle import moe_oracle as O  # noqa: E402
from mixture_experts_layer_62_b200 import inputs  # noqa: E402

ZIPF_S = 1.2
ITERS = 300
ETA = 0.5


def main():
    cfg = inputs.workload("skewed_capacity")
    cfg_nobias = dict(cfg, bias_mode=0)
    x, W_r, _ = inputs.make_routing_inputs(cfg_nobias, seed=0)
    z = O.router_logits(x.float().numpy(), W_r.float().numpy())
    T, E, k = cfg["T"], cfg["E"], cfg["k"]
    target = np.array([1.0 / (i + 1) ** ZIPF_S for i in range(E)])
    target /= target.sum()
    b = np.zeros(E)
    for _ in range(ITERS):
        idx = O.topk_lowest_index(O.selection_key(z, b, O.BIAS_LOGIT), k)
        counts = np.bincount(idx.reshape(-1), minlength=E)
        load = np.maximum(counts / (T * k), 1e-9)
        b += ETA * (np.log(target) - np.log(load))
        b -= b.mean()
    b32 = b.astype(np.float32)
    idx = O.topk_lowest_index(O.selection_key(z, b32.astype(np.float64), O.BIAS_LOGIT), k)
    counts = np.bincount(idx.reshape(-1), minlength=E)
    C = O.capacity(cfg["cf"], T, k, E)
    perm = O.permute(idx, E, C)
    path = os.path.join(HERE, "zipf_bias_skewed.txt")
    with open(path, "w") as fh:
        fh.write("# Selection bias (added to the router logits) of the skewed workload: Mixtral shape,\n")
        fh.write("# T=16384, top-2 of 8, capacity factor 1.25, seed-0 router inputs. Calibrated by\n")
        fh.write("# tests/golden/make_zipf_bias.py toward Zipf(1.2) loads with the per-expert bias\n")
        fh.write("# update of [CME295 W2D2] §4.2 / [CMU 15-779 L21] §2.4 (log-ratio step).\n")
        fh.write("# loads (oracle, fp64 logits): " + " ".join(f"{c / (T * k):.4f}" for c in counts) + "\n")
        fh.write("# targets: " + " ".join(f"{t:.4f}" for t in target) + "\n")
        fh.write(f"# capacity {C}: kept {int(perm.kept.sum())} of {T * k} pairs, "
                 f"dropped {int((perm.counts - perm.kept).sum())}\n")
        fh.write(" ".join(repr(float(v)) for v in b32) + "\n")
    print(path)
    print("loads", np.round(counts / (T * k), 4), "targets", np.round(target, 4))
    print("dropped", int((perm.counts - perm.kept).sum()), "of", T * k)


if __name__ == "__main__":
    main()
