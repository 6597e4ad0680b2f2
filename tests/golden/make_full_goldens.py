"""Write the full-layer oracle results that the full-size GPU tests compare with.

    python tests/golden/make_full_goldens.py [workload ...]

For each named single-layer workload (default: llama7b_attn_proj and
llama7b_mlp_down) this draws the seeded synthetic layer, computes the
activation statistic with the oracle, runs the oracle's grid search over
EVERY output column and every alpha, and writes
tests/golden/full_<workload>.json with all L(alpha), the argmin and a digest
of the input bytes.  It calls only oracle/ (and the input generators); no
value in the files comes from the CUDA path.  Expect minutes per workload on
a many-core host (the oracle is plain fp64 loops, OpenMP over columns).
"""
from __future__ import annotations

import hashlib
import json
import os
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from post_weight_only_b200 import synth  # noqa: E402

DEFAULT = ("llama7b_attn_proj", "llama7b_mlp_down")


def input_digest(X, W) -> str:
    """sha1 of the bf16 bytes of X followed by the fp32 bytes of W."""
    import torch
    h = hashlib.sha1()
    h.update(X.contiguous().view(torch.int16).numpy().tobytes())
    h.update(W.contiguous().numpy().tobytes())
    return h.hexdigest()


def make(name: str) -> dict:
    wl = synth.workload(name)
    assert len(wl.layers) == 1 and len(wl.quant) == 1, "single-layer, single-setting workloads only"
    layer = wl.layers[0]
    bits, group = wl.quant[0]
    X, W = synth.layer_inputs(layer)
    alphas = synth.alpha_grid(wl.n_intervals).numpy()
    a = oracle.act_stats(X).astype(np.float32)
    t0 = time.time()
    L, best = oracle.search(X, W, a, alphas, bits, group)
    dt = time.time() - t0
    cmd = "python tests/golden/make_full_goldens.py " + name
    return {
        "_source": "compassingai.com AWQ concept page, 'full scale-optimisation flow', steps 2-5: "
                   "a_j = mean|X_j|, s = a^alpha for alpha in {0, 0.05, ..., 1}, "
                   "L(alpha) = ||X S^-1 Q(S W) - X W||^2 over the whole layer, alpha* = argmin L.",
        "_how": f"written by `{cmd}`: oracle.act_stats (fp64, rounded to fp32), then oracle.search over all "
                f"{layer.D_out} output columns and {len(alphas)} alphas ({dt:.0f} s on "
                f"{oracle.num_threads()} threads). Inputs: synth.layer_inputs of the workload.",
        "workload": name,
        "N": layer.N, "D_in": layer.D_in, "D_out": layer.D_out, "bits": bits, "group": group,
        "input_sha1": input_digest(X, W),
        "alphas": [float(v) for v in alphas],
        "a_sum": float(np.sum(a.astype(np.float64))),
        "L": [float(v) for v in L],
        "alpha_idx": int(best),
        "alpha_star": float(alphas[best]),
    }


def main(argv):
    names = argv or list(DEFAULT)
    for name in names:
        d = make(name)
        path = os.path.join(HERE, f"full_{name}.json")
        with open(path, "w") as f:
            json.dump(d, f, indent=1)
            f.write("\n")
        print(f"{path}: alpha* = {d['alpha_star']} (index {d['alpha_idx']})", flush=True)


if __name__ == "__main__":
    main(sys.argv[1:])
