"""Write the static E4M3 scales of the layers whose activations are E4M3:
  mixtral_prefill_fp8  Mixtral-shaped prefill, T=4096, H=4096, I=14336, E=8,
                       top-2, E4M3 weights and activations
  dsv3_decode_fp8      DeepSeek-V3-shaped decode, H=7168, I=2048, E=256 top-8
                       sigmoid x2.5 + 1 shared expert, E4M3 weights and
                       activations, calibrated on the 128 seeded tokens and
                       used for every batch of 1..128 of them

Static per-tensor FP8 ("tensor-quantized", as in "Mixture-of-Experts kernel
engineering on Amazon SageMaker AI", backend paragraph) needs one calibrated
scale per activation tensor.  The token scale a1 = amax(x)/448 comes with the
seeded inputs; the hidden scale is calibrated here, once, by the CPU oracle:
a2 = amax(h) / 448 over the routed and shared experts of the calibration
tokens (fp32).  Values of h beyond that amax saturate at 448 * a2 on both
sides.  Only the oracle and the seeded generator run here.

    python tests/golden/make_hidden_scale.py [workload ...]
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle as orc  # noqa: E402
from mixture_experts_layer_22_b200 import synthetic as syn  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))
# workload -> (tokens the layer is calibrated on, batch the tokens come from)
CALIB = {"mixtral_prefill_fp8": (64, None), "dsv3_decode_fp8": (128, 128)}


def write(name):
    n_tok, T = CALIB[name]
    wl = syn.WORKLOADS[name]
    if T is not None:
        wl = wl.with_T(T)
    d = syn.make_inputs(wl)
    amax = orc.hidden_amax(d["x"], d["logits"], d["w13"], E=wl.E, k=wl.k, n_shared=wl.n_shared,
                           gate=wl.gate, renorm=wl.renorm, routed_scale=wl.routed_scale, wdtype=wl.wdtype,
                           adtype=wl.adtype, w13_scale=d["w13_scale"], a1=d["a1"],
                           tokens=np.arange(n_tok, dtype=np.int32))
    a2 = float(np.float32(amax / 448.0))
    rec = {"workload": name, "a1": d["a1"], "a2": a2, "hidden_amax": amax,
           "calibration_tokens": n_tok, "seed": wl.seed,
           "source": "oracle/orc_hidden_amax on the seeded inputs; written by tests/golden/make_hidden_scale.py"}
    with open(os.path.join(HERE, f"{name}_hidden_scale.json"), "w") as f:
        json.dump(rec, f, indent=1)
    print(json.dumps(rec))


if __name__ == "__main__":
    for name in (sys.argv[1:] or sorted(CALIB)):
        write(name)
