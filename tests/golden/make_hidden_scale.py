"""Write the static E4M3 scale of the hidden vector h for the Mixtral-shaped
FP8 prefill layer (T=4096, H=4096, I=14336, E=8, top-2, E4M3 weights and
activations).

Static per-tensor FP8 ("tensor-quantized", as in "Mixture-of-Experts kernel
engineering on Amazon SageMaker AI", backend paragraph) needs one calibrated
scale per activation tensor.  It is calibrated here, once, by the CPU oracle:
a2 = amax(h) / 448 over the routed and shared experts of the first
CALIB_TOKENS seeded tokens (fp32).  Values of h beyond that amax saturate at
448 * a2 on both sides.  Only the oracle and the seeded generator run here.

    python tests/golden/make_hidden_scale.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle as orc  # noqa: E402
from mixture_experts_layer_22_b200 import synthetic as syn  # noqa: E402

CALIB_TOKENS = 64
OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "mixtral_prefill_fp8_hidden_scale.json")


def main():
    wl = syn.WORKLOADS["mixtral_prefill_fp8"]
    d = syn.make_inputs(wl)
    amax = orc.hidden_amax(d["x"], d["logits"], d["w13"], E=wl.E, k=wl.k, n_shared=wl.n_shared,
                           gate=wl.gate, renorm=wl.renorm, routed_scale=wl.routed_scale, wdtype=wl.wdtype,
                           adtype=wl.adtype, w13_scale=d["w13_scale"], a1=d["a1"],
                           tokens=np.arange(CALIB_TOKENS, dtype=np.int32))
    a2 = float(np.float32(amax / 448.0))
    rec = {"workload": "mixtral_prefill_fp8", "a1": d["a1"], "a2": a2, "hidden_amax": amax,
           "calibration_tokens": CALIB_TOKENS, "seed": wl.seed,
           "source": "oracle/orc_hidden_amax on the seeded inputs; written by tests/golden/make_hidden_scale.py"}
    with open(OUT, "w") as f:
        json.dump(rec, f, indent=1)
    print(json.dumps(rec))


if __name__ == "__main__":
    main()
