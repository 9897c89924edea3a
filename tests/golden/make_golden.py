"""Writes tests/golden/tiny_decode_oracle.json: the oracle's decode step on the tiny workload.

Run from the repository root:  python tests/golden/make_golden.py
Only the oracle (oracle/sas_oracle.py) and the seeded input generator (synth/) are used; no
value comes from the CUDA library.  Floats are stored as hexadecimal strings (exact).
"""
from __future__ import annotations

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from oracle import sas_oracle as O  # noqa: E402
from synth import make_config  # noqa: E402

OUT = os.path.join(HERE, "tiny_decode_oracle.json")


def compute():
    import torch

    p = make_config("tiny", seed=0)
    f = lambda t: t.detach().to(torch.float64).numpy()
    q, K, V, M = f(p.q), f(p.K), f(p.V), f(p.M)
    seqlens, ks = p.seqlens.tolist(), p.k.tolist()
    kp = O.build_proj_cache(K, M, seqlens)
    res = O.decode_step(q, kp, K, V, M, seqlens, ks)
    heads = []
    for (b, h), (idx, out, u, keys) in sorted(res.items()):
        heads.append({"b": b, "h": h, "idx": [int(i) for i in idx],
                      "out": [[float(x).hex() for x in row] for row in out]})
    return {"workload": "tiny", "seed": 0, "source": "oracle/sas_oracle.py decode_step on synth.make_config('tiny', seed=0), "
            "projected cache built by the oracle (build_proj_cache)", "heads": heads}


if __name__ == "__main__":
    with open(OUT, "w") as fh:
        json.dump(compute(), fh, indent=0)
    print("wrote", OUT)
