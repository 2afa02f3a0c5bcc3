"""Write oracle_regression.json from the oracle alone (no CUDA code involved)."""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import synth  # noqa: E402
from oracle import chunk_attention as ca  # noqa: E402
from oracle import fp8, mask_cache  # noqa: E402


def build():
    s = synth.tiny(n_chunks=6)
    out = {"workload": "tiny (seed 0), 6 chunks, W=2", "attention": {}}
    for t in (0, 3, 5):
        o = ca.chunk_attention(s.q[t], s.k, s.v, t, s.window)
        out["attention"][str(t)] = [float(x).hex() for x in o.reshape(-1)]
    m, d, tau = mask_cache.token_mask(s.src, s.edit, tau=s.tau)
    out["mask_tau1"] = m.tolist()
    out["dist"] = [float(x).hex() for x in d]
    md, _, taud = mask_cache.token_mask(s.src, s.edit, prune_quantile=0.7)
    out["mask_q070"] = md.tolist()
    out["tau_q070"] = float(taud).hex()
    vals = np.linspace(-500, 500, 257)
    out["e4m3_codes_linspace_-500_500_257"] = fp8.e4m3_encode(vals).tolist()
    return out


if __name__ == "__main__":
    with open(os.path.join(HERE, "oracle_regression.json"), "w") as f:
        json.dump(build(), f)
    print("wrote oracle_regression.json")
