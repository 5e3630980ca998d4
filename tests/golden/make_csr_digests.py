"""Write csr_digests.json: SHA-256 digests of every array of the oracle's CSR
for the large periodic workloads (Fe BCC 65,536 and 524,288 atoms) at seeds
0, 1 and 2.

The GPU parity test (tests/test_gpu_build.py) hashes the device CSR of the
same seeded systems and compares, so that the full-size graphs are checked
edge for edge without running the brute-force oracle (about 2.7e11 pair
tests at 524,288 atoms) on every test run.  This script calls only the
oracle and the seeded input generators; it takes minutes on a few cores:

    python tests/golden/make_csr_digests.py [--keys 3 5] [--seeds 0 1 2]
"""
from __future__ import annotations

import argparse
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
from neighbour_graph_attention_b200 import configs as C  # noqa: E402

OUT = os.path.join(HERE, "csr_digests.json")
ARRAYS = {"row_ptr": np.int64, "src": np.int32, "shift": np.int32, "vec": np.float64,
          "dist": np.float64, "sw": np.float64}


def digests(csr) -> dict:
    """SHA-256 of each CSR array's bytes (C order, the library's dtypes)."""
    out = {}
    for k, dt in ARRAYS.items():
        a = np.ascontiguousarray(csr[k], dtype=dt)
        out[k] = hashlib.sha256(a.tobytes()).hexdigest()
    return out


def main(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--keys", type=int, nargs="+", default=[3, 5])
    p.add_argument("--seeds", type=int, nargs="+", default=[0, 1, 2])
    args = p.parse_args(argv)
    oracle.build()
    table = {}
    if os.path.exists(OUT):
        with open(OUT) as f:
            table = json.load(f).get("graphs", {})
    for key in args.keys:
        w = C.workload(key)
        for seed in args.seeds:
            s = C.system(key, seed)
            t0 = time.time()
            csr = oracle.build_csr(s["coords"], s["box"], s["pbc"], w.rcut, w.r_on, w.nnei_max)
            rec = {"workload": w.name, "n_atoms": w.n_atoms, "rcut": w.rcut, "r_on": w.r_on,
                   "nnei_max": w.nnei_max, "seed": seed, "n_edges": int(csr["row_ptr"][-1]),
                   "n_truncated": int(csr["n_truncated"]), "sha256": digests(csr)}
            table[f"{key}:{seed}"] = rec
            print(f"workload {key} seed {seed}: E = {rec['n_edges']}, "
                  f"{time.time() - t0:.0f} s", flush=True)
            with open(OUT, "w") as f:
                json.dump({"source": "oracle.build_csr (brute force over all images); "
                                     "written by tests/golden/make_csr_digests.py",
                           "graphs": table}, f, indent=1, sort_keys=True)
                f.write("\n")


if __name__ == "__main__":
    main()
