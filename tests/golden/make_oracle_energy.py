"""Writes tests/golden/oracle_energy.json: the CPU oracle's free-running
energy traces on the seeded workloads, for the free-running parity tests at
sizes the oracle cannot redo inside a test.  Calls only oracle/ and the
seeded input generator.  Usage: python tests/golden/make_oracle_energy.py [name ...]
"""
import json
import os
import sys
import time
from concurrent.futures import ProcessPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
OUT = os.path.join(ROOT, "tests", "golden", "oracle_energy.json")


def _workloads():
    from expanded_rank_matrix_b200 import workloads as W
    return {
        "iid256": W.config_small,
        "llm1024_tau0.3": lambda: W.config_llm1024(0.3),
        "llm1024_tau0.5": lambda: W.config_llm1024(0.5),
        "llm1024_tau0.7": lambda: W.config_llm1024(0.7),
        "attn2560": W.config_attn2560,
        "mlp9728_b64": lambda: W.config_mlp9728(64),
        "mlp9728_b1": lambda: W.config_mlp9728(1),
        **{f"blk_{nm}": (lambda i=i: W.config_block_matrices(64)[i])
           for i, (nm, _, _) in enumerate(W.BLOCK_MATRICES)},
    }


def run(name):
    from oracle import ref
    wl = _workloads()[name]()
    t = time.time()
    dec = ref.decompose(wl.a, wl.k, wl.tau, wl.iters, w=wl.w, block=wl.block)
    dt = time.time() - t
    k = wl.k
    marks = sorted(set([0, 1, 2, 3, 7, 15, 31, 63, 127, 255, 511, 1023, 2047, 4095, k // 2, k - 1]))
    marks = [c for c in marks if c < k]
    return name, {
        "m": wl.m, "n": wl.n, "mu": wl.mu, "tau": wl.tau, "iters": wl.iters, "block": wl.block,
        "k": k, "seed": wl.meta.get("seed"), "final_energy": float(dec.energy[-1]),
        "energy_at": {str(c): float(dec.energy[c]) for c in marks},
        "n_fallback": int(dec.n_fallback),
        "zero_frac_B": float((dec.U == 0).mean()), "zero_frac_C": float((dec.V == 0).mean()),
        "oracle_seconds": dt,
    }


if __name__ == "__main__":
    names = sys.argv[1:] or list(_workloads().keys())
    data = json.load(open(OUT)) if os.path.exists(OUT) else {}
    data["_source"] = ("CPU oracle (oracle/externd_ref.cpp), free-running, single thread; "
                       "written by tests/golden/make_oracle_energy.py")
    with ProcessPoolExecutor(max_workers=min(len(names), 7)) as ex:
        for name, rec in ex.map(run, names):
            data[name] = rec
            print(name, rec["final_energy"], f"{rec['oracle_seconds']:.1f}s", flush=True)
            json.dump(data, open(OUT, "w"), indent=1, sort_keys=True)
