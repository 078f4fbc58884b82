"""Writes summary_two_keys.json: a hand-worked landmark summary.

Closed form from the HiLS notes ("Hierarchical Sparse Attention Done Right"),
section 5.1, with d = 1 and scale 1 so the logits are the products l*k_j:
keys [0, ln 3], landmark 1 -> p = [1/4, 3/4], kbar = (3/4) ln 3,
H = ln 4 - (3/4) ln 3; the score at query q is q*kbar + H and the exact
chunk log-mass is ln(1 + 3^q).  Pure arithmetic, no oracle call.
"""
import json
import math
import os

QUERIES = [1.0, 0.0, 2.0]


def main():
    ln3 = math.log(3.0)
    d = {
        "citation": "HiLS notes 'Hierarchical Sparse Attention Done Right', section 5.1 "
                    "(s_j, p_j, k'_c, b'_c); hand-worked with d = 1, scale = 1.",
        "keys": [[0.0], [ln3]],
        "landmark": [1.0],
        "scale": 1.0,
        "p": [0.25, 0.75],
        "kbar": [0.75 * ln3],
        "hbias": math.log(4.0) - 0.75 * ln3,
        "queries": QUERIES,
        "score": [0.75 * ln3 * q + math.log(4.0) - 0.75 * ln3 for q in QUERIES],
        "exact_log_mass": [math.log(1.0 + 3.0 ** q) for q in QUERIES],
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "summary_two_keys.json")
    with open(path, "w") as f:
        json.dump(d, f, indent=1)


if __name__ == "__main__":
    main()
