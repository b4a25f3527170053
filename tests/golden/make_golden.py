"""Writes tests/golden/exact_small.json from the exact-rational oracle.

The pages print no numeric worked example, so the fixtures here are tiny
problems evaluated with no rounding at all (oracle/exact.py, Fractions) from
the update rule as printed: [EXPL] "Fast Weight Attention：用于持续学习的快速
权重注意力", 核心方法 1 (S_t = S_{t-1} - eta grad L, both gradients) and 2 (the
variant table); [NEWS] "借鉴40年前的设想！…", 02 (1) (decay by 1 - eta lambda,
eta normalised by the input scale) and (2) (scalar / per-value-channel /
sliding-window granularity).  Keys are picked with rational norms so that the
L2 feature map stays exact.

Run:  python tests/golden/make_golden.py
"""
from __future__ import annotations

import json
import os
import sys
from fractions import Fraction as Fr

sys.path.insert(0, os.path.join(os.path.dirname(os.path.abspath(__file__)), "..", ".."))
from oracle import exact  # noqa: E402

KEYS3 = [(1, 2, 2), (2, 3, 6), (1, 4, 8), (4, 4, 7), (2, 6, 9), (6, 6, 7), (0, 3, 4), (0, 0, 0),
         (-2, 1, 2)]


def F(*x):
    return Fr(*x)


def case(name, variant, pairing, phi, L, dv, lam, eps, window=1, beta_seed=1, keys=KEYS3):
    dk = len(keys[0])
    k = [[F(c) for c in keys[t % len(keys)]] for t in range(L)]
    q = [[F((t * 3 + c * 5) % 7 - 3, 2) for c in range(dk)] for t in range(L)]
    v = [[F((t * 5 + j * 3 + 1) % 9 - 4, 3) for j in range(dv)] for t in range(L)]
    if variant in ("F2", "F2A"):
        beta = [[F(1 + (t + j + beta_seed) % 4, 5) for j in range(dv)] for t in range(L)]
    else:
        beta = [F(1 + (t + beta_seed) % 4, 5) for t in range(L)]
    out, S = exact.unit(variant, q, k, v, beta, lam, eps, window, pairing, phi)
    s = lambda a: str(a)  # noqa: E731
    return {
        "name": name, "variant": variant, "pairing": pairing, "phi": phi, "window": window,
        "lam": s(lam), "eps": s(eps),
        "q": [[s(c) for c in r] for r in q], "k": [[s(c) for c in r] for r in k],
        "v": [[s(c) for c in r] for r in v],
        "beta": [[s(c) for c in r] if isinstance(r, list) else s(r) for r in beta],
        "out": [[s(c) for c in r] for r in out], "final_state": [[s(c) for c in r] for r in S],
    }


def main():
    cases = []
    for var in ("F1", "F2", "F3", "F1A", "F2A", "F3A"):
        w = 3 if var in ("F3", "F3A") else 1
        cases.append(case("%s-prefix-l2" % var, var, "prefix", "l2", 9, 2, F("1/20"), F("1/1000"), w))
        cases.append(case("%s-same-l2" % var, var, "same_step", "l2", 7, 2, F("1/10"), F(0), w))
        cases.append(case("%s-prefix-identity" % var, var, "prefix", "identity", 6, 3, F("1/8"),
                          F("1/2"), w))
    # positive-decay floor: a tiny key with eps = 0 gives eta = beta/|x|^2 huge, so
    # 1 - eta*lambda < 0 and the clamp alpha = 2^-20 takes over.
    cases.append(case("F1-floor", "F1", "prefix", "identity", 4, 2, F("1/2"), F(0), 1,
                      keys=[(F(1, 1000), 0, 0), (1, 0, 0), (0, F(1, 500), 0)]))
    doc = {
        "source": "exact rational evaluation (oracle/exact.py) of the update printed in "
                  "[EXPL] 核心方法 1-2 and [NEWS] 02 (1)-(2); no numbers are printed on the pages",
        "cases": cases,
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "exact_small.json")
    with open(path, "w") as f:
        json.dump(doc, f, indent=0)
    print("wrote", path, len(cases), "cases")


if __name__ == "__main__":
    main()
