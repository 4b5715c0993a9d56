"""Write the exact-rational fixtures in this folder.

Each fixture is a tiny single-(sequence, head) case of the Gated DeltaNet
recurrence with rational inputs (alpha given directly as a rational decay),
and its exact outputs o_t and final state S_T computed with
``oracle.explicit_product_state(..., exact=True)``: the unrolled product form
S_T = S_0 M_1...M_T + sum_t beta_t v_t k_t^T M_{t+1}...M_T with
M_t = alpha_t (I - beta_t k_t k_t^T), evaluated in fractions.Fraction (no
rounding at all).  o_t = S_t q_t uses the product form over the first t
tokens.  The recurrence is the one of "NovaSky's IsoExec Fixes the Hidden Math
Bug Corrupting AI Training Runs", section "Solving the linear-attention
headache" (CPR keeps the recurrence as the primary algorithm); the pages print
no worked example, so these fixtures are computed, not quoted.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import random
import sys
from fractions import Fraction

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402


def rat(rng, lo, hi, den):
    return Fraction(rng.randint(lo * den, hi * den), den)


def case(seed, T, dk, dv):
    rng = random.Random(seed)
    q = [[rat(rng, -1, 1, 8) for _ in range(dk)] for _ in range(T)]
    k = [[rat(rng, -1, 1, 4) for _ in range(dk)] for _ in range(T)]
    v = [[rat(rng, -2, 2, 8) for _ in range(dv)] for _ in range(T)]
    beta = [Fraction(rng.randint(1, 8), 8) for _ in range(T)]
    alpha = [Fraction(rng.randint(1, 16), 16) for _ in range(T)]
    S0 = [[rat(rng, -1, 1, 4) for _ in range(dk)] for _ in range(dv)]
    o = []
    for t in range(1, T + 1):
        St = oracle.explicit_product_state(S0, k[:t], v[:t], beta[:t], alpha[:t], exact=True)
        o.append([sum((St[r][j] * q[t - 1][j] for j in range(dk)), Fraction(0)) for r in range(dv)])
    ST = oracle.explicit_product_state(S0, k, v, beta, alpha, exact=True)
    enc = lambda M: [[str(x) for x in row] for row in M]  # noqa: E731
    return {
        "what": "Gated DeltaNet recurrence, exact rationals, explicit product form",
        "seed": seed, "T": T, "dk": dk, "dv": dv,
        "q": enc(q), "k": enc(k), "v": enc(v),
        "beta": [str(x) for x in beta], "alpha": [str(x) for x in alpha],
        "S0": enc(S0), "o": enc(o), "S_T": enc(ST.tolist()),
    }


def main():
    for seed, T, dk, dv in [(11, 4, 2, 2), (12, 5, 3, 2), (13, 6, 3, 3), (14, 3, 4, 3)]:
        path = os.path.join(HERE, f"exact_T{T}_dk{dk}_dv{dv}.json")
        with open(path, "w") as f:
            json.dump(case(seed, T, dk, dv), f, indent=0)
        print("wrote", path)


if __name__ == "__main__":
    main()
