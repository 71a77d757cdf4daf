"""Writes tests/golden/tiny_prefix6.json: the brute-force enumeration of the
tiny workload (L=8, k=2, V=1, T=0.5, codebook seed 0, weights seed 1) on its
first 6 steps, every one of its 256 * 4^5 paths summed in fp64.

Source of the definition: "BCJR-QAT: A Differentiable Relaxation of
Trellis-Coded Weight Quantization", Abstract (soft codeword = Boltzmann
expectation over trellis paths) and Technical Summary, "Core Mechanism"
(w_hat_t = sum_s c(s) p_T(s_t = s | w)).  Calls only ``oracle.reference``.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from bcjr_sum_product_b200 import inputs as I  # noqa: E402  (seeded draws only)
from oracle import reference as R  # noqa: E402


def main():
    inp = I.make("tiny")
    w6 = inp.w[:, :6].contiguous()
    out = {"workload": "tiny (L=8,k=2,V=1,T=0.5), first 6 steps", "method": "brute-force path enumeration, fp64",
           "logZ": [], "soft": [], "viterbi_energy_fp64": []}
    for q in range(w6.shape[0]):
        b = R.brute_force(w6[q], inp.c, 8, 2, 1, 0.5)
        out["logZ"].append(b["logZ"])
        out["soft"].append([float(x) for x in b["soft"]])
        out["viterbi_energy_fp64"].append(b["Emin"])
    with open(os.path.join(HERE, "tiny_prefix6.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
