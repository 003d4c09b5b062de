"""Writes the stored expected values under tests/golden/.

Calls only the oracle package (its exact rational brute force), never the CUDA
path.  Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import forms  # noqa: E402

# A hand-sized KDA example (d_k = d_v = 2, three tokens) with rational inputs,
# so that the update of "Hybrid Linear Attention Architecture: Making LLM
# Training and Inference More Efficient", section 3.3, can be followed by hand.
CASE = {
    "q": [[1, 0], [0.5, 0.5], [0, 1]],
    "k": [[0.6, 0.8], [1, 0], [0.8, -0.6]],
    "v": [[1, 2], [-1, 0.5], [0.25, -2]],
    "beta": [0.5, 0.75, 1.0],
    "alpha": [[1.0, 0.5], [0.25, 1.0], [0.5, 0.5]],
    "s0": [[0.5, -1.0], [2.0, 0.25]],
}


def main():
    outs, S = forms.exact_recurrence_fraction(CASE["q"], CASE["k"], CASE["v"], CASE["beta"],
                                              CASE["alpha"], CASE["s0"])
    doc = {
        "source": "KDA update, 'Hybrid Linear Attention Architecture: Making LLM Training and "
                  "Inference More Efficient' section 3.3; read-out after the write, "
                  "'Demystifying Hybrid LLM Architectures' section 2.3. Exact rational arithmetic.",
        "inputs": CASE,
        "o": [[f"{x.numerator}/{x.denominator}" for x in row] for row in outs],
        "final_state": [[f"{x.numerator}/{x.denominator}" for x in row] for row in S],
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "kda_rational_d2_t3.json")
    with open(path, "w") as f:
        json.dump(doc, f, indent=1)
        f.write("\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
