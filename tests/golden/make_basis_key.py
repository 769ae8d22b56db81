"""Writes basis_key_e5.json: the worked example of a basis key, derived by hand from the
definitions of "Technical Summary: ParisKV" (Core Algorithmic Innovations 1 and 2) -- it
calls neither the oracle nor the CUDA library; the only arithmetic is the Sylvester sign rule
and the closed forms written in the fixture's derivation.

    python tests/golden/make_basis_key.py
"""
import json
import math
import os

IDX, SCALE = 5, 3.0


def main():
    # Sylvester H[i][IDX] = (-1)^popcount(i & IDX); within a subspace i = 8b + j and IDX < 8
    neg = [j for j in range(8) if bin(j & IDX).count("1") % 2 == 1]
    own = sum(1 << j for j in neg)
    neigh = sorted(own ^ (1 << j) for j in range(8))[:3]
    fix = {
        "source": "\"Technical Summary: ParisKV\", Methodology, Core Algorithmic Innovations 1 "
                  "(Normalization and Rotation, Analytic Centroids) and 2 (Coarse Candidate "
                  "Generation, Quantization, Calibration, Estimation); readings R1-R8, R11 of "
                  "the design notes",
        "derivation": [
            "k = 3 e_5, all SRHT signs +1: ||k|| = 3, k^ = e_5, y = H e_5 / sqrt(128) = column 5 "
            "of the Sylvester Hadamard matrix / sqrt(128).",
            "Sylvester H[i][5] = (-1)^popcount(i & 5); since 5 = 0b101, for i = 8b + j it is "
            "(-1)^popcount(j & 5): negative for j in {1, 3, 4, 6}.",
            "Bucket id of every subspace (bit j = y_j < 0): 2 + 8 + 16 + 64 = 90.",
            "All |y_j| equal 1/sqrt(128): every magnitude is the top uniform level, 7; the "
            "code's sign bit is the id bit.",
            "Factor f_b = ||k|| * sum_j y_j^2 / sum_j vt_j y_j = 3 * (8/128) / (56/sqrt(128)) "
            "= 3 / (7 sqrt(128)).",
            "Query q = e_5 gives q~ = y and ||q|| = 1: its own pattern 90 has penalty 0; the 8 "
            "patterns one bit away tie at 1/sqrt(128); ties go to the lower id, so with rho = 4 "
            "the vote table holds 90 -> 2 and the three lowest one-bit neighbours -> 1.",
            "Estimate: ||q|| * sum_b f_b <vt_b, q~_b> = 16 * (3 / (7 sqrt(128))) * "
            "(56 / sqrt(128)) = 3 = <k, q>.",
        ],
        "key_scale": SCALE, "basis_index": IDX,
        "ids": [own] * 16,
        "magnitude": 7,
        "negative_dims_in_subspace": neg,
        "factor": SCALE / (7.0 * math.sqrt(128.0)),
        "lut_rho4": {str(own): 2, **{str(c): 1 for c in neigh}},
        "estimate": SCALE,
    }
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "basis_key_e5.json")
    with open(out, "w") as f:
        json.dump(fix, f, indent=1)


if __name__ == "__main__":
    main()
