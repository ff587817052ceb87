"""Writes closed_form_three_tokens.json: a hand-derived decode example.

The expected values are closed forms (see "derivation" in the file); this
script evaluates them with the ``math`` module only.  It calls no library code
and no CUDA path.  Run: ``python tests/golden/make_closed_form.py``.
"""
import json
import math
import os

C = 0.5  # rope contribution shared by every token


def build() -> dict:
    out0 = (0 * 1 + 2 * math.log(2) + 3 * math.log(3)) / 6
    rows = []
    for j, a in enumerate((6.0, 0.0, -6.0)):
        rows.append({"0": math.log(j + 1), "1": a, "2": 1.0, "512": C, "520": 7.0})
    return {
        "citation": ("MLA 和 MHA 的 Kernel 区别 (sealessland.top), section 'Decode 阶段的 HBM 访问模式 / "
                     "MLA Decode': score each cached token against the query, softmax, weighted sum of "
                     "values; absorbed layout: 576-wide row = 512 latent + 64 rope, value = first 512 dims"),
        "derivation": [
            "softmax_scale = 1; q = e_0 + e_512 (one latent dim, one rope dim); L = 3 tokens in one page",
            "k_j[0] = ln(j+1), k_j[1] = (6, 0, -6)[j], k_j[2] = 1, k_j[512] = c = 0.5 (rope), "
            "k_j[520] = 7 (rope, q[520] = 0)",
            "z_j = ln(j+1) + c, so the weights are (1, 2, 3) / 6 and lse = ln 6 + c",
            "value = first 512 dims: out[0] = (0 + 2 ln 2 + 3 ln 3) / 6, out[1] = (6 - 18) / 6 = -2, "
            "out[2] = 1, all other dims 0",
            "the rope dims (512..575) enter the score but not the value",
        ],
        "softmax_scale": 1.0,
        "L": 3,
        "q_nonzero": {"0": 1.0, "512": 1.0},
        "k_rows_nonzero": rows,
        "expected_out_nonzero": {"0": out0, "1": -2.0, "2": 1.0},
        "expected_lse": math.log(6) + C,
    }


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "closed_form_three_tokens.json")
    with open(path, "w") as f:
        json.dump(build(), f, indent=1)
