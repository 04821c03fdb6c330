"""Writes tiny_closed_form.json: the 2-token case of the learned-relative attention
worked out by hand, evaluated from its closed-form expressions with Python's math
module (no oracle, no GPU code).

Case: B = 1, S = Skv = 2, Hq = Hkv = 1, D = 1 (scale 1), one document (positions
0, 1), all valid; q = [1, 1], k = [1, 0], v = [2, 4], profile rows [[0.5, 0], [0, 1]]
(profiles[b,h,i,d], the relative logit of distance d = pos_q - pos_k, added only for
d < relative_extent: Inkling2FlexAttention.forward on the NeMo AutoModel page
"nemo_automodel.components.models.inkling2.flex_attention"), sink = [0, ln 2 rounded
to FP32] (a virtual key with a zero value row: Inkling2Attention.forward on the
"...inkling2.attention" page).

Row 0 sees key 0 at distance 0: z = 1 + 0.5. Row 1 sees key 0 at distance 1
(z = 1 + profiles[1,1] = 2, or 1 when R = 1) and key 1 at distance 0 (z = 0 + 0).
lse = log(exp(sink) + sum exp z); out = sum exp(z - lse) v; with dout = 1:
Dv = out, dS = P (v - Dv), dsink = -exp(sink - lse) Dv, dprofiles[i, d] = dS.

python tests/golden/make_tiny_closed_form.py   (rewrites the file next to it)
"""
import json
import math
import os
import struct

S1 = struct.unpack("f", struct.pack("f", math.log(2.0)))[0]  # ln 2 rounded to FP32


def rows(R):
    z00 = 1.5
    z10 = 2.0 if R >= 2 else 1.0
    z11 = 0.0
    lse0 = math.log(1.0 + math.exp(z00))
    lse1 = math.log(math.exp(S1) + math.exp(z10) + math.exp(z11))
    p00 = math.exp(z00 - lse0)
    p10, p11 = math.exp(z10 - lse1), math.exp(z11 - lse1)
    out0, out1 = 2.0 * p00, 2.0 * p10 + 4.0 * p11
    return dict(lse=[lse0, lse1], out=[out0, out1], p=[p00, p10, p11])


def main():
    r2, r1 = rows(2), rows(1)
    p00, p10, p11 = r2["p"]
    out0, out1 = r2["out"]
    ps0 = math.exp(0.0 - r2["lse"][0])
    ps1 = math.exp(S1 - r2["lse"][1])
    e = math.e
    data = {
        "what": "learned-relative GQA attention, 2-token case worked by hand (see the generating script)",
        "citation": ("Inkling2FlexAttention.forward, NeMo AutoModel page "
                     "nemo_automodel.components.models.inkling2.flex_attention (profiles[b,h,i,d], "
                     "d = pos_q - pos_k, bias only for d < relative_extent, scale head_dim^-0.5); "
                     "Inkling2Attention.forward, ...inkling2.attention page (the sink acts as a virtual key whose value row is zero)"),
        "inputs": {"q": [1.0, 1.0], "k": [1.0, 0.0], "v": [2.0, 4.0], "profiles": [[0.5, 0.0], [0.0, 1.0]],
                   "sink": [0.0, S1], "positions": [0, 1]},
        "R2": {"out": r2["out"], "lse": r2["lse"]},
        "R1_row1": {"out": r1["out"][1], "lse": r1["lse"][1]},
        "plain_causal_zero_profiles_no_sink": {"out": [2.0, (2 * e + 4) / (e + 1)], "lse": [1.0, math.log(e + 1)]},
        "R2_backward_dout_ones": {
            "dsink": [-ps0 * out0, -ps1 * out1],
            "dprofiles_00_11_10": [p00 * (2.0 - out0), p10 * (2.0 - out1), p11 * (4.0 - out1)],
        },
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_closed_form.json")
    with open(path, "w") as f:
        json.dump(data, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
