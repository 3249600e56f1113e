"""Writes closed_forms.json: textbook values used to pin the oracle.

Uses only the Python `math` module (never the oracle or the CUDA path):
  * Bernoulli KL: KL(p||q) = p ln(p/q) + (1-p) ln((1-p)/(1-q))  (definition of
    the Kullback-Leibler divergence for a two-outcome distribution).
  * RMSNorm of [3, 4] with eps = 0 and unit gains: x / sqrt((9 + 16) / 2).
  * SiLU(1) = 1 / (1 + e^-1).
  * Rotate-half rotary embedding of x = [1, 2, 3, 4] (head_dim 4, theta 1e4) at
    position 1: pairs (x0, x2) turn by 1 rad and (x1, x3) by 1e4^(-1/2) rad.
Run: python tests/golden/make_closed_forms.py
"""
import json
import math
import os

out = {}
p, q = 0.7, 0.4
out["bernoulli_kl"] = {"p": [p, 1 - p], "q": [q, 1 - q],
                       "kl": p * math.log(p / q) + (1 - p) * math.log((1 - p) / (1 - q)),
                       "source": "definition of KL divergence, two outcomes"}
r = math.sqrt((9 + 16) / 2)
out["rmsnorm_3_4"] = {"x": [3.0, 4.0], "eps": 0.0, "y": [3 / r, 4 / r],
                      "source": "RMSNorm definition x / sqrt(mean(x^2) + eps)"}
out["silu_1"] = {"x": 1.0, "y": 1.0 / (1.0 + math.exp(-1.0)), "source": "SiLU x*sigmoid(x)"}
a0, a1 = 1.0, 1e4 ** (-0.5)
x = [1.0, 2.0, 3.0, 4.0]
out["rope_dh4_pos1"] = {
    "x": x, "pos": 1, "theta": 1e4,
    "y": [x[0] * math.cos(a0) - x[2] * math.sin(a0), x[1] * math.cos(a1) - x[3] * math.sin(a1),
          x[2] * math.cos(a0) + x[0] * math.sin(a0), x[3] * math.cos(a1) + x[1] * math.sin(a1)],
    "source": "rotate-half rotary embedding, pair (i, i + dh/2) turned by pos * theta^(-2i/dh)"}
with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "closed_forms.json"), "w") as f:
    json.dump(out, f, indent=1)
