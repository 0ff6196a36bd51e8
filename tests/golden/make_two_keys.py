"""Writes two_keys.json: a two-key decode problem whose answer is a closed form.

Every query head h has one nonzero latent coordinate a_h (q_nope[0]) and one nonzero
RoPE coordinate b_h (q_pe[0]).  Cache row t has c_kv[0] = u_t, c_kv[5] = w_t and
k_pe[0] = v_t (column 512 of the 576-wide row); everything else is zero.  Hence

    s_t   = scale * (a_h * u_t + b_h * v_t)
    lse   = ln(e^{s_0} + e^{s_1})
    out[0] = p_0 u_0 + p_1 u_1,  out[5] = p_0 w_0 + p_1 w_1,  p_t = e^{s_t - lse}

and every other output coordinate is 0.  Computed here with the math module only
(no oracle code).  The two rows sit in physical block 1 (block table [1]).
"""
import json
import math
import os

scale = 0.125
u, w, v = [2.0, -1.0], [1.0, 4.0], [0.5, 3.0]
heads = []
for a, b in [(1.0, 0.0), (0.0, 2.0), (4.0, -1.0)]:
    s = [scale * (a * u[t] + b * v[t]) for t in range(2)]
    m = max(s)
    lse = m + math.log(sum(math.exp(x - m) for x in s))
    p = [math.exp(x - lse) for x in s]
    heads.append({
        "q_nope0": a, "q_pe0": b, "lse": lse,
        "out": {"0": p[0] * u[0] + p[1] * u[1], "5": p[0] * w[0] + p[1] * w[1], "1": 0.0, "511": 0.0},
    })
rows = [{"0": u[t], "5": w[t], "512": v[t]} for t in range(2)]
fixture = {"source": "closed form of a two-term softmax (see make_two_keys.py)",
           "scale": scale, "block_table": [1], "rows": rows, "heads": heads}
with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "two_keys.json"), "w") as f:
    json.dump(fixture, f, indent=1)
