"""Writes hand_worked_producer_d1.json: three tokens of the write-term producer with d = 1 and
L = 2, worked step by step (anchor by the width-4 causal convolution, GELU(z) = z Phi(z) with
Phi(z) = (1 + erf(z / sqrt 2)) / 2, residual r <- r - delta), after "PRISM: Parallel Residual
Iterative Sequence Model" (gist.science explainer), technical summary 2.2, and the banbantang.com
PRISM article, section 3(4) (first residual = the input itself).  Plain arithmetic only: it does
not call the oracle it checks."""
import json
import math
import os

phi = lambda z: 0.5 * (1.0 + math.erf(z / math.sqrt(2.0)))
x, v = [1.0, 2.0, -2.0], [1.0, 0.4, 2.0]
c = [1.0, 0.5, 0.0, 0.0]          # c_0 multiplies x_t, c_1 x_{t-1}
Wk, Wp = [2.0, -1.0], [1.0, 1.0]  # per rank l = 1, 2 (d = 1)
beta = [[1.0, 0.5], [0.5, 1.0], [2.0, 1.0]]
derivation, u, w, r_final = [], [], [], []
for t in range(3):
    a = sum(c[j] * x[t - j] for j in range(4) if t - j >= 0)
    r, args, deltas, res = v[t], [], [], [v[t]]
    for l in range(2):
        z = (Wp[l] * a) * r
        dl = z * phi(z)
        args.append(z)
        deltas.append(dl)
        r = r - dl
        res.append(r)
    derivation.append({"t": t, "anchor": a, "gelu_args": args, "deltas": deltas, "residuals": res})
    u.append([[beta[t][l] * deltas[l]] for l in range(2)])
    w.append([[Wk[l] * a] for l in range(2)])
    r_final.append([r])
out = {
    "_what": "d = 1, L = 2, T = 3, one head: anchors 1, 2.5, -1; first GELU arguments 1, 1, -2 "
             "(written by tests/golden/make_hand_worked_producer.py, plain arithmetic)",
    "derivation": derivation,
    "x": [[[[xv]] for xv in x]], "v": [[[[vv]] for vv in v]],
    "conv": [[[cv] for cv in c]],
    "Wk": [[[[Wk[0]]], [[Wk[1]]]]], "Wp": [[[[Wp[0]]], [[Wp[1]]]]],
    "beta": [[[b] for b in beta]],
    "u": [[[ut] for ut in u]], "w": [[[wt] for wt in w]], "r_final": [[[rt] for rt in r_final]],
}
# shapes: x, v [B=1][T][H=1][d=1]; conv [H][4][d]; Wk, Wp [H][L][d][d]; beta [B][T][H][L];
# u, w [B][T][H][L][d]; r_final [B][T][H][d]
out["x"] = [[[[xv]] for xv in x]]
out["v"] = [[[[vv]] for vv in v]]
out["beta"] = [[[beta[t]] for t in range(3)]]
out["u"] = [[[u[t]] for t in range(3)]]
out["w"] = [[[w[t]] for t in range(3)]]
out["r_final"] = [[[r_final[t]] for t in range(3)]]
with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "hand_worked_producer_d1.json"), "w") as f:
    json.dump(out, f, indent=1)
print("written")
