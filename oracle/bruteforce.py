"""Pure-Python loop forms of the oracle for tiny inputs.

TEST INFRASTRUCTURE ONLY.  These are written with explicit loops over
Python floats (no NumPy arithmetic) so that the vectorised oracle can be
checked against an independent spelling of the same definitions:

* codes c_j = sum_i P[i][j] x_i (Half the Memory, section 04);
* attention over reconstructed keys/values, k^_i = sum_j P_k[i][j] c_j,
  with anchors joining the softmax (section 08; OjaKV page anchors);
* one Oja step y = P^T x, P <- P + eta (x - P y) y^T (OjaKV page).
"""
import math


def codes(P, X):
    d, r = len(P), len(P[0])
    return [[sum(P[i][j] * x[i] for i in range(d)) for j in range(r)] for x in X]


def recon(P, C):
    d, r = len(P), len(P[0])
    return [[sum(P[i][j] * c[j] for j in range(r)) for i in range(d)] for c in C]


def attention(q, P_k, P_v, C_k, C_v, K_anc, V_anc, scale):
    """Softmax attention of q over reconstructed latent rows and anchors."""
    keys = recon(P_k, C_k) + [list(k) for k in K_anc]
    vals = recon(P_v, C_v) + [list(v) for v in V_anc]
    d = len(q)
    scores = [sum(q[i] * k[i] for i in range(d)) * scale for k in keys]
    m = max(scores)
    w = [math.exp(s - m) for s in scores]
    tot = sum(w)
    return [sum(w[t] * vals[t][i] for t in range(len(vals))) / tot
            for i in range(d)]


def oja_step(P, x, eta):
    d, r = len(P), len(P[0])
    y = [sum(P[i][j] * x[i] for i in range(d)) for j in range(r)]
    z = [x[i] - sum(P[i][j] * y[j] for j in range(r)) for i in range(d)]
    return [[P[i][j] + eta * z[i] * y[j] for j in range(r)] for i in range(d)]
