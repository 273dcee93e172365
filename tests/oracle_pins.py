"""Independent checks ("pins") of the fp64 oracle, shared by the oracle tests
and by the planted-mistake tests.

Each pin compares an oracle entry point against something that is not the
oracle: scalar loops written from the definition of a matrix product, torch's
own float64 autograd and tanh-GeLU, central finite differences, the erf form
of GELU, or the pages' partition invariant.  Each returns the worst error it
saw so a caller can assert on it (or, for a planted mistake, assert that it is
large).
"""
from __future__ import annotations

import math

import numpy as np
import torch


def tiny_problem(T=3, h=4, f=6, seed=1):
    """A small fp64 problem (values of bf16 magnitude, not rounded)."""
    rng = np.random.default_rng(seed)
    return {
        "X": rng.standard_normal((T, h)),
        "A": rng.standard_normal((h, f)) * 0.5,
        "a": rng.standard_normal(f) * 0.3,
        "B": rng.standard_normal((f, h)) * 0.5,
        "b": rng.standard_normal(h) * 0.3,
        "dY": rng.standard_normal((T, h)),
    }


def rel_err(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    return float(np.max(np.abs(x - ref)) / max(1e-300, np.max(np.abs(ref))))


# ---------------------------------------------------------------- brute force
def brute_force(p):
    """Scalar loops over every index: Z_tj = Σ_k X_tk A_kj + a_j, etc."""
    X, A, a, B, b, dY = (p[k] for k in ("X", "A", "a", "B", "b", "dY"))
    T, h = X.shape
    f = A.shape[1]
    c = math.sqrt(2.0 / math.pi)

    def g(x):
        return 0.5 * x * (1.0 + math.tanh(c * (x + 0.044715 * x ** 3)))

    Z = [[sum(X[t][k] * A[k][j] for k in range(h)) + a[j] for j in range(f)] for t in range(T)]
    H = [[g(Z[t][j]) for j in range(f)] for t in range(T)]
    Y = [[sum(H[t][j] * B[j][n] for j in range(f)) + b[n] for n in range(h)] for t in range(T)]
    # dH by differentiating g numerically is not brute force; use the chain
    # rule on the scalar definition: d/dx [½x(1+tanh u)] with u = c(x + kx³)
    def gp(x):
        u = c * (x + 0.044715 * x ** 3)
        return 0.5 * (1 + math.tanh(u)) + 0.5 * x * (1 - math.tanh(u) ** 2) * c * (1 + 3 * 0.044715 * x * x)

    dG = [[sum(dY[t][n] * B[j][n] for n in range(h)) for j in range(f)] for t in range(T)]
    dH = [[dG[t][j] * gp(Z[t][j]) for j in range(f)] for t in range(T)]
    dX = [[sum(dH[t][j] * A[k][j] for j in range(f)) for k in range(h)] for t in range(T)]
    dA = [[sum(X[t][k] * dH[t][j] for t in range(T)) for j in range(f)] for k in range(h)]
    da = [sum(dH[t][j] for t in range(T)) for j in range(f)]
    dB = [[sum(H[t][j] * dY[t][n] for t in range(T)) for n in range(h)] for j in range(f)]
    db = [sum(dY[t][n] for t in range(T)) for n in range(h)]
    return {k: np.array(v) for k, v in dict(Y=Y, Z=Z, H=H, dX=dX, dA=dA, da=da, dB=dB, db=db).items()}


# ---------------------------------------------------------------- library
def torch_autograd(p):
    """float64 torch: F.gelu(approximate='tanh') and autograd of <Y, dY>."""
    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=(k != "dY")) for k, v in p.items()}
    Z = t["X"] @ t["A"] + t["a"]
    H = torch.nn.functional.gelu(Z, approximate="tanh")
    Y = H @ t["B"] + t["b"]
    (Y * t["dY"]).sum().backward()
    return {"Y": Y.detach().numpy(), "Z": Z.detach().numpy(), "H": H.detach().numpy(),
            "dX": t["X"].grad.numpy(), "dA": t["A"].grad.numpy(), "da": t["a"].grad.numpy(),
            "dB": t["B"].grad.numpy(), "db": t["b"].grad.numpy()}


# ---------------------------------------------------------------- pins
def pin_brute_force(oracle, p):
    ref = brute_force(p)
    out = oracle.forward(p["X"], p["A"], p["a"], p["B"], p["b"])
    out.update(oracle.backward(p["dY"], p["X"], p["A"], p["a"], p["B"]))
    return max(rel_err(out[k], ref[k]) for k in ref)


def pin_autograd(oracle, p):
    ref = torch_autograd(p)
    out = oracle.forward(p["X"], p["A"], p["a"], p["B"], p["b"])
    out.update(oracle.backward(p["dY"], p["X"], p["A"], p["a"], p["B"]))
    return max(rel_err(out[k], ref[k]) for k in ref)


def pin_finite_difference(oracle, p, n_dir=3, eps=1e-6, seed=0):
    """Directional derivatives of L(X,A,a,B,b) = <Y, dY> by central differences
    against <grad, direction> from the oracle's backward."""
    rng = np.random.default_rng(seed)
    grads = oracle.backward(p["dY"], p["X"], p["A"], p["a"], p["B"])
    names = {"X": "dX", "A": "dA", "a": "da", "B": "dB", "b": "db"}

    def loss(q):
        Y = oracle.forward(q["X"], q["A"], q["a"], q["B"], q["b"])["Y"]
        return float(np.sum(Y * q["dY"]))

    worst = 0.0
    for name, gname in names.items():
        for _ in range(n_dir):
            d = rng.standard_normal(p[name].shape)
            qp = dict(p)
            qm = dict(p)
            qp[name] = p[name] + eps * d
            qm[name] = p[name] - eps * d
            fd = (loss(qp) - loss(qm)) / (2 * eps)
            an = float(np.sum(grads[gname] * d))
            worst = max(worst, abs(fd - an) / max(1.0, abs(an)))
    return worst


def pin_partition(oracle, p, t):
    """Sharded sum over t column/row shards equals the unsharded block."""
    full_f = oracle.forward(p["X"], p["A"], p["a"], p["B"], p["b"])
    full_b = oracle.backward(p["dY"], p["X"], p["A"], p["a"], p["B"])
    sf = oracle.forward_sharded(p["X"], p["A"], p["a"], p["B"], p["b"], t)
    sb = oracle.backward_sharded(p["dY"], p["X"], p["A"], p["a"], p["B"], t)
    errs = [rel_err(sf["Y"], full_f["Y"]), rel_err(sf["Z"], full_f["Z"]), rel_err(sf["H"], full_f["H"])]
    errs += [rel_err(sb[k], full_b[k]) for k in ("dX", "dA", "da", "dB", "db")]
    return max(errs)


def pin_gelu_library(oracle):
    x = np.linspace(-12, 12, 4001)
    ref = torch.nn.functional.gelu(torch.tensor(x, dtype=torch.float64), approximate="tanh").numpy()
    return float(np.max(np.abs(oracle.gelu(x) - ref)))


def pin_gelu_grad_fd(oracle):
    x = np.linspace(-8, 8, 1601)
    eps = 1e-5
    fd = (oracle.gelu(x + eps) - oracle.gelu(x - eps)) / (2 * eps)
    return float(np.max(np.abs(oracle.gelu_grad(x) - fd)))
