"""Float64 oracle of the backward pass of one HSTU block (gradients of the
block of "MTGR: Industrial-Scale Generative Recommendation Framework in
Meituan", summary page, Method: the update equations). TEST INFRASTRUCTURE
ONLY (see the package docstring for who may import it).

The forward is the block of ``mtgr.hstu_block`` (variant 0):

  X~ = GroupLN_1(X);  Z = X~ W^T + b = [Q | K | V | U]
  per user and head: S = Q K^T, A = silu(S) (.) M / N, O = A V
  G = O (.) U;  G~ = GroupLN_2(G);  Z1 = G~ W1^T + b1;  H = silu(Z1)
  Y = H W2^T + b2 + X

and ``hstu_block_backward`` takes dY = dL/dY and returns dL/dX and the
gradients of every parameter, each written out by the chain rule in the
forward's notation (no automatic differentiation):

  dW2 = dY^T H, db2 = sum dY, dH = dY W2
  dZ1 = dH (.) silu'(Z1), silu'(z) = s(z) (1 + z (1 - s(z))), s the logistic
  dW1 = dZ1^T G~, db1 = sum dZ1, dG~ = dZ1 W1
  GroupLN backward (per token, xhat = (x - mu) / sigma, sigma = sqrt(var + eps)):
    dgamma_g = sum over the group's tokens of dy (.) xhat, dbeta_g = sum dy,
    dxhat = dy (.) gamma_g,
    dx = (dxhat - mean(dxhat) - xhat mean(dxhat (.) xhat)) / sigma
  dO = dG (.) U, dU = dG (.) O
  dA = dO V^T, dV = A^T dO, dS = dA (.) M / N (.) silu'(S), dQ = dS K, dK = dS^T Q
  dW = dZ^T X~, db = sum dZ, dX~ = dZ W;  dX = dX~ through GroupLN_1 + dY
"""

from __future__ import annotations

import numpy as np
from scipy.special import expit

from .mtgr import EPS, pack_offsets, user_mask


def _silu_grad(z: np.ndarray) -> np.ndarray:
    s = expit(z)
    return s * (1.0 + z * (1.0 - s))


def _gln_forward(x, gid, gamma, beta, eps):
    mu = x.mean(axis=1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=1, keepdims=True)
    sigma = np.sqrt(var + eps)
    xhat = (x - mu) / sigma
    return xhat * gamma[gid] + beta[gid], xhat, sigma


def _gln_backward(dy, xhat, sigma, gid, gamma):
    G = gamma.shape[0]
    dgamma = np.zeros_like(gamma)
    dbeta = np.zeros_like(gamma)
    for g in range(G):
        sel = gid == g
        dgamma[g] = (dy[sel] * xhat[sel]).sum(axis=0)
        dbeta[g] = dy[sel].sum(axis=0)
    dxhat = dy * gamma[gid]
    dx = (dxhat - dxhat.mean(axis=1, keepdims=True)
          - xhat * (dxhat * xhat).mean(axis=1, keepdims=True)) / sigma
    return dx, dgamma, dbeta


def hstu_block_backward(x: np.ndarray, lens: np.ndarray, ts: np.ndarray, p: dict, H: int,
                        dy: np.ndarray, norm: np.ndarray | None = None,
                        eps: float = EPS) -> dict:
    """Gradients of one HSTU block for the upstream gradient ``dy`` [T, d].

    Returns a dict with ``x`` [T, d] and one entry per parameter of ``p``
    (``gln1_gamma``, ``gln1_beta``, ``w_qkvu``, ``b_qkvu``, ``gln2_gamma``,
    ``gln2_beta``, ``w1``, ``b1``, ``w2``, ``b2``); the bias gradients are
    returned whether or not ``p`` holds the biases (absent biases are zero).
    """
    f64 = lambda a: np.asarray(a, np.float64)  # noqa: E731
    x, dy = f64(x), f64(dy)
    lens = np.asarray(lens, np.int64).reshape(-1, 4)
    _, user_off, gid = pack_offsets(lens)
    gid = np.asarray(gid, np.int64)
    T, d = x.shape
    dh = d // H
    g1, b1n, g2, b2n = f64(p["gln1_gamma"]), f64(p["gln1_beta"]), f64(p["gln2_gamma"]), f64(p["gln2_beta"])
    W, W1, W2 = f64(p["w_qkvu"]), f64(p["w1"]), f64(p["w2"])
    bq = f64(p["b_qkvu"]) if p.get("b_qkvu") is not None else np.zeros(4 * d)
    bb1 = f64(p["b1"]) if p.get("b1") is not None else np.zeros(W1.shape[0])
    bb2 = f64(p["b2"]) if p.get("b2") is not None else np.zeros(d)

    # forward, keeping what the backward reads
    xt, xhat1, sig1 = _gln_forward(x, gid, g1, b1n, eps)
    Z = xt @ W.T + bq
    Q, K, V, U = Z[:, :d], Z[:, d:2 * d], Z[:, 2 * d:3 * d], Z[:, 3 * d:]
    O = np.zeros((T, d))
    for b in range(lens.shape[0]):
        s, e = int(user_off[b]), int(user_off[b + 1])
        if e == s:
            continue
        M = user_mask(*(int(v) for v in lens[b]), ts[s:e]).astype(np.float64)
        Nb = float(e - s) if norm is None else float(norm[b])
        for h in range(H):
            c = slice(h * dh, (h + 1) * dh)
            S = Q[s:e, c] @ K[s:e, c].T
            A = S * expit(S) * M / Nb
            O[s:e, c] = A @ V[s:e, c]
    Gm = O * U
    gt, xhat2, sig2 = _gln_forward(Gm, gid, g2, b2n, eps)
    Z1 = gt @ W1.T + bb1
    Hm = Z1 * expit(Z1)

    # backward
    grads = {}
    grads["w2"] = dy.T @ Hm
    grads["b2"] = dy.sum(axis=0)
    dH = dy @ W2
    dZ1 = dH * _silu_grad(Z1)
    grads["w1"] = dZ1.T @ gt
    grads["b1"] = dZ1.sum(axis=0)
    dgt = dZ1 @ W1
    dG, grads["gln2_gamma"], grads["gln2_beta"] = _gln_backward(dgt, xhat2, sig2, gid, g2)
    dO = dG * U
    dU = dG * O
    dQ, dK, dV = np.zeros((T, d)), np.zeros((T, d)), np.zeros((T, d))
    for b in range(lens.shape[0]):
        s, e = int(user_off[b]), int(user_off[b + 1])
        if e == s:
            continue
        M = user_mask(*(int(v) for v in lens[b]), ts[s:e]).astype(np.float64)
        Nb = float(e - s) if norm is None else float(norm[b])
        for h in range(H):
            c = slice(h * dh, (h + 1) * dh)
            S = Q[s:e, c] @ K[s:e, c].T
            A = S * expit(S) * M / Nb
            dA = dO[s:e, c] @ V[s:e, c].T
            dV[s:e, c] = A.T @ dO[s:e, c]
            dS = dA * M / Nb * _silu_grad(S)
            dQ[s:e, c] = dS @ K[s:e, c]
            dK[s:e, c] = dS.T @ Q[s:e, c]
    dZ = np.concatenate([dQ, dK, dV, dU], axis=1)
    grads["w_qkvu"] = dZ.T @ xt
    grads["b_qkvu"] = dZ.sum(axis=0)
    dxt = dZ @ W
    dx1, grads["gln1_gamma"], grads["gln1_beta"] = _gln_backward(dxt, xhat1, sig1, gid, g1)
    grads["x"] = dx1 + dy
    return grads
