"""Pins of the oracle's HSTU-block backward (the chain rule written out in
``oracle/backward.py``): against PyTorch autograd through an independent
float64 PyTorch statement of the forward, against central finite differences
of the oracle's own forward, and two closed forms."""

import numpy as np
import torch
import torch.nn.functional as F

import oracle
import synth

T64 = torch.float64


def _case(seed, bias=True, d=16, H=2, d_ff=24):
    rng = np.random.default_rng(seed)
    lens = np.array([[2, 5, 3, 3], [1, 3, 0, 2], [0, 0, 0, 0], [2, 2, 2, 1]], np.int64)
    ts = synth.make_timestamps(lens, rng)
    x = synth.make_tokens(lens, d, rng).astype(np.float64)
    p = {k: np.asarray(v, np.float64) for k, v in synth.make_block_params(d, d_ff, rng, dtype="f32").items()}
    if bias:
        p["b_qkvu"] = 0.1 * rng.standard_normal(4 * d)
        p["b1"] = 0.1 * rng.standard_normal(d_ff)
        p["b2"] = 0.1 * rng.standard_normal(d)
    dy = rng.standard_normal(x.shape)
    return lens, ts, x, p, H, dy


def _torch_block(x, lens, ts, p, H, eps=1e-5):
    """The block in float64 PyTorch ops (LayerNorm, Linear, SiLU), the mask
    from the oracle's pinned explicit M."""
    _, user_off, gid = oracle.pack_offsets(lens)
    gid = torch.as_tensor(np.asarray(gid, np.int64))
    d = x.shape[1]

    def gln(z, gamma, beta):
        return F.layer_norm(z, (d,), eps=eps) * gamma[gid] + beta[gid]

    xt = gln(x, p["gln1_gamma"], p["gln1_beta"])
    z = F.linear(xt, p["w_qkvu"], p.get("b_qkvu"))
    q, k, v, u = z.split(d, dim=1)
    dh = d // H
    rows = []
    for b in range(lens.shape[0]):
        s, e = int(user_off[b]), int(user_off[b + 1])
        if e == s:
            continue
        M = torch.as_tensor(oracle.user_mask(*(int(t) for t in lens[b]), ts[s:e]), dtype=T64)
        heads = []
        for h in range(H):
            c = slice(h * dh, (h + 1) * dh)
            S = q[s:e, c] @ k[s:e, c].T
            heads.append((F.silu(S) * M / (e - s)) @ v[s:e, c])
        rows.append(torch.cat(heads, dim=1))
    o = torch.cat(rows, dim=0)
    gt = gln(o * u, p["gln2_gamma"], p["gln2_beta"])
    hdn = F.silu(F.linear(gt, p["w1"], p.get("b1")))
    return F.linear(hdn, p["w2"], p.get("b2")) + x


def test_backward_matches_torch_autograd():
    lens, ts, x, p, H, dy = _case(0)
    got = oracle.hstu_block_backward(x, lens, ts, p, H, dy)
    tp = {k: torch.tensor(v, dtype=T64, requires_grad=True) for k, v in p.items()}
    tx = torch.tensor(x, dtype=T64, requires_grad=True)
    y = _torch_block(tx, lens, ts, tp, H)
    y.backward(torch.as_tensor(dy))
    np.testing.assert_allclose(got["x"], tx.grad.numpy(), rtol=1e-9, atol=1e-10)
    for k, v in tp.items():
        np.testing.assert_allclose(got[k], v.grad.numpy(), rtol=1e-9, atol=1e-10, err_msg=k)


def test_forward_of_the_backward_is_the_oracle_block():
    # the torch statement used above computes the oracle's block
    lens, ts, x, p, H, _ = _case(1)
    y = _torch_block(torch.as_tensor(x), lens, ts, {k: torch.as_tensor(v) for k, v in p.items()}, H)
    np.testing.assert_allclose(y.numpy(), oracle.hstu_block(x, lens, ts, p, H), rtol=1e-11, atol=1e-11)


def test_backward_matches_finite_differences():
    # L = sum(dY (.) Y): dL/dtheta by central differences of the oracle's own
    # forward at a handful of coordinates of every tensor
    lens, ts, x, p, H, dy = _case(2)
    got = oracle.hstu_block_backward(x, lens, ts, p, H, dy)
    rng = np.random.default_rng(7)
    h = 1e-6

    def loss(x_, p_):
        return float((oracle.hstu_block(x_, lens, ts, p_, H) * dy).sum())

    for name in ["x"] + sorted(p):
        base = x if name == "x" else p[name]
        for _ in range(4):
            idx = tuple(rng.integers(0, n) for n in base.shape)
            plus, minus = base.copy(), base.copy()
            plus[idx] += h
            minus[idx] -= h
            if name == "x":
                num = (loss(plus, p) - loss(minus, p)) / (2 * h)
            else:
                num = (loss(x, {**p, name: plus}) - loss(x, {**p, name: minus})) / (2 * h)
            ana = got[name][idx]
            assert abs(num - ana) <= 1e-5 * max(1.0, abs(num)), (name, idx, num, ana)


def test_zero_upstream_gradient_gives_zero_gradients():
    lens, ts, x, p, H, dy = _case(3)
    got = oracle.hstu_block_backward(x, lens, ts, p, H, np.zeros_like(dy))
    for k, v in got.items():
        assert not np.any(v), k


def test_output_weight_gradients_closed_form():
    # dW2 = dY^T H and db2 = sum dY whatever the rest of the block; with
    # W2 = 0 the input gradient is exactly dY (nothing flows back through the
    # MLP), and every gradient upstream of W2 vanishes
    lens, ts, x, p, H, dy = _case(4)
    p = dict(p)
    p["w2"] = np.zeros_like(p["w2"])
    got = oracle.hstu_block_backward(x, lens, ts, p, H, dy)
    np.testing.assert_array_equal(got["x"], dy)
    np.testing.assert_allclose(got["b2"], dy.sum(axis=0), rtol=1e-12, atol=1e-12)
    for k in ("w1", "b1", "gln2_gamma", "gln2_beta", "w_qkvu", "b_qkvu", "gln1_gamma", "gln1_beta"):
        assert not np.any(got[k]), k
