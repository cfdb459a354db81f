"""Pins of the oracle's token MLPs and CTR/CTCVR heads (blog posts,
"Converting heterogeneous features into tokens"; summary page, Method;
fun-rec 7.3.3): the packed order from a hand-written fixture, the MLP against
PyTorch's functional layers, closed forms, and candidate independence."""

import os

import numpy as np
import torch
import torch.nn.functional as F
from scipy.special import expit

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "token_layout_two_users.txt")


def _golden():
    lines = [l.strip() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    i = lines.index("lens")
    j = lines.index("order")
    k = lines.index("candidates")
    lens = np.array([[int(v) for v in l.split()] for l in lines[i + 1:j]], np.int64)
    order = lines[j + 1].split()
    cands = [int(v) for v in lines[k + 1].split()]
    return lens, order, cands


def _params(rng, d, f, bias=True):
    p = {}
    for name, fin in zip(oracle.tokens.DOMAINS, f):
        p["w1_" + name] = rng.standard_normal((d, fin)) / np.sqrt(fin)
        p["w2_" + name] = rng.standard_normal((d, d)) / np.sqrt(d)
        p["b1_" + name] = rng.standard_normal(d) * 0.1 if bias else None
        p["b2_" + name] = rng.standard_normal(d) * 0.1 if bias else None
    return p


def test_packed_order_matches_fixture():
    # identity MLPs (F = d, W1 = W2 = I, no bias) make every S/R/C token
    # silu(e); each input row carries a code naming its domain and index
    lens, order, _ = _golden()
    d = 8
    code = {"u": 1000.0, "s": 2000.0, "r": 3000.0, "c": 4000.0}
    e = []
    for g, name in enumerate("usrc"):
        n = int(lens[:, g].sum())
        rows = np.zeros((n, d))
        rows[:, 0] = code[name] + np.arange(n)
        e.append(rows)
    eye = np.eye(d)
    p = {k + "_" + n: (eye if k.startswith("w") else None) for n in "src" for k in ("w1", "b1", "w2", "b2")}
    x = oracle.tokenize(lens, e, p)
    assert x.shape == (len(order), d)
    for row, name in zip(x, order):
        v = code[name[0]] + int(name[1:])
        want = v if name[0] == "u" else v * expit(v)  # silu of a large positive value
        assert row[0] == want, (name, row[0], want)


def test_token_mlp_matches_torch_functional():
    rng = np.random.default_rng(0)
    e = rng.standard_normal((7, 24))
    w1, b1 = rng.standard_normal((16, 24)), rng.standard_normal(16)
    w2, b2 = rng.standard_normal((16, 16)), rng.standard_normal(16)
    t = lambda a: torch.as_tensor(a, dtype=torch.float64)  # noqa: E731
    ref = F.linear(F.silu(F.linear(t(e), t(w1), t(b1))), t(w2), t(b2)).numpy()
    np.testing.assert_allclose(oracle.token_mlp(e, w1, b1, w2, b2), ref, rtol=1e-12, atol=1e-12)
    ref0 = F.linear(F.silu(F.linear(t(e), t(w1))), t(w2)).numpy()
    np.testing.assert_allclose(oracle.token_mlp(e, w1, None, w2, None), ref0, rtol=1e-12, atol=1e-12)


def test_tokenize_domains_use_their_own_weights():
    # zero first-layer weights: a domain's tokens are W2_g silu(b1_g) + b2_g,
    # one constant row per domain; U rows are the inputs
    rng = np.random.default_rng(1)
    lens = np.array([[2, 3, 1, 2], [1, 0, 2, 3]])
    d, f = 8, (16, 8, 24)
    p = _params(rng, d, f)
    for n in "src":
        p["w1_" + n] = np.zeros_like(p["w1_" + n])
    e = [rng.standard_normal((int(lens[:, g].sum()), d if g == 0 else f[g - 1])) for g in range(4)]
    x = oracle.tokenize(lens, e, p)
    _, _, gid = oracle.pack_offsets(lens)
    np.testing.assert_array_equal(x[gid == 0], e[0])
    for g, n in enumerate("src", start=1):
        const = p["w2_" + n] @ (p["b1_" + n] * expit(p["b1_" + n])) + p["b2_" + n]
        np.testing.assert_allclose(x[gid == g], np.broadcast_to(const, (int((gid == g).sum()), d)),
                                   rtol=1e-12, atol=1e-12)


def _head_params(rng, d, d_h, n_tasks=2):
    return dict(w1=rng.standard_normal((n_tasks, d_h, d)) / np.sqrt(d),
                b1=rng.standard_normal((n_tasks, d_h)) * 0.1,
                w2=rng.standard_normal((n_tasks, d_h)) / np.sqrt(d_h),
                b2=rng.standard_normal(n_tasks) * 0.1)


def test_heads_read_candidate_rows_in_order():
    # x[i, 0] = i; task 0 = silu(x_c[0]), task 1 = b2[1] only
    lens, _, cands = _golden()
    T, d = int(lens.sum()), 4
    x = np.zeros((T, d))
    x[:, 0] = np.arange(T)
    w1 = np.zeros((2, 3, d))
    w1[0, 0, 0] = 1.0
    w2 = np.zeros((2, 3))
    w2[0, 0] = 1.0
    out = oracle.candidate_heads(x, lens, dict(w1=w1, b1=None, w2=w2, b2=np.array([0.0, -2.5])))
    c = np.asarray(cands, np.float64)
    np.testing.assert_array_equal(out[:, 0], c * expit(c))
    np.testing.assert_array_equal(out[:, 1], -2.5)


def test_heads_match_torch_and_ignore_context_rows():
    rng = np.random.default_rng(2)
    lens = np.array([[3, 5, 2, 4], [2, 7, 0, 1], [1, 1, 1, 0]])
    T, d, d_h = int(lens.sum()), 12, 10
    x = rng.standard_normal((T, d))
    p = _head_params(rng, d, d_h)
    out = oracle.candidate_heads(x, lens, p)
    _, _, gid = oracle.pack_offsets(lens)
    t = lambda a: torch.as_tensor(a, dtype=torch.float64)  # noqa: E731
    xc = t(x[gid == 3])
    for k in range(2):
        ref = F.linear(F.silu(F.linear(xc, t(p["w1"][k]), t(p["b1"][k]))), t(p["w2"][k][None]),
                       t(p["b2"][k:k + 1])).numpy()[:, 0]
        np.testing.assert_allclose(out[:, k], ref, rtol=1e-12, atol=1e-12)
    # context rows and other candidates do not move a candidate's logits
    x2 = x.copy()
    x2[gid != 3] += 5.0
    x2[np.flatnonzero(gid == 3)[0]] -= 3.0
    out2 = oracle.candidate_heads(x2, lens, p)
    np.testing.assert_array_equal(out2[1:], out[1:])
    assert not np.array_equal(out2[0], out[0])
