"""Float64 oracle of the steps on either side of the HSTU stack: the token
MLPs that bring every feature domain to d_model, and the CTR/CTCVR heads on
the candidates' output rows. TEST INFRASTRUCTURE ONLY (see the package
docstring for who may import it).

Sources, cited by page and section:
  * blog posts "generative recommendation 18: MTGR" (chenhuiyu, zh and en),
    "Converting heterogeneous features into tokens": a scalar feature such as
    age or gender becomes a token of its own; the fields of each sequence item
    are embedded and concatenated, then a domain-specific MLP projects them to
    d_model; a candidate's cross and item features are fused before its token
    is formed; Feat_D = Concat(Feat_U, Feat_S, Feat_R, Feat_I); the hidden
    states at the candidate positions go through MLPs that give the CTR and
    CTCVR logits.
  * summary page (marovi), "Method": each scalar feature of U is one d_model
    token; each item of S and R becomes a token by embedding plus MLP; each
    candidate is one token whose embedding fuses its own features with the
    user-specific cross features.
  * fun-rec "MTGR: Hybrid Paradigm Modeling", 7.3.3: the candidate token is an
    MLP of the concatenated item and cross embeddings.

Readings taken where the pages are silent:
  * U tokens are the feature embeddings themselves, already d_model wide; no
    MLP is applied to them.
  * The token MLP of domain g in {S, R, C} is Linear(F_g, d) -> SiLU ->
    Linear(d, d) with optional biases, with its own weights per domain.
  * Inputs: for each domain, the concatenated field embeddings of that
    domain's tokens, the tokens of user 0 first, then user 1, ..., each user's
    in sequence order (the embedding lookup itself is not part of the path).
  * Each task head (CTR, CTCVR) is Linear(d, d_h) -> SiLU -> Linear(d_h, 1)
    with optional biases; it outputs a logit (no sigmoid). Output rows are
    the candidates in user order, each user's in sequence order.
"""

from __future__ import annotations

import numpy as np

from .mtgr import pack_offsets, silu

DOMAINS = ("s", "r", "c")


def token_mlp(e: np.ndarray, w1, b1, w2, b2) -> np.ndarray:
    """Linear(F, d) -> SiLU -> Linear(d, d) on rows e [n, F]; weights in
    [out, in] layout, biases optional (None)."""
    h = np.asarray(e, np.float64) @ np.asarray(w1, np.float64).T
    if b1 is not None:
        h = h + np.asarray(b1, np.float64)
    y = silu(h) @ np.asarray(w2, np.float64).T
    if b2 is not None:
        y = y + np.asarray(b2, np.float64)
    return y


def tokenize(lens: np.ndarray, e: list, p: dict) -> np.ndarray:
    """The block input X [T, d] of a packed batch.

    ``e`` = [E_U, E_S, E_R, E_C]: E_U [sum N_U, d], E_g [sum N_g, F_g], each
    in user order. ``p`` holds ``w1_g``, ``b1_g``, ``w2_g``, ``b2_g`` for
    g in s, r, c. Each user's rows are its U tokens, then the S, R and
    candidate tokens, as in Feat_D = Concat(Feat_U, Feat_S, Feat_R, Feat_I).
    """
    lens = np.asarray(lens, np.int64).reshape(-1, 4)
    tokens = [np.asarray(e[0], np.float64)]
    for g, name in enumerate(DOMAINS, start=1):
        tokens.append(token_mlp(e[g], p["w1_" + name], p.get("b1_" + name), p["w2_" + name],
                                p.get("b2_" + name)))
    for g in range(4):
        assert tokens[g].shape[0] == int(lens[:, g].sum()), "domain rows do not match lens"
    d = tokens[0].shape[1] if tokens[0].size else tokens[1].shape[1]
    x = np.zeros((int(lens.sum()), d), np.float64)
    seg_off, _, _ = pack_offsets(lens)
    taken = [0, 0, 0, 0]
    for b in range(lens.shape[0]):
        for g in range(4):
            n = int(lens[b, g])
            s = int(seg_off[4 * b + g])
            x[s:s + n] = tokens[g][taken[g]:taken[g] + n]
            taken[g] += n
    return x


def candidate_heads(x: np.ndarray, lens: np.ndarray, p: dict) -> np.ndarray:
    """Logits [K_total, n_tasks] of the candidates' rows of x [T, d].

    ``p``: ``w1`` [n_tasks, d_h, d], ``b1`` [n_tasks, d_h] or None, ``w2``
    [n_tasks, d_h], ``b2`` [n_tasks] or None. Task t's logit of candidate row
    x_c is w2[t] . silu(w1[t] x_c + b1[t]) + b2[t].
    """
    lens = np.asarray(lens, np.int64).reshape(-1, 4)
    seg_off, _, _ = pack_offsets(lens)
    rows = [np.arange(seg_off[4 * b + 3], seg_off[4 * b + 4]) for b in range(lens.shape[0])]
    rows = np.concatenate(rows) if rows else np.zeros(0, np.int64)
    xc = np.asarray(x, np.float64)[rows]
    w1 = np.asarray(p["w1"], np.float64)
    w2 = np.asarray(p["w2"], np.float64)
    n_tasks = w1.shape[0]
    out = np.zeros((xc.shape[0], n_tasks), np.float64)
    for t in range(n_tasks):
        h = xc @ w1[t].T
        if p.get("b1") is not None:
            h = h + np.asarray(p["b1"], np.float64)[t]
        out[:, t] = silu(h) @ w2[t]
        if p.get("b2") is not None:
            out[:, t] += float(np.asarray(p["b2"], np.float64)[t])
    return out
