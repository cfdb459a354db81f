"""Float64 NumPy oracle of the MTGR HSTU block (test infrastructure only).

Sources, cited by page and section:
  * "MTGR: Industrial-Scale Generative Recommendation Framework in Meituan"
    summary page (marovi.ai, zh), section "Method": the sample
    D = [U, S, R, [C,I]_1..K], GroupLN -> Q,K,V,U, the attention update
    V~ = silu(K^T Q) / (N_U + N_S + N_R + N_I) * M * V and
    X <- MLP(GroupLN(V~ (.) U)) + X, and the three mask rules.
  * fun-rec "MTGR: Hybrid Paradigm Modeling", 7.3.3 (GLN formula: per-token
    normalisation with the group's gamma/beta) and 7.3.4 (Rules 1-3 of the
    dynamic mask, with the 12:00/12:30/13:00 leakage example).

Readings taken where the pages are silent or garbled (each is listed in the
design notes of the repository):
  * GLN statistics are per token over d_model; gamma/beta are chosen by group.
  * eps = 1e-5 inside the square root, biased variance (divide by d).
  * No 1/sqrt(dh) scale; the score of query i and key j is q_i . k_j.
  * Q, K, V, U are plain linear projections (no activation), split into H
    contiguous heads of dh = d/H columns each.
  * N is the user's total token count, the same for every query of the user;
    a per-user override replaces it when given.
  * R rule: key j in R is visible to query i iff t_j < t_i (strict) or j == i;
    U queries carry no time and never see R keys; S queries use their own time.
  * A candidate key is visible only to itself. U and S keys are visible to every
    query of the same user. Nothing crosses a user boundary.
  * MLP = Linear(d, d_ff) -> SiLU -> Linear(d_ff, d), no final activation.
"""

from __future__ import annotations

import numpy as np
from scipy.special import expit

EPS = 1e-5
# canonical tile size of the mask metadata (a build artefact, not from the pages)
BM = 128
BN = 128

G_U, G_S, G_R, G_C = 0, 1, 2, 3


def silu(x: np.ndarray) -> np.ndarray:
    """SiLU(x) = x * sigmoid(x), with the logistic sigmoid from SciPy."""
    return x * expit(x)


def pack_offsets(lens: np.ndarray):
    """Jagged packing of users back to back, each in the order U, S, R, C.

    Follows the user-aggregated sample D = [U, S, R, [C,I]_1..K] (summary page,
    Method) and sequence packing without cross-user attention (chenhuiyu blog,
    "training system" list). Returns
      seg_off  int32 [4B+1]: start row of U, S, R, C of each user; last = T
      user_off int32 [B+1]
      group_id int8  [T]: 0 U, 1 S, 2 R, 3 C
    """
    lens = np.asarray(lens, dtype=np.int64).reshape(-1, 4)
    B = lens.shape[0]
    flat = lens.reshape(-1)
    seg_off = np.zeros(4 * B + 1, dtype=np.int64)
    seg_off[1:] = np.cumsum(flat)
    user_off = seg_off[0::4].copy()
    group_id = np.zeros(int(seg_off[-1]), dtype=np.int8)
    for b in range(B):
        for g in range(4):
            group_id[seg_off[4 * b + g]:seg_off[4 * b + g + 1]] = g
    return seg_off.astype(np.int32), user_off.astype(np.int32), group_id


def user_mask(n_u: int, n_s: int, n_r: int, n_k: int, ts: np.ndarray) -> np.ndarray:
    """Visibility matrix M [N, N] of one user (row = query i, column = key j).

    fun-rec 7.3.4, Rules 1-3, and the summary page's mask paragraph:
      Rule 1: keys in U or S are visible to every query of the user.
      Rule 2: a key j in R is visible to query i iff t_j < t_i, or j == i.
      Rule 3: a candidate key is visible only to itself.
    ``ts`` holds the user's N timestamps in layout order; U entries are unused
    because U queries carry no time (they never see an R key).
    """
    N = n_u + n_s + n_r + n_k
    grp = np.repeat(np.array([G_U, G_S, G_R, G_C]), [n_u, n_s, n_r, n_k])
    ts = np.asarray(ts, dtype=np.int64)
    M = np.zeros((N, N), dtype=bool)
    key_static = (grp == G_U) | (grp == G_S)
    M[:, key_static] = True
    key_rt = grp == G_R
    query_has_time = grp != G_U
    earlier = (ts[None, :] < ts[:, None]) & query_has_time[:, None]
    M[:, key_rt] = earlier[:, key_rt]
    idx = np.arange(N)
    M[idx, idx] = True  # every token sees itself (rules 1-3 all include j == i)
    return M


def visible_pairs(lens: np.ndarray, ts: np.ndarray) -> int:
    """Total number of visible (query, key) pairs over all users."""
    seg_off, user_off, _ = pack_offsets(lens)
    total = 0
    for b, (n_u, n_s, n_r, n_k) in enumerate(np.asarray(lens).reshape(-1, 4)):
        s, e = int(user_off[b]), int(user_off[b + 1])
        total += int(user_mask(int(n_u), int(n_s), int(n_r), int(n_k), ts[s:e]).sum())
    return total


def group_layernorm(x: np.ndarray, group_id: np.ndarray, gamma: np.ndarray,
                    beta: np.ndarray, eps: float = EPS) -> np.ndarray:
    """GLN(x_i) = (x_i - mu_i) / sqrt(var_i + eps) * gamma_{g(i)} + beta_{g(i)}.

    fun-rec 7.3.3 (the GLN formula), with per-token statistics over d_model.
    """
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=1, keepdims=True)
    xhat = (x - mu) / np.sqrt(var + eps)
    g = np.asarray(group_id, dtype=np.int64)
    return xhat * np.asarray(gamma, np.float64)[g] + np.asarray(beta, np.float64)[g]


# Block variants the pages leave open (bit flags, combinable):
#   VARIANT_POOLED_GLN: GroupLN statistics pooled over all tokens and features
#     of one group of one user, the reading of the practice article's 3.1 GLN
#     pseudocode (group_mean = mean(group_hidden_states), group_std likewise);
#   VARIANT_SILU_QKVU: Q, K, V, U = silu(X~ W_qkvu^T + b), HSTU's pointwise
#     SiLU on the projections, one reading of the blog posts' "HSTU-style SiLU
#     attention and gating" (it also puts SiLU on U before the gate).
VARIANT_POOLED_GLN = 1
VARIANT_SILU_QKVU = 2
#   VARIANT_RAB: HSTU's relative attention bias, a learned per-head bias added
#     to every score before the SiLU, silu(q_i . k_j + rab_h(i, j)). The pages
#     name the bias only through HSTU; the reading taken: rab_h(i, j) =
#     w_pos[h][clip(i - j, -RAB_MAX_DIST, RAB_MAX_DIST) + RAB_MAX_DIST] +
#     w_time[h][time_bucket(|t_i - t_j|)], with i, j the user-relative
#     positions, time_bucket(0) = 0 and time_bucket(dt) = min(floor(log2 dt)
#     + 1, RAB_TIME_BUCKETS - 1) for dt >= 1, and no time term (bucket 0)
#     when either token is a U token, which carries no time.
VARIANT_RAB = 4
RAB_MAX_DIST = 128
RAB_TIME_BUCKETS = 32


def rab_time_bucket(dt: int) -> int:
    """Bucket of an absolute time difference: 0 for 0, else the number of
    binary digits of dt (floor(log2 dt) + 1), capped at RAB_TIME_BUCKETS - 1."""
    dt = int(dt)
    if dt <= 0:
        return 0
    return min(dt.bit_length(), RAB_TIME_BUCKETS - 1)


def rab_bias(n_u: int, n_s: int, n_r: int, n_k: int, ts: np.ndarray, w_pos: np.ndarray,
             w_time: np.ndarray, h: int) -> np.ndarray:
    """The relative attention bias [N, N] of head h for one user (query i,
    key j), by the VARIANT_RAB reading above, entry by entry."""
    N = n_u + n_s + n_r + n_k
    ts = np.asarray(ts, dtype=np.int64)
    idx = np.arange(N)
    pos = np.clip(idx[:, None] - idx[None, :], -RAB_MAX_DIST, RAB_MAX_DIST) + RAB_MAX_DIST
    dt = np.abs(ts[:, None] - ts[None, :])
    # binary digit count of dt: frexp's exponent (exact for |dt| < 2^53), 0 for dt = 0
    digits = np.frexp(dt.astype(np.float64))[1]
    tb = np.where(dt == 0, 0, np.minimum(digits, RAB_TIME_BUCKETS - 1))
    has_time = idx >= n_u
    tb = np.where(has_time[:, None] & has_time[None, :], tb, 0)
    return np.asarray(w_pos[h], np.float64)[pos] + np.asarray(w_time[h], np.float64)[tb]


def group_layernorm_pooled(x: np.ndarray, lens: np.ndarray, gamma: np.ndarray,
                           beta: np.ndarray, eps: float = EPS) -> np.ndarray:
    """GroupLN with pooled statistics: for every user b and group g, mu and
    var are the mean and the biased variance of all N_{b,g} x d values of that
    group's tokens; y = (x - mu) / sqrt(var + eps) * gamma_g + beta_g."""
    x = np.asarray(x, dtype=np.float64)
    seg_off, _, _ = pack_offsets(lens)
    y = np.zeros_like(x)
    for b in range(np.asarray(lens).reshape(-1, 4).shape[0]):
        for g in range(4):
            s, e = int(seg_off[4 * b + g]), int(seg_off[4 * b + g + 1])
            if e == s:
                continue
            blk = x[s:e]
            mu = blk.mean()
            var = ((blk - mu) ** 2).mean()
            y[s:e] = (blk - mu) / np.sqrt(var + eps) * np.asarray(gamma, np.float64)[g] \
                + np.asarray(beta, np.float64)[g]
    return y


def hstu_attention(qkvu: np.ndarray, lens: np.ndarray, ts: np.ndarray, H: int,
                   norm: np.ndarray | None = None, rab: tuple | None = None) -> np.ndarray:
    """G = (silu(Q K^T) * M / N) V, gated by U, per user and head.

    Summary page, Method: V~ = silu(K^T Q) / (N_U+N_S+N_R+N_I) * M * V and the
    gate V~ (.) U of the update. ``qkvu`` is [T, 4d] with column blocks
    Q | K | V | U; head h owns columns [h*dh, (h+1)*dh) of each block.
    ``rab`` = (w_pos [H, 2 RAB_MAX_DIST + 1], w_time [H, RAB_TIME_BUCKETS])
    adds the relative attention bias of VARIANT_RAB to the scores.
    Returns G [T, d] in float64.
    """
    qkvu = np.asarray(qkvu, dtype=np.float64)
    T, d4 = qkvu.shape
    d = d4 // 4
    dh = d // H
    Q, K, V, U = qkvu[:, :d], qkvu[:, d:2 * d], qkvu[:, 2 * d:3 * d], qkvu[:, 3 * d:]
    lens = np.asarray(lens, dtype=np.int64).reshape(-1, 4)
    _, user_off, _ = pack_offsets(lens)
    out = np.zeros((T, d), dtype=np.float64)
    for b in range(lens.shape[0]):
        s, e = int(user_off[b]), int(user_off[b + 1])
        if e == s:
            continue
        n_u, n_s, n_r, n_k = (int(v) for v in lens[b])
        M = user_mask(n_u, n_s, n_r, n_k, ts[s:e]).astype(np.float64)
        Nb = float(e - s) if norm is None else float(norm[b])
        for h in range(H):
            c = slice(h * dh, (h + 1) * dh)
            scores = Q[s:e, c] @ K[s:e, c].T        # scores[i, j] = q_i . k_j
            if rab is not None:
                scores = scores + rab_bias(n_u, n_s, n_r, n_k, ts[s:e], rab[0], rab[1], h)
            A = silu(scores) * M / Nb
            out[s:e, c] = A @ V[s:e, c]
    return out * U


def hstu_block(x: np.ndarray, lens: np.ndarray, ts: np.ndarray, p: dict, H: int,
               norm: np.ndarray | None = None, eps: float = EPS, variant: int = 0) -> np.ndarray:
    """One HSTU block of MTGR (summary page, Method):

      X~ = GroupLN_1(X);  Q,K,V,U = X~ W_qkvu^T
      G  = (silu(Q K^T) M / N) V (.) U
      X  <- MLP(GroupLN_2(G)) + X,  MLP = Linear -> SiLU -> Linear
    Optional biases ``b_qkvu``, ``b1``, ``b2`` are added when present in ``p``.
    ``variant`` selects the VARIANT_* readings above (0: the block as written).
    """
    x = np.asarray(x, dtype=np.float64)
    _, _, gid = pack_offsets(lens)

    def gln(z, gamma, beta):
        if variant & VARIANT_POOLED_GLN:
            return group_layernorm_pooled(z, lens, gamma, beta, eps)
        return group_layernorm(z, gid, gamma, beta, eps)

    xt = gln(x, p["gln1_gamma"], p["gln1_beta"])
    qkvu = xt @ np.asarray(p["w_qkvu"], np.float64).T
    if p.get("b_qkvu") is not None:
        qkvu = qkvu + np.asarray(p["b_qkvu"], np.float64)
    if variant & VARIANT_SILU_QKVU:
        qkvu = silu(qkvu)
    rab = (p["rab_pos"], p["rab_time"]) if variant & VARIANT_RAB else None
    g = hstu_attention(qkvu, lens, ts, H, norm, rab)
    gt = gln(g, p["gln2_gamma"], p["gln2_beta"])
    h = gt @ np.asarray(p["w1"], np.float64).T
    if p.get("b1") is not None:
        h = h + np.asarray(p["b1"], np.float64)
    h = silu(h)
    y = h @ np.asarray(p["w2"], np.float64).T
    if p.get("b2") is not None:
        y = y + np.asarray(p["b2"], np.float64)
    return x + y


def hstu_stack(x: np.ndarray, lens: np.ndarray, ts: np.ndarray, layers: list, H: int,
               norm: np.ndarray | None = None, eps: float = EPS, variant: int = 0) -> np.ndarray:
    """L stacked HSTU blocks (summary page, Method: "L stacked HSTU blocks")."""
    y = np.asarray(x, dtype=np.float64)
    for p in layers:
        y = hstu_block(y, lens, ts, p, H, norm, eps, variant)
    return y


def mask_meta(lens: np.ndarray, ts: np.ndarray, bm: int = BM, bn: int = BN):
    """Canonical tile list of the mask, read off the explicit M of each user.

    Tiles are bm x bn on the user-relative grid; only in-range cells count. A
    tile with no visible cell is EMPTY and omitted; FULL if every in-range cell
    is visible; PARTIAL otherwise. Q-tiles are listed user-major with the
    q-tile index ascending, and entries of a q-tile by ascending k-tile; each
    entry is (kt << 1) | partial. ``order`` lists the q-tiles user by user,
    users by descending length (ties by ascending user index), each user's
    q-tiles by ascending qt. Returns dict with qtile_desc int32
    [Q,2] (user, qt), row_ptr int32 [Q+1], entries int32 [E], order int32 [Q]
    and the visible-pair count.
    """
    lens = np.asarray(lens, dtype=np.int64).reshape(-1, 4)
    _, user_off, _ = pack_offsets(lens)
    desc, row_ptr, entries = [], [0], []
    vis = 0
    for b in range(lens.shape[0]):
        s, e = int(user_off[b]), int(user_off[b + 1])
        N = e - s
        if N == 0:
            continue
        n_u, n_s, n_r, n_k = (int(v) for v in lens[b])
        M = user_mask(n_u, n_s, n_r, n_k, ts[s:e])
        vis += int(M.sum())
        for qt in range((N + bm - 1) // bm):
            rows = M[qt * bm:min(N, (qt + 1) * bm)]
            for kt in range((N + bn - 1) // bn):
                cells = rows[:, kt * bn:min(N, (kt + 1) * bn)]
                if not cells.any():
                    continue
                entries.append((kt << 1) | (0 if cells.all() else 1))
            desc.append((b, qt))
            row_ptr.append(len(entries))
    Q = len(desc)
    n_user = lens.sum(axis=1)
    order = sorted(range(Q), key=lambda q: (-int(n_user[desc[q][0]]), desc[q][0], desc[q][1]))
    return dict(
        qtile_desc=np.asarray(desc, dtype=np.int32).reshape(-1, 2),
        row_ptr=np.asarray(row_ptr, dtype=np.int32),
        entries=np.asarray(entries, dtype=np.int32),
        order=np.asarray(order, dtype=np.int32),
        visible_pairs=vis,
    )
