"""Pins of the oracle's block variants: GroupLN with statistics pooled over
a user's group (the practice article's 3.1 GLN pseudocode) and SiLU on the
Q|K|V|U projections (HSTU's pointwise SiLU, one reading of the blog posts'
"HSTU-style SiLU attention and gating"). Checked against PyTorch's
layer_norm over whole segments and closed forms in which the attention
reduces to a masked sum."""

import numpy as np
import torch
import torch.nn.functional as F

import oracle
import synth

T64 = torch.float64


def _t(a):
    return torch.as_tensor(np.asarray(a, np.float64), dtype=T64)


def _pooled_torch(x, lens, gamma, beta, eps):
    """layer_norm over each (user, group) segment as one [n, d] block."""
    seg_off, _, _ = oracle.pack_offsets(lens)
    y = torch.zeros(x.shape, dtype=T64)
    xt = _t(x)
    for b in range(lens.shape[0]):
        for g in range(4):
            s, e = int(seg_off[4 * b + g]), int(seg_off[4 * b + g + 1])
            if e > s:
                y[s:e] = F.layer_norm(xt[s:e], (e - s, x.shape[1]), eps=eps) * _t(gamma[g]) + _t(beta[g])
    return y.numpy()


def _case(seed, d=16):
    rng = np.random.default_rng(seed)
    lens = np.array([[2, 6, 4, 5], [3, 4, 0, 3], [1, 0, 2, 1]], np.int64)
    x = synth.make_tokens(lens, d, rng).astype(np.float64)
    gamma = 1.0 + 0.3 * rng.standard_normal((4, d))
    beta = 0.3 * rng.standard_normal((4, d))
    return rng, lens, x, gamma, beta


def test_pooled_gln_matches_torch_layer_norm_over_segments():
    _, lens, x, gamma, beta = _case(0)
    y = oracle.group_layernorm_pooled(x, lens, gamma, beta, 1e-5)
    np.testing.assert_allclose(y, _pooled_torch(x, lens, gamma, beta, 1e-5), rtol=1e-12, atol=1e-12)


def test_pooled_gln_one_token_per_group_is_per_token_gln():
    rng = np.random.default_rng(1)
    lens = np.array([[1, 1, 1, 1], [1, 1, 0, 1]], np.int64)
    d = 8
    x = rng.standard_normal((int(lens.sum()), d)) * 3 + 1
    gamma, beta = rng.standard_normal((4, d)), rng.standard_normal((4, d))
    _, _, gid = oracle.pack_offsets(lens)
    np.testing.assert_allclose(oracle.group_layernorm_pooled(x, lens, gamma, beta),
                               oracle.group_layernorm(x, gid, gamma, beta), rtol=1e-12, atol=1e-12)


def test_pooled_gln_segment_scale_invariance():
    # with eps = 0, scaling and shifting one segment leaves the output unchanged
    _, lens, x, gamma, beta = _case(2)
    seg_off, _, _ = oracle.pack_offsets(lens)
    y = oracle.group_layernorm_pooled(x, lens, gamma, beta, 0.0)
    x2 = x.copy()
    s, e = int(seg_off[1]), int(seg_off[2])  # user 0's S tokens
    x2[s:e] = 7.5 * x2[s:e] - 3.0
    y2 = oracle.group_layernorm_pooled(x2, lens, gamma, beta, 0.0)
    np.testing.assert_allclose(y2, y, rtol=1e-10, atol=1e-10)
    # a per-token GLN would not see the other tokens of the segment; the
    # pooled one does: changing one token moves the others
    x3 = x.copy()
    x3[s] += 10.0
    y3 = oracle.group_layernorm_pooled(x3, lens, gamma, beta, 0.0)
    assert not np.allclose(y3[s + 1], y[s + 1])


def _mlp(z, p):
    h = F.silu(F.linear(_t(z), _t(p["w1"])))
    return F.linear(h, _t(p["w2"])).numpy()


def _ln_tok(z, gid, gamma, beta, eps=1e-5):
    return (F.layer_norm(_t(z), (z.shape[1],), eps=eps) * _t(gamma)[gid] + _t(beta)[gid]).numpy()


def test_silu_qkvu_closed_form():
    # W_qkvu = 0, b_qkvu = c: every projection is silu(c). Per head h the
    # score is s_h = silu(c_q) . silu(c_k) for every pair, so
    # G_i = silu(s_h) * rowsum(M_i) / N_b * silu(c_v) (.) silu(c_u)
    rng, lens, x, _, _ = _case(3)
    d, H = 16, 2
    dh = d // H
    p = synth.make_block_params(d, 40, rng, dtype="f32")
    p = {k: np.asarray(v, np.float64) for k, v in p.items()}
    p["w_qkvu"] = np.zeros((4 * d, d))
    c = 0.7 * rng.standard_normal(4 * d)
    p["b_qkvu"] = c
    ts = synth.make_timestamps(lens, rng)
    y = oracle.hstu_block(x, lens, ts, p, H, variant=oracle.VARIANT_SILU_QKVU)
    sc = F.silu(_t(c)).numpy()
    q, k, v, u = sc[:d], sc[d:2 * d], sc[2 * d:3 * d], sc[3 * d:]
    _, user_off, gid = oracle.pack_offsets(lens)
    g = np.zeros_like(x)
    for b in range(lens.shape[0]):
        s_, e_ = int(user_off[b]), int(user_off[b + 1])
        M = oracle.user_mask(*(int(t) for t in lens[b]), ts[s_:e_])
        rs = M.sum(axis=1)
        for h in range(H):
            cs = slice(h * dh, (h + 1) * dh)
            sh = float(q[cs] @ k[cs])
            silu_s = float(F.silu(torch.tensor(sh, dtype=T64)))
            g[s_:e_, cs] = silu_s * rs[:, None] / (e_ - s_) * (v[cs] * u[cs])[None, :]
    ref = x + _mlp(_ln_tok(g, gid, p["gln2_gamma"], p["gln2_beta"]), p)
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-10)


def test_pooled_block_constant_scores_reduce_to_masked_sum():
    # W_q = W_k = 0 with biases c_q, c_k: the score of every pair of head h
    # is s_h = c_q . c_k, so the attention is silu(s_h)/N_b times M @ V.
    # Both GroupLNs pooled: checked against layer_norm over whole segments.
    rng, lens, x, _, _ = _case(4)
    d, H = 16, 2
    dh = d // H
    p = synth.make_block_params(d, 40, rng, dtype="f32")
    p = {k: np.asarray(v, np.float64) for k, v in p.items()}
    p["w_qkvu"] = p["w_qkvu"].copy()
    p["w_qkvu"][:2 * d] = 0.0
    c = np.zeros(4 * d)
    c[:2 * d] = 0.5 * rng.standard_normal(2 * d)
    p["b_qkvu"] = c
    ts = synth.make_timestamps(lens, rng)
    y = oracle.hstu_block(x, lens, ts, p, H, variant=oracle.VARIANT_POOLED_GLN)
    xt = _pooled_torch(x, lens, p["gln1_gamma"], p["gln1_beta"], 1e-5)
    V = F.linear(_t(xt), _t(p["w_qkvu"][2 * d:3 * d])).numpy()
    U = F.linear(_t(xt), _t(p["w_qkvu"][3 * d:])).numpy()
    _, user_off, _ = oracle.pack_offsets(lens)
    g = np.zeros_like(x)
    for b in range(lens.shape[0]):
        s_, e_ = int(user_off[b]), int(user_off[b + 1])
        M = oracle.user_mask(*(int(t) for t in lens[b]), ts[s_:e_]).astype(np.float64)
        for h in range(H):
            cs = slice(h * dh, (h + 1) * dh)
            sh = float(c[:d][cs] @ c[d:2 * d][cs])
            silu_s = float(F.silu(torch.tensor(sh, dtype=T64)))
            g[s_:e_, cs] = silu_s / (e_ - s_) * (M @ V[s_:e_, cs]) * U[s_:e_, cs]
    gt = _pooled_torch(g, lens, p["gln2_gamma"], p["gln2_beta"], 1e-5)
    ref = x + _mlp(gt, p)
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-10)


# ---------------------------------------------------------------- VARIANT_RAB
def test_rab_time_bucket_is_the_binary_digit_count():
    import math
    assert oracle.rab_time_bucket(0) == 0
    for dt in list(range(1, 70)) + [1000, 65535, 65536, 2 ** 29 + 3, 2 ** 40]:
        want = min(int(math.floor(math.log2(dt))) + 1, oracle.RAB_TIME_BUCKETS - 1)
        assert oracle.rab_time_bucket(dt) == want, dt


def test_rab_bias_matches_hand_worked_user(golden):
    g = golden("rab_tiny_user.txt")
    n_u, n_s, n_r, n_k = g["lens"]
    ts = np.array(g["ts"], np.int64)
    bk = np.array(g["buckets"], np.int64)
    H = 2
    w_pos = np.tile(np.arange(2 * oracle.RAB_MAX_DIST + 1, dtype=np.float64), (H, 1))
    w_time = np.tile(1000.0 * np.arange(oracle.RAB_TIME_BUCKETS), (H, 1))
    w_time[1] *= 2.0  # the heads keep their own tables
    for h in range(H):
        got = oracle.rab_bias(n_u, n_s, n_r, n_k, ts, w_pos, w_time, h)
        i, j = np.meshgrid(np.arange(6), np.arange(6), indexing="ij")
        want = (i - j + oracle.RAB_MAX_DIST) + 1000.0 * (h + 1) * bk
        np.testing.assert_array_equal(got, want)


def test_rab_position_term_clips_far_pairs():
    N = 300
    ts = np.arange(N, dtype=np.int64)
    w_pos = np.arange(2 * oracle.RAB_MAX_DIST + 1, dtype=np.float64)[None, :]
    w_time = np.zeros((1, oracle.RAB_TIME_BUCKETS))
    b = oracle.rab_bias(0, N, 0, 0, ts, w_pos, w_time, 0)
    assert b[299, 0] == 2 * oracle.RAB_MAX_DIST and b[0, 299] == 0.0
    assert b[150, 150 - oracle.RAB_MAX_DIST] == 2 * oracle.RAB_MAX_DIST
    assert b[10, 10] == oracle.RAB_MAX_DIST


def _rab_case(seed=0, H=2, dh=8):
    rng = np.random.default_rng(seed)
    lens = np.array([[2, 7, 4, 3], [1, 5, 0, 2], [0, 4, 3, 0]], np.int32)
    ts = synth.make_timestamps(lens, rng)
    qkvu = rng.standard_normal((int(lens.sum()), 4 * H * dh))
    return lens, ts, qkvu, H


def test_rab_zero_tables_reduce_to_the_plain_attention():
    lens, ts, qkvu, H = _rab_case()
    z = (np.zeros((H, 2 * oracle.RAB_MAX_DIST + 1)), np.zeros((H, oracle.RAB_TIME_BUCKETS)))
    np.testing.assert_array_equal(oracle.hstu_attention(qkvu, lens, ts, H, rab=z),
                                  oracle.hstu_attention(qkvu, lens, ts, H))


def test_rab_constant_bias_with_zero_queries_closed_form():
    # Q = 0 and rab = c everywhere: every visible weight is silu(c) / N, so
    # G_i = silu(c) / N_b sum_j M_ij v_j (.) u_i, with M the mask's own matrix
    lens, ts, qkvu, H = _rab_case(seed=1)
    d = qkvu.shape[1] // 4
    qkvu[:, :d] = 0.0
    c = 0.7
    rab = (np.full((H, 2 * oracle.RAB_MAX_DIST + 1), c), np.zeros((H, oracle.RAB_TIME_BUCKETS)))
    g = oracle.hstu_attention(qkvu, lens, ts, H, rab=rab)
    off = np.concatenate([[0], np.cumsum(lens.sum(1))])
    sc = c / (1.0 + np.exp(-c))
    for b in range(lens.shape[0]):
        s, e = off[b], off[b + 1]
        M = oracle.user_mask(*(int(v) for v in lens[b]), ts[s:e]).astype(np.float64)
        want = sc / (e - s) * (M @ qkvu[s:e, 2 * d:3 * d]) * qkvu[s:e, 3 * d:]
        np.testing.assert_allclose(g[s:e], want, rtol=1e-12, atol=1e-12)


def test_rab_time_term_ignores_u_tokens_and_shifts_scores():
    # a time table that only bucket 3 uses: exactly the pairs the fixture's
    # bucket matrix marks 3 change, by silu(s + w) - silu(s) in their weight
    lens = np.array([[1, 2, 2, 1]], np.int32)
    ts = np.array([0, 5, 9, 12, 20, 13], np.int64)
    H, dh = 1, 4
    rng = np.random.default_rng(3)
    qkvu = rng.standard_normal((6, 4 * dh))
    w_time = np.zeros((H, oracle.RAB_TIME_BUCKETS))
    w_time[0, 3] = 0.5
    b = oracle.rab_bias(1, 2, 2, 1, ts, np.zeros((H, 2 * oracle.RAB_MAX_DIST + 1)), w_time, 0)
    marked = np.array([[0, 0, 0, 0, 0, 0], [0, 0, 1, 1, 0, 0], [0, 1, 0, 0, 0, 1],
                       [0, 1, 0, 0, 0, 0], [0, 0, 0, 0, 0, 1], [0, 0, 1, 0, 1, 0]], bool)
    np.testing.assert_array_equal(b != 0, marked)


def test_rab_bias_matches_the_entrywise_definition():
    # brute force over every (i, j) of random small users against the scalar
    # bucket function and the clip, ties and large gaps included
    rng = np.random.default_rng(9)
    H = 2
    w_pos = rng.standard_normal((H, 2 * oracle.RAB_MAX_DIST + 1))
    w_time = rng.standard_normal((H, oracle.RAB_TIME_BUCKETS))
    for lens in ([3, 40, 9, 5], [0, 150, 2, 140], [1, 0, 0, 1]):
        N = sum(lens)
        ts = rng.integers(0, 3, N) * rng.integers(1, 1 << 40, N)
        for h in range(H):
            b = oracle.rab_bias(*lens, ts, w_pos, w_time, h)
            for i in range(N):
                for j in range(N):
                    p = min(max(i - j, -oracle.RAB_MAX_DIST), oracle.RAB_MAX_DIST) + oracle.RAB_MAX_DIST
                    tb = 0 if (i < lens[0] or j < lens[0]) else oracle.rab_time_bucket(abs(int(ts[i]) - int(ts[j])))
                    assert b[i, j] == w_pos[h][p] + w_time[h][tb]
