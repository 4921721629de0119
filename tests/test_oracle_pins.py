"""Pins of the oracle against facts the pages and mathematics fix (CPU only).

Each test is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign, index or head slice, a transposed weight, the tanh GELU instead of
the erf form) fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import lowram_oracle as orc

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _orthogonal(rng, n):
    q, r = np.linalg.qr(rng.standard_normal((n, n)))
    return q * np.sign(np.diag(r))


# ----------------------------------------------------------------------------- rounding

def test_round_bf16_ties_and_torch():
    r = orc.round_bf16
    assert r(1.0) == 1.0
    assert r(1.0 + 2.0 ** -8) == 1.0                      # tie -> even (1.0)
    assert r(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6      # tie -> even (mantissa ...10)
    assert r(1.0 + 2.0 ** -8 + 2.0 ** -20) == 1.0 + 2.0 ** -7
    assert r(-3.0) == -3.0 and r(0.0) == 0.0
    assert np.isinf(r(3.5e38))
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-30, 30, 20000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(orc.round_bf16(x.astype(np.float64)), ref)


# ----------------------------------------------------------------------------- GELU

def test_gelu_is_exact_erf_form():
    for x, phi in _gold("normal_cdf.json")["values"]:
        assert abs(orc.gelu(x) - x * phi) <= 1e-12 * max(1.0, abs(x))
    # the tanh approximation differs by ~1.6e-4 at x = 1; the pin above rejects it
    tanh_form = 0.5 * (1 + math.tanh(math.sqrt(2 / math.pi) * (1 + 0.044715)))
    assert abs(tanh_form - orc.gelu(1.0)) > 1e-5


# ----------------------------------------------------------------------------- predictor

def test_predict_values_hand_computed():
    # k = [1, -1]; W_lin (out x in) = [[1, 2], [0, 1]] -> k W_lin^T = [1*1 + 2*-1, 0*1 + 1*-1] = [-1, -1]
    # u = k W1^T + b1 with W1 = I, b1 = [0, 0.5] -> [1, -0.5]; g = [Phi(1), -0.5 Phi(-0.5)]
    # W2 (out x in) = [[2, 5], [0, 3]] -> g W2^T = [2 g0 + 5 g1, 3 g1]; b2 = [0.5, -1]
    phi1 = 0.8413447460685429
    phim05 = 1.0 - 0.6914624612740131
    g0, g1 = 1.0 * phi1, -0.5 * phim05
    expect = np.array([-1 + 2 * g0 + 5 * g1 + 0.5, -1 + 3 * g1 - 1.0])
    got = orc.predict_values(np.array([[1.0, -1.0]]), np.array([[1.0, 2.0], [0.0, 1.0]]),
                             np.eye(2), np.array([0.0, 0.5]), np.array([[2.0, 5.0], [0.0, 3.0]]),
                             np.array([0.5, -1.0]))
    np.testing.assert_allclose(got[0], expect, rtol=0, atol=1e-12)


def test_token_errors_squared_l2():
    v = np.array([[3.0, 4.0, 1.0], [0.0, 0.0, 0.0]])
    vh = np.array([[0.0, 0.0, 1.0], [1.0, -2.0, 2.0]])
    np.testing.assert_array_equal(orc.token_errors(v, vh), [25.0, 9.0])


# ----------------------------------------------------------------------------- top-k

def _unique_valid_set(e, k):
    """The one k-subset whose every member ranks above every non-member by (e desc, t asc)."""
    T = len(e)
    found = []
    for S in itertools.combinations(range(T), k):
        s = set(S)
        ok = all((e[i] > e[j]) or (e[i] == e[j] and i < j)
                 for i in s for j in range(T) if j not in s)
        if ok:
            found.append(S)
    assert len(found) == 1
    return np.array(found[0], dtype=np.int64)


@pytest.mark.parametrize("ties", [False, True])
def test_topk_matches_brute_force(ties):
    rng = np.random.default_rng(7 if ties else 3)
    for T in range(0, 11):
        for trial in range(3):
            e = (rng.integers(0, 3, T).astype(float) if ties else rng.random(T))
            for k in range(0, T + 1):
                got = orc.topk_residual_tokens(e, k)
                np.testing.assert_array_equal(got, _unique_valid_set(e, k))
                # the set minimises the error left uncorrected over all k-subsets
                left = e.sum() - e[got].sum()
                best = min((e.sum() - sum(e[list(S)]) for S in itertools.combinations(range(T), k)),
                           default=0.0)
                assert abs(left - best) <= 1e-12


def test_topk_remaining_error_invariant_large():
    rng = np.random.default_rng(11)
    e = rng.random(5000) ** 3
    k = 731
    sel = orc.topk_residual_tokens(e, k)
    left = np.delete(e, sel).sum()
    assert abs(left - np.sort(e)[: 5000 - k].sum()) <= 1e-9
    for _ in range(20):
        rnd = rng.choice(5000, k, replace=False)
        assert left <= np.delete(e, rnd).sum()
    assert np.all(np.diff(sel) > 0)


def test_block_ptr_properties():
    rng = np.random.default_rng(5)
    for T in (1, 63, 64, 65, 1000, 4097):
        for k in (0, 1, min(T, 17), T):
            idx = np.sort(rng.choice(T, k, replace=False))
            ptr = orc.block_ptr(idx, T)
            nblk = (T + 63) // 64
            assert len(ptr) == nblk + 1 and ptr[0] == 0 and ptr[-1] == k
            for j in range(nblk):
                seg = idx[ptr[j]:ptr[j + 1]]
                assert np.all((seg >= 64 * j) & (seg < 64 * j + 64))


# ----------------------------------------------------------------------------- attention pins

def test_dense_attention_hand():
    q = np.array([1.0, 0.0])
    K = np.array([[1.0, 0.0], [0.0, 1.0]])
    V = np.array([[2.0, 0.0], [0.0, 4.0]])
    p0 = math.e / (math.e + 1)
    np.testing.assert_allclose(orc.dense_attention(q, K, V, 1.0), [2 * p0, 4 * (1 - p0)], atol=1e-14)
    np.testing.assert_allclose(orc.dense_attention(q, K[:1], V[:1], 0.3), V[0], atol=1e-15)
    np.testing.assert_allclose(orc.dense_attention(np.zeros(2), K, V, 1.0), V.mean(0), atol=1e-15)
    assert orc.default_scale(64, 0.0) == 0.125 and orc.default_scale(64, 0.5) == 0.5


def _hidden(rng, T, d):
    return rng.standard_normal((T, d))


def test_slim_attention_exact_recovery():
    """Square invertible key projection, zero nonlinear branch: v_hat = v and o = dense attention."""
    rng = np.random.default_rng(21)
    d = hd = 64
    T, G = 300, 2
    W_K = _orthogonal(rng, d) @ np.diag(np.linspace(0.5, 2.0, d))
    W_V = rng.standard_normal((d, hd)) / 8
    W_Q = rng.standard_normal((d, G * hd)) / 8
    x = _hidden(rng, T, d)
    K, V = x @ W_K, x @ W_V
    Bt = _orthogonal(rng, d)                      # full-rank basis (r = D)
    W_lin = (np.linalg.pinv(W_K) @ W_V).T[None, None]
    W1 = rng.standard_normal((1, 1, 32, hd)) * 0.1
    b1 = rng.standard_normal((1, 1, 32))
    W2 = np.zeros((1, 1, hd, 32))
    packed = orc.pack_sequence(K, V[None, :, None, :], Bt, W_lin, W1, b1, W2, None, 0, "f64", 1, hd)
    assert packed["err"].max() <= 1e-18 * np.sum(V * V)
    q = (rng.standard_normal((1, d)) @ W_Q).reshape(G, hd)
    o = orc.decode_sequence(q, packed["A"], Bt, W_lin, W1, b1, W2, None, 0, packed["idx"],
                            packed["val"], None, orc.default_scale(hd, 0), 1, hd)
    for g in range(G):
        ref = orc.dense_attention(q[g], K, V, 1 / math.sqrt(hd))
        np.testing.assert_allclose(o[g], ref, rtol=1e-10, atol=1e-10 * np.abs(ref).max())


def _group_problem(rng, d=64, L=2, Hkv=2, G=2, hd=16, T=200, H=24):
    WK = rng.standard_normal((L, d, Hkv * hd)) / 8
    WV = rng.standard_normal((L, d, Hkv * hd)) / 8
    x = _hidden(rng, T, d)
    K_group = np.concatenate([x @ WK[l] for l in range(L)], axis=1)     # [T, D]
    V = np.stack([(x @ WV[l]).reshape(T, Hkv, hd) for l in range(L)])   # [L, T, Hkv, hd]
    pred = dict(W_lin=rng.standard_normal((L, Hkv, hd, hd)) * 0.3,
                W1=rng.standard_normal((L, Hkv, H, hd)) * 0.3,
                b1=rng.standard_normal((L, Hkv, H)),
                W2=rng.standard_normal((L, Hkv, hd, H)) * 0.3,
                b2=rng.standard_normal((L, Hkv, hd)))
    return K_group, V, pred


def test_full_rank_keys_reproduce_every_head_slice():
    rng = np.random.default_rng(8)
    L, Hkv, hd = 2, 2, 16
    K_group, _, _ = _group_problem(rng, L=L, Hkv=Hkv, hd=hd)
    Bt = _orthogonal(rng, K_group.shape[1])
    A = orc.project_keys(K_group, Bt)
    for l in range(L):
        for h in range(Hkv):
            kt = orc.reconstruct_keys(A, orc.key_slice(Bt, l, h, Hkv, hd))
            c0 = (l * Hkv + h) * hd
            np.testing.assert_allclose(kt, K_group[:, c0:c0 + hd], atol=1e-12)


@pytest.mark.parametrize("selective", [False, True])
def test_full_budget_reproduces_dense_attention(selective):
    """k = T residuals and a full-rank key factor: o = dense attention over (K, V), any predictor."""
    rng = np.random.default_rng(31 + selective)
    L, Hkv, G, hd, T = 2, 2, 2, 16, 200
    K_group, V, pred = _group_problem(rng, L=L, Hkv=Hkv, G=G, hd=hd, T=T)
    Bt = _orthogonal(rng, K_group.shape[1])
    packed = orc.pack_sequence(K_group, V, Bt, pred["W_lin"], pred["W1"], pred["b1"], pred["W2"],
                               pred["b2"], T, "f64", Hkv, hd)
    np.testing.assert_array_equal(packed["idx"][0, 0], np.arange(T))
    blocks = [[0, 3], [1, 2, 3]] if selective else None
    for layer in range(L):
        q = rng.standard_normal((Hkv * G, hd))
        o = orc.decode_sequence(q, packed["A"], Bt, pred["W_lin"], pred["W1"], pred["b1"],
                                pred["W2"], pred["b2"], layer, packed["idx"], packed["val"],
                                blocks, 0.0 + 0.2, Hkv, hd)
        for hq in range(Hkv * G):
            h = hq // G
            S = orc.selected_tokens(T, None if blocks is None else blocks[h])
            c0 = (layer * Hkv + h) * hd
            ref = orc.dense_attention(q[hq], K_group[S, c0:c0 + hd], V[layer][S, h], 0.2)
            np.testing.assert_allclose(o[hq], ref, rtol=1e-10, atol=1e-10)


def test_selection_all_blocks_equals_full_and_empty_is_zero():
    rng = np.random.default_rng(4)
    L, Hkv, G, hd, T = 1, 2, 2, 16, 150
    K_group, V, pred = _group_problem(rng, L=L, Hkv=Hkv, G=G, hd=hd, T=T)
    Bt = _orthogonal(rng, K_group.shape[1])[:, :20]
    packed = orc.pack_sequence(K_group, V, Bt, pred["W_lin"], pred["W1"], pred["b1"], pred["W2"],
                               pred["b2"], 30, "bf16", Hkv, hd)
    q = rng.standard_normal((Hkv * G, hd))
    args = (packed["A"], Bt, pred["W_lin"], pred["W1"], pred["b1"], pred["W2"], pred["b2"], 0,
            packed["idx"], packed["val"])
    full = orc.decode_sequence(q, *args, None, 0.25, Hkv, hd)
    allb = orc.decode_sequence(q, *args, [[0, 1, 2], [0, 1, 2]], 0.25, Hkv, hd)
    np.testing.assert_allclose(full, allb, rtol=1e-13, atol=1e-13)
    empty = orc.decode_sequence(q, *args, [[], [1]], 0.25, Hkv, hd)
    assert np.all(empty[:G] == 0) and np.all(np.isfinite(empty[G:]))


def test_residuals_are_value_minus_prediction_at_worst_tokens():
    rng = np.random.default_rng(9)
    L, Hkv, hd, T, k = 1, 1, 16, 120, 13
    K_group, V, pred = _group_problem(rng, L=L, Hkv=Hkv, hd=hd, T=T)
    Bt = _orthogonal(rng, K_group.shape[1])[:, :10]
    p = orc.pack_sequence(K_group, V, Bt, pred["W_lin"], pred["W1"], pred["b1"], pred["W2"],
                          pred["b2"], k, "f64", Hkv, hd)
    kt = orc.reconstruct_keys(p["A"], orc.key_slice(Bt, 0, 0, Hkv, hd))
    vh = orc.predict_values(kt, pred["W_lin"][0, 0], pred["W1"][0, 0], pred["b1"][0, 0],
                            pred["W2"][0, 0], pred["b2"][0, 0])
    e = ((V[0, :, 0] - vh) ** 2).sum(1)
    worst = np.argsort(-e, kind="stable")[:k]
    np.testing.assert_array_equal(p["idx"][0, 0], np.sort(worst))
    np.testing.assert_allclose(p["val"][0, 0], (V[0, :, 0] - vh)[np.sort(worst)], atol=1e-12)


# ----------------------------------------------------------------------------- accounting pins

def test_worked_memory_example():
    g = _gold("worked_memory_example.json")
    hd, H, ratio = g["head_dim"], g["hidden"], g["ratio"]
    assert orc.predictor_numbers(hd, H) == g["cases"][0]["predictor_numbers"]
    c0, c1, c2 = g["cases"]
    n0 = orc.residual_budget(c0["T"], hd, ratio, H)
    assert c0["T"] * hd == c0["value_numbers"] and c0["T"] * hd // ratio == c0["budget_numbers"]
    assert c0["budget_numbers"] - c0["predictor_numbers"] == c0["remaining_numbers"]
    assert hd + 2 == c0["numbers_per_residual"]
    assert round(n0) == c0["residuals_printed_approx"]
    assert round(100 * n0 / c0["T"]) == c0["fraction_printed_approx_pct"]
    n1 = orc.residual_budget(c1["T"], hd, ratio, H)
    assert round(n1) == c1["residuals_printed_approx"]
    assert round(100 * n1 / c1["T"]) == c1["fraction_printed_approx_pct"]
    share = orc.predictor_numbers(hd, H) / (c2["T"] * hd / ratio)
    assert abs(share - c2["predictor_share_approx"]) < 0.01


def test_dense_cache_bytes():
    g = _gold("dense_cache_size.json")
    b = orc.dense_cache_bytes_per_token(g["n_layers"], g["n_kv_heads"], g["head_dim"], g["elem_bytes"])
    assert round(b / 1000, 2) == g["kb_per_token_printed"]


@pytest.mark.parametrize("selective", [False, True])
def test_tail_joins_the_softmax_as_dense_tokens(selective):
    """Exact recent-token tail: with k = T residuals and a full-rank key factor the cache is
    exact, so decode with a tail equals dense attention over the attended cache tokens
    followed by the tail tokens (explainer: newly generated tokens are stored exactly)."""
    rng = np.random.default_rng(71 + selective)
    L, Hkv, G, hd, T, n_tail = 1, 2, 2, 16, 200, 5
    K_group, V, pred = _group_problem(rng, L=L, Hkv=Hkv, G=G, hd=hd, T=T)
    Bt = _orthogonal(rng, K_group.shape[1])
    packed = orc.pack_sequence(K_group, V, Bt, pred["W_lin"], pred["W1"], pred["b1"], pred["W2"],
                               pred["b2"], T, "f64", Hkv, hd)
    tail_K = rng.standard_normal((Hkv, n_tail, hd))
    tail_V = rng.standard_normal((Hkv, n_tail, hd))
    blocks = [[1], [0, 2, 3]] if selective else None
    q = rng.standard_normal((Hkv * G, hd))
    o = orc.decode_sequence(q, packed["A"], Bt, pred["W_lin"], pred["W1"], pred["b1"], pred["W2"], pred["b2"],
                            0, packed["idx"], packed["val"], blocks, 0.3, Hkv, hd, tail_K, tail_V)
    for hq in range(Hkv * G):
        h = hq // G
        S = orc.selected_tokens(T, None if blocks is None else blocks[h])
        K = np.concatenate([K_group[S, h * hd:(h + 1) * hd], tail_K[h]])
        Vh = np.concatenate([V[0][S, h], tail_V[h]])
        np.testing.assert_allclose(o[hq], orc.dense_attention(q[hq], K, Vh, 0.3), rtol=1e-10, atol=1e-10)


def test_tail_alone_and_tail_order():
    """A single tail token with nothing else attended is the output itself (softmax over one
    element); the tail's order does not matter."""
    rng = np.random.default_rng(5)
    L, Hkv, G, hd, T = 1, 2, 4, 16, 150
    K_group, V, pred = _group_problem(rng, L=L, Hkv=Hkv, G=G, hd=hd, T=T)
    Bt = _orthogonal(rng, K_group.shape[1])[:, :24]
    packed = orc.pack_sequence(K_group, V, Bt, pred["W_lin"], pred["W1"], pred["b1"], pred["W2"],
                               pred["b2"], 10, "bf16", Hkv, hd)
    args = (packed["A"], Bt, pred["W_lin"], pred["W1"], pred["b1"], pred["W2"], pred["b2"], 0,
            packed["idx"], packed["val"])
    q = rng.standard_normal((Hkv * G, hd))
    tK, tV = rng.standard_normal((Hkv, 1, hd)), rng.standard_normal((Hkv, 1, hd))
    only = orc.decode_sequence(q, *args, [[], []], 0.25, Hkv, hd, tK, tV)
    for hq in range(Hkv * G):
        np.testing.assert_array_equal(only[hq], tV[hq // G, 0])
    tK, tV = rng.standard_normal((Hkv, 6, hd)), rng.standard_normal((Hkv, 6, hd))
    perm = rng.permutation(6)
    a = orc.decode_sequence(q, *args, None, 0.25, Hkv, hd, tK, tV)
    b = orc.decode_sequence(q, *args, None, 0.25, Hkv, hd, tK[:, perm], tV[:, perm])
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)
    assert not np.allclose(a, orc.decode_sequence(q, *args, None, 0.25, Hkv, hd))


def test_block_scores_are_rank_space_means_and_selection_is_brute_force():
    """Block scores: the mean of a block's reconstructed keys equals the rank-space mean of
    its A rows times the basis (linearity), so the score can be formed from block means
    of A; a block whose keys are aligned with a query head wins; the selection is the
    brute-force top-n_sel with ties to the lower block id, ascending."""
    rng = np.random.default_rng(12)
    L, Hkv, G, hd, T, r = 1, 2, 2, 16, 300, 24
    K_group, V, pred = _group_problem(rng, L=L, Hkv=Hkv, G=G, hd=hd, T=T)
    Bt = _orthogonal(rng, K_group.shape[1])[:, :r]
    A = orc.project_keys(K_group, Bt)
    q = rng.standard_normal((Hkv * G, hd))
    sc = orc.block_scores(q, A, Bt, 0, Hkv, hd, 0.5)
    assert sc.shape == (Hkv, 5)
    for h in range(Hkv):
        Bh = orc.key_slice(Bt, 0, h, Hkv, hd)
        for j in range(5):
            abar = A[j * 64:min(T, j * 64 + 64)].mean(axis=0)   # the last block has 44 rows
            want = max(0.5 * float(q[h * G + g] @ (Bh @ abar)) for g in range(G))
            assert abs(sc[h, j] - want) <= 1e-12 * max(1.0, abs(want))
    # a planted block: keys of block 3 of head 1 point along query head 3 (G = 2: head 1 reads 2, 3)
    A2 = A.copy()
    B1 = orc.key_slice(Bt, 0, 1, Hkv, hd)
    A2[192:256] += 50.0 * (np.linalg.pinv(B1) @ q[3])
    assert np.argmax(orc.block_scores(q, A2, Bt, 0, Hkv, hd, 1.0)[1]) == 3
    # selection against brute force over all subsets, with ties
    import itertools
    s = np.array([[1.0, 3.0, 3.0, -2.0, 3.0, 0.5], [0.0, 0.0, 0.0, 0.0, 0.0, 0.0]])
    for n_sel in range(0, 7):
        got = orc.select_blocks(s, n_sel)
        for h in range(2):
            best = None
            for sub in itertools.combinations(range(6), n_sel):
                key = (sorted((-s[h, i] for i in sub)), list(sub))
                if best is None or key < best[0]:
                    best = (key, sub)
            # the chosen set has the largest multiset of scores and, among equals, the lowest ids
            assert list(got[h]) == sorted(best[1])


# ----------------------------------------------------------------------------- block means

def test_block_means_against_column_sums_and_block_scores():
    """Block means: a constant block gives that constant; the last block is clipped at T;
    summing mean x block size over the blocks gives the column sums of A; and scoring a
    block through its mean A row equals the oracle's block score over reconstructed keys
    (the rebuild is linear)."""
    rng = np.random.default_rng(21)
    T, r = 300, 10
    A = rng.standard_normal((T, r))
    A[64:128] = np.arange(r)                       # block 1 is constant
    m = orc.block_means(A)
    assert m.shape == (5, r)
    np.testing.assert_array_equal(m[1], np.arange(r, dtype=np.float64))
    sizes = np.array([64, 64, 64, 64, 44.0])
    np.testing.assert_allclose((m * sizes[:, None]).sum(axis=0), A.sum(axis=0), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(m[4] * 44.0, A[256:].sum(axis=0), rtol=1e-12, atol=1e-12)
    L, Hkv, G, hd = 1, 2, 3, 8
    K_group, _, _ = _group_problem(rng, L=L, Hkv=Hkv, G=G, hd=hd, T=T)
    Bt = _orthogonal(rng, K_group.shape[1])[:, :12]
    A2 = orc.project_keys(K_group, Bt)
    q = rng.standard_normal((Hkv * G, hd))
    sc = orc.block_scores(q, A2, Bt, 0, Hkv, hd, 0.3)
    mb = orc.block_means(A2)
    for h in range(Hkv):
        Bh = orc.key_slice(Bt, 0, h, Hkv, hd)
        want = np.max(0.3 * (q[h * G:(h + 1) * G] @ Bh) @ mb.T, axis=0)
        np.testing.assert_allclose(sc[h], want, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- 2-bit residual rows

def test_quantize_residual_rows_hand_values():
    rows = np.array([
        [0.0, 1.0, 2.0, 3.0, 3.0, 2.0, 1.0, 0.0],      # lo 0, step 1: the codes are the values
        [0.0, 0.5, 1.5, 2.5, 3.0, 3.0, 3.0, 3.0],      # ties: 0.5 -> 0, 1.5 -> 2, 2.5 -> 2 (even)
        [2.0, 2.0, 2.0, 2.0, 2.0, 2.0, 2.0, 2.0],      # constant row: step 0, codes 0
        [-3.0, 0.0, 3.0, 1.5, -3.0, -3.0, -3.0, -3.0],  # lo -3, step 2: 1.5, 3, 2.25 -> 2, 3, 2
    ])
    codes, lo, step = orc.quantize_residual_rows(rows)
    np.testing.assert_array_equal(codes[0], [0, 1, 2, 3, 3, 2, 1, 0])
    np.testing.assert_array_equal(codes[1], [0, 0, 2, 2, 3, 3, 3, 3])
    np.testing.assert_array_equal(codes[2], np.zeros(8))
    np.testing.assert_array_equal(codes[3], [0, 2, 3, 2, 0, 0, 0, 0])
    np.testing.assert_array_equal(lo, [0.0, 0.0, 2.0, -3.0])
    np.testing.assert_array_equal(step, [1.0, 1.0, 0.0, 2.0])
    back = orc.dequantize_residual_rows(codes, lo, step)
    np.testing.assert_array_equal(back[0], rows[0])
    np.testing.assert_array_equal(back[2], rows[2])
    assert back[3, 1] == 1.0 and back[3, 2] == 3.0


def test_quantize_residual_rows_nearest_level_and_bound():
    """Every entry gets a nearest level (within fp32 rounding of a tie), the row minimum and
    maximum get codes 0 and 3, and the round trip is within half a step."""
    rng = np.random.default_rng(5)
    rows = orc.round_bf16(rng.standard_normal((200, 128)) * np.exp(rng.uniform(-4, 4, (200, 1))))
    codes, lo, step = orc.quantize_residual_rows(rows)
    back = orc.dequantize_residual_rows(codes, lo, step)
    for i in range(rows.shape[0]):
        levels = lo[i] + np.arange(4) * np.float64(step[i])
        dist = np.abs(rows[i][:, None] - levels[None, :])
        got = dist[np.arange(128), codes[i]]
        assert np.all(got <= dist.min(axis=1) + 1e-6 * step[i])
        assert codes[i][np.argmin(rows[i])] == 0 and codes[i][np.argmax(rows[i])] == 3
        assert np.max(np.abs(back[i] - rows[i])) <= 0.5 * step[i] * (1 + 1e-5) + 1e-6 * np.abs(rows[i]).max()


def test_pack_2bit_layout():
    codes = np.array([[1, 2, 3, 0, 3, 3, 3, 3]], np.uint8)
    packed = orc.pack_2bit(codes)
    assert packed.tolist() == [[1 + (2 << 2) + (3 << 4), 255]]
    rng = np.random.default_rng(3)
    c = rng.integers(0, 4, (9, 128)).astype(np.uint8)
    np.testing.assert_array_equal(orc.unpack_2bit(orc.pack_2bit(c), 128), c)


# ----------------------------------------------------------------------------- test-time fitting

def _fit_problem(rng, T=13, hd=3, H=4, b2=True):
    kt = rng.standard_normal((T, hd))
    v = rng.standard_normal((T, hd))
    p = {"W_lin": rng.standard_normal((hd, hd)), "W1": rng.standard_normal((H, hd)),
         "b1": rng.standard_normal(H), "W2": rng.standard_normal((hd, H)),
         "b2": rng.standard_normal(hd) if b2 else None}
    return kt, v, p


@pytest.mark.parametrize("b2", [True, False])
def test_predictor_grads_match_finite_differences(b2):
    rng = np.random.default_rng(31)
    kt, v, p = _fit_problem(rng, b2=b2)
    gr = orc.predictor_grads(kt, v, p)
    assert set(gr) == {n for n, a in p.items() if a is not None}
    eps = 1e-6
    for name, g in gr.items():
        num = np.zeros_like(g)
        for ix in np.ndindex(g.shape):
            pp = {n: (None if a is None else a.copy()) for n, a in p.items()}
            pm = {n: (None if a is None else a.copy()) for n, a in p.items()}
            pp[name][ix] += eps
            pm[name][ix] -= eps
            num[ix] = (orc.predictor_loss(kt, v, pp) - orc.predictor_loss(kt, v, pm)) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-9, err_msg=name)


def test_fit_zero_steps_descent_and_exact_start():
    rng = np.random.default_rng(32)
    kt, v, p = _fit_problem(rng, T=40, hd=4, H=5)
    same = orc.fit_predictor(kt, v, p, 0, 0.1)
    for n in p:
        np.testing.assert_array_equal(same[n], p[n])
    l0 = orc.predictor_loss(kt, v, p)
    assert orc.predictor_loss(kt, v, orc.fit_predictor(kt, v, p, 1, 1e-3)) < l0
    assert orc.predictor_loss(kt, v, orc.fit_predictor(kt, v, p, 20, 1e-2)) < orc.predictor_loss(
        kt, v, orc.fit_predictor(kt, v, p, 1, 1e-2))
    # a start that already predicts every value exactly is a stationary point
    p0 = dict(p, W2=np.zeros_like(p["W2"]))
    v0 = kt @ p0["W_lin"].T + p0["b2"]
    fitted = orc.fit_predictor(kt, v0, p0, 5, 0.5)
    for n in p0:
        np.testing.assert_array_equal(fitted[n], p0[n])


def test_fit_linear_branch_converges_to_least_squares():
    """With the nonlinear branch switched off (W1 = 0, b1 = 0, W2 = 0 give zero gradients
    to W1, b1 and W2), gradient descent fits the linear map and b2 by least squares."""
    rng = np.random.default_rng(33)
    T, hd, H = 40, 3, 2
    kt = rng.standard_normal((T, hd))
    v = rng.standard_normal((T, hd))
    p = {"W_lin": np.zeros((hd, hd)), "W1": np.zeros((H, hd)), "b1": np.zeros(H),
         "W2": np.zeros((hd, H)), "b2": np.zeros(hd)}
    fitted = orc.fit_predictor(kt, v, p, 3000, 1.0)
    X = np.concatenate([kt, np.ones((T, 1))], axis=1)
    sol, *_ = np.linalg.lstsq(X, v, rcond=None)
    np.testing.assert_allclose(fitted["W_lin"], sol[:hd].T, atol=1e-8)
    np.testing.assert_allclose(fitted["b2"], sol[hd], atol=1e-8)
    np.testing.assert_array_equal(fitted["W1"], 0.0)
    np.testing.assert_array_equal(fitted["W2"], 0.0)
