"""Pins for the CPU oracle: it is checked against things other than itself.

Each test names what fixes the expected value: a figure the LoopVQ pages
print, a hand-worked fixture (tests/golden/hand_worked.json), a closed form,
a library routine computing the same definition by another route (SciPy
cdist, torch scaled_dot_product_attention), or an invariant of softmax
attention.  Chosen so that a dropped term, a wrong sign or index, or a
transposed operand anywhere in the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.spatial.distance import cdist
from scipy.special import logsumexp

import oracle as O
from sub_bit_vector_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _sdpa(q, K, V, scale):
    """torch's fused attention (math backend, fp64) for one query."""
    qt = torch.tensor(q, dtype=torch.float64).reshape(1, 1, 1, -1)
    Kt = torch.tensor(K, dtype=torch.float64).reshape(1, 1, K.shape[0], -1)
    Vt = torch.tensor(V, dtype=torch.float64).reshape(1, 1, V.shape[0], -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)
    return o.reshape(-1).numpy()


# ---------------------------------------------------------------- accounting

def test_page_figures_bits_and_bytes():
    fig = _load("page_figures.json")
    for row in fig["bits_and_compression"]:
        assert O.bits_per_element(row["n_codes"], row["group_elems"]) == row["bits"]
        assert O.compression_vs_bf16(row["n_codes"], row["group_elems"]) == row["compression_vs_bf16"]
    for row in fig["bytes_per_token_and_loop_step"]:
        b = O.bytes_per_token_step(row["head_dim"], row["group_elems"], row["tc"])
        assert b["ratio"] == row["ratio_vs_bf16"]
    # geometry of the configurations used throughout
    g = O.geometry(4, 4, 128, 16)
    assert (g["W"], g["J"], g["NB"], g["bits"]) == (4, 32, 1, 0.5)
    g = O.geometry(4, 4, 128, 32)
    assert (g["W"], g["J"], g["NB"], g["bits"]) == (8, 16, 1, 0.25)
    g = O.geometry(4, 1, 128, 16)
    assert (g["W"], g["J"], g["NB"]) == (16, 8, 4)
    with pytest.raises(ValueError):
        O.geometry(4, 3, 128, 16)


# ---------------------------------------------------------- hand-worked case

def test_hand_worked_example():
    g = _load("hand_worked.json")
    X = np.array(g["X_T_N_H_D"], dtype=np.float64)
    cb = np.array(g["codebook_NB_H_J_C_Tc_W"], dtype=np.float64)
    tc = g["geometry"]["Tc"]
    idx, d1, d2 = O.encode(X, cb, tc)
    np.testing.assert_array_equal(idx, np.array(g["idx_NB_H_N_J"]))
    np.testing.assert_array_equal(d1, np.array(g["d_best_NB_H_N_J"]))
    np.testing.assert_array_equal(d2, np.array(g["d_second_NB_H_N_J"]))
    np.testing.assert_array_equal(O.dequantize(idx, cb, 0, tc), np.array(g["dequant_step0_N_H_D"]))
    np.testing.assert_array_equal(O.dequantize(idx, cb, 1, tc), np.array(g["dequant_step1_N_H_D"]))
    assert O.reconstruction_mse(X, idx, cb, tc) == g["mse"]

    a = g["attention_step1"]
    q = np.array([a["q"]])
    empty = np.zeros((1, 0, 2))
    o, lse = O.decode_attention(q, 1, tc, idx, idx, cb, cb, empty, empty, a["scale"])
    np.testing.assert_allclose(o[0], a["o"], rtol=1e-14)
    assert abs(lse[0] - a["lse"]) < 1e-14

    w = g["attention_step1_with_window"]
    o, lse = O.decode_attention(q, 1, tc, idx, idx, cb, cb, np.array([w["win_k"]]),
                                np.array([w["win_v"]]), a["scale"])
    np.testing.assert_allclose(o[0], w["o"], rtol=1e-14)
    assert abs(lse[0] - w["lse"]) < 1e-14


# -------------------------------------------------------------------- encode

def _subvectors_by_reshape(X, tc, w):
    """Loop-axis sub-vectors by a second route: reshape D into (J, W) and
    move the step axis next to W, giving [NB][N][H][J][Tc*W]."""
    T, N, H, D = X.shape
    J = D // w
    Y = X.reshape(T // tc, tc, N, H, J, w)           # [NB][Tc][N][H][J][W]
    Y = np.moveaxis(Y, 1, 4)                         # [NB][N][H][J][Tc][W]
    return Y.reshape(T // tc, N, H, J, tc * w)


@pytest.mark.parametrize("tc,G", [(4, 16), (4, 32), (1, 16), (2, 8)])
def test_encode_matches_cdist_argmin(tc, G):
    rng = np.random.default_rng(11)
    T, N, H, D, C = 4, 96, 2, 32, 64
    X = rng.standard_normal((T, N, H, D))
    w = G // tc
    cb = rng.standard_normal((T // tc, H, D // w, C, tc, w))
    idx, d1, d2 = O.encode(X, cb, tc)
    sub = _subvectors_by_reshape(X, tc, w)
    for b in range(T // tc):
        for h in range(H):
            for j in range(D // w):
                d = cdist(sub[b, :, h, j], cb[b, h, j].reshape(C, G), "sqeuclidean")
                np.testing.assert_array_equal(idx[b, h, :, j], np.argmin(d, axis=1))
                np.testing.assert_allclose(d1[b, h, :, j], d.min(axis=1), rtol=1e-12)
                np.testing.assert_allclose(d2[b, h, :, j], np.sort(d, axis=1)[:, 1], rtol=1e-12)


def test_exact_codeword_returns_its_index_and_roundtrip():
    rng = np.random.default_rng(5)
    T, tc, H, D, G, C, N = 4, 4, 2, 16, 16, 32, 40
    w = G // tc
    cb = rng.standard_normal((1, H, D // w, C, tc, w))
    codes = rng.integers(0, C, size=(1, H, N, D // w))
    X = np.stack([O.dequantize(codes, cb, t, tc) for t in range(T)])   # [T][N][H][D]
    idx, d1, _ = O.encode(X, cb, tc)
    np.testing.assert_array_equal(idx, codes)
    assert np.all(d1 == 0.0)
    assert O.reconstruction_mse(X, idx, cb, tc) == 0.0


def test_duplicate_codewords_give_lowest_index():
    rng = np.random.default_rng(6)
    cb = rng.standard_normal((1, 1, 2, 8, 2, 2))
    cb[0, 0, :, 5] = cb[0, 0, :, 2]      # codeword 5 duplicates 2
    cb[0, 0, :, 7] = cb[0, 0, :, 2]
    X = np.zeros((2, 3, 1, 4))
    for t in range(2):
        X[t, :, 0, 0:2] = cb[0, 0, 0, 2, t]
        X[t, :, 0, 2:4] = cb[0, 0, 1, 2, t]
    idx, d1, d2 = O.encode(X, cb, 2)
    assert np.all(idx == 2)
    assert np.all(d1 == 0) and np.all(d2 == 0)


def test_tiny_codebook_rows_encode_to_their_own_index():
    K, _ = synth.tiny_kv(seed=0)
    tc, G = 4, 16
    cb = synth.codebook_from_rows(K, tc, G, 256, seed=1)
    idx, d1, _ = O.encode(K, cb, tc)
    rng = np.random.Generator(np.random.PCG64(1))
    rows = rng.permutation(K.shape[1])[:256]       # the draw of slot 0
    np.testing.assert_array_equal(idx[0, 0, rows, 0], np.arange(256))
    assert np.all(d1[0, 0, rows, 0] == 0.0)


def test_loop_axis_code_beats_single_step_code():
    """Project page, 'Method', loop-axis redundancy figure: at equal bits a
    code spanning four loop steps reconstructs with lower error than a code
    spanning one step.  Directional: the pages print no values."""
    X = synth.loop_correlated(seed=4, n_loop=4, n_tokens=2048, n_heads=1, head_dim=32,
                              rho=0.9, bf16=False)
    mse = {}
    for tc in (4, 1):
        cb = synth.codebook_from_rows(X, tc, 16, 256, seed=9)
        idx, _, _ = O.encode(X, cb, tc)
        assert O.bits_per_element(256, 16) == 0.5
        mse[tc] = O.reconstruction_mse(X, idx, cb, tc)
    assert mse[4] < mse[1]


# ----------------------------------------------------------------- attention

def test_window_split_closed_form():
    assert O.window_split(32768, 64, 256, 8) == (64, 32448, 256)
    assert O.window_split(32770, 64, 256, 8) == (64, 32448, 258)
    assert O.window_split(32775, 64, 256, 8) == (64, 32448, 263)
    assert O.window_split(32776, 64, 256, 8) == (64, 32456, 256)
    assert O.window_split(320, 64, 256, 8) == (64, 0, 256)
    assert O.window_split(321, 64, 256, 8) == (64, 0, 257)
    assert O.window_split(300, 64, 256, 8) == (64, 0, 236)
    assert O.window_split(50, 64, 256, 8) == (50, 0, 0)
    assert O.window_split(0, 64, 256, 8) == (0, 0, 0)
    assert O.window_split(512, 0, 0, 8) == (0, 512, 0)
    for ctx in range(321, 2000, 37):
        s, b, r = O.window_split(ctx, 64, 256, 8)
        assert s + b + r == ctx and b % 8 == 0 and 256 <= r <= 263


def test_attention_matches_sdpa_and_logsumexp():
    rng = np.random.default_rng(2)
    q = rng.standard_normal(64)
    K = rng.standard_normal((300, 64))
    V = rng.standard_normal((300, 64))
    scale = 1 / 8
    o, lse = O.attention(q, K, V, scale)
    np.testing.assert_allclose(o, _sdpa(q, K, V, scale), rtol=1e-12, atol=1e-14)
    assert abs(lse - logsumexp(scale * K @ q)) < 1e-12


def test_all_dense_decode_is_textbook_attention():
    """Tc = 1, no body (context within the window): plain softmax attention."""
    rng = np.random.default_rng(3)
    T, H, D, n = 4, 2, 32, 200
    Kw = synth.round_bf16(rng.standard_normal((T, H, n, D)))
    Vw = synth.round_bf16(rng.standard_normal((T, H, n, D)))
    q = rng.standard_normal((T, H, D))
    cb = np.zeros((T, H, D // 16, 256, 1, 16))
    none = np.zeros((T, H, 0, D // 16), dtype=np.int64)
    for t in range(T):
        o, _ = O.decode_attention(q[t], t, 1, none, none, cb, cb, Kw[t], Vw[t], D ** -0.5)
        od, _ = O.dense_decode_attention(q[t], Kw[t], Vw[t], D ** -0.5)
        for h in range(H):
            np.testing.assert_allclose(o[h], _sdpa(q[t, h], Kw[t, h], Vw[t, h], D ** -0.5), rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(od[h], o[h], rtol=1e-14, atol=1e-15)


def test_lossless_vq_equals_dense_attention():
    """Codebook = every token's own sub-vector, so the body reconstructs
    exactly and decode attention from codes equals dense attention."""
    X = synth.loop_correlated(seed=7, n_loop=4, n_tokens=256, n_heads=2, head_dim=32, rho=0.9)
    V = synth.loop_correlated(seed=8, n_loop=4, n_tokens=256, n_heads=2, head_dim=32, rho=0.9)
    tc, G = 4, 16
    cbk = synth.codebook_from_rows(X, tc, G, 256, seed=1)
    cbv = synth.codebook_from_rows(V, tc, G, 256, seed=2)
    ik, dk, _ = O.encode(X, cbk, tc)
    iv, dv, _ = O.encode(V, cbv, tc)
    assert np.all(dk == 0) and np.all(dv == 0)
    q = synth.queries(3, 4, 1, 2, 32)[:, 0]
    # window: the first 16 tokens in bf16, body: the rest from codes
    for t in range(4):
        win_k = np.transpose(X[t, :16], (1, 0, 2))
        win_v = np.transpose(V[t, :16], (1, 0, 2))
        o, lse = O.decode_attention(q[t], t, tc, ik[:, :, 16:], iv[:, :, 16:], cbk, cbv,
                                    win_k, win_v, 32 ** -0.5)
        for h in range(2):
            ref = _sdpa(q[t, h], X[t, :, h], V[t, :, h], 32 ** -0.5)
            np.testing.assert_allclose(o[h], ref, rtol=1e-12, atol=1e-13)
            ref_lse = logsumexp(32 ** -0.5 * X[t, :, h].astype(np.float64) @ q[t, h].astype(np.float64))
            assert abs(lse[h] - ref_lse) < 1e-11


def test_single_token_returns_its_value():
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 16))
    k = rng.standard_normal((1, 1, 16))
    v = rng.standard_normal((1, 1, 16))
    cb = np.zeros((1, 1, 4, 256, 4, 4))
    none = np.zeros((1, 1, 0, 4), dtype=np.int64)
    o, lse = O.decode_attention(q, 0, 4, none, none, cb, cb, k, v, 0.25)
    np.testing.assert_array_equal(o[0], v[0, 0])
    assert abs(lse[0] - 0.25 * float(q[0] @ k[0, 0])) < 1e-15


def test_shift_of_all_keys_leaves_output_unchanged():
    """Adding the same vector u to every key (window keys and K codewords)
    adds scale*q.u to every score, which softmax ignores; lse moves by it."""
    rng = np.random.default_rng(9)
    T, tc, H, D, G, C, nb, nw = 4, 4, 1, 16, 16, 16, 50, 10
    w = G // tc
    cbk = rng.standard_normal((1, H, D // w, C, tc, w))
    cbv = rng.standard_normal((1, H, D // w, C, tc, w))
    ik = rng.integers(0, C, (1, H, nb, D // w))
    iv = rng.integers(0, C, (1, H, nb, D // w))
    wk = rng.standard_normal((H, nw, D))
    wv = rng.standard_normal((H, nw, D))
    q = rng.standard_normal((H, D))
    t = 2
    u = rng.standard_normal(D)
    cbk2 = cbk.copy()
    for j in range(D // w):
        cbk2[0, :, j, :, t, :] += u[j * w:(j + 1) * w]
    o1, l1 = O.decode_attention(q, t, tc, ik, iv, cbk, cbv, wk, wv, 0.3)
    o2, l2 = O.decode_attention(q, t, tc, ik, iv, cbk2, cbv, wk + u, wv, 0.3)
    np.testing.assert_allclose(o1, o2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(l2 - l1, 0.3 * q @ u, rtol=1e-11)


def test_equal_keys_give_mean_of_values():
    rng = np.random.default_rng(10)
    H, D, nb, nw = 2, 8, 30, 5
    cbk = np.zeros((1, H, 2, 4, 4, 4))
    cbk[:, :, :, :, :, :] = 0.7                     # all K codewords equal
    cbv = rng.standard_normal((1, H, 2, 4, 4, 4))
    ik = rng.integers(0, 4, (1, H, nb, 2))
    iv = rng.integers(0, 4, (1, H, nb, 2))
    wk = np.full((H, nw, D), 0.7)
    wv = rng.standard_normal((H, nw, D))
    q = rng.standard_normal((H, D))
    o, lse = O.decode_attention(q, 3, 4, ik, iv, cbk, cbv, wk, wv, 0.5)
    Vb = O.dequantize(iv, cbv, 3, 4)
    for h in range(H):
        mean = np.concatenate([wv[h], Vb[:, h]]).mean(axis=0)
        np.testing.assert_allclose(o[h], mean, rtol=1e-12, atol=1e-14)
        assert abs(lse[h] - (0.5 * 0.7 * q[h].sum() + math.log(nb + nw))) < 1e-12


def test_gqa_head_mapping():
    rng = np.random.default_rng(12)
    H, Hq, D, n = 2, 4, 16, 20
    K = rng.standard_normal((H, n, D))
    V = rng.standard_normal((H, n, D))
    q = rng.standard_normal((Hq, D))
    o, _ = O.dense_decode_attention(q, K, V, 0.25)
    for hq in range(Hq):
        np.testing.assert_allclose(o[hq], _sdpa(q[hq], K[hq // 2], V[hq // 2], 0.25), rtol=1e-12)


def test_dequantize_rejects_out_of_range_codes():
    cb = np.zeros((1, 1, 1, 4, 1, 4))
    with pytest.raises(ValueError):
        O.dequantize(np.full((1, 1, 2, 1), 4), cb, 0, 1)


# ----------------------------------------------------------------- generator

def test_generator_loop_correlation_and_scale():
    X = synth.loop_correlated(seed=1, n_loop=4, n_tokens=4096, n_heads=2, head_dim=64,
                              rho=0.9, bf16=False)
    a = X[:-1].reshape(3, -1)
    b = X[1:].reshape(3, -1)
    for t in range(3):
        assert abs(np.corrcoef(a[t], b[t])[0, 1] - 0.9) < 0.01
    assert abs(X.std() - 1.0) < 0.02
    K = synth.loop_correlated(seed=1, n_loop=4, n_tokens=1024, n_heads=2, head_dim=64,
                              rho=0.9, n_outlier=4, bf16=True)
    per_chan = np.abs(K).mean(axis=(0, 1))           # [H][D]
    assert np.all(np.sort(per_chan, axis=1)[:, -4:].min(axis=1) > 3 * np.median(per_chan))
    assert np.array_equal(K, synth.round_bf16(K))    # already bf16 values


# ---------------------------------------------------------- codebook k-means

def _small_kv(seed, n=600, h=2, d=16):
    return synth.loop_correlated(seed=seed, n_loop=4, n_tokens=n, n_heads=h, head_dim=d, n_outlier=1)


def test_kmeans_one_round_matches_scikit_learn_lloyd():
    """One Lloyd round (nearest-codeword assignment, then means) against
    scikit-learn's Lloyd k-means started from the same centers; the codebook
    is made of data rows, so no cluster is empty."""
    from sklearn.cluster import KMeans
    X = _small_kv(500)
    tc, G, C = 4, 16, 32
    cb = synth.codebook_from_rows(X, tc, G, C, seed=501)
    new, idx, _ = O.kmeans(X, cb, tc, 1)
    W = G // tc
    sub = O.form_subvectors(X, 0, tc, W)
    for h in range(X.shape[2]):
        for j in range(X.shape[3] // W):
            init = cb[0, h, j].reshape(C, G).astype(np.float64)
            km = KMeans(n_clusters=C, init=init, n_init=1, max_iter=1, tol=0.0, algorithm="lloyd")
            km.fit(sub[:, h, j])
            np.testing.assert_allclose(new[0, h, j].reshape(C, G), km.cluster_centers_, rtol=1e-12, atol=1e-12)


def test_kmeans_update_single_member_and_empty_cluster():
    """A codeword with one member becomes that sub-vector exactly; a codeword
    without members keeps its value."""
    X = _small_kv(510, n=8, h=1, d=8)
    tc, G = 4, 8  # W = 2, J = 4
    rng = np.random.default_rng(511)
    cb = rng.standard_normal((1, 1, 4, 16, tc, G // tc))
    idx = np.zeros((1, 1, 8, 4), dtype=np.int64)
    idx[0, 0, :, :] = np.arange(8)[:, None]          # token n -> code n in every slot
    new, counts = O.kmeans_update(X, idx, cb, tc)
    sub = O.form_subvectors(X, 0, tc, G // tc)
    for j in range(4):
        for n in range(8):
            np.testing.assert_array_equal(new[0, 0, j, n].reshape(-1), sub[n, 0, j])
        np.testing.assert_array_equal(new[0, 0, j, 8:], cb[0, 0, j, 8:])
        assert list(counts[0, 0, j]) == [1] * 8 + [0] * 8


def test_kmeans_update_closed_form_two_clusters():
    """Two hand-made groups of sub-vectors: the update is their arithmetic
    means, written out."""
    X = np.zeros((1, 5, 1, 2))
    X[0, :, 0, 0] = [1.0, 2.0, 3.0, 10.0, 14.0]
    X[0, :, 0, 1] = [0.0, 0.0, 3.0, -2.0, -4.0]
    cb = np.zeros((1, 1, 1, 2, 1, 2))
    idx = np.array([0, 0, 0, 1, 1]).reshape(1, 1, 5, 1)
    new, counts = O.kmeans_update(X, idx, cb, 1)
    np.testing.assert_allclose(new[0, 0, 0, 0, 0], [2.0, 1.0])
    np.testing.assert_allclose(new[0, 0, 0, 1, 0], [12.0, -3.0])
    assert list(counts[0, 0, 0]) == [3, 2]


def test_kmeans_update_is_the_distortion_minimiser_and_a_fixed_point():
    """For a fixed assignment the mean minimises the squared error: any
    perturbation of the updated codebook raises the distortion; updating
    again with the same assignment changes nothing."""
    X = _small_kv(520)
    tc, G, C = 2, 8, 16
    cb = synth.codebook_from_rows(X, tc, G, C, seed=521)
    idx, _, _ = O.encode(X, cb, tc)
    new, _ = O.kmeans_update(X, idx, cb, tc)
    base = O.distortion(X, idx, new, tc)
    assert base <= O.distortion(X, idx, cb, tc)
    rng = np.random.default_rng(522)
    for _ in range(3):
        bumped = new + 1e-3 * rng.standard_normal(new.shape)
        assert O.distortion(X, idx, bumped, tc) > base
    again, _ = O.kmeans_update(X, idx, new, tc)
    np.testing.assert_allclose(again, new, rtol=0, atol=1e-13)


def test_distortion_hand_value_and_element_identity():
    """The distortion is the sum, over every sub-vector, of its squared
    distance to its codeword: 1 on the hand-worked fixture (one element off by
    one), the encoder's best distances summed, and -- every element lying in
    exactly one sub-vector -- the mean squared reconstruction error times the
    element count, with several code blocks, heads and slots."""
    g = _load("hand_worked.json")
    X = np.array(g["X_T_N_H_D"], dtype=np.float64)
    cb = np.array(g["codebook_NB_H_J_C_Tc_W"], dtype=np.float64)
    idx = np.array(g["idx_NB_H_N_J"])
    assert O.distortion(X, idx, cb, g["geometry"]["Tc"]) == 1.0
    rng = np.random.default_rng(760)
    T, tc, N, H, D, G, C = 4, 2, 37, 3, 16, 4, 9     # NB = 2 blocks, W = 2, J = 8
    X = rng.standard_normal((T, N, H, D))
    cb = rng.standard_normal((T // tc, H, D // (G // tc), C, tc, G // tc))
    idx, d1, _ = O.encode(X, cb, tc)
    total = O.distortion(X, idx, cb, tc)
    assert total == pytest.approx(float(np.sum(d1)), rel=1e-12)
    assert total == pytest.approx(O.reconstruction_mse(X, idx, cb, tc) * X.size, rel=1e-12)
    # a code that is not the nearest one adds exactly its extra distance
    idx2 = idx.copy()
    idx2[1, 2, 5, 3] = (idx[1, 2, 5, 3] + 1) % C
    sub = X[2:4, 5, 2, 6:8].reshape(-1)   # block 1, token 5, head 2, slot 3: channels 6..7 of steps 2..3, order [t][w]
    extra = np.sum((sub - cb[1, 2, 3, idx2[1, 2, 5, 3]].reshape(-1)) ** 2) - d1[1, 2, 5, 3]
    assert O.distortion(X, idx2, cb, tc) == pytest.approx(total + extra, rel=1e-12)


def test_lloyd_distortion_never_increases():
    X = _small_kv(530)
    cb = synth.codebook_from_rows(X, 4, 16, 32, seed=531)
    _, _, hist = O.kmeans(X, cb, 4, 5)
    assert all(b <= a * (1 + 1e-12) for a, b in zip(hist, hist[1:]))
    assert hist[-1] < hist[0]


# ------------------------------------------ codebook gradient (fine-tuning)

def _grad_case(seed, tc, T=4, H=2, Hq=4, D=8, G=4, n_body=7, n_win=3, n_codes=6, C=256):
    rng = np.random.default_rng(seed)
    W = G // tc
    J = D // W
    NB = T // tc
    cbk = rng.standard_normal((NB, H, J, C, tc, W))
    cbv = rng.standard_normal((NB, H, J, C, tc, W))
    ik = rng.integers(0, n_codes, (NB, H, n_body, J))
    iv = rng.integers(0, n_codes, (NB, H, n_body, J))
    wk = rng.standard_normal((H, n_win, D))
    wv = rng.standard_normal((H, n_win, D))
    q = rng.standard_normal((Hq, D))
    target = 0.3 * rng.standard_normal((Hq, D))
    return cbk, cbv, ik, iv, wk, wv, q, target


def _fd_loss(case, tc, t, scale, weight):
    cbk, cbv, ik, iv, wk, wv, q, target = case
    o, _ = O.decode_attention(q, t, tc, ik, iv, cbk, cbv, wk, wv, scale)
    return weight * float(np.sum((o - target) ** 2))


@pytest.mark.parametrize("tc,t,n_win", [(2, 3, 3), (4, 2, 3), (1, 1, 0)])
def test_codebook_grad_matches_central_differences(tc, t, n_win):
    """Every gradient entry of the codewords in use, in the step's block and
    slice, equals the central difference of the loss computed through
    ``decode_attention``; entries of other slices and blocks and of unused
    codewords move the loss by nothing and are zero."""
    scale, weight, eps = 0.7, 1.3, 1e-6
    case = _grad_case(600 + tc, tc, n_win=n_win)
    cbk, cbv, ik, iv, wk, wv, q, target = case
    loss, gk, gv, out = O.attention_mse_codebook_grad(q, t, tc, ik, iv, cbk, cbv, wk, wv, scale, target, weight)
    assert loss == pytest.approx(_fd_loss(case, tc, t, scale, weight), rel=1e-13)
    np.testing.assert_allclose(out, O.decode_attention(q, t, tc, ik, iv, cbk, cbv, wk, wv, scale)[0], rtol=1e-13)
    b, tt = divmod(t, tc)
    NB, H, J, _, _, W = cbk.shape
    for which, grad in ((0, gk), (1, gv)):
        cb = case[which]
        checked = 0
        for h in range(H):
            for j in range(J):
                for c in range(6):
                    for w in range(W):
                        e = (b, h, j, c, tt, w)
                        keep = cb[e]
                        cb[e] = keep + eps
                        up = _fd_loss(case, tc, t, scale, weight)
                        cb[e] = keep - eps
                        dn = _fd_loss(case, tc, t, scale, weight)
                        cb[e] = keep
                        fd = (up - dn) / (2 * eps)
                        assert grad[e] == pytest.approx(fd, rel=1e-6, abs=1e-8), (which, e)
                        checked += int(abs(fd) > 1e-6)
        assert checked > H * J  # the check is not vacuous
        # other slices / blocks and unused codewords: zero
        mask = np.zeros(grad.shape, dtype=bool)
        mask[b, :, :, :6, tt, :] = True
        assert np.all(grad[~mask] == 0.0)
        e = (NB - 1 - b, 0, 0, 1, (tt + 1) % tc, 0) if tc > 1 or NB > 1 else (b, 0, 0, 7, tt, 0)
        keep = cb[e]
        cb[e] = keep + 1e-3
        assert _fd_loss(case, tc, t, scale, weight) == _fd_loss(case, tc, t, scale, weight)
        moved = _fd_loss(case, tc, t, scale, weight)
        cb[e] = keep
        assert moved == pytest.approx(loss, rel=1e-14)


def test_codebook_grad_zero_at_target_and_empty_body():
    """Target equal to the output: zero loss and zero gradient.  A context of
    window tokens only: zero gradient, loss against the window attention."""
    tc, t, scale = 2, 1, 0.5
    cbk, cbv, ik, iv, wk, wv, q, _ = _grad_case(610, tc)
    o, _ = O.decode_attention(q, t, tc, ik, iv, cbk, cbv, wk, wv, scale)
    loss, gk, gv, _ = O.attention_mse_codebook_grad(q, t, tc, ik, iv, cbk, cbv, wk, wv, scale, o)
    # (decode_attention divides after the sum: the two outputs differ by rounding)
    assert loss < 1e-28 and np.max(np.abs(gk)) < 1e-13 and np.max(np.abs(gv)) < 1e-13
    target = np.ones_like(o)
    e0k, e0v = ik[:, :, :0], iv[:, :, :0]
    loss, gk, gv, out = O.attention_mse_codebook_grad(q, t, tc, e0k, e0v, cbk, cbv, wk, wv, scale, target, 2.0)
    ref = O.dense_decode_attention(q, wk, wv, scale)[0]
    np.testing.assert_allclose(out, ref, rtol=1e-13)
    assert loss == pytest.approx(2.0 * float(np.sum((ref - 1.0) ** 2)), rel=1e-13)
    assert not gk.any() and not gv.any()


# ------------------------------------------- KV-residual 4-bit quantization

def test_quantize4_grid_values_are_exact():
    """Values on the 16-level grid of an fp16-representable min and scale
    come back exactly, with their level as the code; the extremes are codes
    0 and 15."""
    lo, sc = np.float16(-1.25), np.float16(0.125)
    levels = np.array([0, 15, 3, 7, 7, 12, 1, 15, 0, 9], dtype=np.uint8)
    x = np.float32(lo) + levels.astype(np.float32) * np.float32(sc)
    q, l, c = O.quantize4_group(x)
    assert l == lo and c == sc
    np.testing.assert_array_equal(q, levels)
    np.testing.assert_array_equal(O.dequantize4(q, l, c), x)
    # half-way values round to the even level
    half = np.array([0, 15, 2.5, 3.5, 10.5], dtype=np.float32)
    q, _, _ = O.quantize4_group(np.float32(lo) + half * np.float32(sc))
    np.testing.assert_array_equal(q, [0, 15, 2, 4, 10])


def test_quantize4_error_bound_and_constant_group():
    """|x - dequant| is at most half a step plus the fp16 rounding of min and
    scale (times the largest code); a constant group has scale 0, codes 0 and
    reconstructs to its fp16-rounded value."""
    rng = np.random.default_rng(700)
    for _ in range(200):
        x = (rng.standard_normal(32) * rng.uniform(0.01, 10)).astype(np.float32)
        q, l, c = O.quantize4_group(x)
        lo, hi = float(x.min()), float(x.max())
        scale = np.float32(np.float32(hi - lo) / np.float32(15))
        bound = 0.5 * float(c) + abs(float(l) - lo) + 15 * abs(float(c) - float(scale)) + 1e-6 * max(abs(lo), abs(hi))
        assert np.max(np.abs(O.dequantize4(q, l, c) - x)) <= bound
        assert q.max() <= 15
    q, l, c = O.quantize4_group(np.full(32, 0.3, dtype=np.float32))
    assert c == 0 and not q.any() and np.all(O.dequantize4(q, l, c) == np.float32(np.float16(0.3)))


def _residual_hand_worked_inputs(g, kind):
    """The fixture's inputs and hand-derived expectations (closed forms stated
    in tests/golden/residual_hand_worked.json)."""
    T, N, H, D = g["shape_T_N_H_D"]
    n = np.arange(N)[:, None]
    d = np.arange(D)[None, :]
    delta = g["delta"]
    if kind == "k":
        x0 = 0.5 * (n % 16) + 8.0 * (d % 2) + delta * (n == 5)
        code0 = np.broadcast_to(n % 16, (N, D))
        hat0 = 0.5 * (n % 16) + 8.0 * (d % 2)
    else:
        x0 = 0.5 * (d % 16) + 8.0 * (n % 2) + delta * (d == 5)
        code0 = np.broadcast_to(d % 16, (N, D))
        hat0 = 0.5 * (d % 16) + 8.0 * (n % 2)
    code1 = (n + d) % 16
    x1 = hat0 + 0.25 * code1
    X = np.stack([x0, x1])[:, :, None, :].astype(np.float32)      # [T][N][H][D]
    return X, code0, hat0, code1, x1


@pytest.mark.parametrize("kind", ["k", "v"])
def test_residual_hand_worked_two_steps(kind):
    """FlashLoop page, Figure 2 (c) and Figure 3 (c-d), with the readings of
    KIVI's axes and the reconstruction as the residual's reference: a
    two-step case derived by hand.  Coding step 1 against K_0 instead of
    Khat_0, or grouping along the other axis, changes the codes or the
    parameters checked here."""
    g = _load("residual_hand_worked.json")
    X, code0, hat0, code1, x1 = _residual_hand_worked_inputs(g, kind)
    codes, lo, sc, recon = O.residual_encode(X, kind)
    np.testing.assert_array_equal(codes[0, 0], code0)
    np.testing.assert_array_equal(codes[1, 0], code1)
    np.testing.assert_array_equal(recon[0, :, 0], hat0.astype(np.float32))
    np.testing.assert_array_equal(recon[1, :, 0], x1.astype(np.float32))
    e = g["keys" if kind == "k" else "values"]
    par = np.arange(32) % 2
    if kind == "k":     # one token group: lo/scale [T][H][1][D]
        np.testing.assert_array_equal(lo[0, 0, 0], np.array(e["step0"]["lo_per_channel_parity"])[par])
        assert lo.shape == (2, 1, 1, 32)
    else:               # one channel group per token: [T][H][N][1]
        np.testing.assert_array_equal(lo[0, 0, :, 0], np.array(e["step0"]["lo_per_token_parity"])[par])
        assert lo.shape == (2, 1, 32, 1)
    assert np.all(sc[0] == np.float16(e["step0"]["scale"])) and np.all(sc[1] == np.float16(e["step1"]["scale"]))
    assert np.all(lo[1] == np.float16(e["step1"]["lo"]))
    for sp in e["spot"]:
        t, n_, d_ = sp["t"], sp["n"], sp["d"]
        assert X[t, n_, 0, d_] == sp["x"]
        assert codes[t, 0, n_, d_] == sp["code"]
        assert recon[t, n_, 0, d_] == sp["recon"]
        assert O.residual_reconstruct(codes, lo, sc, kind, t)[n_, 0, d_] == sp["recon"]


def test_residual_hand_worked_rejects_the_other_readings():
    """The fixture tells the readings apart: against the raw previous step
    the key residual of channel 11 has its minimum at -delta; grouped along
    the other axis the step-0 scale is fp16(8/15), not 0.5."""
    g = _load("residual_hand_worked.json")
    X, _, _, _, _ = _residual_hand_worked_inputs(g, "k")
    raw_resid = X[1, :, 0, 11] - X[0, :, 0, 11]
    _, lo_raw, _ = O.quantize4_group(raw_resid)
    assert lo_raw == np.float16(-g["delta"])
    # keys grouped per token (the values' axis): token 0 over channels
    _, _, sc_swapped = O.quantize4_group(X[0, 0, 0, :])
    assert sc_swapped == np.float16(8.0 / 15.0) == np.float16(0.533203125)


def test_residual_reconstruction_telescopes():
    """Step 0 codes K_0 itself; the reconstruction read at step t is the sum of
    the dequantized residuals of steps 0..t, and equals the encoder's running
    reconstruction; keys group tokens (ragged last group), values channels."""
    X = synth.loop_correlated(seed=710, n_loop=4, n_tokens=45, n_heads=2, head_dim=64)
    for kind in ("k", "v"):
        codes, lo, sc, recon = O.residual_encode(X, kind)
        assert codes.max() <= 15
        if kind == "k":
            assert lo.shape == (4, 2, 2, 64)
        else:
            assert lo.shape == (4, 2, 45, 2)
        for t in range(4):
            np.testing.assert_array_equal(O.residual_reconstruct(codes, lo, sc, kind, t), recon[t])
        # step 0 alone is plain 4-bit coding of K_0
        c0, l0, s0, r0 = O.residual_encode(X[:1], kind)
        np.testing.assert_array_equal(r0[0], recon[0])


def test_residual_coding_beats_per_step_coding_on_loop_correlated_data():
    """FlashLoop page, Figure 2 (c): coding each step as a residual over the
    previous step's reconstruction reconstructs a loop-correlated cache with
    lower error than coding every loop step's K/V on its own at the same
    bits."""
    X = synth.loop_correlated(seed=720, n_loop=4, n_tokens=96, n_heads=2, head_dim=64, rho=0.95)
    for kind in ("k", "v"):
        _, _, _, recon = O.residual_encode(X, kind)
        err_res = np.mean((recon[1:] - X[1:]) ** 2)
        err_ind = 0.0
        for t in range(1, 4):
            _, _, _, r = O.residual_encode(X[t:t + 1], kind)
            err_ind += np.mean((r[0] - X[t]) ** 2) / 3
        assert err_res < err_ind, (kind, err_res, err_ind)


def test_residual_decode_is_attention_over_the_reconstruction():
    X = synth.loop_correlated(seed=730, n_loop=4, n_tokens=70, n_heads=1, head_dim=64)
    Y = synth.loop_correlated(seed=731, n_loop=4, n_tokens=70, n_heads=1, head_dim=64)
    kc, kl, ks, kr = O.residual_encode(X, "k")
    vc, vl, vs, vr = O.residual_encode(Y, "v")
    q = np.random.default_rng(732).standard_normal((2, 64))
    for t in (0, 3):
        o, lse = O.residual_decode_attention(q, t, kc, kl, ks, vc, vl, vs, 0.125)
        for hq in range(2):
            np.testing.assert_allclose(o[hq], _sdpa(q[hq], kr[t][:, 0], vr[t][:, 0], 0.125), rtol=1e-12, atol=1e-12)
    assert O.residual_bits_per_element() == 5.0
