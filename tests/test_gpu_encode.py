"""GPU loop-axis VQ encode vs the oracle's brute-force argmin, through the C ABI.

Index tolerance: a GPU code i at a position is accepted iff it equals the
oracle's code, or the oracle's top-2 gap is within 1e-5 relative to the
second-best distance and codeword i is itself within that gap of the best
(distances recomputed by the oracle in fp64).
"""
import numpy as np
import pytest
import torch

import oracle as O
from sub_bit_vector_b200 import synth

pytestmark = pytest.mark.gpu

REL = 1e-5


def _L():
    from sub_bit_vector_b200 import loopvq
    return loopvq


def _accept(X, cb, tc, gpu_idx, tokens=None):
    """Checks GPU codes [NB][H][n][J] against the oracle for X[:, tokens]."""
    Xs = X if tokens is None else X[:, tokens]
    idx, d1, d2 = O.encode(Xs, cb, tc)
    mism = np.argwhere(idx != gpu_idx)
    w = cb.shape[-1]
    for (b, h, n, j) in mism:
        sub = O.form_subvectors(Xs[:, n:n + 1], b, tc, w)[0, h, j]
        d = O.subvector_distances(sub[None], cb[b, h, j].reshape(cb.shape[3], -1))[0]
        gap_ok = (d2[b, h, n, j] - d1[b, h, n, j]) <= REL * d2[b, h, n, j]
        near = d[gpu_idx[b, h, n, j]] <= d1[b, h, n, j] + REL * d2[b, h, n, j]
        assert gap_ok and near, f"code mismatch at b={b} h={h} n={n} j={j}: gpu {gpu_idx[b, h, n, j]} oracle {idx[b, h, n, j]}"
    return len(mism)


def _encode_gpu(desc, cb, X_t_n_h_d, kind, pool_tokens, tok_off=0, x_dtype=torch.bfloat16):
    """Packs the codebook, encodes a contiguous [T][N][H][D] tensor into a
    fresh pool and unpacks the codes back to [NB][H][N][J]."""
    L = _L()
    packed = torch.zeros(L.loopvq_codebook_packed_bytes(desc), dtype=torch.uint8, device="cuda")
    cbt = torch.from_numpy(np.ascontiguousarray(cb, dtype=np.float32)).cuda()
    if desc.cb_dtype == L.LOOPVQ_BF16:
        cbt = cbt.to(torch.bfloat16)
    L.loopvq_codebook_pack(desc, cbt, packed)
    x_dev = torch.from_numpy(np.ascontiguousarray(X_t_n_h_d, dtype=np.float32)).cuda().to(x_dtype)
    T, N, H, D = X_t_n_h_d.shape
    pool = torch.zeros(L.loopvq_index_pool_bytes(desc, pool_tokens), dtype=torch.uint8, device="cuda")
    L.loopvq_encode(desc, packed, kind, x_dev, N, N * H * D, H * D, D, pool, tok_off, pool_tokens)
    J = desc.head_dim * desc.tc // desc.group_elems
    codes = torch.zeros((desc.n_loop // desc.tc, desc.n_heads_kv, N, J), dtype=torch.uint8, device="cuda")
    L.loopvq_index_pool_unpack(desc, kind, pool, tok_off, pool_tokens, N, codes)
    torch.cuda.synchronize()
    return codes.cpu().numpy().astype(np.int64), pool


def test_tiny_encode_fp32():
    L = _L()
    K, V = synth.tiny_kv(seed=0)
    for X, seed, kind in ((K, 1, L.LOOPVQ_KEYS), (V, 2, L.LOOPVQ_VALUES)):
        cb = synth.codebook_from_rows(X, 4, 16, 256, seed=seed)
        desc = L.make_desc(4, 4, 1, 64, 16, 256, cb_dtype=L.LOOPVQ_F32)
        g, _ = _encode_gpu(desc, cb, X, kind, 512, x_dtype=torch.float32)
        assert _accept(X, cb, 4, g) == 0   # fp32 data, well-separated codes


_BIG = {}


def _prefill(kind):
    if kind not in _BIG:
        T, N, H, D = 4, 32768, 16, 128
        if kind == "K":
            _BIG[kind] = synth.loop_correlated(seed=40, n_loop=T, n_tokens=N, n_heads=H, head_dim=D, n_outlier=4)
        else:
            _BIG[kind] = synth.loop_correlated(seed=41, n_loop=T, n_tokens=N, n_heads=H, head_dim=D)
    return _BIG[kind]


@pytest.mark.parametrize("kind", ["K", "V"])
@pytest.mark.parametrize("tc,G", [(4, 16), (4, 32), (1, 16)])
def test_prefill_encode_32k_sampled(kind, tc, G):
    """32768 tokens x 16 heads x 128 x 4 loop steps bf16 (rho = 0.9), encoded
    at 0.5 bit and 0.25 bit with Tc = 4 and at 0.5 bit with Tc = 1; the whole
    launch runs, the oracle checks a seeded sample of 384 tokens (all heads,
    slots and blocks) plus the ragged last chunk."""
    L = _L()
    X = _prefill(kind)
    cb = synth.codebook_from_rows(X, tc, G, 256, seed=42 + tc + G)
    desc = L.make_desc(4, tc, 16, 128, G, 256)
    g, _ = _encode_gpu(desc, cb, X, L.LOOPVQ_KEYS if kind == "K" else L.LOOPVQ_VALUES, 32768)
    assert g.max() <= 255
    rng = np.random.Generator(np.random.PCG64(43))
    toks = np.sort(np.concatenate([rng.choice(32768 - 64, 320, replace=False), np.arange(32768 - 64, 32768)]))
    _accept(X, cb, tc, g[:, :, toks], tokens=toks)


def test_tc4_beats_tc1_reconstruction_with_gpu_codes():
    """Project page, "Method" loop-redundancy figure: at 0.5 bit a code
    spanning 4 loop steps reconstructs loop-correlated keys with lower error
    than a code spanning 1 step.  The codes are the GPU's (tensor-core
    encode of bf16 inputs, each accepted against the oracle), dequantized by
    the oracle."""
    L = _L()
    X = synth.round_bf16(_prefill("K")[:, :2048, :2])
    m = {}
    for tc in (4, 1):
        cb = synth.round_bf16(synth.codebook_from_rows(X, tc, 16, 256, seed=44))
        desc = L.make_desc(4, tc, 2, 128, 16, 256)
        g, _ = _encode_gpu(desc, cb, X, L.LOOPVQ_KEYS, 2048)
        _accept(X, cb, tc, g)
        m[tc] = O.reconstruction_mse(X, g, cb, tc)
    assert m[4] < m[1], m


def test_page_encode_from_window_pool_layout():
    """Encode one 8-token page straight out of a [T][H][P][D] window pool
    (strided input) into an index pool at an unaligned token offset; bytes
    outside the page stay untouched."""
    L = _L()
    T, H, D, P, G, tc = 4, 16, 128, 320, 16, 4
    Xw = synth.loop_correlated(seed=50, n_loop=T, n_tokens=P, n_heads=H, head_dim=D, n_outlier=4)  # [T][P][H][D]
    pool_layout = np.ascontiguousarray(Xw.transpose(0, 2, 1, 3))   # [T][H][P][D]
    cb = synth.codebook_from_rows(Xw, tc, G, 256, seed=51)
    desc = L.make_desc(T, tc, H, D, G, 256)
    page0 = 64
    x_dev = torch.from_numpy(pool_layout).cuda().to(torch.bfloat16)
    x_page = x_dev[:, :, page0:page0 + 8]   # view; strides of the pool
    packed = torch.zeros(L.loopvq_codebook_packed_bytes(desc), dtype=torch.uint8, device="cuda")
    L.loopvq_codebook_pack(desc, torch.from_numpy(cb).cuda().to(torch.bfloat16), packed)
    pool_tokens = 128
    pool = torch.full((L.loopvq_index_pool_bytes(desc, pool_tokens),), 7, dtype=torch.uint8, device="cuda")
    tok_off = 40
    L.loopvq_encode(desc, packed, L.LOOPVQ_KEYS, x_page, 8, H * P * D, D, P * D, pool, tok_off, pool_tokens)
    codes = torch.zeros((1, H, 8, 32), dtype=torch.uint8, device="cuda")
    L.loopvq_index_pool_unpack(desc, L.LOOPVQ_KEYS, pool, tok_off, pool_tokens, 8, codes)
    torch.cuda.synchronize()
    _accept(Xw[:, page0:page0 + 8], cb, tc, codes.cpu().numpy().astype(np.int64))
    allc = torch.zeros((1, H, pool_tokens, 32), dtype=torch.uint8, device="cuda")
    L.loopvq_index_pool_unpack(desc, L.LOOPVQ_KEYS, pool, 0, pool_tokens, pool_tokens, allc)
    a = allc.cpu().numpy()
    assert np.all(a[:, :, :tok_off] == 7) and np.all(a[:, :, tok_off + 8:] == 7)


@pytest.mark.parametrize("J,kind", [(8, 0), (16, 0), (32, 0), (8, 1), (16, 1), (32, 1)])
def test_pool_pack_unpack_roundtrip(J, kind):
    L = _L()
    D = 128
    W = D // J
    desc = L.make_desc(4, 4, 3, D, 4 * W, 256)
    rng = np.random.default_rng(J + 10 * kind)
    n, off, pt = 77, 19, 128
    codes = rng.integers(0, 256, (1, 3, n, J), dtype=np.uint8)
    pool = torch.zeros(L.loopvq_index_pool_bytes(desc, pt), dtype=torch.uint8, device="cuda")
    L.loopvq_index_pool_pack(desc, kind, torch.from_numpy(codes).cuda(), n, pool, off, pt)
    back = torch.zeros((1, 3, n, J), dtype=torch.uint8, device="cuda")
    L.loopvq_index_pool_unpack(desc, kind, pool, off, pt, n, back)
    np.testing.assert_array_equal(back.cpu().numpy(), codes)
    # every code landed in its own byte: the pool holds exactly these codes
    assert int((pool != 0).sum()) <= codes.size


def test_codebook_pack_slices():
    L = _L()
    desc = L.make_desc(4, 2, 3, 64, 8, 256, cb_dtype=L.LOOPVQ_F32)
    rng = np.random.default_rng(3)
    can = rng.standard_normal((2, 3, 16, 256, 2, 4)).astype(np.float32)
    packed = torch.zeros(L.loopvq_codebook_packed_bytes(desc), dtype=torch.uint8, device="cuda")
    L.loopvq_codebook_pack(desc, torch.from_numpy(can).cuda(), packed)
    torch.cuda.synchronize()
    raw = packed.cpu().numpy()
    nbytes = can.nbytes
    np.testing.assert_array_equal(raw[:nbytes].view(np.float32).reshape(can.shape), can)
    off = (nbytes + 255) // 256 * 256
    sl = raw[off:off + nbytes].view(np.float32).reshape(4, 3, 256, 16, 4)   # [T][H][C][J][W]
    for t in range(4):
        np.testing.assert_array_equal(sl[t], can[t // 2, :, :, :, t % 2, :].transpose(0, 2, 1, 3))


@pytest.mark.parametrize("tc,G", [(4, 16), (4, 32), (2, 16), (1, 16)])
def test_tensor_core_encode_ragged_all_tokens(tc, G):
    """bf16 encode of 1000 tokens (7 full 128-row tiles and a ragged one of
    104) x 2 heads, written at an unaligned pool offset: every code is
    checked against the oracle, and the pool bytes outside the range stay
    untouched."""
    L = _L()
    T, N, H, D = 4, 1000, 2, 128
    X = synth.loop_correlated(seed=60 + G + tc, n_loop=T, n_tokens=N, n_heads=H, head_dim=D, n_outlier=4)
    cb = synth.codebook_from_rows(X, tc, G, 256, seed=61 + G + tc)
    desc = L.make_desc(T, tc, H, D, G, 256)
    tok_off, pool_tokens = 37, 1088
    packed = torch.zeros(L.loopvq_codebook_packed_bytes(desc), dtype=torch.uint8, device="cuda")
    L.loopvq_codebook_pack(desc, torch.from_numpy(cb).cuda().to(torch.bfloat16), packed)
    x_dev = torch.from_numpy(np.ascontiguousarray(X, dtype=np.float32)).cuda().to(torch.bfloat16)
    pool = torch.full((L.loopvq_index_pool_bytes(desc, pool_tokens),), 3, dtype=torch.uint8, device="cuda")
    faults = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.loopvq_encode(desc, packed, L.LOOPVQ_KEYS, x_dev, N, N * H * D, H * D, D, pool, tok_off, pool_tokens,
                    fault_bits=faults)
    J = D * tc // G
    allc = torch.zeros((T // tc, H, pool_tokens, J), dtype=torch.uint8, device="cuda")
    L.loopvq_index_pool_unpack(desc, L.LOOPVQ_KEYS, pool, 0, pool_tokens, pool_tokens, allc)
    torch.cuda.synchronize()
    a = allc.cpu().numpy().astype(np.int64)
    assert np.all(a[:, :, :tok_off] == 3) and np.all(a[:, :, tok_off + N:] == 3)
    _accept(X, cb, tc, a[:, :, tok_off:tok_off + N])
    assert int(faults.item()) == 0


def test_tensor_core_encode_exact_ties_go_to_lowest_index():
    """Codebooks with duplicated codewords and sub-vectors equal to codewords:
    the distances tie exactly (and are zero for the equal rows), so the
    result must be the oracle's lowest index, not a near-tie alternative."""
    L = _L()
    T, N, H, D, tc, G = 4, 512, 1, 128, 4, 16
    X = synth.loop_correlated(seed=70, n_loop=T, n_tokens=N, n_heads=H, head_dim=D)
    cb = synth.codebook_from_rows(X, tc, G, 256, seed=71)
    # codeword 200 repeats codeword 10, 255 repeats 0, 7 repeats 6
    for hi, lo in ((200, 10), (255, 0), (7, 6)):
        cb[:, :, :, hi] = cb[:, :, :, lo]
    # tokens 0..63 are exactly codewords 0..63 of their slot
    W = G // tc
    Xe = X.copy()
    for j in range(D // W):
        for t in range(tc):
            Xe[t, :64, 0, j * W:(j + 1) * W] = cb[0, 0, j, :64, t, :]
    desc = L.make_desc(T, tc, H, D, G, 256)
    g, _ = _encode_gpu(desc, cb, Xe, L.LOOPVQ_KEYS, 512)
    idx, _, _ = O.encode(Xe, cb, tc)
    expect = np.arange(64)
    expect = np.where(expect == 7, 6, expect)   # codeword 7 duplicates 6
    np.testing.assert_array_equal(idx[0, 0, :64], np.repeat(expect[:, None], D // W, axis=1))
    np.testing.assert_array_equal(g[0, 0, :64], idx[0, 0, :64])
    assert _accept(Xe, cb, tc, g) == 0


def test_tensor_core_encode_near_tie_clusters():
    """Near-duplicate codewords (one element one bf16 step apart) and
    sub-vectors drawn tightly around them: nearly every row's two best fast
    distances fall within the fast path's error bound, so the rows are
    re-solved exactly.  The clusters sit in different top-2 chains (codes 16
    and 40; chains take the code groups (code % 32) // 8), in one chain (24
    and 30) and as a triple over two chains (64, 72 and 65), so both the
    two-head re-solve and the chain re-read run.  Every code must be the
    oracle's nearest, and both members of each cluster must win somewhere."""
    L = _L()
    T, N, H, D, tc, G = 4, 768, 1, 128, 4, 16
    W, J = G // tc, D * tc // G
    X = synth.loop_correlated(seed=72, n_loop=T, n_tokens=N, n_heads=H, head_dim=D)
    cb = synth.codebook_from_rows(X, tc, G, 256, seed=73)

    def nudge(v, e):   # element e of every [tc][W] codeword one bf16 step up in magnitude
        f = np.ascontiguousarray(v, dtype=np.float32).reshape(v.shape[:-2] + (tc * W,)).copy()
        f.view(np.uint32)[..., e] += 0x10000
        return f.reshape(v.shape)

    for c0, dups in {16: [(40, 0)], 24: [(30, 1)], 64: [(72, 2), (65, 3)]}.items():
        for cd, e in dups:
            cb[:, :, :, cd] = nudge(cb[:, :, :, c0], e)
    rng = np.random.default_rng(74)
    sel = np.array([16, 24, 64])[np.arange(N) % 3]
    cs = cb[0, 0][:, sel]                       # [J][N][tc][W]
    Xe = np.empty_like(X)
    for t in range(tc):
        Xe[t, :, 0, :] = cs[:, :, t, :].transpose(1, 0, 2).reshape(N, J * W)
    Xe = synth.round_bf16(Xe + 0.006 * rng.standard_normal(Xe.shape).astype(np.float32))
    desc = L.make_desc(T, tc, H, D, G, 256)
    g, _ = _encode_gpu(desc, cb, Xe, L.LOOPVQ_KEYS, N)
    idx, _, _ = O.encode(Xe, cb, tc)
    for c in (16, 40, 24, 30, 64, 72, 65):
        assert (idx == c).any() and (g == c).any(), c
    assert _accept(Xe, cb, tc, g) == 0


@pytest.mark.parametrize("n", [1, 8, 200])
@pytest.mark.parametrize("tc,G", [(4, 16), (4, 32), (4, 64), (2, 8), (1, 4)])
@pytest.mark.parametrize("xdt", ["bf16", "f32"])
def test_few_token_encode_all_tokens(n, tc, G, xdt):
    """Few-token encode (fewer than 256 tokens: one warp per token, lanes over
    codes) across J = 8, 16 and 32 slots, bf16 and fp32 inputs: every code is
    checked against the oracle."""
    L = _L()
    T, H, D = 4, 3, 128
    X = synth.loop_correlated(seed=80 + n + G, n_loop=T, n_tokens=max(n, 256), n_heads=H, head_dim=D,
                              n_outlier=4)
    cb = synth.codebook_from_rows(X, tc, G, 256, seed=81 + G)
    Xn = np.ascontiguousarray(X[:, :n])
    desc = L.make_desc(T, tc, H, D, G, 256)
    g, _ = _encode_gpu(desc, cb, Xn, L.LOOPVQ_VALUES, 256, tok_off=5,
                       x_dtype=torch.bfloat16 if xdt == "bf16" else torch.float32)
    _accept(Xn, cb, tc, g)
