"""GPU Lloyd codebook update (loopvq_codebook_update) against the oracle.

The update is checked on codes both sides share (drawn by the seeded
generator and packed into an index pool), so the comparison isolates the
means: fp32 codebooks within fp32 summation rounding, bf16 codebooks within
one bf16 unit of the oracle's mean rounded to bf16, member counts exactly,
unused codewords unchanged.  A few full Lloyd rounds (GPU encode + update)
are compared by their distortion history.
"""
import numpy as np
import pytest
import torch

import oracle as O
from sub_bit_vector_b200 import synth

pytestmark = pytest.mark.gpu


def _L():
    from sub_bit_vector_b200 import loopvq
    return loopvq


def _update_gpu(desc, X, codes, cb, tok_off, pool_tokens, x_dtype, cb_dtype, kind=0):
    L = _L()
    T, N, H, D = X.shape
    pool = torch.zeros(L.loopvq_index_pool_bytes(desc, pool_tokens), dtype=torch.uint8, device="cuda")
    L.loopvq_index_pool_pack(desc, kind, torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).cuda(), N,
                             pool, tok_off, pool_tokens)
    x = torch.from_numpy(np.ascontiguousarray(X, dtype=np.float32)).cuda().to(x_dtype)
    cb_in = torch.from_numpy(np.ascontiguousarray(cb, dtype=np.float32)).cuda().to(cb_dtype)
    cb_out = torch.empty_like(cb_in)
    counts = torch.zeros(cb.shape[:4], dtype=torch.int32, device="cuda")
    ws = torch.empty(L.loopvq_codebook_update_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    L.loopvq_codebook_update(desc, kind, x, N, N * H * D, H * D, D, pool, tok_off, pool_tokens, cb_in, cb_out,
                             counts, ws)
    torch.cuda.synchronize()
    return cb_out.float().cpu().numpy().astype(np.float64), counts.cpu().numpy()


@pytest.mark.parametrize("tc,G", [(4, 16), (4, 32), (2, 8), (1, 16)])
@pytest.mark.parametrize("cbt", ["f32", "bf16"])
def test_codebook_update_matches_oracle_means(tc, G, cbt):
    """3000 tokens (one full 2048-token chunk and a ragged one) x 2 heads at an
    unaligned pool offset; codes drawn from [0, 200) so codewords 200..255 are
    unused and must come back unchanged."""
    L = _L()
    T, N, H, D = 4, 3000, 2, 128
    X = synth.loop_correlated(seed=900 + G + tc, n_loop=T, n_tokens=N, n_heads=H, head_dim=D, n_outlier=4)
    W = G // tc
    J = D // W
    NB = T // tc
    cb = synth.codebook_from_rows(X, tc, G, 256, seed=901)
    codes = synth.random_codes(902 + tc, NB, H, N, J, n_codes=200)
    desc = L.make_desc(T, tc, H, D, G, cb_dtype=L.LOOPVQ_F32 if cbt == "f32" else L.LOOPVQ_BF16)
    got, cnt = _update_gpu(desc, X, codes, cb, 40, 3072 + 64, torch.float32,
                           torch.float32 if cbt == "f32" else torch.bfloat16)
    ref, ref_cnt = O.kmeans_update(X, codes.astype(np.int64), cb, tc)
    np.testing.assert_array_equal(cnt, ref_cnt)
    if cbt == "f32":
        np.testing.assert_allclose(got, ref, rtol=2e-5, atol=2e-6)
    else:
        exp = synth.round_bf16(ref.astype(np.float32)).astype(np.float64)
        ulp = np.abs(exp) * 2.0 ** -7 + 1e-30
        assert np.all(np.abs(got - exp) <= ulp), float(np.max(np.abs(got - exp) / ulp))
    np.testing.assert_array_equal(got[:, :, :, 200:], np.asarray(cb, dtype=np.float64)[:, :, :, 200:])


def test_codebook_update_bf16_inputs_and_empty_token_range():
    """bf16 sub-vectors give the same means; zero tokens leave the codebook
    as it was (every codeword unused)."""
    L = _L()
    T, N, H, D, tc, G = 4, 700, 1, 64, 4, 16
    X = synth.loop_correlated(seed=910, n_loop=T, n_tokens=N, n_heads=H, head_dim=D)
    cb = synth.codebook_from_rows(X, tc, G, 256, seed=911)
    codes = synth.random_codes(912, 1, H, N, D * tc // G)
    desc = L.make_desc(T, tc, H, D, G, cb_dtype=L.LOOPVQ_F32)
    got, _ = _update_gpu(desc, X, codes, cb, 0, 704, torch.bfloat16, torch.float32)
    ref, _ = O.kmeans_update(X, codes.astype(np.int64), cb, tc)
    np.testing.assert_allclose(got, ref, rtol=2e-5, atol=2e-6)
    x = torch.from_numpy(np.ascontiguousarray(X, dtype=np.float32)).cuda()
    pool = torch.zeros(L.loopvq_index_pool_bytes(desc, 32), dtype=torch.uint8, device="cuda")
    cb_in = torch.from_numpy(np.ascontiguousarray(cb, dtype=np.float32)).cuda()
    cb_out = torch.full_like(cb_in, float("nan"))
    cnt0 = torch.ones(cb.shape[:4], dtype=torch.int32, device="cuda")
    ws = torch.empty(L.loopvq_codebook_update_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    L.loopvq_codebook_update(desc, 0, x, 0, N * H * D, H * D, D, pool, 0, 32, cb_in, cb_out, cnt0, ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cb_out.cpu().numpy(), cb_in.cpu().numpy())
    assert int(cnt0.sum()) == 0


def test_lloyd_rounds_on_gpu_follow_the_oracle():
    """Three Lloyd rounds on fp32 data and codebooks, each a GPU encode and a
    GPU update: the distortion of every round matches the oracle's Lloyd run
    from the same start and never increases."""
    L = _L()
    T, N, H, D, tc, G = 4, 2500, 2, 64, 4, 16
    X = synth.loop_correlated(seed=920, n_loop=T, n_tokens=N, n_heads=H, head_dim=D, n_outlier=2)
    cb0 = synth.codebook_from_rows(X, tc, G, 256, seed=921).astype(np.float32)
    desc = L.make_desc(T, tc, H, D, G, cb_dtype=L.LOOPVQ_F32)
    J = D * tc // G
    x = torch.from_numpy(np.ascontiguousarray(X, dtype=np.float32)).cuda()
    cb = torch.from_numpy(cb0).cuda()
    packed = torch.zeros(L.loopvq_codebook_packed_bytes(desc), dtype=torch.uint8, device="cuda")
    pool = torch.zeros(L.loopvq_index_pool_bytes(desc, 2528), dtype=torch.uint8, device="cuda")
    ws = torch.empty(L.loopvq_codebook_update_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    codes = torch.zeros((1, H, N, J), dtype=torch.uint8, device="cuda")
    hist = []
    for _ in range(3):
        L.loopvq_codebook_pack(desc, cb, packed)
        L.loopvq_encode(desc, packed, 0, x, N, N * H * D, H * D, D, pool, 0, 2528)
        L.loopvq_index_pool_unpack(desc, 0, pool, 0, 2528, N, codes)
        torch.cuda.synchronize()
        hist.append(O.distortion(X, codes.cpu().numpy().astype(np.int64), cb.cpu().numpy(), tc))
        nxt = torch.empty_like(cb)
        L.loopvq_codebook_update(desc, 0, x, N, N * H * D, H * D, D, pool, 0, 2528, cb, nxt, None, ws)
        cb = nxt
    _, _, ref_hist = O.kmeans(X, cb0, tc, 3)
    np.testing.assert_allclose(hist, ref_hist, rtol=1e-5)
    assert all(b <= a * (1 + 1e-6) for a, b in zip(hist, hist[1:]))
