"""Adjacent-loop KV-residual 4-bit coding on the GPU against the oracle.

Encode: every quantization decision is taken in fp32 with separately
rounded operations on both sides, so codes and the fp16 (min, scale) pairs
must match bit for bit -- keys (token groups, ragged last group) and values
(channel groups), fp32 and bf16 inputs, at an offset inside a larger pool.
Decode: attention over the reconstruction, normwise within 2e-3 of the fp64
oracle (the decode tests' budget) with lse within 2e-3, for every loop step,
GQA 2, ragged and empty requests; both sides read the same codes.
"""
import numpy as np
import pytest
import torch

import oracle as O
from sub_bit_vector_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _L():
    from sub_bit_vector_b200 import loopvq
    return loopvq


def _encode_gpu(desc, kind, X, tok_off, pool, dtype):
    L = _L()
    T, N, H, D = X.shape
    codes = torch.zeros(L.loopvq_residual_codes_bytes(desc, pool), dtype=torch.uint8, device="cuda")
    params = torch.zeros(L.loopvq_residual_params_bytes(desc, kind, pool) // 2, dtype=torch.float16, device="cuda")
    x = torch.from_numpy(np.ascontiguousarray(X, dtype=np.float32)).cuda().to(dtype)
    L.loopvq_residual_encode(desc, kind, x, N, N * H * D, H * D, D, codes, params, tok_off, pool)
    torch.cuda.synchronize()
    return codes, params


def _unpack(desc, codes, params, kind, tok_off, N, pool):
    """Pool bytes -> codes [T][H][N][D] and (min, scale) in the oracle's layout."""
    T, H, D = desc.n_loop, desc.n_heads_kv, desc.head_dim
    c = codes.cpu().numpy().reshape(T, H, pool, D // 2)[:, :, tok_off:tok_off + N]
    full = np.empty((T, H, N, D), dtype=np.uint8)
    full[..., 0::2] = c & 15
    full[..., 1::2] = c >> 4
    pr = params.cpu().numpy()
    if kind == 0:
        pr = pr.reshape(T, H, pool // 32, D, 2)[:, :, tok_off // 32:tok_off // 32 + -(-N // 32)]
    else:
        pr = pr.reshape(T, H, pool, D // 32, 2)[:, :, tok_off:tok_off + N]
    return full, pr[..., 0], pr[..., 1]


@pytest.mark.parametrize("N,H,D,dtype", [(45, 2, 64, torch.float32), (300, 2, 128, torch.bfloat16),
                                         (64, 1, 128, torch.float32)])
@pytest.mark.parametrize("kind", [0, 1])
def test_residual_encode_bit_exact(N, H, D, dtype, kind):
    L = _L()
    T = 4
    X = synth.loop_correlated(seed=800 + N + kind, n_loop=T, n_tokens=N, n_heads=H, head_dim=D,
                              n_outlier=4 if kind == 0 else 0)
    if dtype == torch.bfloat16:
        X = synth.round_bf16(X.astype(np.float32))
    desc = L.make_residual_desc(T, H, D)
    pool, off = 512, 64
    codes, params = _encode_gpu(desc, kind, X, off, pool, dtype)
    got_c, got_lo, got_sc = _unpack(desc, codes, params, kind, off, N, pool)
    ref_c, ref_lo, ref_sc, _ = O.residual_encode(np.asarray(X, dtype=np.float32), "k" if kind == 0 else "v")
    np.testing.assert_array_equal(got_c, ref_c)
    np.testing.assert_array_equal(got_lo.view(np.uint16), ref_lo.view(np.uint16))
    np.testing.assert_array_equal(got_sc.view(np.uint16), ref_sc.view(np.uint16))


@pytest.mark.parametrize("T,D", [(4, 128), (6, 64)])
def test_residual_decode_matches_oracle_every_step(T, D):
    """Every loop step against the oracle: step 0 rebuilds the key row per
    element, later steps score keys with integer digits (D = 128 and D = 64
    instances, up to 6 planes), ragged contexts with a one-token last tile,
    GQA 2."""
    L = _L()
    H, Hq = 2, 4
    ctx = [3000, 301, 45, 1, 0]
    pool = sum(-(-max(c, 1) // 32) * 32 for c in ctx)
    offs = np.cumsum([0] + [-(-max(c, 1) // 32) * 32 for c in ctx])[:-1]
    desc = L.make_residual_desc(T, H, D, n_heads_q=Hq)
    ck = torch.zeros(L.loopvq_residual_codes_bytes(desc, pool), dtype=torch.uint8, device="cuda")
    cv = torch.zeros_like(ck)
    pk = torch.zeros(L.loopvq_residual_params_bytes(desc, 0, pool) // 2, dtype=torch.float16, device="cuda")
    pv = torch.zeros(L.loopvq_residual_params_bytes(desc, 1, pool) // 2, dtype=torch.float16, device="cuda")
    ref_codes = []
    for r, c in enumerate(ctx):
        K = synth.loop_correlated(seed=900 + r, n_loop=T, n_tokens=max(c, 1), n_heads=H, head_dim=D, n_outlier=4)
        V = synth.loop_correlated(seed=950 + r, n_loop=T, n_tokens=max(c, 1), n_heads=H, head_dim=D)
        K, V = K[:, :c], V[:, :c]
        if c:
            for kind, X, cc, pp in ((0, K, ck, pk), (1, V, cv, pv)):
                x = torch.from_numpy(np.ascontiguousarray(X, dtype=np.float32)).cuda().to(torch.bfloat16)
                L.loopvq_residual_encode(desc, kind, x, c, c * H * D, H * D, D, cc, pp, int(offs[r]), pool)
        ref_codes.append((O.residual_encode(np.asarray(K, dtype=np.float32), "k")[:3],
                          O.residual_encode(np.asarray(V, dtype=np.float32), "v")[:3]) if c else None)
    ctx_d = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    off_d = torch.from_numpy(offs.astype(np.int64)).cuda()
    ws = torch.zeros(L.loopvq_residual_decode_workspace_bytes(desc, len(ctx), max(ctx)), dtype=torch.uint8,
                     device="cuda")
    out = torch.zeros((len(ctx), Hq, D), dtype=torch.float32, device="cuda")
    lse = torch.zeros((len(ctx), Hq), dtype=torch.float32, device="cuda")
    rng = np.random.default_rng(960)
    for t in range(T):
        q = synth.round_bf16(rng.standard_normal((len(ctx), Hq, D)).astype(np.float32))
        L.loopvq_residual_decode_attn(desc, len(ctx), max(ctx), ctx_d, off_d, pool, ck, pk, cv, pv,
                                      torch.from_numpy(q).cuda().to(torch.bfloat16), t, D ** -0.5, out, lse, ws)
        torch.cuda.synchronize()
        o, l = out.cpu().numpy(), lse.cpu().numpy()
        for r, c in enumerate(ctx):
            if c == 0:
                assert np.all(o[r] == 0) and np.all(l[r] == -np.inf)
                continue
            (kc, kl, ks), (vc, vl, vs) = ref_codes[r]
            o_ref, l_ref = O.residual_decode_attention(q[r], t, kc, kl, ks, vc, vl, vs, D ** -0.5)
            for hq in range(Hq):
                e = np.max(np.abs(o[r, hq] - o_ref[hq])) / np.max(np.abs(o_ref[hq]))
                assert e <= TOL, (t, r, hq, e)
                assert abs(l[r, hq] - l_ref[hq]) <= TOL * max(1.0, abs(l_ref[hq]))
    assert L.loopvq_read_device_status(ws)[1] == 0


def test_residual_beats_per_step_coding_on_gpu_codes():
    """On the GPU's own codes of a loop-correlated cache: reconstructing step
    t from the residual planes has lower error than 4-bit coding step t alone
    (the page's Figure 2 (c) claim, measured on the library's output)."""
    L = _L()
    T, N, H, D = 4, 256, 2, 128
    X = synth.loop_correlated(seed=970, n_loop=T, n_tokens=N, n_heads=H, head_dim=D, rho=0.95)
    desc = L.make_residual_desc(T, H, D)
    desc1 = L.make_residual_desc(1, H, D)
    for kind in (0, 1):
        codes, params = _encode_gpu(desc, kind, X, 0, N, torch.float32)
        c, lo, sc = _unpack(desc, codes, params, kind, 0, N, N)
        err_res = err_ind = 0.0
        for t in range(1, T):
            rec = O.residual_reconstruct(c, lo, sc, "k" if kind == 0 else "v", t)
            err_res += np.mean((rec - X[t]) ** 2)
            c1, p1 = _encode_gpu(desc1, kind, X[t:t + 1], 0, N, torch.float32)
            u = _unpack(desc1, c1, p1, kind, 0, N, N)
            err_ind += np.mean((O.residual_reconstruct(*u, "k" if kind == 0 else "v", 0) - X[t]) ** 2)
        assert err_res < err_ind, (kind, err_res, err_ind)


def test_residual_decode_most_planes_and_refusal_beyond():
    """16 planes (loop step 15) are the most a 64-token tile stage holds at
    D = 128 next to the key digits: that launch matches the oracle; loop step
    16 is refused before anything is launched (the buffers are real and in
    range all the same)."""
    L = _L()
    T, H, D, c = 17, 1, 128, 40
    pool = 64
    desc = L.make_residual_desc(T, H, D)
    ck = torch.zeros(L.loopvq_residual_codes_bytes(desc, pool), dtype=torch.uint8, device="cuda")
    cv = torch.zeros_like(ck)
    pk = torch.zeros(L.loopvq_residual_params_bytes(desc, 0, pool) // 2, dtype=torch.float16, device="cuda")
    pv = torch.zeros(L.loopvq_residual_params_bytes(desc, 1, pool) // 2, dtype=torch.float16, device="cuda")
    K = synth.loop_correlated(seed=970, n_loop=T, n_tokens=c, n_heads=H, head_dim=D, n_outlier=4)
    V = synth.loop_correlated(seed=971, n_loop=T, n_tokens=c, n_heads=H, head_dim=D)
    for kind, X, cc, pp in ((0, K, ck, pk), (1, V, cv, pv)):
        x = torch.from_numpy(np.ascontiguousarray(X, dtype=np.float32)).cuda().to(torch.bfloat16)
        L.loopvq_residual_encode(desc, kind, x, c, c * H * D, H * D, D, cc, pp, 0, pool)
    (kc, kl, ks), (vc, vl, vs) = (O.residual_encode(np.asarray(K, dtype=np.float32), "k")[:3],
                                  O.residual_encode(np.asarray(V, dtype=np.float32), "v")[:3])
    ctx_d = torch.tensor([c], dtype=torch.int32, device="cuda")
    off_d = torch.zeros(1, dtype=torch.int64, device="cuda")
    ws = torch.zeros(L.loopvq_residual_decode_workspace_bytes(desc, 1, c), dtype=torch.uint8, device="cuda")
    out = torch.zeros((1, H, D), dtype=torch.float32, device="cuda")
    q = synth.round_bf16(np.random.default_rng(972).standard_normal((1, H, D)).astype(np.float32))
    qd = torch.from_numpy(q).cuda().to(torch.bfloat16)
    L.loopvq_residual_decode_attn(desc, 1, c, ctx_d, off_d, pool, ck, pk, cv, pv, qd, 15, D ** -0.5, out, None, ws)
    torch.cuda.synchronize()
    o_ref, _ = O.residual_decode_attention(q[0], 15, kc, kl, ks, vc, vl, vs, D ** -0.5)
    e = np.max(np.abs(out.cpu().numpy()[0, 0] - o_ref[0])) / np.max(np.abs(o_ref[0]))
    assert e <= TOL, e
    with pytest.raises(L.LoopVQError) as err:
        L.loopvq_residual_decode_attn(desc, 1, c, ctx_d, off_d, pool, ck, pk, cv, pv, qd, 16, D ** -0.5, out, None,
                                      ws)
    assert err.value.status == L.LOOPVQ_ERR_UNSUPPORTED
    assert L.loopvq_read_device_status(ws)[1] == 0
