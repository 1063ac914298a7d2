"""GPU codebook gradients (loopvq_codebook_grad) against the oracle.

The forward is the library's decode (fp32 output and lse); the gradient call
adds the gradients of weight * sum ||o - target||^2 with respect to both
codebooks.  The oracle's ``attention_mse_codebook_grad`` (pinned by central
differences) is summed over the requests.  Tolerance: normwise, max |error|
within 2e-3 of max |reference| per codebook -- the gradient is linear in the
output error g and the softmax weights, which the forward already matches
to that budget; with fp32 tables and sums the observed error is ~1e-5.
Entries outside the step's block and slice must stay exactly zero.  A
fine-tuning loop over the library's gradients (normalised gradient steps per
loop step with a growing or halving step size; codes fixed) lowers the
attention error of all four loop steps.
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


def _cache():
    from sub_bit_vector_b200 import cache
    return cache


def _normwise(got, ref):
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


def _cache_case(tc, G, D, ctx, cb_dtype, Hq=4, H=2, T=4, seed=0):
    C = _cache()
    dc = C.DecodeCache(n_loop=T, tc=tc, n_heads_kv=H, head_dim=D, group_elems=G, ctx_lens=ctx, n_heads_q=Hq,
                       cb_dtype=cb_dtype)
    W = G // tc
    J = D // W
    bf = cb_dtype == torch.bfloat16
    cbk = synth.uniform_codebook(seed + 1, T // tc, H, J, 256, tc, W, bf16=bf)
    cbv = synth.uniform_codebook(seed + 2, T // tc, H, J, 256, tc, W, bf16=bf)
    dc.set_codebooks(cbk, cbv)
    rng = np.random.default_rng(seed + 3)
    codes, wins = [], []
    for r, c in enumerate(ctx):
        s, body, rec = dc.splits[r]
        ck = synth.random_codes(seed + 10 + r, T // tc, H, body, J)
        cv = synth.random_codes(seed + 20 + r, T // tc, H, body, J)
        dc.set_request_codes(r, ck, cv)
        wk = synth.round_bf16(rng.standard_normal((T, H, s + rec, D)).astype(np.float32))
        wv = synth.round_bf16(rng.standard_normal((T, H, s + rec, D)).astype(np.float32))
        dc.set_request_window(r, wk, wv)
        codes.append((ck, cv))
        wins.append((wk, wv))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda().to(cb_dtype)
    return dc, cbk, cbv, dev(cbk), dev(cbv), codes, wins


def _oracle_sum(dc, t, cbk, cbv, codes, wins, q, target, scale, weight, requests):
    loss, gk, gv = 0.0, np.zeros(cbk.shape), np.zeros(cbv.shape)
    for r, rr in enumerate(requests):
        ck, cv = codes[rr]
        wk, wv = wins[rr]
        l, a, b, _ = O.attention_mse_codebook_grad(q[r], t, dc.Tc, ck, cv, cbk, cbv, wk[t], wv[t], scale,
                                                   target[r], weight)
        loss += l
        gk += a
        gv += b
    return loss, gk, gv


@pytest.mark.parametrize("tc,G,D,cbt", [(4, 16, 128, torch.bfloat16), (4, 32, 128, torch.float32),
                                        (1, 16, 128, torch.bfloat16), (2, 8, 64, torch.float32)])
def test_codebook_grad_matches_oracle(tc, G, D, cbt):
    """Ragged contexts (several splits, ragged tiles, window-only and empty
    requests), GQA 2, two loop steps of different slices."""
    L = _L()
    ctx = [3000, 700, 333, 64, 0]
    dc, cbk, cbv, cbk_d, cbv_d, codes, wins = _cache_case(tc, G, D, ctx, cbt, seed=100 + G + tc)
    scale, weight = D ** -0.5, 0.75
    rng = np.random.default_rng(5)
    for t in (1, 3):
        q = synth.round_bf16(rng.standard_normal((len(ctx), dc.Hq, D)).astype(np.float32))
        target = (0.05 * rng.standard_normal((len(ctx), dc.Hq, D))).astype(np.float32)
        dc.set_queries(q)
        dc.decode(t, scale)
        gk = torch.zeros(cbk.shape, dtype=torch.float32, device="cuda")
        gv = torch.zeros_like(gk)
        loss = torch.zeros(1, dtype=torch.float32, device="cuda")
        faults = torch.zeros(1, dtype=torch.int32, device="cuda")
        tgt = torch.from_numpy(target).cuda()
        L.loopvq_codebook_grad(dc.desc, cbk_d, cbv_d, dc.layout, dc.idxK, dc.idxV, dc.q, t, scale, dc.out, dc.lse,
                               tgt, weight, gk, gv, loss, faults)
        torch.cuda.synchronize()
        assert int(faults.item()) == 0
        ref_loss, ref_k, ref_v = _oracle_sum(dc, t, cbk.astype(np.float64), cbv.astype(np.float64), codes, wins,
                                             q, target, scale, weight, range(len(ctx)))
        got_k = gk.cpu().numpy().astype(np.float64)
        got_v = gv.cpu().numpy().astype(np.float64)
        assert _normwise(got_k, ref_k) <= 2e-3, _normwise(got_k, ref_k)
        assert _normwise(got_v, ref_v) <= 2e-3, _normwise(got_v, ref_v)
        b, tt = divmod(t, tc)
        mask = np.zeros(got_k.shape, dtype=bool)
        mask[b, :, :, :, tt, :] = True
        assert not got_k[~mask].any() and not got_v[~mask].any()
        assert float(loss.item()) == pytest.approx(ref_loss, rel=2e-3)


def test_requests_sharing_one_cache_sum_their_gradients():
    """Three queries against one cache (the same body and window offsets)
    give the sum of the three single-query gradients; a second call adds on
    top of the first."""
    L = _L()
    T, tc, G, D = 4, 4, 16, 128
    dc, cbk, cbv, cbk_d, cbv_d, codes, wins = _cache_case(tc, G, D, [2500], torch.bfloat16, Hq=2, H=2, seed=300)
    nq, scale, t = 3, D ** -0.5, 2
    ctx = dc.ctx_dev.repeat(nq)
    boff = dc.body_off_dev.repeat(nq)
    woff = dc.win_off_dev.repeat(nq)
    lay = L.make_layout(nq, dc.n_sink, dc.n_recent, dc.page, dc.max_ctx_len, ctx, boff, woff, dc.body_pool_tokens,
                        dc.win_pool_tokens, 0)
    rng = np.random.default_rng(6)
    q = synth.round_bf16(rng.standard_normal((nq, 2, D)).astype(np.float32))
    target = (0.05 * rng.standard_normal((nq, 2, D))).astype(np.float32)
    qd = torch.from_numpy(q).cuda().to(torch.bfloat16)
    out = torch.zeros((nq, 2, D), dtype=torch.float32, device="cuda")
    lse = torch.zeros((nq, 2), dtype=torch.float32, device="cuda")
    ws = torch.zeros(L.loopvq_decode_workspace_bytes(dc.desc, lay), dtype=torch.uint8, device="cuda")
    L.loopvq_decode_attn(dc.desc, dc.cbK, dc.cbV, lay, dc.idxK, dc.idxV, dc.winK, dc.winV, qd, t, scale, out, lse,
                         ws)
    gk = torch.zeros(cbk.shape, dtype=torch.float32, device="cuda")
    gv = torch.zeros_like(gk)
    tgt = torch.from_numpy(target).cuda()
    for _ in range(2):
        L.loopvq_codebook_grad(dc.desc, cbk_d, cbv_d, lay, dc.idxK, dc.idxV, qd, t, scale, out, lse, tgt, 1.0, gk,
                               gv)
    torch.cuda.synchronize()
    _, ref_k, ref_v = _oracle_sum(dc, t, cbk.astype(np.float64), cbv.astype(np.float64), codes, wins, q, target,
                                  scale, 1.0, [0] * nq)
    assert _normwise(gk.cpu().numpy() / 2, ref_k) <= 2e-3
    assert _normwise(gv.cpu().numpy() / 2, ref_v) <= 2e-3


def test_fine_tuning_loop_lowers_attention_error_at_every_step():
    """Codes from the library's encode of a loop-correlated cache, codebooks
    from data rows; target = attention over the full-precision cache (oracle,
    fp64), eight queries per loop step.  Step t's loss depends only on slice
    t of both codebooks (Tc = T = 4), so each step takes its own normalised
    gradient steps on its slice with a step size that grows on success and
    halves on failure (codes fixed).  Fifteen rounds of the library's decode
    and gradient lower every step's squared attention error by >= 15 %."""
    L = _L()
    T, tc, H, D, G, N = 4, 4, 2, 128, 16, 2000
    K = synth.loop_correlated(seed=400, n_loop=T, n_tokens=N, n_heads=H, head_dim=D, n_outlier=4)
    V = synth.loop_correlated(seed=401, n_loop=T, n_tokens=N, n_heads=H, head_dim=D)
    cb0k = synth.codebook_from_rows(K, tc, G, 256, seed=402).astype(np.float32)
    cb0v = synth.codebook_from_rows(V, tc, G, 256, seed=403).astype(np.float32)
    nq = 8
    C = _cache()
    dc = C.DecodeCache(n_loop=T, tc=tc, n_heads_kv=H, head_dim=D, group_elems=G, ctx_lens=[N],
                       cb_dtype=torch.float32)
    s, body, rec = dc.splits[0]
    desc = dc.desc
    xk = torch.from_numpy(K).cuda().to(torch.bfloat16)
    xv = torch.from_numpy(V).cuda().to(torch.bfloat16)
    for kind, x, cb, pool in ((L.LOOPVQ_KEYS, xk, cb0k, dc.idxK), (L.LOOPVQ_VALUES, xv, cb0v, dc.idxV)):
        packed = torch.zeros(L.loopvq_codebook_packed_bytes(desc), dtype=torch.uint8, device="cuda")
        L.loopvq_codebook_pack(desc, torch.from_numpy(cb).cuda(), packed)
        view = x[:, s:s + body]
        L.loopvq_encode(desc, packed, kind, view, body, N * H * D, H * D, D, pool, dc.body_off[0],
                        dc.body_pool_tokens)
    win = list(range(s)) + list(range(s + body, N))
    dc.set_request_window(0, K[:, win].transpose(0, 2, 1, 3), V[:, win].transpose(0, 2, 1, 3))
    rng = np.random.default_rng(404)
    qs = [synth.round_bf16(rng.standard_normal((nq, H, D)).astype(np.float32)) for _ in range(T)]
    scale = D ** -0.5
    targets = []
    for t in range(T):
        Kt = np.asarray(K[t], dtype=np.float64).transpose(1, 0, 2)   # [H][N][D]
        Vt = np.asarray(V[t], dtype=np.float64).transpose(1, 0, 2)
        targets.append(np.stack([O.dense_decode_attention(qs[t][i], Kt, Vt, scale)[0] for i in range(nq)]))
    # the layout holds raw device pointers: keep its arrays alive
    ctx_q, boff_q, woff_q = dc.ctx_dev.repeat(nq), dc.body_off_dev.repeat(nq), dc.win_off_dev.repeat(nq)
    lay = L.make_layout(nq, dc.n_sink, dc.n_recent, dc.page, dc.max_ctx_len, ctx_q, boff_q, woff_q,
                        dc.body_pool_tokens, dc.win_pool_tokens, 0)
    ws = torch.zeros(L.loopvq_decode_workspace_bytes(desc, lay), dtype=torch.uint8, device="cuda")
    out = torch.zeros((nq, H, D), dtype=torch.float32, device="cuda")
    lse = torch.zeros((nq, H), dtype=torch.float32, device="cuda")
    qd = [torch.from_numpy(q).cuda().to(torch.bfloat16) for q in qs]
    td = [torch.from_numpy(x.astype(np.float32)).cuda() for x in targets]
    packed = [torch.zeros(L.loopvq_codebook_packed_bytes(desc), dtype=torch.uint8, device="cuda") for _ in range(2)]

    def losses_and_grads(cb):
        for c, pk in zip(cb, packed):
            L.loopvq_codebook_pack(desc, c, pk)
        grads = [torch.zeros_like(cb[0]), torch.zeros_like(cb[1])]
        losses = torch.zeros(T, dtype=torch.float32, device="cuda")
        for t in range(T):
            L.loopvq_decode_attn(desc, packed[0], packed[1], lay, dc.idxK, dc.idxV, dc.winK, dc.winV, qd[t], t,
                                 scale, out, lse, ws)
            L.loopvq_codebook_grad(desc, cb[0], cb[1], lay, dc.idxK, dc.idxV, qd[t], t, scale, out, lse, td[t], 1.0,
                                   grads[0], grads[1], losses[t:t + 1])
        return losses.cpu().numpy().astype(np.float64), grads

    cb = [torch.from_numpy(cb0k).cuda(), torch.from_numpy(cb0v).cuda()]
    loss, grads = losses_and_grads(cb)
    first = loss.copy()
    eta = np.full(T, 0.05)
    for _ in range(15):
        trial = [c.clone() for c in cb]
        for t in range(T):   # slice t (block 0, step slot t) of both codebooks
            g = torch.cat([grads[0][0, :, :, :, t].flatten(), grads[1][0, :, :, :, t].flatten()])
            gmax = float(g.abs().max())
            assert gmax > 0
            for i in range(2):
                trial[i][0, :, :, :, t] -= (eta[t] / gmax) * grads[i][0, :, :, :, t]
        new_loss, new_grads = losses_and_grads(trial)
        for t in range(T):
            if new_loss[t] < loss[t]:
                for i in range(2):
                    cb[i][0, :, :, :, t] = trial[i][0, :, :, :, t]
                eta[t] *= 1.5
            else:
                eta[t] *= 0.5
        loss, grads = losses_and_grads(cb)
    assert np.all(loss <= 0.85 * first), (first, loss)
    assert L.loopvq_read_device_status(ws)[1] == 0


def test_codebook_grad_paged_layout_matches_contiguous():
    """The same logical cache with the body in shuffled 256-token pages gives
    the same gradients (up to the order of the float atomics)."""
    L = _L()
    T, tc, G, D = 4, 4, 16, 128
    ctx = [3000, 700, 333]
    dc, cbk, cbv, cbk_d, cbv_d, codes, wins = _cache_case(tc, G, D, ctx, torch.bfloat16, Hq=2, H=2, seed=500)
    bpt = 256
    max_pages = -(-max(dc.splits[r][1] for r in range(len(ctx))) // bpt)
    n_phys = len(ctx) * max_pages + 2
    rng = np.random.default_rng(501)
    perm = rng.permutation(n_phys)
    pool_tokens = n_phys * bpt
    idxK = torch.zeros(L.loopvq_index_pool_bytes(dc.desc, pool_tokens), dtype=torch.uint8, device="cuda")
    idxV = torch.zeros_like(idxK)
    pages = np.full((len(ctx), max_pages), -1, dtype=np.int32)
    nxt = 0
    for r in range(len(ctx)):
        body = dc.splits[r][1]
        ck, cv = codes[r]
        for pi in range(-(-body // bpt)):
            pages[r, pi] = perm[nxt]
            nxt += 1
            n = min(bpt, body - pi * bpt)
            for kind, src, pool in ((0, ck, idxK), (1, cv, idxV)):
                t = torch.from_numpy(np.ascontiguousarray(src[:, :, pi * bpt:pi * bpt + n])).cuda()
                L.loopvq_index_pool_pack(dc.desc, kind, t, n, pool, int(pages[r, pi]) * bpt, pool_tokens)
    pages_dev = torch.from_numpy(pages).cuda()
    lay = L.make_layout(len(ctx), dc.n_sink, dc.n_recent, dc.page, dc.max_ctx_len, dc.ctx_dev, dc.body_off_dev,
                        dc.win_off_dev, pool_tokens, dc.win_pool_tokens, L.LOOPVQ_LAYOUT_PAGED_BODY, pages_dev, bpt,
                        max_pages)
    t, scale = 2, D ** -0.5
    q = synth.round_bf16(rng.standard_normal((len(ctx), 2, D)).astype(np.float32))
    dc.set_queries(q)
    dc.decode(t, scale)
    tgt = torch.from_numpy((0.05 * rng.standard_normal((len(ctx), 2, D))).astype(np.float32)).cuda()
    grads = []
    for layout, ik, iv in ((dc.layout, dc.idxK, dc.idxV), (lay, idxK, idxV)):
        gk = torch.zeros(cbk.shape, dtype=torch.float32, device="cuda")
        gv = torch.zeros_like(gk)
        faults = torch.zeros(1, dtype=torch.int32, device="cuda")
        L.loopvq_codebook_grad(dc.desc, cbk_d, cbv_d, layout, ik, iv, dc.q, t, scale, dc.out, dc.lse, tgt, 1.0, gk, gv,
                               None, faults)
        torch.cuda.synchronize()
        assert int(faults.item()) == 0
        grads.append((gk.cpu().numpy(), gv.cpu().numpy()))
    assert _normwise(grads[1][0], grads[0][0]) <= 1e-5
    assert _normwise(grads[1][1], grads[0][1]) <= 1e-5
    assert np.any(grads[0][0] != 0)


def test_codebook_grad_code_out_of_range_sets_fault_and_skips_token():
    """n_codes = 100: a stored code >= 100 raises the code-range bit and its
    token adds nothing; the rest still matches the oracle without it."""
    L = _L()
    C = _cache()
    T, tc, H, D, G, n_codes = 4, 4, 1, 64, 16, 100
    dc = C.DecodeCache(n_loop=T, tc=tc, n_heads_kv=H, head_dim=D, group_elems=G, ctx_lens=[1200], n_codes=n_codes,
                       cb_dtype=torch.float32, q_dtype=torch.float32)
    W = G // tc
    J = D // W
    cbk = synth.uniform_codebook(600, 1, H, J, n_codes, tc, W, bf16=False)
    cbv = synth.uniform_codebook(601, 1, H, J, n_codes, tc, W, bf16=False)
    dc.set_codebooks(cbk, cbv)
    s, body, rec = dc.splits[0]
    ck = synth.random_codes(602, 1, H, body, J, n_codes)
    cv = synth.random_codes(603, 1, H, body, J, n_codes)
    rng = np.random.default_rng(604)
    wk = rng.standard_normal((T, H, s + rec, D)).astype(np.float32)
    wv = rng.standard_normal((T, H, s + rec, D)).astype(np.float32)
    dc.set_request_window(0, wk, wv)
    dc.set_request_codes(0, ck, cv)
    t, scale = 1, D ** -0.5
    q = rng.standard_normal((1, H, D)).astype(np.float32)
    dc.set_queries(q)
    dc.decode(t, scale)                          # forward with valid codes
    bad = ck.copy()
    bad[0, 0, 77, 5] = 200                       # token 77's key code out of range
    dc.set_request_codes(0, bad, cv)
    target = (0.05 * rng.standard_normal((1, H, D))).astype(np.float32)
    gk = torch.zeros(cbk.shape, dtype=torch.float32, device="cuda")
    gv = torch.zeros_like(gk)
    faults = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.loopvq_codebook_grad(dc.desc, torch.from_numpy(cbk).cuda(), torch.from_numpy(cbv).cuda(), dc.layout, dc.idxK,
                           dc.idxV, dc.q, t, scale, dc.out, dc.lse, torch.from_numpy(target).cuda(), 1.0, gk, gv, None,
                           faults)
    torch.cuda.synchronize()
    assert int(faults.item()) & L.LOOPVQ_FAULT_CODE_RANGE
    # oracle over the valid codes; token 77 is skipped on the GPU, so compare
    # every entry that token 77 does not touch (its K and V codeword per slot)
    _, ref_k, ref_v, _ = O.attention_mse_codebook_grad(q[0], t, tc, ck, cv, cbk, cbv, wk[t], wv[t], scale, target[0])
    got_k = gk.cpu().numpy().astype(np.float64)
    got_v = gv.cpu().numpy().astype(np.float64)
    mk = np.ones(got_k.shape, dtype=bool)
    mv = np.ones(got_v.shape, dtype=bool)
    for j in range(J):
        mk[0, 0, j, ck[0, 0, 77, j]] = False
        mv[0, 0, j, cv[0, 0, 77, j]] = False
    scale_k = np.max(np.abs(ref_k))
    scale_v = np.max(np.abs(ref_v))
    assert np.max(np.abs(got_k[mk] - ref_k[mk])) <= 2e-3 * scale_k
    assert np.max(np.abs(got_v[mv] - ref_v[mv])) <= 2e-3 * scale_v
    assert np.all(np.isfinite(got_k)) and np.all(np.isfinite(got_v))
