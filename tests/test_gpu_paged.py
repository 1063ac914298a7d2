"""Paged body, ring window and the fused bf16 write of the current token.

1. A paged + ring layout of the same logical cache as a contiguous layout
   (shuffled physical pages, ring heads that wrap) gives bit-identical
   outputs: the layout changes only where bytes come from.
2. With new_k/new_v the decode uses the given current-token K/V (the pool
   row holds garbage) and stores them in the token's window slot.
3. An incremental run of PagedCache (prompt, then generated tokens that cross
   several page evictions, the new token written by the decode itself) is
   checked at every token and loop step against the oracle on the logical
   cache, and its body codes against the oracle's encode.
"""
import numpy as np
import pytest
import torch

import oracle as O
from sub_bit_vector_b200 import synth

pytestmark = pytest.mark.gpu

NS, NR, PG = 64, 256, 8


def _L():
    from sub_bit_vector_b200 import loopvq
    return loopvq


def _cache():
    from sub_bit_vector_b200 import cache
    return cache


def test_paged_ring_layout_equals_contiguous_layout():
    L, C = _L(), _cache()
    T, tc, H, D, G = 4, 4, 2, 128, 16
    ctx = [5000, 3000, 333, 70]
    dc = C.DecodeCache(n_loop=T, tc=tc, n_heads_kv=H, head_dim=D, group_elems=G, ctx_lens=ctx)
    W = G // tc
    J = D // W
    cbk = synth.uniform_codebook(1, 1, H, J, 256, tc, W, outlier_channels=synth.key_outlier_channels(2, H, D))
    cbv = synth.uniform_codebook(3, 1, H, J, 256, tc, W)
    dc.set_codebooks(cbk, cbv)
    rng = np.random.default_rng(7)
    wins, codes = [], []
    for r, c in enumerate(ctx):
        s, body, rec = dc.splits[r]
        ck = synth.random_codes(10 + r, 1, H, body, J)
        cv = synth.random_codes(20 + r, 1, H, body, J)
        dc.set_request_codes(r, ck, cv)
        wk = synth.round_bf16(rng.standard_normal((T, H, s + rec, D)).astype(np.float32))
        wv = synth.round_bf16(rng.standard_normal((T, H, s + rec, D)).astype(np.float32))
        dc.set_request_window(r, wk, wv)
        wins.append((wk, wv))
        codes.append((ck, cv))

    # the same cache, paged and in rings
    bpt, ring = 256, NR + PG
    max_pages = -(-max(dc.splits[r][1] for r in range(len(ctx))) // bpt)
    n_phys = len(ctx) * max_pages + 3
    perm = rng.permutation(n_phys)
    desc = dc.desc
    idxK = torch.zeros(L.loopvq_index_pool_bytes(desc, n_phys * bpt), dtype=torch.uint8, device="cuda")
    idxV = torch.zeros_like(idxK)
    pages = np.full((len(ctx), max_pages), -1, dtype=np.int32)
    heads = np.zeros(len(ctx), dtype=np.int32)
    stride = NS + ring
    P = len(ctx) * stride
    winK = torch.zeros((T, H, P, D), dtype=torch.bfloat16, device="cuda")
    winV = torch.zeros_like(winK)
    nxt = 0
    for r in range(len(ctx)):
        s, body, rec = dc.splits[r]
        ck, cv = codes[r]
        for pi in range(-(-body // bpt)):
            pages[r, pi] = perm[nxt]
            nxt += 1
            n = min(bpt, body - pi * bpt)
            for kind, src, pool in ((0, ck, idxK), (1, cv, idxV)):
                t = torch.from_numpy(np.ascontiguousarray(src[:, :, pi * bpt:pi * bpt + n])).cuda()
                L.loopvq_index_pool_pack(desc, kind, t, n, pool, int(pages[r, pi]) * bpt, n_phys * bpt)
        heads[r] = [200, 8, 256, 0][r] if rec else 0
        wk, wv = wins[r]
        for i in range(s + rec):
            row = r * stride + (i if i < s else NS + (heads[r] + i - s) % ring)
            winK[:, :, row] = torch.from_numpy(wk[:, :, i]).cuda().to(torch.bfloat16)
            winV[:, :, row] = torch.from_numpy(wv[:, :, i]).cuda().to(torch.bfloat16)
    assert any(h + dc.splits[r][2] > ring for r, h in enumerate(heads))   # at least one ring wraps
    pages_dev = torch.from_numpy(pages).cuda()
    heads_dev = torch.from_numpy(heads).cuda()
    win_off = torch.arange(len(ctx), dtype=torch.int64, device="cuda") * stride
    lay = L.make_layout(len(ctx), NS, NR, PG, max(ctx), dc.ctx_dev, dc.body_off_dev, win_off, n_phys * bpt, P,
                        L.LOOPVQ_LAYOUT_PAGED_BODY | L.LOOPVQ_LAYOUT_RING_WINDOW, pages_dev, bpt, max_pages,
                        heads_dev, ring)
    ws = torch.zeros(L.loopvq_decode_workspace_bytes(desc, lay), dtype=torch.uint8, device="cuda")
    out = torch.zeros_like(dc.out)
    lse = torch.zeros_like(dc.lse)
    for t in range(T):
        dc.set_queries(rng.standard_normal((len(ctx), H, D)))
        dc.decode(t)
        L.loopvq_decode_attn(desc, dc.cbK, dc.cbV, lay, idxK, idxV, winK, winV, dc.q, t, D ** -0.5, out, lse, ws)
        torch.cuda.synchronize()
        assert torch.equal(out, dc.out) and torch.equal(lse, dc.lse)
    assert L.loopvq_read_device_status(ws)[1] == 0


def test_new_token_is_used_and_stored():
    L, C = _L(), _cache()
    T, tc, H, D, G = 4, 4, 2, 64, 16
    ctx = [400, 5]
    dc = C.DecodeCache(n_loop=T, tc=tc, n_heads_kv=H, head_dim=D, group_elems=G, ctx_lens=ctx, n_heads_q=4)
    W = G // tc
    J = D // W
    cb = synth.uniform_codebook(5, 1, H, J, 256, tc, W)
    dc.set_codebooks(cb, cb)
    rng = np.random.default_rng(8)
    for r, c in enumerate(ctx):
        s, body, rec = dc.splits[r]
        dc.set_request_codes(r, synth.random_codes(30 + r, 1, H, body, J), synth.random_codes(40 + r, 1, H, body, J))
        dc.set_request_window(r, rng.standard_normal((T, H, s + rec, D)), rng.standard_normal((T, H, s + rec, D)))
    t = 2
    dc.set_queries(rng.standard_normal((2, 4, D)))
    dc.decode(t)
    torch.cuda.synchronize()
    ref = dc.out.clone()
    last = [dc.win_off[r] + dc.splits[r][0] + dc.splits[r][2] - 1 for r in range(2)]
    nk = torch.stack([dc.winK[t, :, last[r]] for r in range(2)]).contiguous()   # [batch][H][D]
    nv = torch.stack([dc.winV[t, :, last[r]] for r in range(2)]).contiguous()
    for r in range(2):  # garbage in the pool rows of the current tokens
        dc.winK[t, :, last[r]] = 1e4
        dc.winV[t, :, last[r]] = -1e4
    lay = L.make_layout(2, NS, NR, PG, max(ctx), dc.ctx_dev, dc.body_off_dev, dc.win_off_dev,
                        dc.body_pool_tokens, dc.win_pool_tokens, 0, new_k=nk, new_v=nv)
    L.loopvq_decode_attn(dc.desc, dc.cbK, dc.cbV, lay, dc.idxK, dc.idxV, dc.winK, dc.winV, dc.q, t, D ** -0.5,
                         dc.out, dc.lse, dc.workspace)
    torch.cuda.synchronize()
    assert torch.equal(dc.out, ref)
    for r in range(2):
        assert torch.equal(dc.winK[t, :, last[r]], nk[r]) and torch.equal(dc.winV[t, :, last[r]], nv[r])


def test_incremental_paged_cache_matches_oracle_every_token():
    C = _cache()
    L = _L()
    T, tc, H, D, G = 4, 4, 2, 128, 16
    W = G // tc
    J = D // W
    prompts, n_new = [300, 317], 40        # crosses 320, 328, 336, 344 and 352
    total = [p + n_new for p in prompts]
    K = [synth.loop_correlated(seed=60 + r, n_loop=T, n_tokens=total[r], n_heads=H, head_dim=D, n_outlier=4)
         for r in range(2)]
    V = [synth.loop_correlated(seed=70 + r, n_loop=T, n_tokens=total[r], n_heads=H, head_dim=D) for r in range(2)]
    cbk = synth.codebook_from_rows(K[0], tc, G, 256, seed=80)
    cbv = synth.codebook_from_rows(V[0], tc, G, 256, seed=81)
    pc = C.PagedCache(n_loop=T, tc=tc, n_heads_kv=H, head_dim=D, group_elems=G, batch=2, max_ctx_len=max(total),
                      body_page_tokens=32, spare_pages=2)
    pc.set_codebooks(cbk, cbv)
    # the oracle's codes of every token (encoding is per token)
    ok = [O.encode(K[r], cbk, tc)[0] for r in range(2)]
    ov = [O.encode(V[r], cbv, tc)[0] for r in range(2)]
    for r in range(2):
        pc.prefill(r, torch.from_numpy(K[r][:, :prompts[r]]), torch.from_numpy(V[r][:, :prompts[r]]))
    rng = np.random.default_rng(90)
    for step in range(n_new):
        for r in range(2):
            pc.begin_token(r)
        for t in range(T):
            q = synth.round_bf16(rng.standard_normal((2, H, D)).astype(np.float32))
            pc.set_queries(q)
            cur = [pc.ctx[r] - 1 for r in range(2)]
            nk = torch.from_numpy(np.stack([K[r][t, cur[r]] for r in range(2)])).cuda().to(torch.bfloat16)
            nv = torch.from_numpy(np.stack([V[r][t, cur[r]] for r in range(2)])).cuda().to(torch.bfloat16)
            pc.decode(t, nk.contiguous(), nv.contiguous())
            torch.cuda.synchronize()
            out = pc.out.cpu().numpy()
            for r in range(2):
                s, body, rec = pc.split(r)
                n = pc.ctx[r]
                win = list(range(s)) + list(range(s + body, n))
                wk = K[r][t][win].transpose(1, 0, 2)    # [H][n_win][D]
                wv = V[r][t][win].transpose(1, 0, 2)
                o_ref, _ = O.decode_attention(q[r], t, tc, ok[r][:, :, s:s + body], ov[r][:, :, s:s + body],
                                              cbk, cbv, wk, wv, D ** -0.5)
                err = np.max(np.abs(out[r] - o_ref), axis=1) / np.max(np.abs(o_ref), axis=1)
                assert np.all(err <= 2e-3), (step, t, r, float(err.max()))
    assert pc.device_status()[1] == 0
    # body codes written by the page encodes match the oracle's (up to near-ties)
    for r in range(2):
        s, body, _ = pc.split(r)
        assert body > 0
        for kind, ref in ((L.LOOPVQ_KEYS, ok[r]), (L.LOOPVQ_VALUES, ov[r])):
            got = pc.body_codes(r, kind).astype(np.int64)
            mism = np.mean(got != ref[:, :, s:s + body])
            assert mism < 1e-3, mism
