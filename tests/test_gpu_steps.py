"""Several loop steps in one launch (loopvq_decode_attn_steps).

Step t of a multi-step launch computes what loopvq_decode_attn computes at
loop step t: checked against the fp64 oracle (tolerance of the decode tests)
for all four steps at once and for a range that crosses code blocks (Tc = 2),
bit-identical to the single-step launches where both plan the same splits
(64K context, 16 heads), and with the current token's K/V per step stored
into every step's window.
"""
import numpy as np
import pytest
import torch

from sub_bit_vector_b200 import synth
from test_gpu_decode import TOL, Case, _err

pytestmark = pytest.mark.gpu


def _L():
    from sub_bit_vector_b200 import loopvq
    return loopvq


def _run_steps(case, first, n):
    L = _L()
    c = case.c
    B = len(c.ctx_lens)
    q = torch.from_numpy(np.ascontiguousarray(case.q[first:first + n], dtype=np.float32)).cuda().to(c.q.dtype)
    out = torch.zeros((n, B, c.Hq, c.D), dtype=torch.float32, device="cuda")
    lse = torch.zeros((n, B, c.Hq), dtype=torch.float32, device="cuda")
    ws = torch.zeros(L.loopvq_decode_steps_workspace_bytes(c.desc, c.layout, n), dtype=torch.uint8, device="cuda")
    L.loopvq_decode_attn_steps(c.desc, c.cbK, c.cbV, c.layout, c.idxK, c.idxV, c.winK, c.winV, q, first, n,
                               c.D ** -0.5, out, lse, ws)
    torch.cuda.synchronize()
    assert L.loopvq_read_device_status(ws)[1] == 0
    return out.cpu().numpy(), lse.cpu().numpy()


def _check(case, first, n, out, lse):
    for i in range(n):
        t = first + i
        for r in sorted(case.keep):
            o_ref, l_ref = case.oracle(t, r)
            for hq in range(case.Hq):
                assert _err(out[i, r, hq], o_ref[hq]) <= TOL, (t, r, hq)
                if np.isfinite(l_ref[hq]):
                    assert abs(lse[i, r, hq] - l_ref[hq]) <= TOL * max(1.0, abs(l_ref[hq]))
                else:
                    assert lse[i, r, hq] == -np.inf


def test_all_steps_in_one_launch_match_oracle():
    case = Case(seed=31, ctx_lens=[5000, 1200, 333, 64, 0], H=2, Hq=4)
    out, lse = _run_steps(case, 0, 4)
    _check(case, 0, 4, out, lse)


def test_step_range_across_code_blocks():
    """Tc = 2: steps 1 and 2 read code blocks 0 and 1."""
    case = Case(seed=32, ctx_lens=[3000, 700], H=2, Tc=2, G=8)
    out, lse = _run_steps(case, 1, 2)
    _check(case, 1, 2, out, lse)
    out1, lse1 = _run_steps(case, 3, 1)
    _check(case, 3, 1, out1, lse1)


def test_steps_launch_bit_identical_to_single_steps_at_64k():
    """With 16 heads at 64K both launches cut 16 body splits per head, so the
    arithmetic is the same and so are the bits."""
    from sub_bit_vector_b200 import cache
    L = _L()
    c = cache.DecodeCache(n_loop=4, tc=4, n_heads_kv=16, head_dim=128, group_elems=16, ctx_lens=[65536])
    cb = synth.uniform_codebook(1, 1, 16, 32, 256, 4, 4)
    c.set_codebooks(cb, cb)
    c.idxK.copy_(synth.device_codes(2, c.idxK.numel()))
    c.idxV.copy_(synth.device_codes(3, c.idxV.numel()))
    c.winK.normal_()
    c.winV.normal_()
    q = torch.randn((4, 1, 16, 128), device="cuda").to(torch.bfloat16)
    single = []
    for t in range(4):
        c.q.copy_(q[t])
        c.decode(t)
        single.append((c.out.clone(), c.lse.clone()))
    out = torch.zeros((4, 1, 16, 128), dtype=torch.float32, device="cuda")
    lse = torch.zeros((4, 1, 16), dtype=torch.float32, device="cuda")
    ws = torch.zeros(L.loopvq_decode_steps_workspace_bytes(c.desc, c.layout, 4), dtype=torch.uint8, device="cuda")
    L.loopvq_decode_attn_steps(c.desc, c.cbK, c.cbV, c.layout, c.idxK, c.idxV, c.winK, c.winV, q, 0, 4,
                               128 ** -0.5, out, lse, ws)
    torch.cuda.synchronize()
    for t in range(4):
        assert torch.equal(out[t], single[t][0]) and torch.equal(lse[t], single[t][1]), t
    assert L.loopvq_read_device_status(ws)[1] == 0 and c.device_status()[1] == 0


def test_new_token_per_step_is_used_and_stored():
    L = _L()
    case = Case(seed=33, ctx_lens=[400, 5], H=2, Hq=4, D=64)
    c = case.c
    ref, ref_lse = _run_steps(case, 0, 4)
    last = [c.win_off[r] + c.splits[r][0] + c.splits[r][2] - 1 for r in range(2)]
    nk = torch.stack([torch.stack([c.winK[t, :, last[r]] for r in range(2)]) for t in range(4)]).contiguous()
    nv = torch.stack([torch.stack([c.winV[t, :, last[r]] for r in range(2)]) for t in range(4)]).contiguous()
    for r in range(2):
        c.winK[:, :, last[r]] = 1e4
        c.winV[:, :, last[r]] = -1e4
    lay = L.make_layout(2, c.n_sink, c.n_recent, c.page, c.max_ctx_len, c.ctx_dev, c.body_off_dev, c.win_off_dev,
                        c.body_pool_tokens, c.win_pool_tokens, 0, new_k=nk, new_v=nv)
    q = torch.from_numpy(np.ascontiguousarray(case.q, dtype=np.float32)).cuda().to(torch.bfloat16)
    out = torch.zeros((4, 2, 4, 64), dtype=torch.float32, device="cuda")
    lse = torch.zeros((4, 2, 4), dtype=torch.float32, device="cuda")
    ws = torch.zeros(L.loopvq_decode_steps_workspace_bytes(c.desc, lay, 4), dtype=torch.uint8, device="cuda")
    L.loopvq_decode_attn_steps(c.desc, c.cbK, c.cbV, lay, c.idxK, c.idxV, c.winK, c.winV, q, 0, 4, 64 ** -0.5, out,
                               lse, ws)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), ref) and np.array_equal(lse.cpu().numpy(), ref_lse)
    for t in range(4):
        for r in range(2):
            assert torch.equal(c.winK[t, :, last[r]], nk[t, r]) and torch.equal(c.winV[t, :, last[r]], nv[t, r])


def test_steps_launch_over_paged_body_and_ring_window():
    """All four steps in one launch over a paged body (shuffled 256-token
    pages) and ring windows that wrap: every step matches the oracle."""
    L = _L()
    case = Case(seed=34, ctx_lens=[5000, 700, 333], H=2, Hq=4)
    c = case.c
    rng = np.random.default_rng(35)
    bpt, ns, nr, pg = 256, 64, 256, 8
    ring = nr + pg
    B = len(c.ctx_lens)
    max_pages = -(-max(c.splits[r][1] for r in range(B)) // bpt)
    n_phys = B * max_pages + 3
    perm = rng.permutation(n_phys)
    idxK = torch.zeros(L.loopvq_index_pool_bytes(c.desc, n_phys * bpt), dtype=torch.uint8, device="cuda")
    idxV = torch.zeros_like(idxK)
    pages = np.full((B, max_pages), -1, dtype=np.int32)
    heads = np.array([200, 8, 0], dtype=np.int32)
    stride = ns + ring
    winK = torch.zeros((c.T, c.H, B * stride, c.D), dtype=torch.bfloat16, device="cuda")
    winV = torch.zeros_like(winK)
    nxt = 0
    for r in range(B):
        s, body, rec = c.splits[r]
        wk, wv, ck, cv = case.req[r]
        for pi in range(-(-body // bpt)):
            pages[r, pi] = perm[nxt]
            nxt += 1
            n = min(bpt, body - pi * bpt)
            for kind, src, pool in ((0, ck, idxK), (1, cv, idxV)):
                t = torch.from_numpy(np.ascontiguousarray(src[:, :, pi * bpt:pi * bpt + n])).cuda()
                L.loopvq_index_pool_pack(c.desc, kind, t, n, pool, int(pages[r, pi]) * bpt, n_phys * bpt)
        for i in range(s + rec):
            row = r * stride + (i if i < s else ns + (heads[r] + i - s) % ring)
            winK[:, :, row] = torch.from_numpy(np.ascontiguousarray(wk[:, :, i], dtype=np.float32)).cuda().to(
                torch.bfloat16)
            winV[:, :, row] = torch.from_numpy(np.ascontiguousarray(wv[:, :, i], dtype=np.float32)).cuda().to(
                torch.bfloat16)
    assert heads[0] + c.splits[0][2] > ring   # request 0's ring wraps
    pages_dev = torch.from_numpy(pages).cuda()
    heads_dev = torch.from_numpy(heads).cuda()
    win_off = torch.arange(B, dtype=torch.int64, device="cuda") * stride
    lay = L.make_layout(B, ns, nr, pg, c.max_ctx_len, c.ctx_dev, c.body_off_dev, win_off, n_phys * bpt, B * stride,
                        L.LOOPVQ_LAYOUT_PAGED_BODY | L.LOOPVQ_LAYOUT_RING_WINDOW, pages_dev, bpt, max_pages,
                        heads_dev, ring)
    q = torch.from_numpy(np.ascontiguousarray(case.q, dtype=np.float32)).cuda().to(torch.bfloat16)
    out = torch.zeros((4, B, c.Hq, c.D), dtype=torch.float32, device="cuda")
    lse = torch.zeros((4, B, c.Hq), dtype=torch.float32, device="cuda")
    ws = torch.zeros(L.loopvq_decode_steps_workspace_bytes(c.desc, lay, 4), dtype=torch.uint8, device="cuda")
    L.loopvq_decode_attn_steps(c.desc, c.cbK, c.cbV, lay, idxK, idxV, winK, winV, q, 0, 4, c.D ** -0.5, out, lse, ws)
    torch.cuda.synchronize()
    assert L.loopvq_read_device_status(ws)[1] == 0
    _check(case, 0, 4, out.cpu().numpy(), lse.cpu().numpy())
