"""Host-side bookkeeping of PagedCache, on the CPU (no kernel runs): over a
long run of generated tokens the ring slots of the live window tokens never
collide, every page that leaves the window is 8 contiguous ring slots
starting at a page boundary, and body tokens get distinct index-pool
positions in the request's own pages."""
import numpy as np
import torch

from sub_bit_vector_b200 import cache, loopvq as L


def test_ring_and_page_bookkeeping(monkeypatch):
    calls = []

    def fake_encode(desc, cb, kind, x, n, st, sn, sh, pool, tok_off, pool_tokens, stream=None, x_dtype=None):
        calls.append((kind, n, tok_off, x.data_ptr()))

    monkeypatch.setattr(L, "loopvq_encode", fake_encode)
    pc = cache.PagedCache(n_loop=4, tc=4, n_heads_kv=1, head_dim=64, group_elems=16, batch=2, max_ctx_len=2000,
                          body_page_tokens=64, device="cpu")
    pc.ctx = [10, 300]
    for r in range(2):
        pc._sync_state(r)
    positions = [dict(), dict()]
    for _ in range(1500):
        for r in range(2):
            if pc.ctx[r] >= 2000:
                continue
            s0, body0, _ = pc.split(r)
            head0 = pc.head[r]
            n_calls = len(calls)
            pc.begin_token(r)
            s, body, rec = pc.split(r)
            assert s + body + rec == pc.ctx[r]
            if body > body0:
                assert body - body0 == 8 and head0 % 8 == 0
                assert len(calls) == n_calls + 2 and all(c[1] == 8 for c in calls[-2:])
                pos = calls[-1][2]
                assert pos == pc._body_pos(r, body0)
                for p in range(body0, body):
                    q = pc._body_pos(r, p)
                    assert q not in positions[r].values()
                    positions[r][p] = q
            slots = [pc._slot_row(r, i) for i in range(s + rec)]
            assert len(set(slots)) == len(slots)
            assert all(r * pc.win_stride <= x < (r + 1) * pc.win_stride for x in slots)
            assert int(pc.ctx_dev[r]) == pc.ctx[r] and int(pc.head_dev[r]) == pc.head[r]
    # the two requests never share a page
    assert not set(pc.pages[0]) & set(pc.pages[1])
    assert torch.equal(pc.pages_dev[0, :len(pc.pages[0])], torch.tensor(pc.pages[0], dtype=torch.int32))
