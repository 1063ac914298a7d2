"""The allocation-free decode entry point against the regular one.

loopvq_decode_attn_noalloc exists for callers that cannot allocate device
memory themselves: a plugin loaded into a host process whose allocator owns
the whole GPU, or a hot path that must not call cudaMalloc because it
synchronizes the device.  It takes no workspace and keeps its split partials
in a fixed array inside the library.  This file checks, through the C ABI,
that two calls in a row give the regular entry point's outputs within the
decode tolerance of the other tests, and that a layout too large for the
fixed array is refused up front.  The file name makes pytest collect it
last; it builds all its own inputs, so it also passes in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle as O
from sub_bit_vector_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _err(o, ref):
    den = np.max(np.abs(ref))
    return float(np.max(np.abs(o - ref)) / (den if den > 0 else 1.0))


def test_noalloc_matches_workspace_entry_on_two_calls():
    from sub_bit_vector_b200 import cache, loopvq as L
    T, Tc, H, Hq, D, G = 4, 4, 4, 8, 128, 16
    ctx = [5000, 9000, 300, 4416]
    c = cache.DecodeCache(n_loop=T, tc=Tc, n_heads_kv=H, head_dim=D, group_elems=G, ctx_lens=ctx, n_heads_q=Hq)
    W, J = G // Tc, D * Tc // G
    outl = synth.key_outlier_channels(31, H, D)
    cbk = synth.uniform_codebook(32, 1, H, J, 256, Tc, W, outlier_channels=outl)
    cbv = synth.uniform_codebook(33, 1, H, J, 256, Tc, W)
    c.set_codebooks(cbk, cbv)
    reqs = []
    for r, (s, b, rc) in enumerate(c.splits):
        wk, wv, ck, cv = synth.decode_request(34 + r, T, H, D, J, 1, s + rc, b, outlier_channels=outl)
        c.set_request_window(r, wk, wv)
        c.set_request_codes(r, ck, cv)
        reqs.append((wk, wv, ck, cv))
    q = synth.queries(35, T, len(ctx), Hq, D)
    out2 = torch.zeros_like(c.out)
    lse2 = torch.zeros_like(c.lse)
    fault = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t in (1, 2):                      # two calls in a row
        c.set_queries(q[t])
        c.decode(t)                       # regular entry point, caller-owned workspace
        L.loopvq_decode_attn_noalloc(c.desc, c.cbK, c.cbV, c.layout, c.idxK, c.idxV, c.winK, c.winV, c.q, t,
                                     D ** -0.5, out2, lse2, fault)
        torch.cuda.synchronize()
        ref, lref = c.out.cpu().numpy(), c.lse.cpu().numpy()
        got, lgot = out2.cpu().numpy(), lse2.cpu().numpy()
        for r in range(len(ctx)):
            for h in range(Hq):
                assert _err(got[r, h], ref[r, h]) <= TOL, (t, r, h)
        np.testing.assert_allclose(lgot, lref, atol=TOL, rtol=TOL)
        assert int(fault.item()) == 0
        # and on its own against the fp64 oracle, request 0 (all query heads)
        wk, wv, ck, cv = reqs[0]
        o_ref, _ = O.decode_attention(q[t, 0], t, Tc, ck, cv, cbk, cbv, wk[t], wv[t], D ** -0.5)
        for h in range(Hq):
            assert _err(got[0, h], o_ref[h]) <= TOL, (t, h)
    assert c.device_status()[1] == 0

    # a fault only the device can see lands in the caller's word: a context
    # longer than the layout's max_ctx_len is reported and that request gets
    # a zero output, the others are unaffected
    bad_ctx = torch.tensor([ctx[0], c.max_ctx_len + 100, ctx[2], ctx[3]], dtype=torch.int32, device="cuda")
    lay = L.make_layout(len(ctx), c.n_sink, c.n_recent, c.page, c.max_ctx_len, bad_ctx, c.body_off_dev,
                        c.win_off_dev, c.body_pool_tokens, c.win_pool_tokens, 0)
    fault.zero_()
    L.loopvq_decode_attn_noalloc(c.desc, c.cbK, c.cbV, lay, c.idxK, c.idxV, c.winK, c.winV, c.q, 2,
                                 D ** -0.5, out2, lse2, fault)
    torch.cuda.synchronize()
    assert int(fault.item()) & L.LOOPVQ_FAULT_CTX_RANGE
    got = out2.cpu().numpy()
    assert np.all(got[1] == 0) and np.all(np.isneginf(lse2.cpu().numpy()[1]))
    for h in range(Hq):
        assert _err(got[0, h], ref[0, h]) <= TOL


def test_noalloc_refuses_layout_beyond_its_scratch():
    from sub_bit_vector_b200 import loopvq as L
    desc = L.make_desc(4, 4, 16, 128, 16, n_heads_q=64)
    fake = 1 << 20
    # 4096 requests x 64 query heads need far more than the fixed 8 MiB
    layout = L.make_layout(4096, 64, 256, 8, 65536, fake, fake, fake, 1 << 20, 1 << 20)
    assert L.loopvq_decode_workspace_bytes(desc, layout) > 8 << 20
    with pytest.raises(L.LoopVQError) as e:
        L.loopvq_decode_attn_noalloc(desc, fake, fake, layout, fake, fake, fake, fake,
                                     torch.zeros(1, dtype=torch.bfloat16, device="cuda"), 0, 0.1,
                                     torch.zeros(1, dtype=torch.float32, device="cuda"), None)
    assert e.value.status == L.LOOPVQ_ERR_WORKSPACE_TOO_SMALL
