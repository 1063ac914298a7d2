"""Host-side plumbing for one layer's LoopVQ decode cache on the device.

Allocates the pools, windows, codebooks, queries, outputs and workspace of
a decode batch as torch device tensors, copies per-request host arrays into
them at the offsets the cache layout prescribes, and calls the library.  It
does no arithmetic of the method: codes, windows and codebooks are inputs, and
every step of encode and decode runs in libloopvq's kernels.
"""
from __future__ import annotations

import numpy as np
import torch

from . import loopvq as L


def _round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


class DecodeCache:
    """Device buffers of one layer (K and V) for a batch of decode requests.

    ``ctx_lens`` are the per-request context lengths (current token
    included).  Bodies are laid out back to back in the index pools at
    32-token-aligned offsets; windows back to back in the window pools.
    """

    def __init__(self, *, n_loop, tc, n_heads_kv, head_dim, group_elems, ctx_lens, n_sink=64, n_recent=256,
                 page=8, n_codes=256, n_heads_q=None, cb_dtype=torch.bfloat16, q_dtype=torch.bfloat16,
                 out_dtype=torch.float32, device="cuda", max_ctx_len=None, pool_slack_tokens=0,
                 static_inputs=False):
        self.device = torch.device(device)
        self.T, self.Tc, self.H, self.D, self.G = n_loop, tc, n_heads_kv, head_dim, group_elems
        self.Hq = n_heads_q or n_heads_kv
        self.W = group_elems // tc
        self.J = head_dim // self.W
        self.NB = n_loop // tc
        self.C = n_codes
        self.n_sink, self.n_recent, self.page = n_sink, n_recent, page
        self.cb_dtype = cb_dtype
        self.desc = L.make_desc(n_loop, tc, n_heads_kv, head_dim, group_elems, n_codes, self.Hq,
                                L.LOOPVQ_BF16 if cb_dtype == torch.bfloat16 else L.LOOPVQ_F32)
        self.ctx_lens = [int(c) for c in ctx_lens]
        self.batch = len(self.ctx_lens)
        self.splits = [L.loopvq_ctx_split(c, n_sink, n_recent, page) for c in self.ctx_lens]
        body_off, win_off = [], []
        b = w = 0
        for (s, body, rec) in self.splits:
            body_off.append(b)
            win_off.append(w)
            b += _round_up(body, 32)
            w += s + rec
        self.body_off = body_off
        self.win_off = win_off
        self.body_pool_tokens = max(32, _round_up(b + pool_slack_tokens, 32))
        self.win_pool_tokens = max(1, w)
        self.max_ctx_len = max(self.ctx_lens) if max_ctx_len is None else max_ctx_len
        dev = self.device
        pool_bytes = L.loopvq_index_pool_bytes(self.desc, self.body_pool_tokens)
        self.idxK = torch.zeros(pool_bytes, dtype=torch.uint8, device=dev)
        self.idxV = torch.zeros(pool_bytes, dtype=torch.uint8, device=dev)
        self.winK = torch.zeros((self.T, self.H, self.win_pool_tokens, self.D), dtype=torch.bfloat16, device=dev)
        self.winV = torch.zeros_like(self.winK)
        pb = L.loopvq_codebook_packed_bytes(self.desc)
        self.cbK = torch.zeros(pb, dtype=torch.uint8, device=dev)
        self.cbV = torch.zeros(pb, dtype=torch.uint8, device=dev)
        self.q = torch.zeros((self.batch, self.Hq, self.D), dtype=q_dtype, device=dev)
        self.out = torch.zeros((self.batch, self.Hq, self.D), dtype=out_dtype, device=dev)
        self.lse = torch.zeros((self.batch, self.Hq), dtype=torch.float32, device=dev)
        self.ctx_dev = torch.tensor(self.ctx_lens, dtype=torch.int32, device=dev)
        self.body_off_dev = torch.tensor(body_off, dtype=torch.int64, device=dev)
        self.win_off_dev = torch.tensor(win_off, dtype=torch.int64, device=dev)
        # static_inputs: this cache's layout arrays, index pools and codebooks
        # are not written by kernels that may still run when a decode starts
        self.flags = L.LOOPVQ_LAYOUT_STATIC_INPUTS if static_inputs else 0
        self.layout = self._make_layout(None, None)
        ws = L.loopvq_decode_workspace_bytes(self.desc, self.layout)
        if ws == 0:
            raise ValueError("invalid cache layout")
        self.workspace = torch.zeros(_round_up(ws, 256), dtype=torch.uint8, device=dev)

    def _make_layout(self, new_k, new_v):
        return L.make_layout(self.batch, self.n_sink, self.n_recent, self.page, self.max_ctx_len, self.ctx_dev,
                             self.body_off_dev, self.win_off_dev, self.body_pool_tokens, self.win_pool_tokens,
                             self.flags, new_k=new_k, new_v=new_v)

    # ------------------------------------------------------------ inputs
    def set_codebooks(self, cb_k: np.ndarray, cb_v: np.ndarray) -> None:
        """Canonical codebooks [NB][H][J][C][Tc][W] (host arrays) -> packed."""
        for src, dst in ((cb_k, self.cbK), (cb_v, self.cbV)):
            t = torch.from_numpy(np.ascontiguousarray(src, dtype=np.float32)).to(self.cb_dtype).to(self.device)
            L.loopvq_codebook_pack(self.desc, t, dst)
        torch.cuda.current_stream().synchronize()

    def set_request_codes(self, r: int, codes_k: np.ndarray, codes_v: np.ndarray) -> None:
        """Body codes of request r, [NB][H][n_body][J] uint8 (token-major)."""
        n = self.splits[r][1]
        if codes_k.shape[2] != n or codes_v.shape[2] != n:
            raise ValueError(f"request {r}: expected {n} body tokens")
        if n == 0:
            return
        for kind, src, pool in ((L.LOOPVQ_KEYS, codes_k, self.idxK), (L.LOOPVQ_VALUES, codes_v, self.idxV)):
            t = torch.from_numpy(np.ascontiguousarray(src, dtype=np.uint8)).to(self.device)
            L.loopvq_index_pool_pack(self.desc, kind, t, n, pool, self.body_off[r], self.body_pool_tokens)
            torch.cuda.current_stream().synchronize()

    def set_request_window(self, r: int, win_k: np.ndarray, win_v: np.ndarray) -> None:
        """Window tokens (sink then recent) of request r, [T][H][n_win][D] values
        (rounded to bf16 on upload)."""
        s, _, rec = self.splits[r]
        n = s + rec
        if win_k.shape[2] != n:
            raise ValueError(f"request {r}: expected {n} window tokens")
        o = self.win_off[r]
        self.winK[:, :, o:o + n] = torch.from_numpy(np.ascontiguousarray(win_k, dtype=np.float32)).to(
            self.device, torch.bfloat16)
        self.winV[:, :, o:o + n] = torch.from_numpy(np.ascontiguousarray(win_v, dtype=np.float32)).to(
            self.device, torch.bfloat16)

    def set_queries(self, q: np.ndarray) -> None:
        """Queries [batch][Hq][D] of the loop step about to run."""
        self.q.copy_(torch.from_numpy(np.ascontiguousarray(q, dtype=np.float32)).to(self.device, self.q.dtype))

    # ------------------------------------------------------------ compute
    def decode(self, loop_step: int, softmax_scale: float | None = None, stream=None, new_k=None,
               new_v=None) -> None:
        """Decode attention at loop_step.  new_k/new_v ([batch][H][D] bf16
        device tensors) are the current token's K and V at this step: the
        kernel uses them and stores them in the token's window slot."""
        scale = self.D ** -0.5 if softmax_scale is None else softmax_scale
        layout = self.layout if new_k is None else self._make_layout(new_k, new_v)
        L.loopvq_decode_attn(self.desc, self.cbK, self.cbV, layout, self.idxK, self.idxV, self.winK,
                             self.winV, self.q, loop_step, scale, self.out, self.lse, self.workspace, stream)

    def device_status(self):
        return L.loopvq_read_device_status(self.workspace)

    def clear_status(self) -> None:
        L.loopvq_clear_device_status(self.workspace)

    def unpack_codes(self, r: int, kind: int) -> np.ndarray:
        n = self.splits[r][1]
        out = torch.empty((self.NB, self.H, n, self.J), dtype=torch.uint8, device=self.device)
        if n:
            L.loopvq_index_pool_unpack(self.desc, kind, self.idxK if kind == L.LOOPVQ_KEYS else self.idxV,
                                       self.body_off[r], self.body_pool_tokens, n, out)
        return out.cpu().numpy()

    def algorithmic_bytes(self) -> int:
        """Bytes one decode launch must move: index rows (K and V) of every body
        token, bf16 K and V of every window token, the query and the fp32
        output, summed over requests and query heads' KV streams."""
        idx = sum(b for (_, b, _) in self.splits) * self.H * 2 * self.J
        win = sum(s + r for (s, _, r) in self.splits) * self.H * 2 * self.D * 2
        qo = self.batch * self.Hq * self.D * (self.q.element_size() + self.out.element_size())
        return idx + win + qo


class PagedCache:
    """Incremental serving cache of one layer (K and V) for a batch of requests.

    LoopVQ project page, "Serving in SGLang": a new token's keys and values
    enter the cache in bf16; the ``n_sink`` sink tokens and the recent window
    are kept in bf16; for each ``page`` new tokens the page leaving the recent
    window is coded; decode reads the coded body from the indices.  Here the body lives in fixed-size pages
    of the index pools (``body_page_tokens`` tokens each, taken from a free
    list, listed per request in a page table) and the recent tokens in a ring
    of ``n_recent + page`` slots per request, so nothing is ever moved.

    Per generated token: ``begin_token(r)`` advances request r's length and,
    when its body grows, encodes the page leaving the recent window (one
    ``loopvq_encode`` per K and V, straight from the ring); then, for each
    loop step t, ``decode(t, new_k, new_v)`` attends with the new token's K/V
    written into its ring slot by the decode kernel itself.
    """

    def __init__(self, *, n_loop, tc, n_heads_kv, head_dim, group_elems, batch, max_ctx_len, n_sink=64,
                 n_recent=256, page=8, body_page_tokens=256, n_codes=256, n_heads_q=None,
                 cb_dtype=torch.bfloat16, q_dtype=torch.bfloat16, out_dtype=torch.float32, device="cuda",
                 spare_pages=0):
        if body_page_tokens % 32 or body_page_tokens % page:
            raise ValueError("body_page_tokens must be a multiple of 32 and of page")
        self.device = torch.device(device)
        self.T, self.Tc, self.H, self.D, self.G = n_loop, tc, n_heads_kv, head_dim, group_elems
        self.Hq = n_heads_q or n_heads_kv
        self.W = group_elems // tc
        self.J = head_dim // self.W
        self.NB = n_loop // tc
        self.n_sink, self.n_recent, self.page = n_sink, n_recent, page
        self.bpt = body_page_tokens
        self.ring = n_recent + page
        self.batch = batch
        self.max_ctx_len = max_ctx_len
        self.cb_dtype = cb_dtype
        self.desc = L.make_desc(n_loop, tc, n_heads_kv, head_dim, group_elems, n_codes, self.Hq,
                                L.LOOPVQ_BF16 if cb_dtype == torch.bfloat16 else L.LOOPVQ_F32)
        max_body = L.loopvq_ctx_split(max_ctx_len, n_sink, n_recent, page)[1]
        self.max_pages = max(1, -(-max_body // self.bpt))
        self.n_phys = batch * self.max_pages + spare_pages
        self.body_pool_tokens = self.n_phys * self.bpt
        self.win_stride = n_sink + self.ring
        self.win_pool_tokens = batch * self.win_stride
        dev = self.device
        pool_bytes = L.loopvq_index_pool_bytes(self.desc, self.body_pool_tokens)
        self.idxK = torch.zeros(pool_bytes, dtype=torch.uint8, device=dev)
        self.idxV = torch.zeros(pool_bytes, dtype=torch.uint8, device=dev)
        self.winK = torch.zeros((self.T, self.H, self.win_pool_tokens, self.D), dtype=torch.bfloat16, device=dev)
        self.winV = torch.zeros_like(self.winK)
        pb = L.loopvq_codebook_packed_bytes(self.desc)
        self.cbK = torch.zeros(pb, dtype=torch.uint8, device=dev)
        self.cbV = torch.zeros(pb, dtype=torch.uint8, device=dev)
        self.q = torch.zeros((batch, self.Hq, self.D), dtype=q_dtype, device=dev)
        self.out = torch.zeros((batch, self.Hq, self.D), dtype=out_dtype, device=dev)
        self.lse = torch.zeros((batch, self.Hq), dtype=torch.float32, device=dev)
        # host state
        self.ctx = [0] * batch
        self.head = [0] * batch
        self.pages = [[] for _ in range(batch)]
        self.free = list(range(self.n_phys))[::-1]
        # device copies of the host state
        self.ctx_dev = torch.zeros(batch, dtype=torch.int32, device=dev)
        self.head_dev = torch.zeros(batch, dtype=torch.int32, device=dev)
        self.pages_dev = torch.full((batch, self.max_pages), -1, dtype=torch.int32, device=dev)
        self.win_off_dev = torch.arange(batch, dtype=torch.int64, device=dev) * self.win_stride
        self.body_off_dev = torch.zeros(batch, dtype=torch.int64, device=dev)
        self._flags = L.LOOPVQ_LAYOUT_PAGED_BODY | L.LOOPVQ_LAYOUT_RING_WINDOW
        ws = L.loopvq_decode_workspace_bytes(self.desc, self._layout(None, None))
        if ws == 0:
            raise ValueError("invalid cache layout")
        self.workspace = torch.zeros(_round_up(ws, 256), dtype=torch.uint8, device=dev)

    def _layout(self, new_k, new_v):
        return L.make_layout(self.batch, self.n_sink, self.n_recent, self.page, self.max_ctx_len, self.ctx_dev,
                             self.body_off_dev, self.win_off_dev, self.body_pool_tokens, self.win_pool_tokens,
                             self._flags, self.pages_dev, self.bpt, self.max_pages, self.head_dev, self.ring,
                             new_k, new_v)

    def _sync_state(self, r):
        self.ctx_dev[r] = self.ctx[r]
        self.head_dev[r] = self.head[r]
        row = self.pages[r] + [-1] * (self.max_pages - len(self.pages[r]))
        self.pages_dev[r].copy_(torch.tensor(row, dtype=torch.int32))

    def split(self, r):
        """(sink, body, recent) of request r's current length."""
        return L.loopvq_ctx_split(self.ctx[r], self.n_sink, self.n_recent, self.page)

    # -------------------------------------------------------------- setup
    def set_codebooks(self, cb_k, cb_v) -> None:
        """Canonical codebooks [NB][H][J][C][Tc][W] (host arrays) -> packed."""
        for src, dst in ((cb_k, self.cbK), (cb_v, self.cbV)):
            t = torch.from_numpy(np.ascontiguousarray(src, dtype=np.float32)).to(self.cb_dtype).to(self.device)
            L.loopvq_codebook_pack(self.desc, t, dst)
        torch.cuda.current_stream().synchronize()

    def _slot_row(self, r, i):
        """Window-pool row of window token i of request r (sink, then ring)."""
        s = self.split(r)[0]
        base = r * self.win_stride
        return base + i if i < s else base + self.n_sink + (self.head[r] + i - s) % self.ring

    def _body_pos(self, r, p):
        """Index-pool position of body token p of request r (allocating its page)."""
        pi = p // self.bpt
        while len(self.pages[r]) <= pi:
            if not self.free:
                raise RuntimeError("index pool out of pages")
            self.pages[r].append(self.free.pop())
        return self.pages[r][pi] * self.bpt + p % self.bpt

    def prefill(self, r, K, V) -> None:
        """Prompt keys and values [T][N][H][D] (torch, any device, any float
        dtype): the window tokens are stored in bf16, the body is encoded into
        pages.  N is the request's new length."""
        N = K.shape[1]
        self.ctx[r], self.head[r] = N, 0
        s, body, rec = self.split(r)
        kb = K.to(self.device, torch.bfloat16)
        vb = V.to(self.device, torch.bfloat16)
        for i in list(range(s)) + list(range(s + body, N)):
            row = self._slot_row(r, i if i < s else i - body)
            self.winK[:, :, row] = kb[:, i]
            self.winV[:, :, row] = vb[:, i]
        H, D = self.H, self.D
        p = 0
        while p < body:
            n = min(body - p, self.bpt - p % self.bpt)
            pos = self._body_pos(r, p)
            for kind, x, pool in ((L.LOOPVQ_KEYS, kb, self.idxK), (L.LOOPVQ_VALUES, vb, self.idxV)):
                xs = x[:, s + p:s + p + n]
                L.loopvq_encode(self.desc, self.cbK if kind == L.LOOPVQ_KEYS else self.cbV, kind, xs, n,
                                xs.stride(0), xs.stride(1), xs.stride(2), pool, pos, self.body_pool_tokens)
            p += n
        self._sync_state(r)

    # -------------------------------------------------------------- per token
    def begin_token(self, r) -> None:
        """Request r grows by one token.  When its body grows, the oldest
        recent page is encoded from the ring into the body pages first."""
        s0, body0, rec0 = self.split(r)
        self.ctx[r] += 1
        s1, body1, rec1 = self.split(r)
        grown = body1 - body0
        if grown:
            if grown != self.page or self.head[r] % self.page:
                raise RuntimeError("unexpected window transition")
            pos = self._body_pos(r, body0)
            base = r * self.win_stride + self.n_sink + self.head[r]
            P = self.win_pool_tokens
            for kind, win, pool, cb in ((L.LOOPVQ_KEYS, self.winK, self.idxK, self.cbK),
                                        (L.LOOPVQ_VALUES, self.winV, self.idxV, self.cbV)):
                view = win[:, :, base:base + self.page]
                L.loopvq_encode(self.desc, cb, kind, view, self.page, self.H * P * self.D, self.D, P * self.D,
                                pool, pos, self.body_pool_tokens)
            self.head[r] = (self.head[r] + self.page) % self.ring
        self._sync_state(r)

    def set_queries(self, q) -> None:
        """Queries [batch][Hq][D] (host array or torch tensor) of the loop step about to run."""
        t = q if isinstance(q, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(q, dtype=np.float32))
        self.q.copy_(t.to(self.device, self.q.dtype))

    def decode(self, loop_step, new_k=None, new_v=None, softmax_scale=None, stream=None) -> None:
        """Decode attention at loop_step for every request.  new_k/new_v are
        the current token's bf16 K and V at this step ([batch][H][D] device
        tensors): the kernel stores them in the token's ring slot and uses
        them.  Without them the slot must already hold the token."""
        scale = self.D ** -0.5 if softmax_scale is None else softmax_scale
        layout = self._layout(new_k, new_v)
        L.loopvq_decode_attn(self.desc, self.cbK, self.cbV, layout, self.idxK, self.idxV, self.winK, self.winV,
                             self.q, loop_step, scale, self.out, self.lse, self.workspace, stream)

    def device_status(self):
        return L.loopvq_read_device_status(self.workspace)

    def body_codes(self, r, kind) -> np.ndarray:
        """Body codes of request r in logical order, [NB][H][n_body][J]."""
        body = self.split(r)[1]
        out = np.zeros((self.NB, self.H, body, self.J), dtype=np.uint8)
        pool = self.idxK if kind == L.LOOPVQ_KEYS else self.idxV
        p = 0
        while p < body:
            n = min(body - p, self.bpt - p % self.bpt)
            pos = self.pages[r][p // self.bpt] * self.bpt + p % self.bpt
            t = torch.empty((self.NB, self.H, n, self.J), dtype=torch.uint8, device=self.device)
            L.loopvq_index_pool_unpack(self.desc, kind, pool, pos, self.body_pool_tokens, n, t)
            out[:, :, p:p + n] = t.cpu().numpy()
            p += n
        return out
