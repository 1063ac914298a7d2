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
        # static_inputs: this cache's layout arrays, pools and codebooks are not
        # written by kernels that may still run when a decode starts
        self.layout = L.make_layout(self.batch, n_sink, n_recent, page, self.max_ctx_len, self.ctx_dev,
                                    self.body_off_dev, self.win_off_dev, self.body_pool_tokens,
                                    self.win_pool_tokens,
                                    L.LOOPVQ_LAYOUT_STATIC_INPUTS if static_inputs else 0)
        ws = L.loopvq_decode_workspace_bytes(self.desc, self.layout)
        if ws == 0:
            raise ValueError("invalid cache layout")
        self.workspace = torch.zeros(_round_up(ws, 256), dtype=torch.uint8, device=dev)

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
    def decode(self, loop_step: int, softmax_scale: float | None = None, stream=None) -> None:
        scale = self.D ** -0.5 if softmax_scale is None else softmax_scale
        L.loopvq_decode_attn(self.desc, self.cbK, self.cbV, self.layout, self.idxK, self.idxV, self.winK,
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
