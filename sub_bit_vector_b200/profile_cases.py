"""Small, self-contained launches of each kernel, for profilers.

``python -m sub_bit_vector_b200.profile_cases <case>`` runs one case on
``cuda:0`` and prints its device status; every input is seeded and drawn on
the device.  The cases are sized so that a profiler replaying one launch
holds well under 2 GB on the device:

- ``decode``  : 32768-token context, batch 1, 16 KV heads x 128, 4 loop
                steps, Tc = 4, G = 16 (0.5 bit): one decode launch per loop
                step (4 launches).
- ``decode-q``: the same at G = 32 (0.25 bit).
- ``decode-gqa``: the same context with 8 KV heads and 16 query heads
                (GQA ratio 2), 4 launches.
- ``decode-steps``: the ``decode`` case as one launch of all 4 loop steps
                (loopvq_decode_attn_steps), 2 launches.
- ``encode``  : loop-axis encode of a [4][32768][16][128] bf16 tensor at
                Tc = 4, G = 16 (tensor-core kernel), 2 launches.
- ``encode-f32``: the same tensor in fp32 (CUDA-core kernel), 2 launches.
- ``residual``: adjacent-loop residual 4-bit coding of [4][32768][16][128]
                bf16 keys and values, then one decode per loop step (4
                launches of the decode kernel).
- ``page``    : encode of one 8-token page out of a [4][16][320][128] bf16
                window pool (few-token kernel), 4 launches.
"""
import sys

import torch

from . import cache, loopvq as L, synth


def _decode(G):
    c = cache.DecodeCache(n_loop=4, tc=4, n_heads_kv=16, head_dim=128, group_elems=G, ctx_lens=[32768])
    W = G // 4
    J = 128 // W
    cb = synth.uniform_codebook(1, 1, 16, J, 256, 4, W)
    c.set_codebooks(cb, cb)
    c.idxK.copy_(synth.device_codes(2, c.idxK.numel()))
    c.idxV.copy_(synth.device_codes(3, c.idxV.numel()))
    c.winK.normal_()
    c.winV.normal_()
    c.q.normal_()
    for t in range(4):
        c.decode(t)
    torch.cuda.synchronize()
    print("decode status", c.device_status(), "algorithmic bytes per launch", c.algorithmic_bytes())


def _decode_gqa():
    c = cache.DecodeCache(n_loop=4, tc=4, n_heads_kv=8, head_dim=128, group_elems=16, ctx_lens=[32768], n_heads_q=16)
    cb = synth.uniform_codebook(1, 1, 8, 32, 256, 4, 4)
    c.set_codebooks(cb, cb)
    c.idxK.copy_(synth.device_codes(2, c.idxK.numel()))
    c.idxV.copy_(synth.device_codes(3, c.idxV.numel()))
    c.winK.normal_()
    c.winV.normal_()
    c.q.normal_()
    for t in range(4):
        c.decode(t)
    torch.cuda.synchronize()
    print("decode-gqa status", c.device_status(), "algorithmic bytes per launch", c.algorithmic_bytes())


def _decode_steps():
    c = cache.DecodeCache(n_loop=4, tc=4, n_heads_kv=16, head_dim=128, group_elems=16, ctx_lens=[32768])
    cb = synth.uniform_codebook(1, 1, 16, 32, 256, 4, 4)
    c.set_codebooks(cb, cb)
    c.idxK.copy_(synth.device_codes(2, c.idxK.numel()))
    c.idxV.copy_(synth.device_codes(3, c.idxV.numel()))
    c.winK.normal_()
    c.winV.normal_()
    q = synth.device_normal(4, (4, 1, 16, 128)).to(torch.bfloat16)
    out = torch.zeros((4, 1, 16, 128), dtype=torch.float32, device="cuda")
    lse = torch.zeros((4, 1, 16), dtype=torch.float32, device="cuda")
    ws = torch.zeros(L.loopvq_decode_steps_workspace_bytes(c.desc, c.layout, 4), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        L.loopvq_decode_attn_steps(c.desc, c.cbK, c.cbV, c.layout, c.idxK, c.idxV, c.winK, c.winV, q, 0, 4,
                                   128 ** -0.5, out, lse, ws)
    torch.cuda.synchronize()
    print("decode-steps status", L.loopvq_read_device_status(ws))


def _encode(dtype):
    T, N, H, D, tc, G = 4, 32768, 16, 128, 4, 16
    x = synth.device_normal(1, (T, N, H, D)).to(dtype)
    desc = L.make_desc(T, tc, H, D, G)
    W = G // tc
    J = D // W
    cb = synth.device_normal(2, (T // tc, H, J, 256, tc, W))
    packed = torch.zeros(L.loopvq_codebook_packed_bytes(desc), dtype=torch.uint8, device="cuda")
    L.loopvq_codebook_pack(desc, cb, packed)
    pool = torch.zeros(L.loopvq_index_pool_bytes(desc, N), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        L.loopvq_encode(desc, packed, L.LOOPVQ_KEYS, x, N, N * H * D, H * D, D, pool, 0, N)
    torch.cuda.synchronize()
    print("encode faults", L.loopvq_read_encode_faults())


def _residual():
    T, N, H, D = 4, 32768, 16, 128
    desc = L.make_residual_desc(T, H, D)
    bufs = []
    for kind in (L.LOOPVQ_KEYS, L.LOOPVQ_VALUES):
        codes = torch.zeros(L.loopvq_residual_codes_bytes(desc, N), dtype=torch.uint8, device="cuda")
        params = torch.zeros(L.loopvq_residual_params_bytes(desc, kind, N) // 2, dtype=torch.float16, device="cuda")
        x = synth.device_normal(20 + kind, (T, N, H, D))
        L.loopvq_residual_encode(desc, kind, x, N, N * H * D, H * D, D, codes, params, 0, N)
        bufs.append((codes, params))
        del x
    ctx = torch.tensor([N], dtype=torch.int32, device="cuda")
    off = torch.zeros(1, dtype=torch.int64, device="cuda")
    q = synth.device_normal(30, (1, H, D))
    out = torch.zeros((1, H, D), dtype=torch.float32, device="cuda")
    ws = torch.zeros(L.loopvq_residual_decode_workspace_bytes(desc, 1, N), dtype=torch.uint8, device="cuda")
    for t in range(T):
        L.loopvq_residual_decode_attn(desc, 1, N, ctx, off, N, bufs[0][0], bufs[0][1], bufs[1][0], bufs[1][1], q, t,
                                      D ** -0.5, out, None, ws)
    torch.cuda.synchronize()
    print("residual decode status", L.loopvq_read_device_status(ws))


def _page():
    T, H, P, D, tc, G = 4, 16, 320, 128, 4, 16
    win = synth.device_normal(3, (T, H, P, D))
    desc = L.make_desc(T, tc, H, D, G)
    W = G // tc
    J = D // W
    cb = synth.device_normal(2, (T // tc, H, J, 256, tc, W))
    packed = torch.zeros(L.loopvq_codebook_packed_bytes(desc), dtype=torch.uint8, device="cuda")
    L.loopvq_codebook_pack(desc, cb, packed)
    pool = torch.zeros(L.loopvq_index_pool_bytes(desc, 32), dtype=torch.uint8, device="cuda")
    view = win[:, :, 64:72]
    for _ in range(4):
        L.loopvq_encode(desc, packed, L.LOOPVQ_KEYS, view, 8, H * P * D, D, P * D, pool, 0, 32)
    torch.cuda.synchronize()
    print("page encode faults", L.loopvq_read_encode_faults())


CASES = {
    "decode": lambda: _decode(16),
    "decode-q": lambda: _decode(32),
    "decode-gqa": _decode_gqa,
    "decode-steps": _decode_steps,
    "encode": lambda: _encode(torch.bfloat16),
    "encode-f32": lambda: _encode(torch.float32),
    "page": _page,
    "residual": _residual,
}


def main(argv):
    if len(argv) != 1 or argv[0] not in CASES:
        print("usage: python -m sub_bit_vector_b200.profile_cases {" + ",".join(CASES) + "}")
        return 2
    CASES[argv[0]]()
    return 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
