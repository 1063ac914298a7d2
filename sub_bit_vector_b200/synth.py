"""Seeded synthetic inputs shared by the tests, the bench and the smoke run.

This module draws random numbers and arranges them in the library's input
shapes.  It holds none of the method's arithmetic (no distances, no argmin,
no dequantization, no softmax): both the CUDA path and the CPU oracle take
its outputs as plain inputs.  Every generator takes an explicit seed and uses
NumPy's PCG64.

Workload shapes follow the LoopVQ pages: Ouro-1.4B/2.6B layers with 16 KV
heads of head_dim 128 and 4 loop steps (the Ouro "R4" setting), 256-entry
codebooks at 0.5 bit (16-element sub-vectors) or 0.25 bit (32-element),
a bf16 window of the first 64 and the most recent 256 tokens, and contexts
from 4K to 64K tokens.  Keys and values of successive loop steps are strongly
correlated (project page, "Method", loop-axis redundancy figure); that is
modelled as an AR(1) process across loop steps with correlation rho.
"""
from __future__ import annotations

import numpy as np

try:  # torch is only used for exact bf16 round-to-nearest-even
    import torch
except Exception:  # pragma: no cover
    torch = None

__all__ = [
    "round_bf16",
    "tiny_kv",
    "loop_correlated",
    "codebook_from_rows",
    "random_codes",
    "ragged_context_lengths",
    "queries",
    "uniform_codebook",
    "key_outlier_channels",
    "decode_request",
    "device_codes",
    "device_normal",
]


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp32/fp64 values to bf16 (nearest-even) and return them as fp32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if torch is not None:
        return torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    u = x.view(np.uint32).astype(np.uint64)
    rounded = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return rounded.astype(np.uint32).view(np.float32)


def tiny_kv(seed: int = 0, n_loop: int = 4, n_tokens: int = 512, n_heads: int = 1,
            head_dim: int = 64, noise: float = 0.3):
    """The small fp32 case: per token a base vector ~N(0,1) shared by all
    loop steps plus independent N(0, noise^2) per loop step, for K and V.

    Returns ``(K, V)`` each ``[T][N][H][D]`` float32.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    out = []
    for _ in range(2):
        base = rng.standard_normal((n_tokens, n_heads, head_dim))
        eps = rng.standard_normal((n_loop, n_tokens, n_heads, head_dim))
        out.append((base[None] + noise * eps).astype(np.float32))
    return out[0], out[1]


def loop_correlated(seed: int, n_loop: int, n_tokens: int, n_heads: int, head_dim: int,
                    rho: float = 0.9, n_outlier: int = 0, outlier_scale: float = 8.0,
                    outlier_dof: float = 4.0, bf16: bool = True,
                    outlier_channels: np.ndarray | None = None) -> np.ndarray:
    """Ouro-shaped cache tensor ``[T][N][H][D]`` with loop-step correlation rho.

    x_0 ~ N(0,1); x_t = rho * x_{t-1} + sqrt(1 - rho^2) * e_t, so every step
    has unit variance and adjacent steps correlate by rho.  For keys,
    ``n_outlier`` channels per head start from a Student-t draw and are scaled
    by ``outlier_scale`` at every step (heavy-tailed key outlier channels).
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    x = np.empty((n_loop, n_tokens, n_heads, head_dim), dtype=np.float32)
    z0 = rng.standard_normal((n_tokens, n_heads, head_dim)).astype(np.float32)
    chans = None
    if outlier_channels is not None:
        chans = np.asarray(outlier_channels)
        n_outlier = chans.shape[1]
    elif n_outlier > 0:
        chans = np.stack([rng.choice(head_dim, size=n_outlier, replace=False) for _ in range(n_heads)])
    if chans is not None:
        t0 = rng.standard_t(outlier_dof, size=(n_tokens, n_heads, n_outlier)).astype(np.float32)
        for h in range(n_heads):
            z0[:, h, chans[h]] = t0[:, h, :]
    x[0] = z0
    a = np.float32(rho)
    b = np.float32(np.sqrt(1.0 - rho * rho))
    for t in range(1, n_loop):
        x[t] = a * x[t - 1] + b * rng.standard_normal((n_tokens, n_heads, head_dim)).astype(np.float32)
    if chans is not None:
        for h in range(n_heads):
            x[:, :, h, chans[h]] *= np.float32(outlier_scale)
    return round_bf16(x) if bf16 else x


def codebook_from_rows(X: np.ndarray, tc: int, group_elems: int, n_codes: int, seed: int,
                       token_lo: int = 0, token_hi: int | None = None) -> np.ndarray:
    """Synthetic codebook made of data rows, in the library's canonical layout
    ``[NB][H][J][C][Tc][W]``.

    For every (Tc-block b, head h, slot j) draw ``n_codes`` distinct token
    positions in ``[token_lo, token_hi)`` by a seeded permutation and take, as
    codeword c, the cache values of token rows[c] at channels j*W..j*W+W-1 of
    loop steps b*Tc..b*Tc+Tc-1.  This is the stand-in for the pages'
    fine-tuned codebooks, which need model weights and data.
    """
    T, N, H, D = X.shape
    W = group_elems // tc
    J = D // W
    NB = T // tc
    hi = N if token_hi is None else token_hi
    rng = np.random.Generator(np.random.PCG64(seed))
    cb = np.empty((NB, H, J, n_codes, tc, W), dtype=X.dtype)
    for b in range(NB):
        for h in range(H):
            for j in range(J):
                rows = token_lo + rng.permutation(hi - token_lo)[:n_codes]
                for t in range(tc):
                    cb[b, h, j, :, t, :] = X[b * tc + t, rows, h, j * W:(j + 1) * W]
    return cb


def key_outlier_channels(seed: int, n_heads: int, head_dim: int, n_outlier: int = 4) -> np.ndarray:
    """Seeded choice of ``n_outlier`` heavy-tailed key channels per head: [H][n]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return np.stack([rng.choice(head_dim, size=n_outlier, replace=False) for _ in range(n_heads)])


def uniform_codebook(seed: int, n_blocks: int, n_heads: int, n_slots: int, n_codes: int,
                     tc: int, w: int, bf16: bool = True, outlier_channels: np.ndarray | None = None,
                     outlier_scale: float = 8.0) -> np.ndarray:
    """Random N(0, 1) codebook ``[NB][H][J][C][Tc][W]`` for cases whose body
    codes are drawn directly (too large to encode on the host).  Channels
    listed in ``outlier_channels`` ([H][n], channel = j*W + w) are scaled by
    ``outlier_scale``, like the key outlier channels of the cache."""
    rng = np.random.Generator(np.random.PCG64(seed))
    cb = rng.standard_normal((n_blocks, n_heads, n_slots, n_codes, tc, w)).astype(np.float32)
    if outlier_channels is not None:
        for h in range(n_heads):
            for ch in np.asarray(outlier_channels)[h]:
                cb[:, h, ch // w, :, :, ch % w] *= np.float32(outlier_scale)
    return round_bf16(cb) if bf16 else cb


def decode_request(seed: int, n_loop: int, n_heads: int, head_dim: int, n_slots: int, n_blocks: int,
                   n_win: int, n_body: int, n_codes: int = 256, rho: float = 0.9,
                   outlier_channels: np.ndarray | None = None):
    """One request of a decode batch: bf16 window keys/values
    ``[T][H][n_win][D]`` (loop-correlated, keys with outlier channels) and
    body codes ``[NB][H][n_body][J]`` uint8 (uniform)."""
    wk = loop_correlated(seed, n_loop, n_win, n_heads, head_dim, rho=rho, outlier_channels=outlier_channels)
    wv = loop_correlated(seed + 7919, n_loop, n_win, n_heads, head_dim, rho=rho)
    ck = random_codes(seed + 104729, n_blocks, n_heads, n_body, n_slots, n_codes)
    cv = random_codes(seed + 1299709, n_blocks, n_heads, n_body, n_slots, n_codes)
    return (np.ascontiguousarray(wk.transpose(0, 2, 1, 3)), np.ascontiguousarray(wv.transpose(0, 2, 1, 3)), ck, cv)


def random_codes(seed: int, n_blocks: int, n_heads: int, n_tokens: int, n_slots: int,
                 n_codes: int = 256) -> np.ndarray:
    """Uniform random codes ``[NB][H][N][J]`` uint8 (stand-in for encoded data)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(0, n_codes, size=(n_blocks, n_heads, n_tokens, n_slots), dtype=np.uint8)


def ragged_context_lengths(batch: int, prompt: int = 2048, gen_lo: int = 4096,
                           gen_hi: int = 16384, seed_base: int = 3000) -> np.ndarray:
    """Per-request context = prompt + generated length U{gen_lo..gen_hi},
    request r drawn from seed ``seed_base + r`` (batched serving decode)."""
    out = np.empty(batch, dtype=np.int64)
    for r in range(batch):
        rng = np.random.Generator(np.random.PCG64(seed_base + r))
        out[r] = prompt + int(rng.integers(gen_lo, gen_hi + 1))
    return out


def queries(seed: int, n_loop: int, batch: int, n_heads_q: int, head_dim: int,
            bf16: bool = True) -> np.ndarray:
    """One decode query per loop step: ``[T][batch][Hq][D]`` ~ N(0,1)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = rng.standard_normal((n_loop, batch, n_heads_q, head_dim)).astype(np.float32)
    return round_bf16(q) if bf16 else q


# --------------------------------------------------------------------------
# device-side draws for large benchmark inputs (torch's seeded CUDA RNG);
# these never feed the oracle
# --------------------------------------------------------------------------

def device_codes(seed: int, n: int, device="cuda"):
    """n uniform uint8 codes drawn on the device."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randint(0, 256, (n,), generator=g, dtype=torch.uint8, device=device)


def device_normal(seed: int, shape, dtype=None, device="cuda"):
    """N(0,1) values drawn on the device, rounded to ``dtype`` (bf16 default)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    return x.to(dtype or torch.bfloat16)
