"""LoopVQ oracle: plain fp64 NumPy, CPU only.  TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` and
``--impl reference`` legs of ``bench.py`` may import this module.  It shares
no code with the CUDA library.

Sources (all from the LoopVQ web pages):

* LoopVQ project page (mscheong01.github.io/loopvq), section "Method",
  figure "Overview of LoopVQ": a code covers G/Tc channels of each of Tc
  loop steps; one index serves all of them; at inference each loop step reads
  the shared index through its own slice of the codebook.
* Same page, "Component 1 -- Loop-axis vector quantization": one index
  covers channels of several *consecutive* loop steps.
* Same page, "Serving in SGLang" -- "Write in bf16", "Encode in pages",
  "Attend from indices": a new token's K/V enter the cache in bf16; the sink
  tokens and the recent window are kept in bf16 for every loop step; for
  each 8 new tokens, the page leaving the recent window is coded; at step t
  the attention reads the coded body through slice B_t and combines it with
  the bf16 part.
* Same page, "Results -- Long-context retrieval": n_sink = 64 and
  n_recent = 256.
* Same page, "Highlights" and "Efficiency": 0.5 / 0.25 bit per element is
  32x / 64x compression; bytes read per token and loop step are 8x / 16x
  fewer than the bf16 keys and values.

Readings taken where the pages are silent (each is stated where it is used):
one codebook per (Tc-block, KV head, slot); slots are contiguous channel
groups; a codeword is stored step-major ``[Tc][W]``; Tc-blocks are the
consecutive steps ``b*Tc .. b*Tc+Tc-1``; plain unweighted L2; ties go to the
lowest index; the recent window holds ``n_recent + ((ctx - n_sink - n_recent)
mod page)`` tokens so that the body is whole pages.

Array conventions (all C-order):

* ``X``        keys or values of one layer, ``[T][N][H][D]``
* ``codebook`` ``[NB][H][J][C][Tc][W]`` with NB = T/Tc, W = G/Tc, J = D/W
* ``idx``      ``[NB][H][N][J]`` integer codes

Parity: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, hand-worked fixtures under ``tests/golden/``, brute-force and
library cross-checks, invariants).  No function is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "geometry",
    "bits_per_element",
    "compression_vs_bf16",
    "bytes_per_token_step",
    "form_subvectors",
    "subvector_distances",
    "encode",
    "dequantize",
    "window_split",
    "attention",
    "decode_attention",
    "dense_decode_attention",
    "reconstruction_mse",
    "kmeans_update",
    "kmeans",
    "distortion",
    "attention_mse_codebook_grad",
    "quantize4_group",
    "dequantize4",
    "residual_encode",
    "residual_reconstruct",
    "residual_decode_attention",
    "residual_bits_per_element",
]


# --------------------------------------------------------------------------
# geometry and accounting
# --------------------------------------------------------------------------

def geometry(n_loop: int, tc: int, head_dim: int, group_elems: int, n_codes: int = 256) -> dict:
    """Derived sizes of one loop-axis VQ configuration.

    Project page, "Overview of LoopVQ": a code spans G/Tc channels of each of
    Tc loop steps.  So W = G/Tc channels per step per code, J = D/W code slots
    per head, and NB = T/Tc groups of consecutive loop steps.
    """
    if tc <= 0 or n_loop % tc:
        raise ValueError("n_loop must be a multiple of tc")
    if group_elems % tc:
        raise ValueError("group_elems must be a multiple of tc")
    w = group_elems // tc
    if head_dim % w:
        raise ValueError("head_dim must be a multiple of group_elems / tc")
    return {
        "T": n_loop,
        "Tc": tc,
        "NB": n_loop // tc,
        "G": group_elems,
        "W": w,
        "D": head_dim,
        "J": head_dim // w,
        "C": n_codes,
        "bits": bits_per_element(n_codes, group_elems),
    }


def bits_per_element(n_codes: int, group_elems: int) -> float:
    """An index into n_codes codewords stands for G elements: log2(C)/G bits.

    Project page, "Overview of LoopVQ" (one index serves G elements) and
    "Highlights" (0.5 and 0.25 bit per element).  Codebooks and the bf16 window
    are not counted, which is how the pages' 32x / 64x figures come out.
    """
    return math.log2(n_codes) / group_elems


def compression_vs_bf16(n_codes: int, group_elems: int) -> float:
    """Ratio of bf16's 16 bits to the quantized bits per element.

    Project page, "Highlights": 32-64x KV cache compression at 0.5 and 0.25 bit.
    """
    return 16.0 / bits_per_element(n_codes, group_elems)


def bytes_per_token_step(head_dim: int, group_elems: int, tc: int, n_codes: int = 256) -> dict:
    """Bytes a decode step reads per (token, KV head, loop step).

    bf16 keys and values: 2 tensors x D elements x 2 bytes.  Quantized: one
    index byte per slot for K and one for V, the index row being read once per
    loop step (project page, "Serving in SGLang": each loop step reads the
    shared index row through its own slice).  Project page, "Efficiency":
    8x fewer bytes at 0.5 bit, 16x at 0.25 bit.
    """
    w = group_elems // tc
    j = head_dim // w
    index_bytes_per_code = math.ceil(math.log2(n_codes) / 8)
    bf16 = 2 * head_dim * 2
    vq = 2 * j * index_bytes_per_code
    return {"bf16": bf16, "vq": vq, "ratio": bf16 / vq}


# --------------------------------------------------------------------------
# encode
# --------------------------------------------------------------------------

def form_subvectors(X: np.ndarray, block: int, tc: int, w: int) -> np.ndarray:
    """Loop-axis sub-vectors of Tc-block ``block``: returns ``[N][H][J][Tc*W]``.

    Project page, "Overview of LoopVQ" and "Component 1": the sub-vector of
    slot j gathers channels j*W .. j*W+W-1 of each of the Tc consecutive loop
    steps block*Tc .. block*Tc+Tc-1; element (t, w) sits at position t*W + w.
    """
    T, N, H, D = X.shape
    J = D // w
    out = np.empty((N, H, J, tc * w), dtype=np.float64)
    for t in range(tc):
        step = np.asarray(X[block * tc + t], dtype=np.float64)  # [N][H][D]
        for j in range(J):
            out[:, :, j, t * w:(t + 1) * w] = step[:, :, j * w:(j + 1) * w]
    return out


def subvector_distances(x: np.ndarray, codewords: np.ndarray) -> np.ndarray:
    """Squared L2 distance of every sub-vector to every codeword, by definition.

    ``x`` is ``[n][G]``, ``codewords`` ``[C][G]``; returns ``[n][C]`` with
    d[i, c] = sum_g (x[i, g] - codewords[c, g])**2, computed from the
    differences (no ||x||^2 - 2 x.c + ||c||^2 expansion).
    """
    x = np.asarray(x, dtype=np.float64)
    cw = np.asarray(codewords, dtype=np.float64)
    diff = x[:, None, :] - cw[None, :, :]
    return np.sum(diff * diff, axis=2)


def encode(X: np.ndarray, codebook: np.ndarray, tc: int, chunk: int = 1024):
    """Brute-force nearest-codeword encoding, ties to the lowest index.

    Project page, "Component 1": each loop-axis sub-vector is replaced by the
    index of a codeword.  The pages fix no distance; the plain reading is the
    nearest codeword in unweighted squared L2.  ``np.argmin`` returns the
    first minimum, i.e. the lowest index on ties.

    Returns ``(idx, d_best, d_second)``, each ``[NB][H][N][J]``; ``d_second``
    is the second-smallest distance (equal to ``d_best`` on an exact tie) and
    serves the near-tie tolerance of the parity tests.
    """
    T, N, H, D = X.shape
    NB, H2, J, C, tc2, w = codebook.shape
    if tc2 != tc or NB * tc != T or H2 != H or J * w != D:
        raise ValueError("codebook shape does not match X")
    cb = np.asarray(codebook, dtype=np.float64).reshape(NB, H, J, C, tc * w)
    idx = np.empty((NB, H, N, J), dtype=np.int64)
    d_best = np.empty((NB, H, N, J), dtype=np.float64)
    d_second = np.empty((NB, H, N, J), dtype=np.float64)
    for b in range(NB):
        sub = form_subvectors(X, b, tc, w)  # [N][H][J][G]
        for h in range(H):
            for j in range(J):
                for n0 in range(0, N, chunk):
                    n1 = min(N, n0 + chunk)
                    d = subvector_distances(sub[n0:n1, h, j], cb[b, h, j])
                    k = np.argmin(d, axis=1)
                    idx[b, h, n0:n1, j] = k
                    d_best[b, h, n0:n1, j] = d[np.arange(n1 - n0), k]
                    if C > 1:
                        d_second[b, h, n0:n1, j] = np.partition(d, 1, axis=1)[:, 1]
                    else:
                        d_second[b, h, n0:n1, j] = np.inf
    return idx, d_best, d_second


def dequantize(idx: np.ndarray, codebook: np.ndarray, loop_step: int, tc: int) -> np.ndarray:
    """Reconstruction seen by loop step t: ``[N][H][D]`` in fp64.

    Project page, "Overview of LoopVQ": each loop step reads the shared index
    through its own slice of the codebook.  Step t belongs to Tc-block
    b = t // Tc and reads slice t - b*Tc: channel j*W + w of token n is
    codebook[b][h][j][idx[b][h][n][j]][t - b*Tc][w].
    """
    NB, H, J, C, tc2, w = codebook.shape
    b, tt = divmod(loop_step, tc)
    N = idx.shape[2]
    out = np.empty((N, H, J * w), dtype=np.float64)
    cb = np.asarray(codebook, dtype=np.float64)
    for h in range(H):
        for j in range(J):
            codes = idx[b, h, :, j]
            if np.any(codes < 0) or np.any(codes >= C):
                raise ValueError("code out of range")
            out[:, h, j * w:(j + 1) * w] = cb[b, h, j, codes, tt, :]
    return out


# --------------------------------------------------------------------------
# decode attention
# --------------------------------------------------------------------------

def window_split(ctx_len: int, n_sink: int, n_recent: int, page: int):
    """Split a context of ``ctx_len`` tokens into (sink, body, recent) counts.

    Project page, "Serving in SGLang": the sink tokens and the recent window
    are kept in bf16 for every loop step, and for each 8 new tokens the page
    leaving the recent window is coded.  Read as: the recent window
    holds n_recent .. n_recent+page-1 tokens, so the encoded body is whole
    pages; a context no longer than n_sink + n_recent is all bf16.  The
    current token is counted in ``ctx_len`` and sits in the recent window.
    """
    if ctx_len < 0:
        raise ValueError("ctx_len must be >= 0")
    if ctx_len <= n_sink + n_recent:
        sink = min(ctx_len, n_sink)
        return sink, 0, ctx_len - sink
    extra = (ctx_len - n_sink - n_recent) % page if page > 0 else 0
    recent = n_recent + extra
    body = ctx_len - n_sink - recent
    return n_sink, body, recent


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float):
    """Naive softmax attention of one query: returns ``(o, lse)``.

    s_n = scale * q.k_n; o = sum_n exp(s_n - m) v_n / sum_n exp(s_n - m) with
    m = max_n s_n; lse = m + log(sum_n exp(s_n - m)) (natural log).
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], dtype=np.float64), -np.inf
    s = scale * (K @ q)
    m = np.max(s)
    p = np.exp(s - m)
    l = np.sum(p)
    o = (p @ V) / l
    return o, m + math.log(l)


def decode_attention(q, loop_step, tc, idx_k, idx_v, codebook_k, codebook_v,
                     win_k, win_v, scale):
    """Decode attention of one request at loop step t over window + body.

    Project page, "Serving in SGLang -- Attend from indices": body keys and
    values come from the shared indices through slice B_t of the K and V
    codebooks; the bf16 sink/recent window is used as stored; the two are
    merged into one softmax.

    q        ``[Hq][D]`` query of loop step t (any float dtype; used in fp64)
    idx_k/v  ``[NB][H][n_body][J]`` body codes of this request
    win_k/v  ``[H][n_win][D]`` bf16 window keys/values of loop step t
    returns  ``(o [Hq][D], lse [Hq])``; query head hq reads KV head
    hq // (Hq / H).
    """
    q = np.asarray(q, dtype=np.float64)
    Hq, D = q.shape
    H = codebook_k.shape[1]
    group = Hq // H
    Kb = dequantize(idx_k, codebook_k, loop_step, tc)  # [n_body][H][D]
    Vb = dequantize(idx_v, codebook_v, loop_step, tc)
    out = np.empty((Hq, D), dtype=np.float64)
    lse = np.empty(Hq, dtype=np.float64)
    for hq in range(Hq):
        h = hq // group
        K = np.concatenate([np.asarray(win_k[h], dtype=np.float64), Kb[:, h, :]], axis=0)
        V = np.concatenate([np.asarray(win_v[h], dtype=np.float64), Vb[:, h, :]], axis=0)
        out[hq], lse[hq] = attention(q[hq], K, V, scale)
    return out, lse


def dense_decode_attention(q, K, V, scale):
    """Plain decode attention over bf16 keys/values: the dense comparator.

    q ``[Hq][D]``, K/V ``[H][n][D]`` of one loop step; returns (o, lse).
    """
    q = np.asarray(q, dtype=np.float64)
    Hq = q.shape[0]
    H = K.shape[0]
    group = Hq // H
    out = np.empty(q.shape, dtype=np.float64)
    lse = np.empty(Hq, dtype=np.float64)
    for hq in range(Hq):
        out[hq], lse[hq] = attention(q[hq], K[hq // group], V[hq // group], scale)
    return out, lse


def reconstruction_mse(X: np.ndarray, idx: np.ndarray, codebook: np.ndarray, tc: int) -> float:
    """Mean squared error of the reconstruction over all loop steps and elements.

    Project page, "Method" figure on loop-axis redundancy: at the same bit
    width, a code spanning four loop steps reconstructs the cache with lower
    error than a code spanning one step.
    """
    T = X.shape[0]
    acc = 0.0
    count = 0
    for t in range(T):
        Xh = dequantize(idx, codebook, t, tc)
        diff = np.asarray(X[t], dtype=np.float64) - Xh
        acc += float(np.sum(diff * diff))
        count += diff.size
    return acc / count


# --------------------------------------------------------------------------
# codebook construction (Lloyd's k-means on the loop-axis sub-vectors)
# --------------------------------------------------------------------------
# The pages fine-tune codebooks against the full-precision model and do not
# say where the fine-tuning starts.  The plain data-driven start is Lloyd's
# k-means on the same loop-axis sub-vectors the encoder codes, seeded from
# data rows: alternate the nearest-codeword assignment (``encode``) with the
# update below.

def kmeans_update(X: np.ndarray, idx: np.ndarray, codebook: np.ndarray, tc: int):
    """One Lloyd update of every codebook, by definition.

    Codeword c of (block b, head h, slot j) becomes the mean of the
    sub-vectors (``form_subvectors``) of the tokens whose code ``idx[b][h][n][j]``
    is c; a codeword that no token uses keeps its value.  Returns
    ``(new_codebook, counts)``: the codebook in fp64, same layout
    ``[NB][H][J][C][Tc][W]``, and the member counts ``[NB][H][J][C]``.
    """
    NB, H, J, C, tc2, w = codebook.shape
    if tc2 != tc:
        raise ValueError("codebook Tc does not match")
    new = np.array(codebook, dtype=np.float64).reshape(NB, H, J, C, tc * w)
    counts = np.zeros((NB, H, J, C), dtype=np.int64)
    for b in range(NB):
        sub = form_subvectors(X, b, tc, w)  # [N][H][J][G]
        for h in range(H):
            for j in range(J):
                codes = np.asarray(idx[b, h, :, j], dtype=np.int64)
                for c in np.unique(codes):
                    members = sub[codes == c, h, j]
                    new[b, h, j, c] = members.sum(axis=0) / len(members)
                    counts[b, h, j, c] = len(members)
    return new.reshape(NB, H, J, C, tc, w), counts


def distortion(X: np.ndarray, idx: np.ndarray, codebook: np.ndarray, tc: int) -> float:
    """Sum over all sub-vectors of the squared distance to their codeword."""
    NB, H, J, C, tc2, w = codebook.shape
    cb = np.asarray(codebook, dtype=np.float64).reshape(NB, H, J, C, tc * w)
    total = 0.0
    for b in range(NB):
        sub = form_subvectors(X, b, tc, w)
        for h in range(H):
            for j in range(J):
                diff = sub[:, h, j] - cb[b, h, j, idx[b, h, :, j]]
                total += float(np.sum(diff * diff))
    return total


def kmeans(X: np.ndarray, codebook: np.ndarray, tc: int, n_iter: int):
    """Lloyd's algorithm from ``codebook``: ``n_iter`` rounds of nearest-codeword
    assignment (``encode``, ties to the lowest index) then ``kmeans_update``.

    Returns ``(codebook, idx, history)`` where ``history[i]`` is the
    distortion of round i's assignment against the codebook it was made
    with (non-increasing in i).
    """
    cb = np.asarray(codebook, dtype=np.float64)
    history = []
    idx = None
    for _ in range(n_iter):
        idx, _, _ = encode(X, cb, tc)
        history.append(distortion(X, idx, cb, tc))
        cb, _ = kmeans_update(X, idx, cb, tc)
    return cb, idx, history


# --------------------------------------------------------------------------
# codebook gradient of the attention-output error (fine-tuning stand-in)
# --------------------------------------------------------------------------
# Project page, "Method" -- "Component 2, Loop-aware codebook fine-tuning":
# the codebooks are tuned so that the quantized model's output matches the
# full-precision model's while every loop step reads the quantized cache.
# Without weights or data, the stand-in objective is one attention layer:
# at loop step t, the squared error between decode attention over the
# quantized cache and a target output (attention over the full-precision
# cache), with a weight per step for the steps' unequal sensitivity.  Its
# gradient with respect to both codebooks follows by the chain rule through
# softmax attention.

def attention_mse_codebook_grad(q, loop_step, tc, idx_k, idx_v, codebook_k, codebook_v,
                                win_k, win_v, scale, target, weight=1.0):
    """Loss and codebook gradients of one request's decode attention at step t.

    L = weight * sum_hq ||o_hq - target_hq||^2 with o from ``decode_attention``
    (same arguments).  Chain rule, per query head hq reading KV head h over
    the window and body tokens n with scores s_n = scale q.k_n, softmax
    weights p_n and o = sum_n p_n v_n:

    * dL/do        g = 2 weight (o - target)
    * dL/dv_n      p_n g
    * dL/ds_n      p_n (g.v_n - g.o)   (softmax Jacobian)
    * dL/dk_n      dL/ds_n * scale * q

    A body token's k_n channels jW+w are codebook entries
    B^K[b][h][j][idx_k[b][h][n][j]][t - b*Tc][w] (``dequantize``), so each
    token's dL/dk_n and dL/dv_n slices are added into the entry its code
    selects; window tokens are stored bf16 and reach no codebook entry.

    target  ``[Hq][D]``; returns ``(loss, grad_k, grad_v, o)`` with the
    gradients in codebook layout ``[NB][H][J][C][Tc][W]`` (fp64, non-zero
    only in block b = t // Tc, slice t - b*Tc) and o ``[Hq][D]``.
    """
    q = np.asarray(q, dtype=np.float64)
    target = np.asarray(target, dtype=np.float64)
    Hq, D = q.shape
    NB, H, J, C, tc2, w = codebook_k.shape
    group = Hq // H
    b, tt = divmod(loop_step, tc)
    Kb = dequantize(idx_k, codebook_k, loop_step, tc)  # [n_body][H][D]
    Vb = dequantize(idx_v, codebook_v, loop_step, tc)
    n_body = Kb.shape[0]
    grad_k = np.zeros(codebook_k.shape, dtype=np.float64)
    grad_v = np.zeros(codebook_v.shape, dtype=np.float64)
    out = np.empty((Hq, D), dtype=np.float64)
    loss = 0.0
    for hq in range(Hq):
        h = hq // group
        wk = np.asarray(win_k[h], dtype=np.float64)
        wv = np.asarray(win_v[h], dtype=np.float64)
        K = np.concatenate([wk, Kb[:, h, :]], axis=0)
        V = np.concatenate([wv, Vb[:, h, :]], axis=0)
        if K.shape[0] == 0:
            out[hq] = 0.0
            loss += weight * float(np.sum(target[hq] ** 2))
            continue
        s = scale * (K @ q[hq])
        p = np.exp(s - np.max(s))
        p /= np.sum(p)
        o = p @ V
        out[hq] = o
        diff = o - target[hq]
        loss += weight * float(diff @ diff)
        g = 2.0 * weight * diff
        ds = p * (V @ g - g @ o)
        nw = wk.shape[0]
        p_body = p[nw:]
        ds_body = ds[nw:]
        for j in range(J):
            sl = slice(j * w, (j + 1) * w)
            ck = np.asarray(idx_k[b, h, :n_body, j], dtype=np.int64)
            cv = np.asarray(idx_v[b, h, :n_body, j], dtype=np.int64)
            # one row per body token, added into the entry its code selects
            np.add.at(grad_k[b, h, j, :, tt, :], ck, np.outer(ds_body, scale * q[hq, sl]))
            np.add.at(grad_v[b, h, j, :, tt, :], cv, np.outer(p_body, g[sl]))
    return loss, grad_k, grad_v, out


# --------------------------------------------------------------------------
# second workload: adjacent-loop KV-residual quantization (4-bit)
# --------------------------------------------------------------------------
# FlashLoop page (thelatestinai.com, "Figure 2 (c)", "Figure 3 (c-d)", "Table
# 2", "Figure 4"): the change of K/V from one loop step to the next gets
# smaller deeper in the loop, so coding each step as a residual over the
# previous step loses less than coding each step's K/V on its own; the page
# codes these residuals with 4 bits, on the axes KIVI's 4-bit quantizer uses.  Readings where the
# page is silent: KIVI's quantizer (asymmetric, 16 levels, min and scale per
# group of 32; keys grouped per channel over 32 consecutive tokens, values
# per token over 32 consecutive channels; min and scale stored in fp16);
# step 0 codes K_0 itself and step t codes R_t = K_t - Khat_{t-1}, the
# residual against the previous step's reconstruction, so that Khat_t =
# Khat_{t-1} + Q(R_t) and errors do not pile up.  Every quantization decision
# is taken in fp32 with separately rounded operations (the kernel's
# precision), so codes and parameters are exact.

RESIDUAL_GROUP = 32


def quantize4_group(x):
    """4-bit asymmetric quantization of one group (KIVI's quantizer).

    lo = min x, scale = (max x - lo) / 15 in fp32; both are stored in fp16
    (round to nearest even); code = clamp(rint((x - lo_h) / scale_h), 0, 15)
    with fp32 subtraction and division, or 0 when scale_h is 0.  Returns
    ``(codes uint8, lo_h, scale_h)`` (the last two as np.float16).
    """
    x = np.asarray(x, dtype=np.float32)
    lo = np.min(x)
    hi = np.max(x)
    scale = np.float32(np.float32(hi - lo) / np.float32(15.0))
    lo_h = np.float16(lo)
    sc_h = np.float16(scale)
    lo32 = np.float32(lo_h)
    sc32 = np.float32(sc_h)
    if sc32 == 0:
        q = np.zeros(x.shape, dtype=np.uint8)
    else:
        q = np.clip(np.rint(np.float32(x - lo32) / sc32), 0, 15).astype(np.uint8)
    return q, lo_h, sc_h


def dequantize4(q, lo_h, sc_h):
    """lo + code * scale in fp32 (multiply, then add, each rounded)."""
    prod = np.float32(np.asarray(q, dtype=np.float32) * np.float32(sc_h))
    return np.float32(np.float32(lo_h) + prod)


def residual_encode(X: np.ndarray, kind: str, group: int = RESIDUAL_GROUP):
    """Recursive 4-bit coding of the adjacent-loop residuals of ``X [T][N][H][D]``.

    kind "k": groups of ``group`` consecutive tokens per (step, head, channel);
    kind "v": groups of ``group`` consecutive channels per (step, head, token).
    The last token group may be shorter.  Returns ``(codes, lo, scale, recon)``:
    codes ``[T][H][N][D]`` uint8 in 0..15; lo/scale fp16 ``[T][H][ceil(N/g)][D]``
    for keys, ``[T][H][N][D/g]`` for values; recon ``[T][N][H][D]`` fp32, the
    reconstruction each step reads (Khat_t).
    """
    T, N, H, D = X.shape
    if D % group:
        raise ValueError("head_dim must be a multiple of the group")
    codes = np.zeros((T, H, N, D), dtype=np.uint8)
    ng = -(-N // group)
    if kind == "k":
        lo = np.zeros((T, H, ng, D), dtype=np.float16)
        sc = np.zeros((T, H, ng, D), dtype=np.float16)
    elif kind == "v":
        lo = np.zeros((T, H, N, D // group), dtype=np.float16)
        sc = np.zeros((T, H, N, D // group), dtype=np.float16)
    else:
        raise ValueError("kind must be 'k' or 'v'")
    acc = np.zeros((N, H, D), dtype=np.float32)
    recon = np.zeros((T, N, H, D), dtype=np.float32)
    for t in range(T):
        r = np.float32(np.asarray(X[t], dtype=np.float32) - acc)   # [N][H][D]
        deq = np.zeros_like(r)
        for h in range(H):
            if kind == "k":
                for g in range(ng):
                    n0, n1 = g * group, min(N, (g + 1) * group)
                    for d in range(D):
                        q, l, c = quantize4_group(r[n0:n1, h, d])
                        codes[t, h, n0:n1, d] = q
                        lo[t, h, g, d], sc[t, h, g, d] = l, c
                        deq[n0:n1, h, d] = dequantize4(q, l, c)
            else:
                for n in range(N):
                    for g in range(D // group):
                        d0, d1 = g * group, (g + 1) * group
                        q, l, c = quantize4_group(r[n, h, d0:d1])
                        codes[t, h, n, d0:d1] = q
                        lo[t, h, n, g], sc[t, h, n, g] = l, c
                        deq[n, h, d0:d1] = dequantize4(q, l, c)
        acc = np.float32(acc + deq)
        recon[t] = acc
    return codes, lo, sc, recon


def residual_reconstruct(codes, lo, sc, kind: str, loop_step: int, group: int = RESIDUAL_GROUP):
    """Khat_t ``[N][H][D]`` fp32 from stored codes: the dequantized residuals
    of steps 0..t added in step order (fp32)."""
    T, H, N, D = codes.shape
    acc = np.zeros((N, H, D), dtype=np.float32)
    for t in range(loop_step + 1):
        for h in range(H):
            if kind == "k":
                lo_e = np.repeat(lo[t, h], group, axis=0)[:N]          # [N][D]
                sc_e = np.repeat(sc[t, h], group, axis=0)[:N]
            else:
                lo_e = np.repeat(lo[t, h], group, axis=1)              # [N][D]
                sc_e = np.repeat(sc[t, h], group, axis=1)
            acc[:, h, :] = np.float32(acc[:, h, :] + dequantize4(codes[t, h], lo_e, sc_e))
    return acc


def residual_decode_attention(q, loop_step, k_codes, k_lo, k_sc, v_codes, v_lo, v_sc, scale):
    """Decode attention of one request at loop step t over the reconstructed
    residual-coded cache (every token quantized); q ``[Hq][D]``; returns
    ``(o [Hq][D], lse [Hq])`` in fp64, query head hq reading KV head
    hq // (Hq / H)."""
    q = np.asarray(q, dtype=np.float64)
    Hq = q.shape[0]
    K = residual_reconstruct(k_codes, k_lo, k_sc, "k", loop_step)
    V = residual_reconstruct(v_codes, v_lo, v_sc, "v", loop_step)
    H = K.shape[1]
    group = Hq // H
    out = np.empty(q.shape, dtype=np.float64)
    lse = np.empty(Hq, dtype=np.float64)
    for hq in range(Hq):
        out[hq], lse[hq] = attention(q[hq], K[:, hq // group, :], V[:, hq // group, :], scale)
    return out, lse


def residual_bits_per_element(group: int = RESIDUAL_GROUP) -> float:
    """4 code bits plus an fp16 min and an fp16 scale shared by ``group``
    elements."""
    return 4.0 + 32.0 / group
