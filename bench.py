"""Benchmark of the LoopVQ decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl loopvq|reference]

Workload: Ouro-1.4B-shaped decode attention of one layer -- batch 1, 16 KV
heads x head_dim 128, 4 loop steps, Tc = 4, context 32768 tokens, 0.5 bit
(256-entry codebooks over 4 channels x 4 steps), first 64 and last 256 tokens
in bf16.  One step = one generated token through that layer: the four loop
steps' decode-attention launches, plus, every 8th step, the 8-token page
encode of K and V (in the serving scheme of the LoopVQ project page, one page
leaves the bf16 recent window and is coded for each 8 new tokens).  Eight distinct
layer caches (~350 MB) rotate across steps so no launch reads warm L2.

Metric: KV tokens/s = (context tokens x loop steps attended) / time.  The
roofline object reports the decode kernel against the measured HBM copy
bandwidth; its algorithmic bytes per launch are the index rows (K and V) of
every body token, the bf16 K and V of every window token, the query and the
fp32 output.

Multi-GPU: every rank runs its own copy of the workload (independent
requests; no data-path collective), the time is the max over ranks and the
value sums the ranks' tokens ("weak" scaling).

--impl reference times the CPU oracle (fp64 NumPy) on the machine's host cores
on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "VQ-KV decode attention: KV tokens/s at 32K ctx, 0.5 bit; % of HBM roofline"
UNIT = "KV tokens/s"
T, TC, H, D, G, CTX = 4, 4, 16, 128, 16, 32768
N_SINK, N_RECENT, PAGE = 64, 256, 8
N_LAYERS = 8
WORKLOAD = "ouro1.4b-layer decode attention, batch 1, 16x128, 4 loop steps, Tc=4, ctx 32768, 0.5 bit"


def _config():
    return {"workload": WORKLOAD, "batch": 1, "ctx_len": CTX, "n_heads": H, "head_dim": D, "n_loop": T,
            "tc": TC, "group_elems": G, "bits": 0.5, "n_sink": N_SINK, "n_recent": N_RECENT, "page": PAGE,
            "step": "4 loop-step decode launches (each stores the new token's bf16 K/V into the window) + "
                    "8-token page encode (K,V) every 8th step",
            "l2": f"inputs larger than L2: {N_LAYERS} rotating layer caches"}


# ----------------------------------------------------------------- oracle legs

def _oracle_task(args):
    """One (KV head, loop step) of the workload through the CPU oracle;
    inputs are built from seeds inside the worker, only the oracle is timed."""
    head, t, seed = args
    import numpy as np
    import oracle as O
    from sub_bit_vector_b200 import synth
    s, b, r = O.window_split(CTX, N_SINK, N_RECENT, PAGE)
    W = G // TC
    J = D // W
    outl = synth.key_outlier_channels(seed, 1, D)
    cbk = synth.uniform_codebook(seed + 1, T // TC, 1, J, 256, TC, W, outlier_channels=outl)
    cbv = synth.uniform_codebook(seed + 2, T // TC, 1, J, 256, TC, W)
    wk, wv, ck, cv = synth.decode_request(seed + head, T, 1, D, J, T // TC, s + r, b, outlier_channels=outl)
    q = synth.queries(seed + 3, T, 1, 1, D)[t, 0]
    t0 = time.perf_counter()
    O.decode_attention(q, t, TC, ck, cv, cbk, cbv, wk[t], wv[t], D ** -0.5)
    return time.perf_counter() - t0


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:  # pragma: no cover
        return os.cpu_count() or 1


def cpu_baseline(budget_s: float = 15.0):
    """Oracle throughput on the host cores: a spawn pool over (head, step)
    tasks of the workload, sized to about `budget_s` seconds of CPU work."""
    import multiprocessing as mp
    cores = _cores()
    ctx = mp.get_context("spawn")
    with ctx.Pool(cores) as pool:
        per = pool.map(_oracle_task, [(i % H, 0, 1) for i in range(cores)])   # warm the workers
        # size the timed sample to ~budget_s of wall time on all cores
        rounds = max(1, min(16, int(budget_s / max(max(per), 1e-3))))
        n_tasks = rounds * cores
        tasks = [(i % H, (i // H) % T, 1) for i in range(n_tasks)]
        t0 = time.perf_counter()
        pool.map(_oracle_task, tasks, chunksize=1)
        wall = time.perf_counter() - t0
    per_task = sorted(per)[len(per) // 2]
    return {"value": n_tasks * CTX / wall, "unit": UNIT, "cores": cores, "kind": "oracle",
            "single_core_value": CTX / per_task,
            "sample": f"{n_tasks} (KV head, loop step) decode-attention problems of the 32K workload "
                      f"(each 1 head x {CTX} tokens), spawn pool of {cores} processes, {wall:.1f} s wall; "
                      f"single_core_value from the median warm-up task"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import multiprocessing as mp
    cores = _cores()
    ctx = mp.get_context("spawn")
    per_step = cores
    with ctx.Pool(cores) as pool:
        step = 0

        def one_step():
            nonlocal step
            tasks = [((step * per_step + i) % H, (step * per_step + i) // H % T, 1) for i in range(per_step)]
            step += 1
            pool.map(_oracle_task, tasks)

        for _ in range(args.warmup):
            one_step()
        t0 = time.perf_counter()
        for _ in range(args.steps):
            one_step()
        wall = time.perf_counter() - t0
    value = args.steps * per_step * CTX / wall
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": wall / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"each step: {per_step} (KV head, loop step) problems of the 32K "
                                       f"workload on a spawn pool of {cores} processes"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- GPU helpers

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join(ROOT, f".clocks_{os.getpid()}.csv")   # removed again by stop()

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for ln in open(self.path):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = sorted(float(r[1]) for r in rows if r[1].replace(".", "").isdigit())
        mx = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for i, n in enumerate(names):
                if r[5 + i].lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(rows)}


def _decode_src_hash():
    h = hashlib.sha256()
    for f in ("decode.cu", "common.cuh"):
        with open(os.path.join(ROOT, "sub_bit_vector_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _profiled_traffic():
    """DRAM bytes per decode launch from the committed ncu summary, if it was
    taken on the current kernel source (the summary names the source hash)."""
    p = os.path.join(ROOT, "profiles", "decode_kernel_ouro14_32k_half_bit.md")
    try:
        text = open(p).read()
    except OSError:
        return None
    m_t = re.search(r"traffic_bytes_per_launch:\s*(\d+)", text)
    m_h = re.search(r"decode_src_sha256_16:\s*([0-9a-f]{16})", text)
    if not m_t or not m_h or m_h.group(1) != _decode_src_hash():
        return None
    return int(m_t.group(1))


def _peak_hbm():
    try:
        m = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return float(m["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def build_layers(device, n_layers):
    import torch
    from sub_bit_vector_b200 import cache, synth
    layers = []
    W = G // TC
    J = D // W
    for i in range(n_layers):
        # the layer's pools, windows and codebooks are not written by other
        # kernels while its decodes run (the page encode below writes a
        # separate pool; the new token reaches the window through the
        # decode's own new_k/new_v write), so a launch may start streaming
        # them while the previous launch finishes
        c = cache.DecodeCache(n_loop=T, tc=TC, n_heads_kv=H, head_dim=D, group_elems=G, ctx_lens=[CTX],
                              n_sink=N_SINK, n_recent=N_RECENT, page=PAGE, device=device, static_inputs=True)
        outl = synth.key_outlier_channels(100 + i, H, D)
        c.set_codebooks(synth.uniform_codebook(200 + i, T // TC, H, J, 256, TC, W, outlier_channels=outl),
                        synth.uniform_codebook(300 + i, T // TC, H, J, 256, TC, W))
        c.idxK.copy_(synth.device_codes(400 + i, c.idxK.numel(), device))
        c.idxV.copy_(synth.device_codes(500 + i, c.idxV.numel(), device))
        c.winK.copy_(synth.device_normal(600 + i, tuple(c.winK.shape), device=device))
        c.winV.copy_(synth.device_normal(700 + i, tuple(c.winV.shape), device=device))
        c.q.copy_(synth.device_normal(800 + i, tuple(c.q.shape), dtype=c.q.dtype, device=device))
        # the current token's K and V at each loop step, [2][T][batch=1][H][D]
        c.new_kv = synth.device_normal(850 + i, (2, T, 1, H, D), device=device)
        # the recent page to encode every 8 steps: [T][H][8][D] view of the window pool
        c.page_view = c.winK[:, :, N_SINK:N_SINK + PAGE]
        c.page_view_v = c.winV[:, :, N_SINK:N_SINK + PAGE]
        c.page_pool_tokens = 32
        from sub_bit_vector_b200 import loopvq as L
        c.page_pool = torch.zeros(L.loopvq_index_pool_bytes(c.desc, 32), dtype=torch.uint8, device=device)
        c.page_pool_v = torch.zeros_like(c.page_pool)
        layers.append(c)
    torch.cuda.synchronize()
    return layers


def encode_page(c, stream):
    """Loop-axis encode of the oldest recent page (8 tokens) for K and V."""
    from sub_bit_vector_b200 import loopvq as L
    P = c.win_pool_tokens
    L.loopvq_encode(c.desc, c.cbK, L.LOOPVQ_KEYS, c.page_view, PAGE, H * P * D, D, P * D, c.page_pool, 0,
                    c.page_pool_tokens, stream)
    L.loopvq_encode(c.desc, c.cbV, L.LOOPVQ_VALUES, c.page_view_v, PAGE, H * P * D, D, P * D, c.page_pool_v, 0,
                    c.page_pool_tokens, stream)


def dense_comparator(device, reps=50):
    """Dense bf16 decode kernel on the same shape (one loop step's cache),
    rotating over enough caches to exceed L2."""
    import torch
    from sub_bit_vector_b200 import loopvq as L, synth
    n_buf = 2
    ks = [synth.device_normal(900 + i, (H, CTX, D), device=device) for i in range(n_buf)]
    vs = [synth.device_normal(950 + i, (H, CTX, D), device=device) for i in range(n_buf)]
    q = synth.device_normal(999, (1, H, D), device=device)
    out = torch.zeros((1, H, D), dtype=torch.float32, device=device)
    ws = torch.zeros(L.loopvq_dense_decode_workspace_bytes(1, H, D, CTX) + 256, dtype=torch.uint8, device=device)
    ctx = torch.tensor([CTX], dtype=torch.int32, device=device)
    off = torch.zeros(1, dtype=torch.int64, device=device)
    s = torch.cuda.current_stream()
    for i in range(4):
        L.loopvq_dense_decode_attn(1, H, H, D, CTX, ctx, off, CTX, ks[i % n_buf], vs[i % n_buf], q, D ** -0.5, out,
                                   None, ws, s)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(s)
    for i in range(reps):
        L.loopvq_dense_decode_attn(1, H, H, D, CTX, ctx, off, CTX, ks[i % n_buf], vs[i % n_buf], q, D ** -0.5, out,
                                   None, ws, s)
    e1.record(s)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / reps
    by = 2 * H * CTX * D * 2 + H * D * 2 + H * D * 4
    return {"us_per_launch": us, "bytes_per_launch": by, "GB_per_s": by / us / 1e3,
            "kv_tokens_per_s": CTX / (us * 1e-6)}


def sdpa_comparator(device, reps=50):
    """torch's scaled_dot_product_attention on the bf16 cache of one loop step
    (batch 1, 16 heads x 32768 tokens x 128, one query), for context."""
    import torch
    from sub_bit_vector_b200 import synth
    n_buf = 2
    ks = [synth.device_normal(1900 + i, (1, H, CTX, D), device=device) for i in range(n_buf)]
    vs = [synth.device_normal(1950 + i, (1, H, CTX, D), device=device) for i in range(n_buf)]
    q = synth.device_normal(1999, (1, H, 1, D), device=device)
    f = torch.nn.functional.scaled_dot_product_attention
    for i in range(4):
        f(q, ks[i % n_buf], vs[i % n_buf])
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for i in range(reps):
        f(q, ks[i % n_buf], vs[i % n_buf])
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / reps
    return {"us_per_launch": us, "kv_tokens_per_s": CTX / (us * 1e-6), "what": "torch SDPA, bf16 K/V, 1 query"}


def all_steps_measurement(layers, device, reps=400):
    """All T loop steps of a layer in one launch (loopvq_decode_attn_steps):
    for callers that hold every step's query at once, not loop-sequential
    decoding.  The steps of one code block share each index row, so a launch
    moves the codes once and every step's window, query and output."""
    import torch
    from sub_bit_vector_b200 import loopvq as L, synth
    s = torch.cuda.Stream(device)
    bufs = []
    for i, c in enumerate(layers):
        q = synth.device_normal(1700 + i, (T, 1, H, D), device=device)
        out = torch.zeros((T, 1, H, D), dtype=torch.float32, device=device)
        lse = torch.zeros((T, 1, H), dtype=torch.float32, device=device)
        ws = torch.zeros(L.loopvq_decode_steps_workspace_bytes(c.desc, c.layout, T), dtype=torch.uint8,
                         device=device)
        bufs.append((c, q, out, lse, ws))

    def launch(b):
        c, q, out, lse, ws = b
        L.loopvq_decode_attn_steps(c.desc, c.cbK, c.cbV, c.layout, c.idxK, c.idxV, c.winK, c.winV, q, 0, T,
                                   D ** -0.5, out, lse, ws, s)
    with torch.cuda.stream(s):
        for b in bufs:
            launch(b)
    torch.cuda.synchronize()
    graphs = []
    for b in bufs:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            launch(b)
        graphs.append(g)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):   # replay() launches on the current stream
        for i in range(2 * len(graphs)):
            graphs[i % len(graphs)].replay()
        torch.cuda.synchronize()
        e0.record(s)
        for i in range(reps):
            graphs[i % len(graphs)].replay()
        e1.record(s)
    torch.cuda.synchronize()
    us_launch = e0.elapsed_time(e1) * 1e3 / reps
    faults = max(L.loopvq_read_device_status(b[4])[1] for b in bufs)
    c = layers[0]
    per_step = c.algorithmic_bytes()
    codes = sum(b for (_, b, _) in c.splits) * H * 2 * (D * TC // G)
    by = codes + T * (per_step - codes)      # codes once, window + q/out per step
    del graphs
    return {"us_per_launch": us_launch, "us_per_loop_step": us_launch / T,
            "kv_tokens_per_s_per_step": CTX * T / (us_launch * 1e-6), "algorithmic_bytes_per_launch": by,
            "GB_per_s": by / us_launch / 1e3, "launches_timed": reps, "device_fault_bits": faults,
            "what": f"{T} loop steps per launch (every step's query given at once), graph of 1 launch per layer, "
                    f"{len(layers)} rotating layer caches"}


def residual_measurement(device, n_layers=4, reps=40):
    """Second workload on the same shape: adjacent-loop KV-residual 4-bit
    coding of one layer's [4][32768][16][128] keys and values, then decode
    attention at each loop step (every token coded, no bf16 window); rotating
    over layer caches larger than L2."""
    import torch
    from sub_bit_vector_b200 import loopvq as L, synth
    desc = L.make_residual_desc(T, H, D)
    layers = []
    enc_ms = None
    for i in range(n_layers):
        bufs = []
        for kind in (L.LOOPVQ_KEYS, L.LOOPVQ_VALUES):
            codes = torch.zeros(L.loopvq_residual_codes_bytes(desc, CTX), dtype=torch.uint8, device=device)
            params = torch.zeros(L.loopvq_residual_params_bytes(desc, kind, CTX) // 2, dtype=torch.float16,
                                 device=device)
            x = synth.device_normal(1500 + 2 * i + kind, (T, CTX, H, D), device=device)
            L.loopvq_residual_encode(desc, kind, x, CTX, CTX * H * D, H * D, D, codes, params, 0, CTX)
            if i == 0 and kind == L.LOOPVQ_KEYS:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                torch.cuda.synchronize()
                e0.record()
                L.loopvq_residual_encode(desc, kind, x, CTX, CTX * H * D, H * D, D, codes, params, 0, CTX)
                e1.record()
                torch.cuda.synchronize()
                enc_ms = e0.elapsed_time(e1)
            bufs.append((codes, params))
            del x
        ws = torch.zeros(L.loopvq_residual_decode_workspace_bytes(desc, 1, CTX), dtype=torch.uint8, device=device)
        layers.append((bufs, ws))
    ctx = torch.tensor([CTX], dtype=torch.int32, device=device)
    off = torch.zeros(1, dtype=torch.int64, device=device)
    q = synth.device_normal(1599, (1, H, D), device=device)
    out = torch.zeros((1, H, D), dtype=torch.float32, device=device)
    per_step = []
    for t in range(T):
        def run(b):
            (ck, pk), (cv, pv) = b[0]
            L.loopvq_residual_decode_attn(desc, 1, CTX, ctx, off, CTX, ck, pk, cv, pv, q, t, D ** -0.5, out, None,
                                          b[1])
        for b in layers:
            run(b)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(reps):
            run(layers[i % n_layers])
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / reps
        by = (t + 1) * H * CTX * (D // 2 * 2 + (D // 32) * 4 + D * 4 // 32) + H * D * 6
        per_step.append({"loop_step": t, "us_per_launch": us, "algorithmic_bytes": by, "GB_per_s": by / us / 1e3,
                         "kv_tokens_per_s": CTX / (us * 1e-6)})
    faults = max(L.loopvq_read_device_status(b[1])[1] for b in layers)
    return {"encode_keys_ms_per_tensor": enc_ms, "decode": per_step, "device_fault_bits": faults,
            "what": "4-bit residuals between adjacent loop steps (fp16 min/scale per 32), decode rebuilding step t "
                    "from t+1 planes; batch 1, 16x128, ctx 32768"}


def encode_measurement(device, with_oracle, sm_mhz=None, reps=5):
    """Prefill encode on its stated inputs: loop-correlated (rho = 0.9) bf16
    keys (4 heavy-tailed outlier channels per head) and values
    [4][32768][16][128], codebooks of seeded data rows, encoded at 0.5 bit
    (G = 16) and 0.25 bit (G = 32) with Tc = 4, and at 0.5 bit with Tc = 1 (16
    channels of one step) for the reconstruction comparison.  Per tensor: ms,
    the fraction of the argmin ALU floor (2 integer operations per candidate
    codeword on 148 SMs x 128 lanes at the SM clock) and of the HBM floor
    (bf16 input + codes at the measured copy bandwidth).  with_oracle adds,
    on a seeded 1/64 token sample on the host: the reconstruction MSE of the
    GPU's codes (dequantized by the oracle) and the oracle's encode rate."""
    import numpy as np
    import torch
    from sub_bit_vector_b200 import loopvq as L, synth
    peak, _ = _peak_hbm()
    f_hz = (sm_mhz or 1965.0) * 1e6
    rng = np.random.Generator(np.random.PCG64(11))
    toks = np.sort(rng.choice(CTX, CTX // 64, replace=False))
    out = {"what": "[4][32768][16][128] bf16 K (4 outlier channels x8) and V, rho 0.9, data-row codebooks; "
                   "MSE on a 1/64 token sample (GPU codes, oracle dequantization)",
           "alu_floor": "2 ops per candidate codeword / (148 SMs x 128 lanes x SM clock); alu_pipe_floor: the "
                        "same over the integer ALU pipe's 64 lanes per clock, which min/max and key formation use",
           "tensors": []}
    for kind_name, seed, n_out in (("K", 40, 4), ("V", 41, 0)):
        X = synth.loop_correlated(seed=seed, n_loop=T, n_tokens=CTX, n_heads=H, head_dim=D, n_outlier=n_out)
        x_dev = torch.from_numpy(X).to(device).to(torch.bfloat16)
        kind = L.LOOPVQ_KEYS if kind_name == "K" else L.LOOPVQ_VALUES
        mse = {}
        for tc, g in ((4, 16), (4, 32), (1, 16)):
            cb = synth.codebook_from_rows(X, tc, g, 256, seed=seed + 2 + tc + g)
            desc = L.make_desc(T, tc, H, D, g)
            packed = torch.zeros(L.loopvq_codebook_packed_bytes(desc), dtype=torch.uint8, device=device)
            L.loopvq_codebook_pack(desc, torch.from_numpy(cb).to(device).to(torch.bfloat16), packed)
            pool = torch.zeros(L.loopvq_index_pool_bytes(desc, CTX), dtype=torch.uint8, device=device)
            faults = torch.zeros(1, dtype=torch.int32, device=device)
            args = (desc, packed, kind, x_dev, CTX, CTX * H * D, H * D, D, pool, 0, CTX)
            for _ in range(2):
                L.loopvq_encode(*args, fault_bits=faults)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record()
            for _ in range(reps):
                L.loopvq_encode(*args, fault_bits=faults)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / reps
            J = D * tc // g
            cand = (T // tc) * H * J * CTX * 256
            alu_ms = cand * 2 / (148 * 128 * f_hz) * 1e3
            alu_pipe_ms = cand * 2 / (148 * 64 * f_hz) * 1e3   # the integer ALU pipe's 64 lanes per clock
            by = T * CTX * H * D * 2 + (T // tc) * H * J * CTX
            hbm_ms = by / (peak * 1e9) * 1e3
            rec = {"tensor": kind_name, "tc": tc, "group_elems": g, "bits": 8.0 / g, "ms_per_tensor": ms,
                   "candidates": cand, "alu_floor_ms": alu_ms, "alu_floor_frac": alu_ms / ms,
                   "alu_pipe_floor_ms": alu_pipe_ms, "alu_pipe_floor_frac": alu_pipe_ms / ms,
                   "hbm_floor_ms": hbm_ms, "hbm_floor_frac": hbm_ms / ms, "fault_bits": int(faults.item())}
            if with_oracle:
                import oracle as O
                codes = torch.zeros((T // tc, H, CTX, J), dtype=torch.uint8, device=device)
                L.loopvq_index_pool_unpack(desc, kind, pool, 0, CTX, CTX, codes)
                idx = codes.cpu().numpy()[:, :, toks].astype(np.int64)
                xs = synth.round_bf16(X[:, toks])
                rec["mse_sample"] = O.reconstruction_mse(xs, idx, synth.round_bf16(cb), tc)
                mse[(tc, g)] = rec["mse_sample"]
                if tc == 4 and g == 16 and kind_name == "K":
                    t0 = time.perf_counter()
                    O.encode(xs, synth.round_bf16(cb), tc)
                    wall = time.perf_counter() - t0
                    rec["oracle_subvectors_per_s"] = len(toks) * H * J / wall
                    rec["oracle_sample"] = f"{len(toks)} of {CTX} tokens (1/64, all heads and slots), 1 process"
            out["tensors"].append(rec)
            del pool
        if with_oracle:
            out[f"mse_{kind_name}_tc4_over_tc1_at_half_bit"] = mse[(4, 16)] / mse[(1, 16)]
        del x_dev
    return out


def decode_config_measurement(device, name, ctx_lens, group_elems, n_layers, reps):
    """One decode configuration timed the way the headline is: a CUDA graph
    of the 4 loop-step launches per layer, rotating over n_layers layer
    caches (larger than L2 together), device-drawn codes, windows and
    queries.  Returns us per launch, algorithmic bytes, GB/s, the fraction of
    the measured HBM copy bandwidth and KV tokens/s."""
    import torch
    from sub_bit_vector_b200 import cache, synth
    peak, _ = _peak_hbm()
    W = group_elems // TC
    J = D // W
    caches = []
    for i in range(n_layers):
        c = cache.DecodeCache(n_loop=T, tc=TC, n_heads_kv=H, head_dim=D, group_elems=group_elems, ctx_lens=ctx_lens,
                              n_sink=N_SINK, n_recent=N_RECENT, page=PAGE, device=device, static_inputs=True)
        outl = synth.key_outlier_channels(3100 + i, H, D)
        c.set_codebooks(synth.uniform_codebook(3200 + i, T // TC, H, J, 256, TC, W, outlier_channels=outl),
                        synth.uniform_codebook(3300 + i, T // TC, H, J, 256, TC, W))
        c.idxK.copy_(synth.device_codes(3400 + i, c.idxK.numel(), device))
        c.idxV.copy_(synth.device_codes(3500 + i, c.idxV.numel(), device))
        c.winK.copy_(synth.device_normal(3600 + i, tuple(c.winK.shape), device=device))
        c.winV.copy_(synth.device_normal(3700 + i, tuple(c.winV.shape), device=device))
        c.q.copy_(synth.device_normal(3800 + i, tuple(c.q.shape), dtype=c.q.dtype, device=device))
        caches.append(c)
    s = torch.cuda.Stream(device)
    with torch.cuda.stream(s):
        for c in caches:
            c.decode(0, stream=s)
    torch.cuda.synchronize()
    graphs = []
    for c in caches:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for t in range(T):
                c.decode(t, stream=s)
        graphs.append(g)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        for i in range(2 * n_layers):
            graphs[i % n_layers].replay()
        torch.cuda.synchronize()
        e0.record(s)
        for i in range(reps):
            graphs[i % n_layers].replay()
        e1.record(s)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (reps * T)
    by = caches[0].algorithmic_bytes()
    faults = max(c.device_status()[1] for c in caches)
    del graphs, caches
    torch.cuda.empty_cache()
    return {"config": name, "bits": 8.0 / group_elems, "batch": len(ctx_lens), "kv_tokens": int(sum(ctx_lens)),
            "us_per_launch": us, "algorithmic_bytes_per_launch": by, "GB_per_s": by / us / 1e3,
            "frac_of_measured_hbm": by / us / 1e3 / peak, "kv_tokens_per_s": sum(ctx_lens) / (us * 1e-6),
            "launches_timed": reps * T, "layer_caches": n_layers, "device_fault_bits": faults}


def other_configs_measurement(device):
    """The quarter-bit context sweep (4K..64K, batch 1) and the batch-128
    ragged serving step (2048 + U{4096..16384} tokens per request, 0.5 bit),
    each with the headline's timing method."""
    from sub_bit_vector_b200 import synth
    res = []
    for ctx in (4096, 8192, 16384, 32768, 65536):
        res.append(decode_config_measurement(device, f"0.25 bit, ctx {ctx}", [ctx], 32,
                                             n_layers=8 if ctx <= 32768 else 4, reps=200))
    ragged = [int(x) for x in synth.ragged_context_lengths(128)]
    res.append(decode_config_measurement(device, "0.5 bit, batch 128 ragged (2048 + U[4096, 16384])", ragged, 16,
                                         n_layers=2, reps=20))
    return res


def reduce_over_ranks(values, world, device=None):
    """Max over ranks of per-rank device timings (ms); every rank takes the
    same collective step.  Returns the list of maxima."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def aggregate_value(world, steps, tokens_per_step, elapsed_ms):
    """Whole-job throughput: every rank processed `steps` steps of its own
    workload (weak scaling) within the max-over-ranks time."""
    return world * steps * tokens_per_step / (elapsed_ms * 1e-3)


def run_gpu(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}), flush=True)
        return 1
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.cpu_budget)

    from sub_bit_vector_b200 import loopvq as L
    layers = build_layers(device, N_LAYERS)
    stream = torch.cuda.Stream(device=device)
    decode_graphs, encode_graphs = [], []
    with torch.cuda.stream(stream):
        for c in layers:          # one eager pass (sets attributes, warms caches)
            for t in range(T):
                c.decode(t, stream=stream, new_k=c.new_kv[0, t], new_v=c.new_kv[1, t])
            encode_page(c, stream)
    torch.cuda.synchronize()
    for c in layers:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for t in range(T):
                c.decode(t, stream=stream, new_k=c.new_kv[0, t], new_v=c.new_kv[1, t])
        decode_graphs.append(g)
        ge = torch.cuda.CUDAGraph()
        with torch.cuda.graph(ge, stream=stream):
            encode_page(c, stream)
        encode_graphs.append(ge)
    torch.cuda.synchronize()

    def step(i, ev=None):
        li = i % N_LAYERS
        if ev is not None:
            ev[0].record(stream)
        decode_graphs[li].replay()
        if ev is not None:
            ev[1].record(stream)
        if i % PAGE == PAGE - 1:
            encode_graphs[li].replay()

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        start.record(stream)
        for i in range(args.steps):
            step(i, evs[i])
        end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    elapsed_ms = start.elapsed_time(end)
    decode_ms = sum(a.elapsed_time(b) for a, b in evs)
    n_enc_steps = sum(1 for i in range(args.steps) if i % PAGE == PAGE - 1)
    elapsed_ms, decode_ms = reduce_over_ranks([elapsed_ms, decode_ms], world, device)

    status = [c.device_status()[1] for c in layers]
    tokens_per_step = CTX * T
    value = aggregate_value(world, args.steps, tokens_per_step, elapsed_ms)
    algo = layers[0].algorithmic_bytes()
    us_launch = decode_ms * 1e3 / (args.steps * T)
    peak, peak_kind = _peak_hbm()
    achieved = algo / (us_launch * 1e-6) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": _profiled_traffic(), "kernel": "loopvq::decode_kernel<32,128,bf16>",
                "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else peak_kind,
                "algorithmic_bytes_per_launch": algo, "us_per_launch": us_launch,
                "frac_of_8TBps_spec": achieved / 8000.0}

    # ---- end to end through the public API with host buffers: every step
    # copies the 4 loop steps' queries and the new token's bf16 K and V from
    # pinned host memory in one transfer, runs the 4 decode calls -- each
    # writes the new token's K/V of its step into the recent window itself
    # (the layout's new_k/new_v) -- plus the page encode every 8th step, and
    # reads the 4 fp32 outputs back into pinned host memory.
    e2e_steps = min(args.steps, 2000)
    n_q = T * H * D
    in_host = torch.randn(3 * n_q, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16).pin_memory()
    out_host = torch.empty((T, 1, H, D), dtype=torch.float32).pin_memory()
    in_dev = torch.empty(3 * n_q, dtype=torch.bfloat16, device=device)
    q_dev = in_dev[:n_q].view(T, 1, H, D)
    k_dev = in_dev[n_q:2 * n_q].view(T, 1, H, D)
    v_dev = in_dev[2 * n_q:].view(T, 1, H, D)
    out_dev = torch.empty((T, 1, H, D), dtype=torch.float32, device=device)
    lse_dev = torch.empty((T, 1, H), dtype=torch.float32, device=device)
    h2d = in_host.numel() * 2
    d2h = out_host.numel() * 4
    calls = []
    for c in layers:
        per = []
        for t in range(T):
            lay = L.make_layout(1, N_SINK, N_RECENT, PAGE, c.max_ctx_len, c.ctx_dev, c.body_off_dev, c.win_off_dev,
                                c.body_pool_tokens, c.win_pool_tokens,
                                L.LOOPVQ_LAYOUT_STATIC_INPUTS,
                                new_k=k_dev[t], new_v=v_dev[t])
            per.append(L.prepare_decode_attn(c.desc, c.cbK, c.cbV, lay, c.idxK, c.idxV, c.winK, c.winV, q_dev[t], t,
                                             D ** -0.5, out_dev[t], lse_dev[t], c.workspace, stream))
        calls.append(per)
    with torch.cuda.stream(stream):
        def e2e_step(i):
            li = i % N_LAYERS
            in_dev.copy_(in_host, non_blocking=True)
            for t in range(T):
                calls[li][t]()
            if i % PAGE == PAGE - 1:
                encode_page(layers[li], stream)
            out_host.copy_(out_dev, non_blocking=True)
            stream.synchronize()
        for i in range(min(args.warmup, 50)):
            e2e_step(i)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for i in range(e2e_steps):
            e2e_step(i)
        s1.record(stream)
        torch.cuda.synchronize()
    e2e_ms = reduce_over_ranks([s0.elapsed_time(s1)], world, device)[0]
    e2e = {"value": aggregate_value(world, e2e_steps, tokens_per_step, e2e_ms), "unit": UNIT,
           "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": e2e_steps,
           "path": "pinned host queries + new-token K/V -> device in one copy, 4 loopvq_decode_attn calls that "
                   "also write the new token into the window (+ page encode every 8th step), fp32 outputs -> "
                   "pinned host, stream sync per step"}

    steps_fused = all_steps_measurement(layers, device) if not args.no_extras else None
    residual = None
    if not args.no_extras:
        try:
            residual = residual_measurement(device)
        except Exception as exc:   # a context figure: report, never lose the line for it
            residual = {"error": f"{type(exc).__name__}: {exc}"}
    others = other_configs_measurement(device) if not args.no_extras else None
    dense = dense_comparator(device) if not args.no_extras else None
    sdpa = sdpa_comparator(device) if not args.no_extras else None
    enc = (encode_measurement(device, with_oracle=(rank == 0 and world == 1 and not args.no_cpu_baseline),
                              sm_mhz=clocks.get("sm_mhz"))
           if not args.no_extras else None)
    launches = args.steps * T * 2 + 2 * n_enc_steps   # decode + merge kernel per loop step; K and V page encodes
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "u8 codes, f32 accumulate", "data": "synthetic",
                "config": dict(_config(), parallelism=f"replicas x{world}" if world > 1 else "single GPU"),
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
                "clocks": clocks, "other_configs": others, "all_steps_one_launch": steps_fused, "kv_residual_4bit": residual, "dense_bf16_comparator": dense, "torch_sdpa_bf16": sdpa, "encode": enc,
                "device_fault_bits": max(status)}
        print(json.dumps(line), flush=True)
    del decode_graphs, encode_graphs
    if world > 1:
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------ profile cases
# Small, self-contained launches of each kernel for a profiler:
# ``python bench.py --profile-case NAME`` runs one case on cuda:0 and prints
# its device status; inputs are seeded and drawn on the device, and each case
# holds well under 2 GB so that a profiler replaying one launch stays small.
#   decode       32768-token context, batch 1, 16 KV heads x 128, 4 loop
#                steps, Tc = 4, G = 16 (0.5 bit): one launch per loop step
#   decode-q     the same at G = 32 (0.25 bit)
#   decode-gqa   8 KV heads, 16 query heads (GQA ratio 2), 4 launches
#   decode-steps the decode case as one launch of all 4 loop steps, 2 launches
#   encode       loop-axis encode of [4][32768][16][128] bf16, Tc = 4, G = 16
#                (tensor-core kernel), 2 launches; encode-f32: fp32 input
#                (CUDA-core kernel)
#   residual     residual 4-bit coding of [4][32768][16][128] keys and values,
#                then one decode per loop step
#   page         encode of one 8-token page out of a [4][16][320][128] window

def _pc_decode(G=16, Hkv=16, Hq=None):
    import torch
    from sub_bit_vector_b200 import cache, synth
    c = cache.DecodeCache(n_loop=T, tc=TC, n_heads_kv=Hkv, head_dim=D, group_elems=G, ctx_lens=[CTX], n_heads_q=Hq)
    W = G // TC
    J = D // W
    cb = synth.uniform_codebook(1, 1, Hkv, J, 256, TC, W)
    c.set_codebooks(cb, cb)
    c.idxK.copy_(synth.device_codes(2, c.idxK.numel()))
    c.idxV.copy_(synth.device_codes(3, c.idxV.numel()))
    c.winK.normal_()
    c.winV.normal_()
    c.q.normal_()
    for t in range(T):
        c.decode(t)
    torch.cuda.synchronize()
    print("decode status", c.device_status(), "algorithmic bytes per launch", c.algorithmic_bytes())


def _pc_decode_steps():
    import torch
    from sub_bit_vector_b200 import cache, loopvq as L, synth
    c = cache.DecodeCache(n_loop=T, tc=TC, n_heads_kv=H, head_dim=D, group_elems=G, ctx_lens=[CTX])
    cb = synth.uniform_codebook(1, 1, H, D * TC // G, 256, TC, G // TC)
    c.set_codebooks(cb, cb)
    c.idxK.copy_(synth.device_codes(2, c.idxK.numel()))
    c.idxV.copy_(synth.device_codes(3, c.idxV.numel()))
    c.winK.normal_()
    c.winV.normal_()
    q = synth.device_normal(4, (T, 1, H, D)).to(torch.bfloat16)
    out = torch.zeros((T, 1, H, D), dtype=torch.float32, device="cuda")
    lse = torch.zeros((T, 1, H), dtype=torch.float32, device="cuda")
    ws = torch.zeros(L.loopvq_decode_steps_workspace_bytes(c.desc, c.layout, T), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        L.loopvq_decode_attn_steps(c.desc, c.cbK, c.cbV, c.layout, c.idxK, c.idxV, c.winK, c.winV, q, 0, T,
                                   D ** -0.5, out, lse, ws)
    torch.cuda.synchronize()
    print("decode-steps status", L.loopvq_read_device_status(ws))


def _pc_encode(dtype_name):
    import torch
    from sub_bit_vector_b200 import loopvq as L, synth
    x = synth.device_normal(1, (T, CTX, H, D)).to(getattr(torch, dtype_name))
    desc = L.make_desc(T, TC, H, D, G)
    W = G // TC
    cb = synth.device_normal(2, (T // TC, H, D // W, 256, TC, W))
    packed = torch.zeros(L.loopvq_codebook_packed_bytes(desc), dtype=torch.uint8, device="cuda")
    L.loopvq_codebook_pack(desc, cb, packed)
    pool = torch.zeros(L.loopvq_index_pool_bytes(desc, CTX), dtype=torch.uint8, device="cuda")
    faults = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        L.loopvq_encode(desc, packed, L.LOOPVQ_KEYS, x, CTX, CTX * H * D, H * D, D, pool, 0, CTX, fault_bits=faults)
    torch.cuda.synchronize()
    print("encode fault bits", int(faults.item()))


def _pc_residual():
    import torch
    from sub_bit_vector_b200 import loopvq as L, synth
    desc = L.make_residual_desc(T, H, D)
    bufs = []
    for kind in (L.LOOPVQ_KEYS, L.LOOPVQ_VALUES):
        codes = torch.zeros(L.loopvq_residual_codes_bytes(desc, CTX), dtype=torch.uint8, device="cuda")
        params = torch.zeros(L.loopvq_residual_params_bytes(desc, kind, CTX) // 2, dtype=torch.float16, device="cuda")
        x = synth.device_normal(20 + kind, (T, CTX, H, D))
        L.loopvq_residual_encode(desc, kind, x, CTX, CTX * H * D, H * D, D, codes, params, 0, CTX)
        bufs.append((codes, params))
        del x
    ctx = torch.tensor([CTX], dtype=torch.int32, device="cuda")
    off = torch.zeros(1, dtype=torch.int64, device="cuda")
    q = synth.device_normal(30, (1, H, D))
    out = torch.zeros((1, H, D), dtype=torch.float32, device="cuda")
    ws = torch.zeros(L.loopvq_residual_decode_workspace_bytes(desc, 1, CTX), dtype=torch.uint8, device="cuda")
    for t in range(T):
        L.loopvq_residual_decode_attn(desc, 1, CTX, ctx, off, CTX, bufs[0][0], bufs[0][1], bufs[1][0], bufs[1][1],
                                      q, t, D ** -0.5, out, None, ws)
    torch.cuda.synchronize()
    print("residual decode status", L.loopvq_read_device_status(ws))


def _pc_page():
    import torch
    from sub_bit_vector_b200 import loopvq as L, synth
    P = 320
    win = synth.device_normal(3, (T, H, P, D))
    desc = L.make_desc(T, TC, H, D, G)
    W = G // TC
    cb = synth.device_normal(2, (T // TC, H, D // W, 256, TC, W))
    packed = torch.zeros(L.loopvq_codebook_packed_bytes(desc), dtype=torch.uint8, device="cuda")
    L.loopvq_codebook_pack(desc, cb, packed)
    pool = torch.zeros(L.loopvq_index_pool_bytes(desc, 32), dtype=torch.uint8, device="cuda")
    faults = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(4):
        L.loopvq_encode(desc, packed, L.LOOPVQ_KEYS, win[:, :, 64:72], 8, H * P * D, D, P * D, pool, 0, 32,
                        fault_bits=faults)
    torch.cuda.synchronize()
    print("page encode fault bits", int(faults.item()))


PROFILE_CASES = {
    "decode": lambda: _pc_decode(16),
    "decode-q": lambda: _pc_decode(32),
    "decode-gqa": lambda: _pc_decode(16, Hkv=8, Hq=16),
    "decode-steps": _pc_decode_steps,
    "encode": lambda: _pc_encode("bfloat16"),
    "encode-f32": lambda: _pc_encode("float32"),
    "page": _pc_page,
    "residual": _pc_residual,
}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=100)
    ap.add_argument("--impl", choices=["loopvq", "reference"], default="loopvq")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES), default=None,
                    help="run one small launch set of a kernel for a profiler and exit")
    args = ap.parse_args(argv)
    if args.profile_case:
        PROFILE_CASES[args.profile_case]()
        return 0
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
