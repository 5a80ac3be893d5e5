"""Benchmark of the CoWA hot path on B200: one step = cowa_fwd + cowa_bwd on the 32K
training layer plus cowa_decode on the 128K decode cache.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cowa|reference]

Prints one JSON line (rank 0).  `value` is visible TFLOP/s of the training part
(forward 4*d and backward 10*d FLOPs per visible query-key pair, summed over all
ranks) divided by the max-over-ranks device time of the whole step (decode
included); `parts` gives each call's CUDA-event time and the decode GB/s over the
visible K/V bytes, and also carries the other configurations, each kernel timed alone
(see `config_parts`): the 32K layer's dense-causal mode and SWA + sinks, the 128K layer
and its dense-causal mode, and the 128K decode in the dense-causal mode, over the
compacted cache and over E4M3 caches; --sweep adds the 8K prefill D sweep.
Inputs are larger than L2 (126 MB), so no flush is needed between steps.

N > 1: one process per GPU (torchrun); every rank runs the same per-GPU workload on
its own batch element and seeds (weak scaling: batch sharding, no exchange step in
the op), timed between barriers, max over ranks.

--impl reference times the CPU fp64 oracle (test infrastructure, not the product) on a
bounded sample of the same workload, on the host cores of rank 0.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "CoWA fwd/bwd TFLOP/s (visible) + decode GB/s at 32K/128K, % of B200 roofline"

# Train 32K layer (B=1 per GPU) and decode 128K cache (B=16 per GPU)
TRAIN = dict(B=1, N=32768, Hq=40, Hkv=8, d=128, S=128, L=2048, T=32768, D=8)
DECODE = dict(B=16, Hq=40, Hkv=8, d=128, T_cap=131072, S=128, L=4096, T=131072, D=8, pos=131071)


# ------------------------------------------------------------------------------ accounting
def visible_pairs(N, S, L, T, D, Hkv, Hq, B=1, h_kv_global=None):
    """Sum over b, query heads and positions of |visible keys| (closed form per position)."""
    import numpy as np

    H = h_kv_global or Hkv
    grp = Hq // Hkv
    bnd = [S + (i * (T - S)) // H for i in range(H + 1)]
    t = np.arange(N, dtype=np.int64)
    total = 0
    for g in range(Hkv):
        p = (g % D) * (H // D)
        lo, hi = bnd[p], bnd[p + 1]
        sink = np.minimum(S, t + 1)
        band_lo = np.maximum(0, t - L + 1)
        band = t + 1 - band_lo
        lr_hi = np.minimum(hi, t + 1)
        lr = np.maximum(0, lr_hi - lo)
        sb = np.maximum(0, np.minimum(S, t + 1) - band_lo)               # sink & band
        lb = np.maximum(0, lr_hi - np.maximum(lo, band_lo))              # interval & band
        ls = np.maximum(0, np.minimum(S, lr_hi) - lo)                    # interval & sink (0: lo >= S)
        total += int((sink + band + lr - sb - lb - ls).sum())
    return total * grp * B


def decode_visible_tokens(pos, S, L, T, D, Hkv, h_kv_global=None):
    H = h_kv_global or Hkv
    bnd = [S + (i * (T - S)) // H for i in range(H + 1)]
    out = []
    for g in range(Hkv):
        p = (g % D) * (H // D)
        lo, hi = bnd[p], bnd[p + 1]
        ranges = sorted([(0, min(S, pos + 1)), (max(0, pos - L + 1), pos + 1), (lo, min(hi, pos + 1))])
        n, cur = 0, None
        for a, b in ranges:
            if a >= b:
                continue
            if cur is None or a > cur[1]:
                if cur:
                    n += cur[1] - cur[0]
                cur = [a, b]
            else:
                cur[1] = max(cur[1], b)
        n += cur[1] - cur[0]
        out.append(n)
    return out


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return pk["bf16_tflops"], pk["bf16_tflops_sustained"], pk["hbm_gbs"], "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


def _traffic_record(kernel: str, kernel_file: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary (profiles/traffic.txt:
    kernel, source file, sha256 prefix of that file when captured, bytes per launch), or None
    when the source has changed since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    src = os.path.join(ROOT, "structured_sparse_attention_cowa_b200", "csrc", kernel_file)
    try:
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        for line in open(path):
            parts = line.split()
            if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel and parts[1] == kernel_file \
                    and parts[2] == sha:
                return float(parts[3])
    except Exception:
        pass
    return None


# ------------------------------------------------------------------------------ multi-rank
def rank_seed_extra(rank: int) -> int:
    """Each rank draws its own batch element (weak scaling by batch sharding)."""
    return rank


def max_over_ranks(x: float, dist=None, device=None) -> float:
    """The slowest rank's time: every multi-GPU number is the max over ranks."""
    if dist is None:
        return x
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(world: int, flop_per_rank: float, ms_per_step: float) -> float:
    """Whole-job throughput: all ranks' work over the max-over-ranks step time."""
    return world * flop_per_rank / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while active."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"cowa_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return None
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for line in open(self.path):
                p = [x.strip() for x in line.split(",")]
                if len(p) < 9:
                    continue
                sm.append(float(p[1]))
                mx = float(p[2])
                for n, v in zip(names, p[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        except Exception:
            return None
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------ CPU oracle
_KV_CACHE = {}


def cpu_oracle_sample(target_s: float, seed_extra: int = 0):
    """Time the fp64 oracle on random blocks of the 32K layer for about target_s seconds of CPU
    work (input generation is outside the timed part), half on the forward and half on the
    backward, and return the whole step's rate at those speeds.

    Forward: attention_fwd_rows on 32-row blocks, 4*d FLOPs credited per visible pair.
    Backward: attention_bwd_rows on 32-row blocks (the row-local part of the backward: S, dP, dS
    and dQ), 6*d FLOPs credited per visible pair; that rate stands for the whole 10*d backward
    (the column-local dK/dV part is the same kind of dense fp64 work).
    Returns (step TFLOP/s = (fwd + bwd FLOPs of a step) / (the time the oracle would take for
    them at the two measured rates), fwd TFLOP/s, bwd TFLOP/s, description, threads, seconds)."""
    import numpy as np

    from oracle import cowa_oracle as orc
    from structured_sparse_attention_cowa_b200 import synth

    c = TRAIN
    pat = orc.Pattern(S=c["S"], L=c["L"], T=c["T"], D=c["D"])
    rng = np.random.default_rng(99 + seed_extra)
    Hkv, Hq, d, N = c["Hkv"], c["Hq"], c["d"], c["N"]
    grp = Hq // Hkv

    class Rows:
        """A seeded bf16 tensor widened to float64 on access (the oracle reads slices)."""

        def __init__(self, name, H):
            self.bits = synth.normal_bf16_bits((1, N, H, d), synth.seed_of(name, seed_extra))
            self.shape = self.bits.shape

        def __getitem__(self, idx):
            return orc.bf16_bits_to_f64(self.bits[idx])

    if seed_extra not in _KV_CACHE:  # generated once per seed, outside the timed parts
        _KV_CACHE[seed_extra] = (Rows("k", Hkv), Rows("v", Hkv))
    k, v = _KV_CACHE[seed_extra]

    class QRows:
        """Query-side rows (q, dO) drawn per accessed block of rows and head: only the sampled
        rows are ever generated (a few milliseconds per block, against the oracle's ~0.1 s)."""

        shape = (1, N, Hq, d)

        def __init__(self, name):
            self.seed = synth.seed_of(name, seed_extra)

        def __getitem__(self, idx):
            _, rows, h, _ = idx
            rows = np.atleast_1d(rows)
            return orc.bf16_bits_to_f64(synth.normal_bf16_bits((len(rows), d), self.seed + 7919 * int(rows[0]) + h))

    q, do = QRows("q"), QRows("do")

    def row_pairs(rows):
        return sum(int(orc.visible_mask(rows, int(rows[-1]) + 1, pat, g, Hkv).sum()) for g in range(Hkv)) * grp

    f_flop = f_t = b_flop = b_t = 0.0
    nf = nb = 0
    while (f_t + b_t) < target_s and nf + nb < 1024:
        t0 = int(rng.integers(0, N - 32))
        rows = np.arange(t0, t0 + 32)
        st = time.perf_counter()
        if f_t <= b_t:
            orc.attention_fwd_rows(q, k, v, pat, rows, b=0)
            f_t += time.perf_counter() - st
            f_flop += 4.0 * d * row_pairs(rows)
            nf += 1
        else:
            orc.attention_bwd_rows(q, k, v, do, pat, rows, b=0)
            b_t += time.perf_counter() - st
            b_flop += 6.0 * d * row_pairs(rows)
            nb += 1
    try:
        from threadpoolctl import threadpool_info

        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        threads = os.cpu_count() or 1
    f_rate, b_rate = f_flop / f_t, b_flop / b_t
    pairs = visible_pairs(N, c["S"], c["L"], c["T"], c["D"], Hkv, Hq, c["B"])
    step_flop = 14.0 * d * pairs
    step_s = 4.0 * d * pairs / f_rate + 10.0 * d * pairs / b_rate
    desc = (f"oracle (fp64 numpy, explicit mask) on the 32K layer, all {Hq} query heads: forward of {nf} "
            f"random 32-row blocks (4*d per visible pair) and the row-local backward (S, dP, dS, dQ) of {nb} "
            f"random 32-row blocks (6*d per pair); value = a step's visible FLOPs (fwd 4*d + bwd 10*d per "
            f"pair) over the time the oracle takes for them at those two rates")
    return step_flop / step_s / 1e12, f_rate / 1e12, b_rate / 1e12, desc, threads, f_t + b_t


# ------------------------------------------------------------------------------ other configurations
# (key, B, N, Hq, Hkv, d, S, L, T, D, time the backward too, in the default report)
CONFIGS = [
    ("train_32k", 1, 32768, 40, 8, 128, 128, 2048, 32768, 8, True, True),
    ("train_32k_dense_causal", 1, 32768, 40, 8, 128, 128, 32768, 32768, 8, True, True),
    ("train_32k_swa_sinks", 1, 32768, 40, 8, 128, 128, 2048, 128, 8, True, True),
    ("long_128k", 1, 131072, 40, 8, 128, 128, 4096, 131072, 8, True, True),
    ("long_128k_dense_causal", 1, 131072, 40, 8, 128, 128, 131072, 131072, 8, True, True),
    ("prefill_8k_D8", 2, 8192, 32, 8, 128, 128, 1024, 8192, 8, True, False),
    ("prefill_8k_D4", 2, 8192, 32, 8, 128, 128, 1024, 8192, 4, False, False),
    ("prefill_8k_D2", 2, 8192, 32, 8, 128, 128, 1024, 8192, 2, False, False),
    ("prefill_8k_D1", 2, 8192, 32, 8, 128, 128, 1024, 8192, 1, False, False),
]


def config_parts(dev, kc, vc, peak_tf, hbm_gbs, sweep=False, reps=2):
    """Each kernel alone (CUDA events, median of `reps` after one warm-up; fractions of the
    measured burst bf16 peak and of the HBM copy rate) on the other configurations: the 32K
    layer itself, its dense-causal mode (L >= T, the FullAttn comparison) and SWA + sinks
    (T = S), the 128K layer and its dense-causal mode, and the 128K decode over the full
    cache, in the dense-causal mode, over the compacted cache and over E4M3 caches; `sweep`
    adds the 8K prefill D sweep.  The decodes run first (before the long training kernels warm the
    GPU into its power-capped state).  Returns {key: row}."""
    import ctypes

    import torch

    from structured_sparse_attention_cowa_b200 import cowa as cw
    from structured_sparse_attention_cowa_b200 import synth

    out = {}

    def timed(fn, inner=1):
        """Median over `reps` of the per-call time of `inner` back-to-back calls between one pair
        of events (inner > 1 for sub-millisecond calls, so that host launch gaps between the
        calls overlap the device work instead of being timed)."""
        fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(max(1, reps)):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(inner):
                fn()
            b.record(); torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) / inner)
        return statistics.median(ts)

    # decode at 128K (B = 16, pos = 131071): the CoWA pattern over the full cache, the
    # dense-causal mode (every cached token up to pos visible), the CoWA pattern over the
    # compacted cache, and over E4M3 caches (full and compacted) quantised from the same values;
    # all timed alike: explicit workspaces, 10 back-to-back calls per event pair
    dc = DECODE
    L_ = cw.lib()
    qt = synth.cuda_normal_bf16((dc["B"], dc["Hq"], dc["d"]), synth.seed_of("q_t"), dev)
    pos = torch.full((dc["B"],), dc["pos"], dtype=torch.int32, device=dev)
    od = torch.empty((dc["B"], dc["Hq"], dc["d"]), dtype=torch.bfloat16, device=dev)
    lsed = torch.empty((dc["B"], dc["Hq"]), dtype=torch.float32, device=dev)
    ws_of = lambda n: torch.zeros(max(256, n), dtype=torch.uint8, device=dev)
    pat_c = cw.Pattern(dc["S"], dc["L"], dc["T"], dc["D"])
    toks = decode_visible_tokens(dc["pos"], dc["S"], dc["L"], dc["T"], dc["D"], dc["Hkv"])
    vbytes = float(sum(toks)) * dc["B"] * dc["d"] * 2 * 2
    shape = (dc["B"], dc["Hq"], dc["Hkv"], dc["d"], dc["T_cap"])
    wss = []

    def dec_row(key, ms, nbytes, **extra):
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[key] = {"B": dc["B"], "pos": dc["pos"], "decode_ms": ms, "bytes": nbytes, "decode_gbs": gbs,
                    "decode_frac_hbm": gbs / hbm_gbs, **extra}

    ws_c = ws_of(L_.cowa_decode_workspace_size(ctypes.byref(pat_c.c()), *shape)); wss.append(ws_c)
    ms = timed(lambda: cw.cowa_decode(qt, kc, vc, pos, pat_c, out=od, lse=lsed, workspace=ws_c), inner=10)
    dec_row("decode_128k", ms, vbytes)
    full_ms = ms

    dpat = cw.Pattern(dc["S"], dc["T"], dc["T"], dc["D"])
    ws_dd = ws_of(L_.cowa_decode_workspace_size(ctypes.byref(dpat.c()), *shape)); wss.append(ws_dd)
    ms = timed(lambda: cw.cowa_decode(qt, kc, vc, pos, dpat, out=od, lse=lsed, workspace=ws_dd), inner=10)
    dec_row("decode_128k_dense_causal", ms, float(dc["pos"] + 1) * dc["B"] * dc["Hkv"] * dc["d"] * 2 * 2,
            cowa_speedup=ms / full_ms)

    kc_c, vc_c = cw.compact_cache(kc.transpose(1, 2), vc.transpose(1, 2), pat_c)
    rows = cw.compact_rows(pat_c, dc["Hkv"])
    ws_k = ws_of(L_.cowa_decode_compact_workspace_size(ctypes.byref(pat_c.c()), *shape[:4])); wss.append(ws_k)
    ms = timed(lambda: cw.cowa_decode_compact(qt, kc_c, vc_c, pos, pat_c, out=od, lse=lsed, workspace=ws_k),
               inner=10)
    cache_full = 2.0 * dc["B"] * dc["Hkv"] * dc["T_cap"] * dc["d"] * 2
    dec_row("decode_128k_compact", ms, vbytes, cache_rows_per_head=rows, cache_bytes=cache_full * rows / dc["T_cap"],
            full_cache_bytes=cache_full)
    del kc_c, vc_c

    # E4M3 caches: one scale per tensor (the inputs are N(0,1): |x| < 7 maps below 448 at 1/64)
    scale = 1.0 / 64
    kq, vq = cw.quantize_e4m3(kc, scale), cw.quantize_e4m3(vc, scale)
    ws_8 = ws_of(L_.cowa_decode_fp8_workspace_size(ctypes.byref(pat_c.c()), *shape)); wss.append(ws_8)
    ms = timed(lambda: cw.cowa_decode_fp8(qt, kq, vq, pos, pat_c, scale, scale, out=od, lse=lsed, workspace=ws_8),
               inner=10)
    dec_row("decode_128k_e4m3", ms, vbytes / 2, bf16_decode_ms=full_ms, cache_bytes=cache_full / 2)
    k8c, v8c = cw.compact_cache_fp8(kq.transpose(1, 2), vq.transpose(1, 2), pat_c)
    del kq, vq
    ws_8c = ws_of(L_.cowa_decode_fp8_compact_workspace_size(ctypes.byref(pat_c.c()), *shape[:4])); wss.append(ws_8c)
    ms = timed(lambda: cw.cowa_decode_fp8_compact(qt, k8c, v8c, pos, pat_c, scale, scale, out=od, lse=lsed,
                                                  workspace=ws_8c), inner=10)
    dec_row("decode_128k_e4m3_compact", ms, vbytes / 2, cache_bytes=cache_full * rows / dc["T_cap"] / 2)
    del k8c, v8c
    for w in wss:
        if cw.workspace_status(w) != 0:
            raise RuntimeError("device status set in the decode configurations")
    torch.cuda.empty_cache()

    for key, B, N, Hq, Hkv, d, S, L, T, D, do_bwd, default in CONFIGS:
        if not (default or sweep):
            continue
        pat = cw.Pattern(S, L, T, D)
        q = synth.cuda_normal_bf16((B, N, Hq, d), synth.seed_of("q"), dev)
        k = synth.cuda_normal_bf16((B, N, Hkv, d), synth.seed_of("k"), dev)
        v = synth.cuda_normal_bf16((B, N, Hkv, d), synth.seed_of("v"), dev)
        o = torch.empty_like(q)
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
        n_ws = cw.lib().cowa_fwd_workspace_size(ctypes.byref(pat.c()), B, N, Hq, Hkv, d)
        ws_f = torch.zeros(max(256, n_ws), dtype=torch.uint8, device=dev)
        pairs = visible_pairs(N, S, L, T, D, Hkv, Hq, B)
        f_ms = timed(lambda: cw.cowa_fwd(q, k, v, pat, out=o, lse=lse, workspace=ws_f))
        row = {"B": B, "N": N, "Hq": Hq, "Hkv": Hkv, "d": d, "S": S, "L": L, "T": T, "D": D,
               "visible_pairs": pairs, "fwd_ms": f_ms, "fwd_tflops": 4.0 * d * pairs / (f_ms * 1e-3) / 1e12}
        row["fwd_frac_burst"] = row["fwd_tflops"] / peak_tf
        if do_bwd:
            do = synth.cuda_normal_bf16((B, N, Hq, d), synth.seed_of("do"), dev)
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
            n = cw.lib().cowa_bwd_workspace_size(ctypes.byref(pat.c()), B, N, Hq, Hkv, d)
            ws = torch.zeros(n, dtype=torch.uint8, device=dev)
            stage = lambda st: cw.cowa_bwd(q, k, v, o, lse, do, pat, dq=dq, dk=dk, dv=dv, workspace=ws, stages=st)
            st_ms = {nm: timed(lambda st=st: stage(st)) for nm, st in
                     (("preprocess", cw.BWD_PREPROCESS), ("dkdv", cw.BWD_DKDV), ("dq", cw.BWD_DQ))}
            b_ms = sum(st_ms.values())
            row.update({"bwd_ms": b_ms, "bwd_stages_ms": st_ms, "bwd_tflops": 10.0 * d * pairs / (b_ms * 1e-3) / 1e12})
            row["bwd_frac_burst"] = row["bwd_tflops"] / peak_tf
            if cw.workspace_status(ws) != 0:
                raise RuntimeError(f"device status set in configuration {key}")
            del do, dq, dk, dv, ws
        if cw.workspace_status(ws_f) != 0:
            raise RuntimeError(f"device status set in configuration {key}")
        out[key] = row
        del q, k, v, o, lse, ws_f
        torch.cuda.empty_cache()
    for key in ("train_32k_dense_causal", "long_128k_dense_causal"):
        base = key.replace("_dense_causal", "")
        if key in out and base in out:  # CoWA against the dense-causal mode of the same kernels
            out[key]["cowa_fwd_speedup"] = out[key]["fwd_ms"] / out[base]["fwd_ms"]
            if "bwd_ms" in out[key] and "bwd_ms" in out[base]:
                out[key]["cowa_bwd_speedup"] = out[key]["bwd_ms"] / out[base]["bwd_ms"]

    return out


# ------------------------------------------------------------------------------ KV-head TP
class TpRank:
    """One rank's share of the layer under KV-head tensor parallelism (--shard heads).

    The rank owns runs of consecutive global KV heads (`shard.kv_head_runs`); per run it holds its
    own q, k, v, dO (the run's query heads and KV heads), outputs, decode cache and workspaces,
    and each call passes kv_head_base = the run's first global head and h_kv_global = the layer's
    KV-head count, so that its intervals are the ones those heads have in the whole layer."""

    def __init__(self, cw, synth, torch, dev, rank: int, world: int, order: str, c=None, dc=None):
        import ctypes

        from structured_sparse_attention_cowa_b200 import shard

        c, dc = c or TRAIN, dc or DECODE
        H, grp, B, N, d = c["Hkv"], c["Hq"] // c["Hkv"], c["B"], c["N"], c["d"]
        self.cw = cw
        self.runs = shard.kv_head_runs(rank, world, H, grp, order)
        lib = cw.lib()
        self.bufs = []
        for run in self.runs:
            nq, nk = run.n * grp, run.n
            ex = 100 + run.G0  # each run's heads draw their own inputs
            pat = shard.run_pattern(cw.Pattern(c["S"], c["L"], c["T"], c["D"]), run, H)
            dpat = shard.run_pattern(cw.Pattern(dc["S"], dc["L"], dc["T"], dc["D"]), run, H)
            rnd = lambda shape, name: synth.cuda_normal_bf16(shape, synth.seed_of(name, ex), dev)
            b = {"run": run, "pat": pat, "dpat": dpat,
                 "q": rnd((B, N, nq, d), "q"), "k": rnd((B, N, nk, d), "k"), "v": rnd((B, N, nk, d), "v"),
                 "do": rnd((B, N, nq, d), "do"),
                 "kc": rnd((dc["B"], nk, dc["T_cap"], dc["d"]), "k_cache"),
                 "vc": rnd((dc["B"], nk, dc["T_cap"], dc["d"]), "v_cache"),
                 "qt": rnd((dc["B"], nq, dc["d"]), "q_t"),
                 "pos": torch.full((dc["B"],), dc["pos"], dtype=torch.int32, device=dev)}
            b["o"] = torch.empty_like(b["q"])
            b["lse"] = torch.empty((B, nq, N), dtype=torch.float32, device=dev)
            b["dq"], b["dk"], b["dv"] = torch.empty_like(b["q"]), torch.empty_like(b["k"]), torch.empty_like(b["v"])
            b["od"] = torch.empty((dc["B"], nq, dc["d"]), dtype=torch.bfloat16, device=dev)
            b["lsed"] = torch.empty((dc["B"], nq), dtype=torch.float32, device=dev)
            cp, cpd = pat.c(), dpat.c()
            ws = lambda n: torch.zeros(max(256, n), dtype=torch.uint8, device=dev)
            b["ws_f"] = ws(lib.cowa_fwd_workspace_size(ctypes.byref(cp), B, N, nq, nk, d))
            n_b = lib.cowa_bwd_workspace_size(ctypes.byref(cp), B, N, nq, nk, d)
            b["ws_b"] = ws(n_b)
            # a workspace larger than header + row statistics means the call splits its long key
            # tiles: two more launches (the chunk table and the reduction of the partials)
            stats = 256 + (2 * B * nq * ((N + 127) // 128 * 128) * 4 + 255) // 256 * 256
            b["split"] = n_b > stats
            b["ws_d"] = ws(lib.cowa_decode_workspace_size(ctypes.byref(cpd), dc["B"], nq, nk, dc["d"], dc["T_cap"]))
            self.bufs.append(b)

    def fwd(self):
        for b in self.bufs:
            self.cw.cowa_fwd(b["q"], b["k"], b["v"], b["pat"], out=b["o"], lse=b["lse"], workspace=b["ws_f"])

    def bwd(self):
        for b in self.bufs:
            self.cw.cowa_bwd(b["q"], b["k"], b["v"], b["o"], b["lse"], b["do"], b["pat"], dq=b["dq"], dk=b["dk"],
                             dv=b["dv"], workspace=b["ws_b"])

    def dec(self):
        for b in self.bufs:
            self.cw.cowa_decode(b["qt"], b["kc"], b["vc"], b["pos"], b["dpat"], out=b["od"], lse=b["lsed"],
                                workspace=b["ws_d"])

    def statuses(self):
        return [self.cw.workspace_status(b[w]) for b in self.bufs for w in ("ws_f", "ws_b", "ws_d")]

    @property
    def launches_per_step(self) -> int:
        # per run: forward 1, backward 3 (+ 2 when it splits long key tiles), decode 2
        return sum(6 + (2 if b["split"] else 0) for b in self.bufs)


def tp_projection(P: int, order: str, steps: int, warmup: int, dev) -> dict:
    """KV-head tensor parallelism projected on one GPU (a `parts` entry of the default line): the
    P ranks' calls (the 32K layer's fwd + bwd and the 128K decode, split by KV head) run one rank
    after another; with no exchange step each rank's time is the time it would take on its own
    GPU, so the slowest rank's time is the P-GPU step."""
    import torch

    from structured_sparse_attention_cowa_b200 import cowa as cw
    from structured_sparse_attention_cowa_b200 import synth

    rank_ms = []
    for r in range(P):
        tr = TpRank(cw, synth, torch, dev, r, P, order)
        for _ in range(warmup):
            tr.fwd(); tr.bwd(); tr.dec()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            tr.fwd(); tr.bwd(); tr.dec()
        b.record()
        torch.cuda.synchronize()
        bad = [x for x in tr.statuses() if x != 0]
        if bad:
            raise RuntimeError(f"device status {bad[0]} in the TP projection (rank {r})")
        rank_ms.append(a.elapsed_time(b) / steps)
        del tr
        torch.cuda.empty_cache()
    return {"P": P, "order": order, "projected_step_ms": max(rank_ms), "rank_ms": rank_ms,
            "slowest_over_mean": max(rank_ms) / statistics.mean(rank_ms),
            "note": "ranks run in turn on this GPU; the slowest rank's time is the P-GPU step"}


def run_cowa_tp(args, world, rank, local):
    """--shard heads: the whole 32K layer and the whole 128K decode batch split by KV head over P
    ranks (strong scaling), each rank's calls over its own runs of global KV heads.  Under
    torchrun every process is one rank (P = WORLD_SIZE) and the step time is the max over ranks.
    In one process, --tp-ranks P runs the P ranks' calls one rank after another on the one GPU:
    the op has no exchange step, so each rank's device time there is the time it would take on
    its own GPU, and `tp.projected` gives the P-GPU step as the slowest rank's time; `value` stays
    what the one GPU did (all the work over the sum of the ranks' times)."""
    import torch

    from structured_sparse_attention_cowa_b200 import cowa as cw
    from structured_sparse_attention_cowa_b200 import shard, synth

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    P = world if world > 1 else max(1, args.tp_ranks)
    my_ranks = [rank] if world > 1 else list(range(P))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    c, dc = TRAIN, DECODE
    H, grp = c["Hkv"], c["Hq"] // c["Hkv"]
    K, W = args.steps, max(3, args.warmup)

    def barrier():
        if dist is not None:
            dist.barrier()

    rows, launches = [], 0
    with ClockSampler(local) as clk:
        for r in my_ranks:
            tr = TpRank(cw, synth, torch, dev, r, P, args.shard_order)
            for _ in range(W):
                tr.fwd(); tr.bwd(); tr.dec()
            torch.cuda.synchronize()
            ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier()
            torch.cuda.synchronize()
            a.record()
            for s in range(K):
                e = ev[s]
                e[0].record(); tr.fwd()
                e[1].record(); tr.bwd()
                e[2].record(); tr.dec()
                e[3].record()
            b.record()
            torch.cuda.synchronize()
            barrier()
            bad = [x for x in tr.statuses() if x != 0]
            if bad:
                raise RuntimeError(f"device status {bad[0]} after the timed region (rank {r})")
            avg = lambda i, j: statistics.mean(e[i].elapsed_time(e[j]) for e in ev)
            pairs = shard.rank_visible_pairs(cw.Pattern(c["S"], c["L"], c["T"], c["D"]), r, P, H, grp, c["N"],
                                             c["B"], args.shard_order)
            rows.append({"rank": r, "runs": [[x.G0, x.n] for x in tr.runs], "ms": a.elapsed_time(b) / K,
                         "fwd_ms": avg(0, 1), "bwd_ms": avg(1, 2), "decode_ms": avg(2, 3),
                         "visible_pairs": pairs})
            launches += K * tr.launches_per_step
            del tr
            torch.cuda.empty_cache()

    step_ms = max_over_ranks(max(x["ms"] for x in rows), dist, dev)
    pairs_all = visible_pairs(c["N"], c["S"], c["L"], c["T"], c["D"], c["Hkv"], c["Hq"], c["B"])
    flop = 14.0 * c["d"] * pairs_all  # forward 4*d + backward 10*d per visible pair, the whole layer
    if dist is not None:
        gathered = [None] * world
        dist.all_gather_object(gathered, rows)
        rows = [x for part in gathered for x in part]
        dist.destroy_process_group()
    if rank != 0:
        return 0
    rank_ms = [x["ms"] for x in rows]
    rank_pairs = [x["visible_pairs"] for x in rows]
    if world > 1:
        value, ms_line = flop / (step_ms * 1e-3) / 1e12, step_ms
    else:
        ms_line = sum(rank_ms)
        value = flop / (ms_line * 1e-3) / 1e12
    tp = {"order": args.shard_order, "P": P, "ranks": rows,
          "balance_pairs": statistics.mean(rank_pairs) / max(rank_pairs),
          "balance_ms": statistics.mean(rank_ms) / max(rank_ms)}
    if world == 1 and P > 1:
        tp["projected"] = {"step_ms": max(rank_ms), "tflops": flop / (max(rank_ms) * 1e-3) / 1e12,
                           "note": "each rank on its own GPU: the slowest rank's time (no exchange step)"}
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": ms_line, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "train 32K layer fwd+bwd + decode 128K cache, whole layer split by KV head",
                       "train": TRAIN, "decode": DECODE, "l2": "inputs larger than L2 (126 MB); no flush",
                       "parallelism": f"kv-head TP x{P} ({args.shard_order})" + (", ranks run in turn on one GPU"
                                                                                 if world == 1 and P > 1 else "")},
            "tp": tp, "roofline": None, "e2e": None, "cpu_baseline": None, "gpu_launches": launches,
            "clocks": clk.summary()}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="cowa", choices=["cowa", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-outputs", default="all", choices=["results", "all"],
                    help="all (default): every step copies o, lse, dq, dk, dv and the decode output/lse back to "
                         "the host, and the line also gives the results-only figure; results: only the forward "
                         "lse and the decode output/lse (o, dq, dk, dv stay on the device as in training)")
    ap.add_argument("--no-parts", action="store_true",
                    help="skip the other configurations (dense-causal mode, SWA + sinks, 128K layer, decode "
                         "variants) that the line reports under 'parts'")
    ap.add_argument("--shard", default="batch", choices=["batch", "heads"],
                    help="batch: every rank runs the per-GPU workload on its own batch element (weak scaling); "
                         "heads: the one layer split by KV head over the ranks (strong scaling, see run_cowa_tp)")
    ap.add_argument("--shard-order", default="folded", choices=["folded", "contiguous"],
                    help="--shard heads: which global KV heads each rank owns (shard.head_owner)")
    ap.add_argument("--tp-ranks", type=int, default=1,
                    help="--shard heads in one process: run this many ranks' calls in turn on the one GPU")
    ap.add_argument("--sweep", action="store_true", help="also time the 8K prefill D sweep (one GPU only)")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, world, rank)
    if args.shard == "heads":
        return run_cowa_tp(args, world, rank, local)
    return run_cowa(args, world, rank, local)


def run_reference(args, world, rank):
    """The reference arm: the fp64 oracle (test infrastructure) on the host cores, on bounded
    samples of the same 32K layer (cpu_oracle_sample), one sample per step; rank 0 only."""
    if rank != 0:
        return 0
    steps, warm = max(1, args.steps), max(0, args.warmup)
    per = max(1.0, min(20.0, 120.0 / (steps + warm)))
    vals = []
    for i in range(warm + steps):
        v, f_cpu, b_cpu, desc, threads, used = cpu_oracle_sample(per, seed_extra=i % 3)
        if i >= warm:
            vals.append((v, f_cpu, b_cpu, used))
    value = statistics.median(x[0] for x in vals)
    ms = statistics.mean(x[3] for x in vals) * 1e3
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": steps, "warmup": warm, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "train 32K layer fwd+bwd, oracle on row samples", **TRAIN},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc,
                             "fwd_tflops": statistics.median(x[1] for x in vals),
                             "bwd_tflops": statistics.median(x[2] for x in vals)},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_cowa(args, world, rank, local):
    import torch

    from structured_sparse_attention_cowa_b200 import cowa as cw
    from structured_sparse_attention_cowa_b200 import synth

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    c, dc = TRAIN, DECODE
    pat = cw.Pattern(c["S"], c["L"], c["T"], c["D"])
    dpat = cw.Pattern(dc["S"], dc["L"], dc["T"], dc["D"])

    # ---- inputs (per rank: its own batch element / seeds), outputs, workspaces
    ex = rank_seed_extra(rank)
    q = synth.cuda_normal_bf16((c["B"], c["N"], c["Hq"], c["d"]), synth.seed_of("q", ex), dev)
    k = synth.cuda_normal_bf16((c["B"], c["N"], c["Hkv"], c["d"]), synth.seed_of("k", ex), dev)
    v = synth.cuda_normal_bf16((c["B"], c["N"], c["Hkv"], c["d"]), synth.seed_of("v", ex), dev)
    do = synth.cuda_normal_bf16((c["B"], c["N"], c["Hq"], c["d"]), synth.seed_of("do", ex), dev)
    kc = synth.cuda_normal_bf16((dc["B"], dc["Hkv"], dc["T_cap"], dc["d"]), synth.seed_of("k_cache", ex), dev)
    vc = synth.cuda_normal_bf16((dc["B"], dc["Hkv"], dc["T_cap"], dc["d"]), synth.seed_of("v_cache", ex), dev)
    qt = synth.cuda_normal_bf16((dc["B"], dc["Hq"], dc["d"]), synth.seed_of("q_t", ex), dev)
    pos = torch.full((dc["B"],), dc["pos"], dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((c["B"], c["Hq"], c["N"]), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    od = torch.empty((dc["B"], dc["Hq"], dc["d"]), dtype=torch.bfloat16, device=dev)
    lsed = torch.empty((dc["B"], dc["Hq"]), dtype=torch.float32, device=dev)
    import ctypes

    L = cw.lib()
    cp = pat.c()
    cpd = dpat.c()
    ws_f = torch.zeros(max(256, L.cowa_fwd_workspace_size(ctypes.byref(cp), c["B"], c["N"], c["Hq"], c["Hkv"], c["d"])),
                       dtype=torch.uint8, device=dev)
    ws_b = torch.zeros(L.cowa_bwd_workspace_size(ctypes.byref(cp), c["B"], c["N"], c["Hq"], c["Hkv"], c["d"]),
                       dtype=torch.uint8, device=dev)
    ws_d = torch.zeros(L.cowa_decode_workspace_size(ctypes.byref(cpd), dc["B"], dc["Hq"], dc["Hkv"], dc["d"],
                                                    dc["T_cap"]), dtype=torch.uint8, device=dev)

    def fwd():
        cw.cowa_fwd(q, k, v, pat, out=o, lse=lse, workspace=ws_f)

    def bwd_stage(st):
        cw.cowa_bwd(q, k, v, o, lse, do, pat, dq=dq, dk=dk, dv=dv, workspace=ws_b, stages=st)

    def bwd():
        cw.cowa_bwd(q, k, v, o, lse, do, pat, dq=dq, dk=dk, dv=dv, workspace=ws_b)

    def dec():
        cw.cowa_decode(qt, kc, vc, pos, dpat, out=od, lse=lsed, workspace=ws_d)

    def barrier():
        if dist is not None:
            dist.barrier()

    def maxr(x: float) -> float:
        return max_over_ranks(x, dist, dev)

    # ---- warm-up
    for _ in range(max(3, args.warmup)):
        fwd(); bwd(); dec()
    torch.cuda.synchronize()

    # ---- timed region: K steps, events between the calls (the backward as its three stages,
    # each one kernel, so that every hot kernel gets its own device time)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(K)]
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        e_start.record()
        for s in range(K):
            e = ev[s]
            e[0].record(); fwd()
            e[1].record(); bwd_stage(cw.BWD_PREPROCESS)
            e[2].record(); bwd_stage(cw.BWD_DKDV)
            e[3].record(); bwd_stage(cw.BWD_DQ)
            e[4].record(); dec()
            e[5].record()
        e_end.record()
        torch.cuda.synchronize()
        barrier()
    total_ms = maxr(e_start.elapsed_time(e_end))
    avg = lambda a_, b_: statistics.mean(e[a_].elapsed_time(e[b_]) for e in ev)
    fwd_ms, pre_ms, dkdv_ms, dq_ms, dec_ms = avg(0, 1), avg(1, 2), avg(2, 3), avg(3, 4), avg(4, 5)
    bwd_ms = pre_ms + dkdv_ms + dq_ms
    for st in (cw.workspace_status(ws_f), cw.workspace_status(ws_b), cw.workspace_status(ws_d)):
        if st != 0:
            raise RuntimeError(f"device status {st} after the timed region")

    pairs = visible_pairs(c["N"], c["S"], c["L"], c["T"], c["D"], c["Hkv"], c["Hq"], c["B"])
    fwd_flop = 4.0 * c["d"] * pairs
    bwd_flop = 10.0 * c["d"] * pairs
    toks = decode_visible_tokens(dc["pos"], dc["S"], dc["L"], dc["T"], dc["D"], dc["Hkv"])
    dec_bytes = float(sum(toks)) * dc["B"] * dc["d"] * 2 * 2  # K and V rows, bf16
    ms_step = total_ms / K
    value = aggregate_tflops(world, fwd_flop + bwd_flop, ms_step)

    burst, sustained, hbm, peak_src = _peaks()
    parts = {
        "fwd": {"ms": fwd_ms, "tflops_visible": fwd_flop / (fwd_ms * 1e-3) / 1e12},
        "bwd": {"ms": bwd_ms, "tflops_visible": bwd_flop / (bwd_ms * 1e-3) / 1e12,
                "stages_ms": {"preprocess": pre_ms, "dkdv": dkdv_ms, "dq": dq_ms}},
        "decode": {"ms": dec_ms, "gbs_visible": dec_bytes / (dec_ms * 1e-3) / 1e9,
                   "frac_hbm": dec_bytes / (dec_ms * 1e-3) / 1e9 / hbm, "visible_bytes": dec_bytes},
    }
    for p in ("fwd", "bwd"):
        parts[p]["frac_peak"] = parts[p]["tflops_visible"] / burst

    # ---- roofline of the dominant kernel (longest device time in the step).  Algorithmic work per
    # launch: forward 2 GEMMs (4*d per visible pair), dK/dV 4 GEMMs (S^T, dP^T, dV, dK: 8*d per
    # pair), dQ 3 GEMMs (S, dP, dQ: 6*d per pair), decode the visible K/V bytes once.
    kernels = {
        "cowa_fwd_kernel<128>": (fwd_ms, fwd_flop, "tensor", "cowa_fwd.cu", "4*d"),
        "bwd_dkdv_kernel<128>": (dkdv_ms, 8.0 * c["d"] * pairs, "tensor", "cowa_bwd.cu", "8*d"),
        "bwd_dq_kernel<128>": (dq_ms, 6.0 * c["d"] * pairs, "tensor", "cowa_bwd.cu", "6*d"),
        "decode_split_kernel<5,128>": (dec_ms, dec_bytes, "hbm", "cowa_decode.cu", None),
    }
    top = max(kernels, key=lambda kname: kernels[kname][0])
    t_ms, work, bound, src, per = kernels[top]
    if bound == "tensor":
        achieved = work / (t_ms * 1e-3) / 1e12
        roofline = {"kernel": top, "bound": "tensor", "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                    "frac": achieved / burst, "frac_of_sustained": achieved / sustained,
                    "traffic": _traffic_record(top, src),
                    "peak_source": f"{peak_src} bf16 dense, burst (the timed region is under a second)",
                    "algorithmic": f"{work:.4e} FLOP per launch = {per} x visible pairs ({pairs:.4e})"}
    else:
        achieved = work / (t_ms * 1e-3) / 1e9
        roofline = {"kernel": top, "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                    "frac": achieved / hbm, "traffic": _traffic_record(top, src),
                    "peak_source": f"{peak_src} HBM copy",
                    "algorithmic": f"{work:.4e} visible K/V bytes per call"}
    roofline["all_kernels_ms"] = {kname: v[0] for kname, v in kernels.items()}

    # ---- end to end: host buffers, copies inside the timed region.  Every step copies its inputs
    # (q, k, v, dO of the layer, q_t and pos of the decode; the KV cache is resident device state)
    # in from pinned host memory and reads its results back into pinned host memory: by default
    # every result (o, lse, dq, dk, dv and the decode output and lse); the line also gives the
    # figure with only the results a host reads in training and serving (the forward's lse, the
    # per-row log-partition a loss is formed from, and the decode output and lse), o, dq, dk, dv
    # staying on the device for the next layer and the optimizer.  Steps are pipelined the way a
    # training or serving loop prefetches:
    # three streams (copy-in, compute, copy-out) and two device buffer sets, so step i+1's
    # inputs land while step i computes and step i's results leave while step i+1 computes.
    # Within a step the forward starts once q, k, v are in (dO lands meanwhile).
    e2e = None
    if not args.no_e2e:
        pin = lambda t: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        names_in = ("q", "k", "v", "do", "qt")
        h_in = {n: pin(x) for n, x in zip(names_in, (q, k, v, do, qt))}
        for n, x in zip(names_in, (q, k, v, do, qt)):
            h_in[n].copy_(x)
        h_pos = pos.cpu().pin_memory()

        def run_e2e(all_out):
            names_out = ("lse", "od", "lsed") + (("o", "dq", "dk", "dv") if all_out else ())
            dev_out = {"lse": lse, "od": od, "lsed": lsed, "o": o, "dq": dq, "dk": dk, "dv": dv}
            h_out = {n: pin(dev_out[n]) for n in names_out}
            h2d = sum(x.numel() * x.element_size() for x in h_in.values()) + h_pos.numel() * 4
            d2h = sum(x.numel() * x.element_size() for x in h_out.values())

            def buffer_set():
                st = {n: torch.empty_like(x) for n, x in zip(names_in + ("pos",), (q, k, v, do, qt, pos))}
                st.update({n: torch.empty_like(x) for n, x in dev_out.items()})
                st.update({n: torch.zeros_like(x) for n, x in (("ws_f", ws_f), ("ws_b", ws_b), ("ws_d", ws_d))})
                return st

            sets = [buffer_set(), buffer_set()]
            s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
            inputs_free = [None, None]   # compute of the step that last used the set has read its inputs
            outputs_free = [None, None]  # copy-out of the step that last used the set is done
            new_ev = lambda: torch.cuda.Event()

            def e2e_step(i):
                st = sets[i % 2]
                j = i % 2
                with torch.cuda.stream(s_in):
                    if inputs_free[j] is not None:
                        s_in.wait_event(inputs_free[j])
                    for n in ("q", "k", "v"):
                        st[n].copy_(h_in[n], non_blocking=True)
                    e_qkv = new_ev(); e_qkv.record(s_in)
                    st["do"].copy_(h_in["do"], non_blocking=True)
                    e_do = new_ev(); e_do.record(s_in)
                    st["qt"].copy_(h_in["qt"], non_blocking=True)
                    st["pos"].copy_(h_pos, non_blocking=True)
                    e_dec_in = new_ev(); e_dec_in.record(s_in)
                with torch.cuda.stream(s_cmp):
                    s_cmp.wait_event(e_qkv)
                    if outputs_free[j] is not None:
                        s_cmp.wait_event(outputs_free[j])
                    cw.cowa_fwd(st["q"], st["k"], st["v"], pat, out=st["o"], lse=st["lse"], workspace=st["ws_f"])
                    e_fwd = new_ev(); e_fwd.record(s_cmp)
                    s_cmp.wait_event(e_do)
                    cw.cowa_bwd(st["q"], st["k"], st["v"], st["o"], st["lse"], st["do"], pat, dq=st["dq"], dk=st["dk"],
                                dv=st["dv"], workspace=st["ws_b"])
                    e_bwd = new_ev(); e_bwd.record(s_cmp)
                    s_cmp.wait_event(e_dec_in)
                    cw.cowa_decode(st["qt"], kc, vc, st["pos"], dpat, out=st["od"], lse=st["lsed"], workspace=st["ws_d"])
                    e_cmp = new_ev(); e_cmp.record(s_cmp)
                    inputs_free[j] = e_cmp
                with torch.cuda.stream(s_out):
                    s_out.wait_event(e_fwd)
                    h_out["lse"].copy_(st["lse"], non_blocking=True)
                    if all_out:
                        h_out["o"].copy_(st["o"], non_blocking=True)
                    s_out.wait_event(e_bwd)
                    if all_out:
                        for n in ("dq", "dk", "dv"):
                            h_out[n].copy_(st[n], non_blocking=True)
                    s_out.wait_event(e_cmp)
                    h_out["od"].copy_(st["od"], non_blocking=True)
                    h_out["lsed"].copy_(st["lsed"], non_blocking=True)
                    e_o = new_ev(); e_o.record(s_out)
                    outputs_free[j] = e_o

            KE = max(2, K)  # the same number of steps as the device-timed region: pipeline fill amortised alike
            e2e_step(0); e2e_step(1); torch.cuda.synchronize()
            barrier()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            main_s = torch.cuda.current_stream(dev)
            a.record(main_s)
            for st_ in (s_in, s_cmp, s_out):
                st_.wait_stream(main_s)
            for i in range(KE):
                e2e_step(i)
            for st_ in (s_in, s_cmp, s_out):
                main_s.wait_stream(st_)
            b.record(main_s); torch.cuda.synchronize()
            barrier()
            for st_ in sets:
                for n in ("ws_f", "ws_b", "ws_d"):
                    if cw.workspace_status(st_[n]) != 0:
                        raise RuntimeError("device status set during the end-to-end steps")
            e_ms = maxr(a.elapsed_time(b)) / KE

            # The same host<->device copies with no kernels between them (copy-in and copy-out on
            # their own streams, as in the steps above): the PCIe ceiling of this e2e number.
            def copy_step(i):
                st = sets[i % 2]
                with torch.cuda.stream(s_in):
                    for n in names_in:
                        st[n].copy_(h_in[n], non_blocking=True)
                    st["pos"].copy_(h_pos, non_blocking=True)
                with torch.cuda.stream(s_out):
                    for n in names_out:
                        h_out[n].copy_(st[n], non_blocking=True)

            copy_step(0); torch.cuda.synchronize()
            barrier()
            a.record(main_s)
            for st_ in (s_in, s_out):
                st_.wait_stream(main_s)
            for i in range(KE):
                copy_step(i)
            for st_ in (s_in, s_out):
                main_s.wait_stream(st_)
            b.record(main_s); torch.cuda.synchronize()
            barrier()
            c_ms = maxr(a.elapsed_time(b)) / KE
            # the results that came back to the host equal the device-timed path's, bit for bit
            # (same inputs, deterministic kernels)
            match = all(torch.equal(h_out[n].to(dev), dev_out[n]) for n in names_out)
            res = {"value": aggregate_tflops(world, fwd_flop + bwd_flop, e_ms), "unit": "TFLOP/s",
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms, "steps": KE,
                   "pipelined": "copy-in / compute / copy-out streams, two device buffer sets",
                   "outputs_read": list(names_out),
                   "copy_only_ms_per_step": c_ms, "frac_of_copy_bound": c_ms / e_ms,
                   "outputs_match_device_path": match,
                   "copy_gbs": {"h2d": h2d / c_ms / 1e6, "d2h": d2h / c_ms / 1e6}}
            del sets
            return res

        e2e = run_e2e(args.e2e_outputs == "all")
        if args.e2e_outputs == "all":
            r = run_e2e(False)
            e2e["results_only"] = {k_: r[k_] for k_ in ("value", "ms_per_step", "h2d_bytes_per_step",
                                                         "d2h_bytes_per_step", "outputs_read",
                                                         "copy_only_ms_per_step", "frac_of_copy_bound",
                                                         "outputs_match_device_path")}

    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        v_cpu, f_cpu, b_cpu, desc, threads, _ = cpu_oracle_sample(args.cpu_seconds)
        cpu = {"value": v_cpu, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc,
               "fwd_tflops": f_cpu, "bwd_tflops": b_cpu, "host_cpus": os.cpu_count()}

    # ---- the other configurations, each kernel timed alone (burst peak), one GPU only
    if world == 1 and not args.no_parts:
        parts.update(config_parts(dev, kc, vc, burst, hbm, sweep=args.sweep))
        parts["kv_head_tp4_projected"] = tp_projection(4, "folded", 3, 3, dev)

    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "train 32K layer fwd+bwd + decode 128K cache, per GPU",
                       "train": TRAIN, "decode": DECODE, "l2": "inputs larger than L2 (126 MB); no flush",
                       "parallelism": f"batch-sharded x{world} (weak)"},
            "parts": parts, "roofline": roofline, "e2e": e2e, "cpu_baseline": cpu,
            "gpu_launches": K * 6, "clocks": clk.summary()}  # fwd 1 + bwd 3 + decode 2 per step
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
