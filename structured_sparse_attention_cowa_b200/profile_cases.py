"""Small, fixed invocations of each hot kernel for profiling with ncu.

    python -m structured_sparse_attention_cowa_b200.profile_cases
        {fwd32k,bwd32k,bwd32k_one_head,decode128k_b4,decode128k_e4m3_b4,all}
        [--reps R]

Each case allocates its seeded inputs on cuda:0 (a few GB at most), calls the C ABI
`reps` times (the first launch warms up; profile with `-s 1 -c 1` on the kernel name) and
checks the device status word.  Shapes follow the 32K training layer (B=1, N=32768,
H_q=40, H_kv=8, d=128, S=128, L=2048, D=8) and the 128K decode cache at 4 sequences
(H_q=40, H_kv=8, d=128, T_cap=131072, pos=131071, S=128, L=4096, D=8), in bf16 or quantised to
E4M3 (scale 1/64).
"""

from __future__ import annotations

import argparse
import sys

import torch

from . import cowa as cw
from . import synth


def _inputs_train(dev):
    B, N, Hq, Hkv, d = 1, 32768, 40, 8, 128
    q = synth.cuda_normal_bf16((B, N, Hq, d), synth.seed_of("q"), dev)
    k = synth.cuda_normal_bf16((B, N, Hkv, d), synth.seed_of("k"), dev)
    v = synth.cuda_normal_bf16((B, N, Hkv, d), synth.seed_of("v"), dev)
    do = synth.cuda_normal_bf16((B, N, Hq, d), synth.seed_of("do"), dev)
    return q, k, v, do


def case_fwd32k(dev, reps):
    q, k, v, _ = _inputs_train(dev)
    pat = cw.Pattern(128, 2048, 32768, 8)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    for _ in range(reps):
        cw.cowa_fwd(q, k, v, pat, workspace=ws)
    return [ws]


def case_bwd32k(dev, reps):
    q, k, v, do = _inputs_train(dev)
    pat = cw.Pattern(128, 2048, 32768, 8)
    o, lse = cw.cowa_fwd(q, k, v, pat)
    ws = None
    wss = []
    for _ in range(reps):
        import ctypes

        if ws is None:
            n = cw.lib().cowa_bwd_workspace_size(ctypes.byref(pat.c()), 1, 32768, 40, 8, 128)
            ws = torch.zeros(n, dtype=torch.uint8, device=dev)
            wss.append(ws)
        cw.cowa_bwd(q, k, v, o, lse, do, pat, workspace=ws)
    return wss


def case_bwd32k_one_head(dev, reps):
    """One KV head of the 32K layer (a rank of KV-head tensor parallelism: kv_head_base = 0,
    h_kv_global = 8): the backward splits its long key tiles (121 chunks of 78 query tiles)."""
    import ctypes

    B, N, Hq, Hkv, d = 1, 32768, 5, 1, 128
    q = synth.cuda_normal_bf16((B, N, Hq, d), synth.seed_of("q"), dev)
    k = synth.cuda_normal_bf16((B, N, Hkv, d), synth.seed_of("k"), dev)
    v = synth.cuda_normal_bf16((B, N, Hkv, d), synth.seed_of("v"), dev)
    do = synth.cuda_normal_bf16((B, N, Hq, d), synth.seed_of("do"), dev)
    pat = cw.Pattern(128, 2048, 32768, 8, kv_head_base=0, h_kv_global=8)
    o, lse = cw.cowa_fwd(q, k, v, pat)
    n = cw.lib().cowa_bwd_workspace_size(ctypes.byref(pat.c()), B, N, Hq, Hkv, d)
    ws = torch.zeros(n, dtype=torch.uint8, device=dev)
    for _ in range(reps):
        cw.cowa_bwd(q, k, v, o, lse, do, pat, workspace=ws)
    return [ws]


def case_decode128k_b4(dev, reps):
    B, Hq, Hkv, d, Tc = 4, 40, 8, 128, 131072
    pat = cw.Pattern(128, 4096, 131072, 8)
    kc = synth.cuda_normal_bf16((B, Hkv, Tc, d), synth.seed_of("k_cache"), dev)
    vc = synth.cuda_normal_bf16((B, Hkv, Tc, d), synth.seed_of("v_cache"), dev)
    qt = synth.cuda_normal_bf16((B, Hq, d), synth.seed_of("q_t"), dev)
    pos = torch.full((B,), Tc - 1, dtype=torch.int32, device=dev)
    import ctypes

    n = cw.lib().cowa_decode_workspace_size(ctypes.byref(pat.c()), B, Hq, Hkv, d, Tc)
    ws = torch.zeros(n, dtype=torch.uint8, device=dev)
    for _ in range(reps):
        cw.cowa_decode(qt, kc, vc, pos, pat, workspace=ws)
    return [ws]


def case_decode128k_e4m3_b4(dev, reps):
    B, Hq, Hkv, d, Tc = 4, 40, 8, 128, 131072
    pat = cw.Pattern(128, 4096, 131072, 8)
    scale = 1.0 / 64
    kc = cw.quantize_e4m3(synth.cuda_normal_bf16((B, Hkv, Tc, d), synth.seed_of("k_cache"), dev), scale)
    vc = cw.quantize_e4m3(synth.cuda_normal_bf16((B, Hkv, Tc, d), synth.seed_of("v_cache"), dev), scale)
    qt = synth.cuda_normal_bf16((B, Hq, d), synth.seed_of("q_t"), dev)
    pos = torch.full((B,), Tc - 1, dtype=torch.int32, device=dev)
    import ctypes

    n = cw.lib().cowa_decode_fp8_workspace_size(ctypes.byref(pat.c()), B, Hq, Hkv, d, Tc)
    ws = torch.zeros(n, dtype=torch.uint8, device=dev)
    for _ in range(reps):
        cw.cowa_decode_fp8(qt, kc, vc, pos, pat, scale, scale, workspace=ws)
    return [ws]


CASES = {"fwd32k": case_fwd32k, "bwd32k": case_bwd32k, "bwd32k_one_head": case_bwd32k_one_head,
         "decode128k_b4": case_decode128k_b4, "decode128k_e4m3_b4": case_decode128k_e4m3_b4}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=list(CASES) + ["all"])
    ap.add_argument("--reps", type=int, default=2)
    args = ap.parse_args(argv)
    dev = torch.device("cuda:0")
    names = list(CASES) if args.case == "all" else [args.case]
    for name in names:
        wss = CASES[name](dev, args.reps)
        torch.cuda.synchronize()
        for ws in wss:
            st = cw.workspace_status(ws)
            if st != 0:
                print(f"{name}: device status {st}", file=sys.stderr)
                return 1
        print(f"{name}: ok", flush=True)
        torch.cuda.empty_cache()
    return 0


if __name__ == "__main__":
    sys.exit(main())
