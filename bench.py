#!/usr/bin/env python
"""Throughput of the streaming pyramid denoising round (PersonaLive) on B200.

One step = one whole round at 512x512 geometry: ring push of the new window,
16 reference-attention layers in the SD-UNet layout (64x64/C320, 32x32/C640,
16x16/C1280, 8x8/C1280, 8 heads) over [own ; bank x4] with the motion
cross-attention after each, the pyramid DDIM step on 16x4x64x64 latents with
the pop of the t=0 window, and the bank check of the 4 new motion embeddings.
All inputs are seeded synthetic tensors of the pages' shapes (no weights or
datasets exist here); per-round inputs (about 0.4 GB of hidden states) are
larger than the 126 MB L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). N > 1 runs N independent replicas (one stream
per GPU; the path has no exchange step), timed as the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic as S  # noqa: E402

METRIC = "pyramid rounds/s & output frames/s; attn TFLOP/s as % of B200 FP16 peak"
WORKLOAD = ("full round at 512x512 geometry: 16 reference-attention layers in SD-UNet layout "
            "(64x64/C320 x5, 32x32/C640 x5, 16x16/C1280 x5, 8x8/C1280 x1; 8 heads), "
            "KV = own + bank x4, motion x-attn 32x16-d per layer, DDIM on 16x4x64x64, bank check")
SEED = S.SEEDS["full"]
L2_NOTE = "per-step inputs (~0.4 GB hidden + bank K/V) exceed the 126 MB L2; no flush"


def bench_config(world: int) -> dict:
    """The `config` both arms print (the same dict, so the two lines name one workload)."""
    return {"workload": WORKLOAD,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": L2_NOTE}


def attn_flops_layer(N: int, C: int, kv_entries: int = 5, frames: int = 16) -> float:
    """Algorithmic attention-core FLOPs of one layer: 4 * Nq * Nkv * head_dim per (frame, head)."""
    hd = C // S.HEADS
    return 4.0 * frames * S.HEADS * N * (kv_entries * N) * hd


def exp2_level64(N: int = 4096, kv_entries: int = 5, frames: int = 16) -> float:
    """exp2 evaluations of one 64x64-level attention launch: one per (frame, head, query, key)."""
    return float(frames * S.HEADS * N * kv_entries * N)


def round_attn_flops() -> float:
    return sum(attn_flops_layer(side * side, C) for _, side, C in S.LAYERS)


def round_proj_flops() -> float:
    """QKV + O projections and motion Q + O projections, 2*M*N*K each."""
    tot = 0.0
    for _, side, C in S.LAYERS:
        M = 16 * side * side
        tot += 2.0 * M * C * (3 * C) + 3 * (2.0 * M * C * C)
    return tot


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d["hbm_gbs"]), "measured"
    except Exception:
        return 1590.0, 6650.0, "fallback"


def kernel_hash() -> str:
    h = hashlib.sha256()
    for f in ("attn.cu", "attn.cuh", "ptx.cuh", "fastmath.cuh"):
        with open(os.path.join(ROOT, "denoise_step_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic():
    """DRAM bytes per launch of the timed attention kernel from the committed ncu summary,
    or None when the kernel source changed since it was captured."""
    path = os.path.join(ROOT, "profiles", "attn_level64_bank4_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("kernel_hash") != kernel_hash():
        return None
    return d.get("dram_bytes_per_launch")


# --------------------------------------------------------------------------- workload

class Workload:
    """Seeded inputs of the full round, uploaded to the device once."""

    def __init__(self, torch, device):
        self.torch = torch
        L = S.LAYERS
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        self.weights = []
        for name, side, C in L:
            w = S.layer_weights(SEED, name, C, np.float16)
            self.weights.append({
                "w_qkv": dev(np.concatenate([w["wq"], w["wk"], w["wv"]], 1)), "w_o": dev(w["wo"]),
                "m_q": dev(w["mq"]), "m_kv": dev(np.concatenate([w["mk"], w["mv"]], 1)),
                "m_o": dev(w["mo"])})
        self.ref_feats = [dev(S.bank_features(SEED, n, 0, s * s, C)) for n, s, C in L]
        self.anchors = [dev(S.bank_features(SEED, n, a, s * s, C)) for a in (1, 2, 3) for n, s, C in L]
        self.ref_latent = dev(S.normal(SEED, "ref_latent", (4, 64, 64), 1.0, np.float32))
        self.prefill_eps = dev(S.normal(SEED, "prefill_eps", (12, 4, 64, 64), 1.0, np.float32))
        e0 = S.normal(SEED, "walk/e0", (512,), 1.0, np.float64)
        self.ref_motion = dev(e0.astype(np.float32))
        self.drive0 = dev(S.normal(SEED, "drive0", (512,), 1.0, np.float32))
        # per-round inputs (host copies kept pinned for the end-to-end leg)
        self.h_hidden = [S.layer_hidden(SEED, n, 1, 16, s * s, C) for n, s, C in L]
        steps = S.normal(SEED, "walk/steps", (4, 512), 3.0)
        self.h_motion = (e0[None] + np.cumsum(steps, 0)).astype(np.float32)
        self.h_noise = S.normal(SEED, "noise", (4, 4, 64, 64), 1.0, np.float32)
        self.h_eps = S.normal(SEED, "eps", (16, 4, 64, 64), 1.0, np.float32)
        self.hidden = [dev(h) for h in self.h_hidden]
        self.motion, self.noise, self.eps = dev(self.h_motion), dev(self.h_noise), dev(self.h_eps)
        self.out = torch.empty((4, 4, 64, 64), dtype=torch.float32, device=device)
        self.flags = torch.zeros(4, dtype=torch.uint8, device=device)
        self.layer_out = [torch.empty((16, s * s, C), dtype=torch.float16, device=device)
                          for _, s, C in L]


def clocks_sampler(device_index: int, path: str):
    q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    try:
        f = open(path, "w")
        return subprocess.Popen(["nvidia-smi", f"--id={device_index}", f"--query-gpu={q}",
                                 "--format=csv,noheader,nounits", "-lms", "200"],
                                stdout=f, stderr=subprocess.DEVNULL), f
    except Exception:
        return None, None


def clocks_summary(path: str):
    try:
        rows = [r.split(",") for r in open(path).read().strip().splitlines() if r.strip()]
    except Exception:
        return None
    sm, mx, reasons = [], 0.0, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for r in rows:
        try:
            sm.append(float(r[1]))
            mx = max(mx, float(r[2]))
        except (ValueError, IndexError):
            continue
        for n, v in zip(names, r[5:9]):
            if v.strip().lower() == "active":
                reasons.add(n)
    if not sm:
        return None
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
            "samples": len(sm)}


# --------------------------------------------------------------------------- CPU oracle arm

def oracle_round_sample():
    """Time the fp64 oracle on a bounded sample of one round and extrapolate to a round.

    Sample: every layer, frame 0, R = 8 and R = 32 query rows (the per-frame K/V
    projection of [own ; bank x4] is the fixed part, the per-row attention the
    linear part), extrapolated to 16 frames x all rows; plus the full pile
    DDIM step and bank check. Returns (seconds per round, sample description).
    """
    import oracle as O
    rng_rows = (8, 32)
    total = 0.0
    tok = O.motion_tokens(S.normal(SEED, "walk/e0", (512,)))
    for name, side, C in S.LAYERS:
        N = side * side
        w = S.layer_weights(SEED, name, C, np.float16)
        h = S.normal(SEED, f"{name}/hidden/sample", (N, C), 1.0, np.float16)
        bank = [S.bank_features(SEED, name, b, N, C) for b in range(4)]
        ts = []
        for R in rng_rows:
            rows = np.arange(min(R, N))
            t0 = time.perf_counter()
            O.layer_forward_frame(h, w, bank, tok, S.HEADS, rows=rows)
            ts.append(time.perf_counter() - t0)
        r1, r2 = min(rng_rows[0], N), min(rng_rows[1], N)
        per_row = max(ts[1] - ts[0], 0.0) / max(r2 - r1, 1)
        fixed = max(ts[0] - r1 * per_row, 0.0)
        total += 16 * (fixed + N * per_row)
    ref = S.normal(SEED, "ref_latent", (4, 64, 64))
    pe = S.normal(SEED, "prefill_eps", (12, 4, 64, 64))
    st = O.PyramidStream(ref, pe, S.normal(SEED, "walk/e0", (512,)), S.normal(SEED, "drive0", (512,)))
    noise = S.normal(SEED, "noise", (4, 4, 64, 64))
    eps = S.normal(SEED, "eps", (16, 4, 64, 64))
    mot = S.normal(SEED, "mot", (4, 512), 3.0)
    t0 = time.perf_counter()
    st.round(noise, mot, eps)
    total += time.perf_counter() - t0
    desc = ("per layer: frame 0 with 8 and 32 query rows (fixed K/V projection + per-row "
            "attention), extrapolated linearly to 16 frames x all rows; full DDIM/pile/bank")
    return total, desc


def blas_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max(int(i.get("num_threads", 1)) for i in info) if info else 1
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, rank):
    if rank != 0:
        return 0
    for _ in range(args.warmup):
        oracle_round_sample()
    secs = []
    desc = ""
    t0 = time.perf_counter()
    for _ in range(args.steps):
        s, desc = oracle_round_sample()
        secs.append(s)
    wall = time.perf_counter() - t0
    per_round = sum(secs) / len(secs)
    value = 1.0 / per_round
    # a step is one bounded sample of a round: ms_per_step is its measured wall
    # time, and it stands for rounds_per_step of a round's work
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "rounds/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": wall / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(args.gpus), "frames_per_s": 4 * value,
        "rounds_per_step": wall / args.steps / per_round,
        "extrapolated_ms_per_round": per_round * 1e3,
        "cpu_baseline": {"value": value, "unit": "rounds/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "rounds/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- GPU arm

def time_attention_kernel(torch, P, wl, stream, reps=10):
    """Average duration of the dominant kernel: the 64x64-level attention over [own ; bank x4]
    (16 frames x 8 heads x 4096 queries x 20480 keys, head_dim 40), launched as in the round."""
    N, C = 4096, 320
    qkv = torch.randn((16, N, 3 * C), device="cuda", dtype=torch.float16,
                      generator=torch.Generator(device="cuda").manual_seed(SEED))
    bank = torch.randn((4, N, 2 * C), device="cuda", dtype=torch.float16,
                       generator=torch.Generator(device="cuda").manual_seed(SEED + 1))
    segs = [(qkv[:, :, C:2 * C], qkv[:, :, 2 * C:])] + [(bank[b, :, :C], bank[b, :, C:]) for b in range(4)]
    out = torch.empty((16, N, C), device="cuda", dtype=torch.float16)
    q = qkv[:, :, :C]
    with torch.cuda.stream(stream):
        for _ in range(3):
            P.segment_attention(q, segs, 8, 40, out=out, stream=stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            P.segment_attention(q, segs, 8, 40, out=out, stream=stream)
        e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / reps / 1e3


def max_over_ranks(torch, dist, seconds: float, device) -> float:
    """Largest per-rank time (all ranks take part; every rank gets the result)."""
    if dist is None:
        return seconds
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world: int, steps: int, max_seconds: float) -> float:
    """Whole-job rounds/s of `world` independent replicas, each doing `steps` rounds."""
    return world * steps / max_seconds


def _event_time(torch, fn, reps, stream):
    with torch.cuda.stream(stream):
        fn()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) / reps / 1e3


def sessions_round(torch, P, wl, stream, sessions, single_ms):
    """`sessions` streams of the full round served by one context (one launch per
    kernel for all of them); each session gets the workload's inputs (timing only:
    the content does not change the work). Rounds timed through the captured graph."""
    L = S.LAYERS
    rep = lambda t: t.unsqueeze(0).expand(sessions, *t.shape).contiguous()
    cfg = P.make_config((64, 64), [(s * s, C) for _, s, C in L], sessions=sessions)
    st = P.Stream(cfg)
    st.bank_init(wl.weights, [rep(t) for t in wl.ref_feats], [rep(t) for t in wl.anchors],
                 rep(wl.ref_motion), rep(wl.drive0), rep(wl.ref_latent), rep(wl.prefill_eps),
                 stream=stream)
    hidden = [rep(t) for t in wl.hidden]
    noise, motion, eps = rep(wl.noise), rep(wl.motion), rep(wl.eps)
    out = torch.empty((sessions, 4, 4, 64, 64), dtype=torch.float32, device="cuda")
    flags = torch.zeros((sessions, 4), dtype=torch.uint8, device="cuda")
    t = _event_time(torch, lambda: st.round(noise, motion, hidden, eps, out, flags, None,
                                            stream=stream), 5, stream)
    st.close()
    del hidden, noise, motion, eps, out
    torch.cuda.synchronize()
    return {"sessions": sessions, "ms_per_round": t * 1e3, "rounds_per_s": sessions / t,
            "frames_per_s": 4 * sessions / t, "speedup_vs_one_session": sessions * single_ms / (t * 1e3)}


def sink_stream_step(torch, P, stream):
    """PR-Sink cache at the C5 sizes (4096 tokens x 40 heads x 128, pool of 64
    pose-descriptor blocks of 64-d): steps with the cache full (own + sink + 3
    rolling + 1 retrieved = 6 x 4096 keys), each timed by CUDA events around
    pl_sink_step alone (the caller's K/V writes stay outside)."""
    n, heads, hd, pool, dim = 4096, 40, 128, 64, 64
    g = torch.Generator(device="cuda").manual_seed(SEED)
    sink = P.Sink(n, heads, hd, pool, dim)
    q = torch.randn((n, heads * hd), device="cuda", dtype=torch.float16, generator=g)
    kv = torch.randn((2, n, heads * hd), device="cuda", dtype=torch.float16, generator=g)
    poses = torch.randn((16, dim), device="cuda", generator=g)
    out = torch.empty_like(q)
    times = []
    with torch.cuda.stream(stream):
        for t in range(12):
            kd, vd = sink.block_kv()
            kd.copy_(kv[0])
            vd.copy_(kv[1])
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            sink.step(q, poses[t], out=out, stream=stream)
            e1.record(stream)
            times.append((e0, e1))
    stream.synchronize()
    st = sink.state(stream)
    sink.close()
    steady = [a.elapsed_time(b) for a, b in times[6:]]     # pool non-empty from step 5
    ms = sum(steady) / len(steady)
    fl = 4.0 * n * 6 * n * hd * heads
    return {"ms_per_step": ms, "tflops": fl / ms / 1e9, "steps_timed": len(steady),
            "pool_count": st["pool_count"], "n_roll": st["n_roll"]}


def lpm_window_step(torch, P, stream):
    """LPM window cache with the window full: 1024 reference tokens + 3 sink + 2
    sliding + the current chunk of 4096 tokens (25600 keys), 40 heads x 128; the
    rotary code applied in the kernel. Timed by CUDA events around pl_lpm_step
    alone, next to the same attention without the rotary code."""
    R, L, heads, hd = 1024, 4096, 40, 128
    C = heads * hd
    g = torch.Generator(device="cuda").manual_seed(SEED)
    lpm = P.Lpm(R, L, heads, hd)
    rk, rv = lpm.ref_kv()
    rk.copy_(torch.randn((R, C), device="cuda", dtype=torch.float16, generator=g))
    rv.copy_(torch.randn((R, C), device="cuda", dtype=torch.float16, generator=g))
    q = torch.randn((L, C), device="cuda", dtype=torch.float16, generator=g)
    kv = torch.randn((2, L, C), device="cuda", dtype=torch.float16, generator=g)
    out = torch.empty_like(q)
    times = []
    with torch.cuda.stream(stream):
        for t in range(10):
            kd, vd = lpm.chunk_kv()
            kd.copy_(kv[0])
            vd.copy_(kv[1])
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            lpm.step(q, out=out, stream=stream)
            e1.record(stream)
            times.append((e0, e1))
    stream.synchronize()
    st = lpm.state()
    steady = [a.elapsed_time(b) for a, b in times[5:]]      # window full from step 5
    ms = sum(steady) / len(steady)
    # the same window without the rotary code
    segs = [(kv[0][:R], kv[1][:R])] + [(kv[0], kv[1])] * 6
    t_plain = _event_time(torch, lambda: P.segment_attention(q[None], segs, heads, hd,
                                                             out=out[None], stream=stream),
                          5, stream)
    lpm.close()
    fl = 4.0 * L * (R + 6 * L) * hd * heads
    return {"ms_per_step": ms, "tflops": fl / ms / 1e9, "keys": R + 6 * L,
            "ms_without_rotary": t_plain * 1e3, "n_sink": st["n_sink"], "n_slide": st["n_slide"]}


def pose_front(torch, P, stream, hbm_peak):
    """Pose path front: keypoints and dot images of a round's 4 new frames at
    512 x 512, and of 64 frames (a 201 MB image batch, past L2) for the HBM
    fraction. Synthetic poses (N(0, 15 deg) angles, N(0, 0.1) translations)."""
    g = torch.Generator(device="cuda").manual_seed(SEED)
    canon = 0.3 * torch.randn((21, 3), device="cuda", generator=g)
    cols = [[1, 0, 0], [0, 1, 0], [0, 0, 1], [1, 1, 0], [1, 0, 1], [0, 1, 1], [0.5, 0.5, 0.5]]
    sel = [0, 3, 5, 8, 11, 15, 20]
    out = {}
    for frames in (4, 64):
        poses = torch.cat([15 * torch.randn((frames, 3), device="cuda", generator=g),
                           0.1 * torch.randn((frames, 3), device="cuda", generator=g)], 1)
        kps = torch.empty((frames, 7, 3), dtype=torch.float64, device="cuda")
        img = torch.empty((frames, 3, 512, 512), dtype=torch.float32, device="cuda")

        def fn():
            P.pose_keypoints(canon, 0.9, poses, sel, out=kps, stream=stream)
            P.pose_dots(kps, cols, 6.0, 512, 512, out=img, stream=stream)

        t = _event_time(torch, fn, 10, stream)
        byts = img.numel() * 4.0
        out[f"frames_{frames}"] = {"us": t * 1e6, "gbs": byts / t / 1e9,
                                   "frac_hbm": byts / t / 1e9 / hbm_peak}
    return out


def tiny_round(torch, P, stream):
    """C1: the round at the tiny geometry (one 8x8-token level, C 1280, 8 heads of
    160, KV = own + bank x1, motion x-attn, DDIM on 16x4x8x8, bank check of 4
    new embeddings) through pl_stream_round with device-resident inputs, and the
    context-free bank check of 4 N(0,4) queries against 8 stored N(0,4) vectors;
    microseconds per call by CUDA events over back-to-back calls."""
    seed, H, W, N, C = S.SEEDS["tiny"], 8, 8, 64, 1280
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    w = S.layer_weights(seed, "m", C, np.float16)
    pw = {"w_qkv": dev(np.concatenate([w["wq"], w["wk"], w["wv"]], 1)), "w_o": dev(w["wo"]),
          "m_q": dev(w["mq"]), "m_kv": dev(np.concatenate([w["mk"], w["mv"]], 1)),
          "m_o": dev(w["mo"])}
    st = P.Stream(P.make_config((H, W), [(N, C)]))
    ref_m = S.normal(seed, "walk/e0", (512,), 1.0, np.float32)
    st.bank_init([pw], [dev(S.bank_features(seed, "m", 0, N, C))], None, dev(ref_m),
                 dev(S.normal(seed, "drive0", (512,), 1.0, np.float32)),
                 dev(S.normal(seed, "ref_latent", (4, H, W), 1.0, np.float32)),
                 dev(S.normal(seed, "prefill_eps", (12, 4, H, W), 1.0, np.float32)), stream=stream)
    hidden = [dev(S.layer_hidden(seed, "m", 1, 16, N, C))]
    noise = dev(S.normal(seed, "noise1", (4, 4, H, W), 1.0, np.float32))
    mot = dev((ref_m[None] + S.normal(seed, "walk/step1", (4, 512), 3.0).cumsum(0)).astype(np.float32))
    eps = dev(S.normal(seed, "eps1", (16, 4, H, W), 1.0, np.float32))
    out = torch.empty((4, 4, H, W), dtype=torch.float32, device="cuda")
    flags = torch.zeros(4, dtype=torch.uint8, device="cuda")
    reps = 200
    t = _event_time(torch, lambda: st.round(noise, mot, hidden, eps, out, flags, None,
                                            stream=stream), reps, stream)
    st.close()
    bank = dev(S.normal(seed, "bank8", (8, 512), 2.0, np.float32))
    qs = dev(S.normal(seed, "bankq", (4, 512), 2.0, np.float32))
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    app = torch.zeros(1, dtype=torch.int32, device="cuda")

    def check():
        cnt.fill_(8)
        app.fill_(0)
        P.motion_bank_check(bank, cnt, app, qs, 17.0, 3, stream=stream)

    tb = _event_time(torch, check, reps, stream)
    return {"us_per_round": t * 1e6, "rounds_per_s": 1.0 / t, "frames_per_s": 4.0 / t,
            "bank_check_8x512_us": tb * 1e6,
            "note": "bank check timed with two 4-byte fills of its counters per call"}


def level64_bank1(torch, P, stream, tf_peak):
    """C2: one 64x64 level (16 frames x 4096 tokens, C 320, 8 heads of 40, KV =
    own + bank x1 = 8192) through pl_ref_attention (QKV projection, bank K/V
    projection, attention core, O projection), the attention core alone at that
    shape, and the pile DDIM step on 16x4x64x64 (ring push + step)."""
    seed, F, N, C, heads = S.SEEDS["level64"], 16, 4096, 320, 8
    hd = C // heads
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    w = S.layer_weights(seed, "L", C, np.float16)
    w_qkv = dev(np.concatenate([w["wq"], w["wk"], w["wv"]], 1))
    w_o = dev(w["wo"])
    h = dev(S.normal(seed, "hidden", (F, N, C), 1.0, np.float16))
    bank = [dev(S.bank_features(seed, "L", 0, N, C))]
    out = torch.empty_like(h)
    need = P.sz()
    P.check(P.lib.pl_ref_attention_workspace_bytes(F, N, C, 1, P.C.byref(need)), "ws")
    ws = torch.empty(need.value, dtype=torch.uint8, device="cuda")
    t_layer = _event_time(torch, lambda: P.ref_attention(h, w_qkv, w_o, bank, heads, out=out,
                                                         workspace=ws, stream=stream), 10, stream)
    core = 4.0 * F * heads * N * (2 * N) * hd
    proj = 2.0 * F * N * C * (3 * C) + 2.0 * F * N * C * C + 2.0 * N * C * (2 * C)
    # attention core alone on the layer's own Q/K/V (the workspace's first 3 F N C halves)
    qkv = ws[: 2 * 3 * F * N * C].view(torch.float16).view(F, N, 3 * C)
    bkv = torch.randn((N, 2 * C), device="cuda", dtype=torch.float16,
                      generator=torch.Generator(device="cuda").manual_seed(seed))
    segs = [(qkv[:, :, C:2 * C], qkv[:, :, 2 * C:]), (bkv[:, :C], bkv[:, C:])]
    o2 = torch.empty((F, N, C), device="cuda", dtype=torch.float16)
    t_core = _event_time(torch, lambda: P.segment_attention(qkv[:, :, :C], segs, heads, hd, out=o2,
                                                            stream=stream), 10, stream)
    # pile DDIM step at the configuration size
    st = P.Stream(P.make_config((64, 64), []))
    g = torch.Generator(device="cuda").manual_seed(seed)
    mkf = lambda *sh: torch.randn(sh, device="cuda", generator=g)
    st.bank_init([], [], None, mkf(512), mkf(512), mkf(4, 64, 64), mkf(12, 4, 64, 64), stream=stream)
    noise, mot, eps = mkf(4, 4, 64, 64), mkf(4, 512), mkf(16, 4, 64, 64)
    xo = torch.empty((4, 4, 64, 64), device="cuda")

    def ddim_round():
        st.ring_push(noise, mot, stream=stream)
        st.ddim_step(eps, xo, stream=stream)

    t_ddim = _event_time(torch, ddim_round, 50, stream)
    st.close()
    fe = 4 * 64 * 64
    byts = 4.0 * fe * (8 + 48)
    return {"layer_ms": t_layer * 1e3, "layer_tflop": (core + proj) / 1e12,
            "layer_tflops": (core + proj) / t_layer / 1e12,
            "layer_frac_of_peak": (core + proj) / t_layer / 1e12 / tf_peak,
            "core_ms": t_core * 1e3, "core_tflops": core / t_core / 1e12,
            "core_frac_of_peak": core / t_core / 1e12 / tf_peak,
            "ddim_push_step_us": t_ddim * 1e6, "ddim_gbs": byts / t_ddim / 1e9,
            "ddim_note": "3.2 MB step, L2-resident and latency-bound at this size"}


def secondary_measurements(torch, P, stream, hbm_peak):
    """The other workloads' kernels, timed live (CUDA events on their stream):
    the PR-Sink block (4096 tokens x 40 heads x 128, KV own + sink + retrieved
    of 64 + 3 rolling), the pile DDIM step on a scaled latent grid (1024 x 1024:
    ring + epsilon 512 MB, past L2), the nearest-vector search over a 1 GB
    store and the motion-bank check of 4 embeddings over a 512 MB bank.
    Inputs are seeded torch tensors (timing only)."""
    g = torch.Generator(device="cuda").manual_seed(SEED)
    out = {}
    # PR-Sink
    n, heads, hd = 4096, 40, 128
    Cc = heads * hd
    mk = lambda *sh: torch.randn(sh, device="cuda", dtype=torch.float16, generator=g)
    q = mk(n, Cc)
    own, snk = (mk(n, Cc), mk(n, Cc)), (mk(n, Cc), mk(n, Cc))
    pool = (mk(64, n, Cc), mk(64, n, Cc))
    roll = [(mk(n, Cc), mk(n, Cc)) for _ in range(3)]
    store = torch.randn((64, 64), device="cuda", generator=g)
    pq = torch.randn((64,), device="cuda", generator=g)
    o = torch.empty_like(q)
    ret = torch.zeros(1, dtype=torch.int32, device="cuda")
    t = _event_time(torch, lambda: P.pr_sink_attention(q, own, snk, pool, store, pq, roll, heads,
                                                       hd, out=o, retrieved=ret, stream=stream),
                    5, stream)
    fl = 4.0 * n * 6 * n * hd * heads
    out["pr_sink_block"] = {"ms": t * 1e3, "tflops": fl / t / 1e12}
    del q, own, snk, pool, roll, o
    # DDIM pile step on a scaled latent grid
    H = W = 1024
    fe = 4 * H * W
    st = P.Stream(P.make_config((H, W), []))
    mkf = lambda *sh: torch.randn(sh, device="cuda", generator=g)
    st.bank_init([], [], None, mkf(512), mkf(512), mkf(4, H, W), mkf(12, 4, H, W), stream=stream)
    noise, mot, eps = mkf(4, 4, H, W), mkf(4, 512), mkf(16, 4, H, W)
    xo = torch.empty((4, 4, H, W), device="cuda")

    def ddim_round():
        st.ring_push(noise, mot, stream=stream)
        st.ddim_step(eps, xo, stream=stream)

    t = _event_time(torch, ddim_round, 10, stream)
    byts = 4.0 * fe * (8 + 48)   # push: 4 frames in + out; step: x, eps of 16 frames in, 16 out
    out["ddim_pile_1024x1024"] = {"ms": t * 1e3, "gbs": byts / t / 1e9,
                                  "frac_hbm": byts / t / 1e9 / hbm_peak}
    st.close()
    del noise, eps, xo
    # nearest vector over a large store
    count, dim = 1 << 21, 128
    store = torch.randn((count, dim), device="cuda", generator=g)
    qv = torch.randn((dim,), device="cuda", generator=g)
    am = torch.zeros(1, dtype=torch.int64, device="cuda")
    md = torch.zeros(1, dtype=torch.float64, device="cuda")
    t = _event_time(torch, lambda: P.nearest(store, qv, am, md, stream=stream), 10, stream)
    byts = 4.0 * count * dim
    out["nearest_2M_x128"] = {"ms": t * 1e3, "gbs": byts / t / 1e9,
                              "frac_hbm": byts / t / 1e9 / hbm_peak}
    del store
    # motion-bank check at scale: 4 round embeddings checked in order against a
    # full bank of 262144 x 512 (512 MB, past L2; full, so no append changes
    # the work between calls)
    count, dim = 1 << 18, 512
    bank = 2.0 * torch.randn((count, dim), device="cuda", generator=g)
    qs = 2.0 * torch.randn((4, dim), device="cuda", generator=g)
    cnt = torch.full((1,), count, dtype=torch.int32, device="cuda")
    app = torch.zeros(1, dtype=torch.int32, device="cuda")
    need = P.sz()
    P.check(P.lib.pl_motion_bank_check_workspace_bytes(count, dim, 4, P.C.byref(need)), "ws")
    ws = torch.empty(need.value, dtype=torch.uint8, device="cuda")
    t = _event_time(torch, lambda: P.motion_bank_check(bank, cnt, app, qs, 17.0, 3, workspace=ws,
                                                       stream=stream), 10, stream)
    byts = 4.0 * (count + 4) * dim
    out["bank_check_256k_x512_q4"] = {"ms": t * 1e3, "gbs": byts / t / 1e9,
                                      "frac_hbm": byts / t / 1e9 / hbm_peak}
    del bank
    torch.cuda.synchronize()
    return out


def run_ours(args, rank, world, local_rank):
    import torch
    import denoise_step_b200 as P
    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    wl = Workload(torch, "cuda")
    cfg = P.make_config((64, 64), [(s * s, C) for _, s, C in S.LAYERS])
    st = P.Stream(cfg)
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    st.bank_init(wl.weights, wl.ref_feats, wl.anchors, wl.ref_motion, wl.drive0, wl.ref_latent,
                 wl.prefill_eps, stream=stream)

    def step():
        st.round(wl.noise, wl.motion, wl.hidden, wl.eps, wl.out, wl.flags, wl.layer_out,
                 stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            step()
    stream.synchronize()
    state = st.state(stream)
    if state["bank_count"] != 4 or state["device_status"] != 0:
        raise RuntimeError(f"unexpected state after warm-up: {state}")

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    clk_dir = tempfile.mkdtemp(prefix="pl_bench_clocks_")
    clk_path = os.path.join(clk_dir, f"clocks_r{rank}.csv")
    proc, fh = clocks_sampler(local_rank, clk_path)
    time.sleep(0.3)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
    barrier()
    if proc is not None:
        proc.terminate()
        proc.wait()
        fh.close()
    elapsed = max_over_ranks(torch, dist, e0.elapsed_time(e1) / 1e3, "cuda")
    if st.device_status(stream) != 0:
        raise RuntimeError("device status word set during the timed region")
    # kernels of one timed round, counted by the library in the captured round graph
    launches_per_round = st.round_kernels()

    # end to end through the public API: pinned host inputs in, x0 frames out, every step
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    h_hidden = [pin(h) for h in wl.h_hidden]
    h_noise, h_motion, h_eps = pin(wl.h_noise), pin(wl.h_motion), pin(wl.h_eps)
    h_out = torch.empty((4, 4, 64, 64), dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in h_hidden + [h_noise, h_motion, h_eps])
    d2h = h_out.numel() * h_out.element_size()

    def e2e_step():
        # pl_stream_round_host: this round's inputs go up on the context's copy
        # stream (into one of two staging sets) while the previous round
        # computes; the x0 frames come back on `stream`
        st.round_host(h_noise, h_motion, h_hidden, h_eps, h_out, stream=stream)

    e2e_steps = max(3, min(args.steps, 20))
    with torch.cuda.stream(stream):
        for _ in range(2):          # one capture per staging set, outside the timed region
            e2e_step()
        stream.synchronize()
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        f1.record(stream)
    barrier()
    e2e_elapsed = max_over_ranks(torch, dist, f0.elapsed_time(f1) / 1e3, "cuda")

    # dominant kernel, timed alone on the stream it is launched on
    attn_s = time_attention_kernel(torch, P, wl, stream)
    attn_fl = attn_flops_layer(4096, 320)
    tf_peak, hbm_peak, peak_kind = peaks()
    achieved = attn_fl / attn_s / 1e12

    value = job_rate(world, args.steps, elapsed)
    line = {
        "metric": METRIC, "value": value, "unit": "rounds/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": bench_config(world),
        "frames_per_s": 4 * value,
        "detail": {
            "round_attn_tflop": round_attn_flops() / 1e12,
            "round_proj_tflop": round_proj_flops() / 1e12,
            "round_tflops_effective": (round_attn_flops() + round_proj_flops()) * args.steps / elapsed / 1e12 / world,
            "attn_tflops_level64": achieved,
            "attn_frac_fp16_peak": {"measured": achieved / tf_peak, "spec_2250": achieved / 2250.0},
            # the same launch counted in exp2 evaluations (one per score; at
            # head_dim 40 the exp2 units, not the tensor pipe, bound it): 11 of
            # every 16 go to the MUFU (16 per clock per SM), the rest to an
            # FMA-pipe polynomial
            "attn_exp2_level64": {
                "exp2_per_s": exp2_level64() / attn_s,
                "mufu_exp2_per_s": exp2_level64() * 11 / 16 / attn_s,
                "mufu_peak_per_s": 16 * 148 * 1.965e9,
                "mufu_frac": exp2_level64() * 11 / 16 / attn_s / (16 * 148 * 1.965e9)},
        },
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": tf_peak, "unit": "TFLOP/s",
                     "frac": achieved / tf_peak, "traffic": ncu_traffic(),
                     "kernel": "attn_kernel<40> (64x64 level, KV own + bank x4)",
                     "peak_kind": f"{peak_kind} bf16 burst (fp16 dense rate is the same)",
                     "launch_ms": attn_s * 1e3},
        "e2e": {"value": job_rate(world, e2e_steps, e2e_elapsed), "unit": "rounds/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": "pl_stream_round_host (pinned host in/out; round k+1's upload "
                       "overlaps round k on a copy stream)"},
        "gpu_launches": launches_per_round * args.steps,
    }
    if rank == 0 and not args.no_secondary:
        sec = secondary_measurements(torch, P, stream, hbm_peak)
        sec["c1_tiny_round"] = tiny_round(torch, P, stream)
        sec["c2_level64_bank1"] = level64_bank1(torch, P, stream, tf_peak)
        sec["sessions_4"] = sessions_round(torch, P, wl, stream, 4, elapsed / args.steps * 1e3)
        sec["pr_sink_cache_step"] = sink_stream_step(torch, P, stream)
        sec["lpm_window_step"] = lpm_window_step(torch, P, stream)
        sec["pose_front_512"] = pose_front(torch, P, stream, hbm_peak)
        line["detail"]["secondary"] = sec
    clk = clocks_summary(clk_path)
    try:
        os.remove(clk_path)
        os.rmdir(clk_dir)
    except OSError:
        pass
    if clk is not None:
        line["clocks"] = clk
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        secs, desc = oracle_round_sample()
        line["cpu_baseline"] = {"value": 1.0 / secs, "unit": "rounds/s", "cores": blas_threads(),
                                "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    st.close()
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)
    return run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
