"""Run one kernel of the round on a chosen shape (for timing and ncu captures).

    python -m denoise_step_b200.microbench attn --frames 16 --n 4096 --c 320 --bank 4 --reps 3
    python -m denoise_step_b200.microbench gemm --m 65536 --n 960 --k 320 --reps 3
    python -m denoise_step_b200.microbench ddim --h 64 --w 64 --reps 3
    python -m denoise_step_b200.microbench sink --n 4096 --c 5120 --heads 40 --pool 64 --reps 3
    python -m denoise_step_b200.microbench nearest --count 1048576 --dim 128 --reps 10
    python -m denoise_step_b200.microbench motion --frames 16 --n 4096 --c 320 --heads 8 --reps 10
    python -m denoise_step_b200.microbench bank --count 4 --dim 512 --queries 4 --reps 10

Inputs are seeded torch tensors on the device; prints the mean CUDA-event time
per launch and the algorithmic throughput.
"""
from __future__ import annotations

import argparse
import json

import torch

import denoise_step_b200 as P


def _time(fn, reps, stream):
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


def attn(a, stream):
    g = torch.Generator(device="cuda").manual_seed(a.seed)
    C, N, F, hd = a.c, a.n, a.frames, a.c // a.heads
    qkv = torch.randn((F, N, 3 * C), device="cuda", dtype=torch.float16, generator=g)
    bank = torch.randn((max(a.bank, 1), N, 2 * C), device="cuda", dtype=torch.float16, generator=g)
    segs = [(qkv[:, :, C:2 * C], qkv[:, :, 2 * C:])]
    segs += [(bank[b, :, :C], bank[b, :, C:]) for b in range(a.bank)]
    out = torch.empty((F, N, C), device="cuda", dtype=torch.float16)
    fn = lambda: P.segment_attention(qkv[:, :, :C], segs, a.heads, hd, out=out, stream=stream)
    t = _time(fn, a.reps, stream)
    flops = 4.0 * F * a.heads * N * (N * (1 + a.bank)) * hd
    return {"kernel": f"attn hd{hd}", "s": t, "tflops": flops / t / 1e12}


def sink(a, stream):
    """PR-Sink block: 4096 tokens, 40 heads x 128, KV = own + sink + retrieved + 3 rolling."""
    g = torch.Generator(device="cuda").manual_seed(a.seed)
    n, heads, hd, n_pool = a.n, a.heads, a.c // a.heads, a.pool
    Cc = heads * hd
    mk = lambda *s: torch.randn(s, device="cuda", dtype=torch.float16, generator=g)
    q = mk(n, Cc)
    own, snk = (mk(n, Cc), mk(n, Cc)), (mk(n, Cc), mk(n, Cc))
    pool = (mk(n_pool, n, Cc), mk(n_pool, n, Cc))
    roll = [(mk(n, Cc), mk(n, Cc)) for _ in range(3)]
    store = torch.randn((n_pool, 64), device="cuda", generator=g)
    pq = torch.randn((64,), device="cuda", generator=g)
    out = torch.empty_like(q)
    ret = torch.zeros(1, dtype=torch.int32, device="cuda")
    fn = lambda: P.pr_sink_attention(q, own, snk, pool, store, pq, roll, heads, hd, out=out,
                                     retrieved=ret, stream=stream)
    t = _time(fn, a.reps, stream)
    flops = 4.0 * n * (6 * n) * hd * heads
    return {"kernel": f"pr-sink attn hd{hd} x{heads}", "s": t, "tflops": flops / t / 1e12}


def nearest(a, stream):
    """argmin over a large fp32 store (one read): algorithmic bytes = count * dim * 4."""
    g = torch.Generator(device="cuda").manual_seed(a.seed)
    store = torch.randn((a.count, a.dim), device="cuda", generator=g)
    q = torch.randn((a.dim,), device="cuda", generator=g)
    am = torch.zeros(1, dtype=torch.int64, device="cuda")
    md = torch.zeros(1, dtype=torch.float64, device="cuda")
    need = P.sz()
    P.check(P.lib.pl_nearest_workspace_bytes(a.count, P.C.byref(need)), "ws")
    ws = torch.empty(need.value, dtype=torch.uint8, device="cuda")
    t = _time(lambda: P.nearest(store, q, am, md, ws, stream=stream), a.reps, stream)
    return {"kernel": "nearest", "s": t, "gbs": 4.0 * a.count * a.dim / t / 1e9}


def gemm(a, stream):
    g = torch.Generator(device="cuda").manual_seed(a.seed)
    A = torch.randn((a.m, a.k), device="cuda", dtype=torch.float16, generator=g)
    B = torch.randn((a.k, a.n), device="cuda", dtype=torch.float16, generator=g) / a.k ** 0.5
    Cm = torch.empty((a.m, a.n), device="cuda", dtype=torch.float16)
    t = _time(lambda: P.gemm(A, B, out=Cm, stream=stream), a.reps, stream)
    return {"kernel": "gemm", "s": t, "tflops": 2.0 * a.m * a.n * a.k / t / 1e12,
            "gbs": 2.0 * (a.m * a.k + a.k * a.n + a.m * a.n) / t / 1e9}


def motion(a, stream):
    """Motion cross-attention of one layer: Mq GEMM (fp32 out), 32-token attention, Mo GEMM."""
    g = torch.Generator(device="cuda").manual_seed(a.seed)
    F, N, Cc = a.frames, a.n, a.c
    x = torch.randn((F, N, Cc), device="cuda", dtype=torch.float16, generator=g)
    mot = torch.randn((F, 512), device="cuda", dtype=torch.float32, generator=g)
    w = lambda r, c: torch.randn((r, c), device="cuda", dtype=torch.float16, generator=g) / r ** 0.5
    m_q, m_kv, m_o = w(Cc, Cc), w(16, 2 * Cc), w(Cc, Cc)
    out = torch.empty_like(x)
    need = P.sz()
    P.check(P.lib.pl_motion_xattn_workspace_bytes(F, N, Cc, P.C.byref(need)), "ws")
    ws = torch.empty(need.value, dtype=torch.uint8, device="cuda")
    t = _time(lambda: P.motion_xattn(x, mot, m_q, m_kv, m_o, a.heads, out=out, workspace=ws,
                                     stream=stream), a.reps, stream)
    return {"kernel": f"motion xattn C{Cc}", "s": t}


def ddim(a, stream):
    st = P.Stream(P.make_config((a.h, a.w), []))
    fe = 4 * a.h * a.w
    g = torch.Generator(device="cuda").manual_seed(a.seed)
    mk = lambda *s: torch.randn(s, device="cuda", dtype=torch.float32, generator=g)
    st.bank_init([], [], None, mk(512), mk(512), mk(4, a.h, a.w), mk(12, 4, a.h, a.w), stream=stream)
    noise, mot, eps = mk(4, 4, a.h, a.w), mk(4, 512), mk(16, 4, a.h, a.w)
    out = torch.empty((4, 4, a.h, a.w), device="cuda", dtype=torch.float32)

    def fn():
        st.ring_push(noise, mot, stream=stream)
        st.ddim_step(eps, out, stream=stream)

    t = _time(fn, a.reps, stream)
    # algorithmic bytes of the step: read x and eps of 16 frames, write 12 x_prev + 4 x0 (fp32)
    byts = 4.0 * fe * (16 + 16 + 16)
    return {"kernel": "ring push + ddim", "s": t, "gbs_ddim_bytes": byts / t / 1e9}


def bank(a, stream):
    """Motion-bank check: `queries` N(0, 4) embeddings checked in order against
    `count` stored N(0, 4) vectors of `dim` (no room to append, so every call
    does the same work); algorithmic bytes = (count + queries) * dim * 4."""
    g = torch.Generator(device="cuda").manual_seed(a.seed)
    store = 2.0 * torch.randn((a.count, a.dim), device="cuda", generator=g)
    qs = 2.0 * torch.randn((a.queries, a.dim), device="cuda", generator=g)
    cnt = torch.full((1,), a.count, dtype=torch.int32, device="cuda")
    app = torch.zeros(1, dtype=torch.int32, device="cuda")
    fn = lambda: P.motion_bank_check(store, cnt, app, qs, 17.0, 3, stream=stream)
    t = _time(fn, a.reps, stream)
    return {"kernel": "bank check", "s": t, "us": t * 1e6,
            "gbs": 4.0 * (a.count + a.queries) * a.dim / t / 1e9}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("what", choices=["attn", "gemm", "ddim", "sink", "nearest", "motion", "bank"])
    ap.add_argument("--queries", type=int, default=4)
    ap.add_argument("--count", type=int, default=1 << 20)
    ap.add_argument("--dim", type=int, default=128)
    ap.add_argument("--pool", type=int, default=64)
    ap.add_argument("--frames", type=int, default=16)
    ap.add_argument("--n", type=int, default=4096)
    ap.add_argument("--c", type=int, default=320)
    ap.add_argument("--heads", type=int, default=8)
    ap.add_argument("--bank", type=int, default=4)
    ap.add_argument("--m", type=int, default=65536)
    ap.add_argument("--k", type=int, default=320)
    ap.add_argument("--h", type=int, default=64)
    ap.add_argument("--w", type=int, default=64)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--seed", type=int, default=1002)
    a = ap.parse_args()
    stream = torch.cuda.Stream()
    r = {"attn": attn, "gemm": gemm, "ddim": ddim, "sink": sink, "nearest": nearest,
         "motion": motion, "bank": bank}[a.what](a, stream)
    print(json.dumps(r))


if __name__ == "__main__":
    main()
