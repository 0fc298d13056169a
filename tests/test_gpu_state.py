"""Checkpoint / resume of a stream and per-layer profiling, on the GPU.

A stream run for three rounds (the walk appends all three anchors in round
1), exported, imported into a fresh context after its pl_bank_init and run
for three more rounds must give the uninterrupted stream's frames, flags,
layer outputs and state bit for bit. Snapshots that do not fit the context
or hold an impossible state are refused before anything is written. A
profiled round (events around each layer, outside the graph) gives the
graph round's outputs and positive layer times.
"""
import numpy as np
import pytest

import synthetic as S
from _gpu_util import dev, host, layer_weights_np, pack_weights

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def P():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import denoise_step_b200 as P
    return P


LAYERS = [("m", 8, 1280), ("d20", 16, 1280)]


def _inputs(seed):
    w = [pack_weights(layer_weights_np(seed, n, C)) for n, _, C in LAYERS]
    ref = [dev(S.bank_features(seed, n, 0, s * s, C)) for n, s, C in LAYERS]
    anchors = [dev(S.bank_features(seed, n, a, s * s, C)) for a in (1, 2, 3) for n, s, C in LAYERS]
    fixed = [dev(S.normal(seed, "walk/e0", (512,), 1.0, np.float32)),
             dev(S.normal(seed, "drive0", (512,), 1.0, np.float32)),
             dev(S.normal(seed, "ref_latent", (4, 8, 8), 1.0, np.float32)),
             dev(S.normal(seed, "prefill_eps", (12, 4, 8, 8), 1.0, np.float32))]
    return w, ref, anchors, fixed


def _round_inputs(seed, r):
    hidden = [dev(S.layer_hidden(seed, n, r, 16, s * s, C)) for n, s, C in LAYERS]
    noise = dev(S.normal(seed, f"noise{r}", (4, 4, 8, 8), 1.0, np.float32))
    mot = dev((S.normal(seed, "walk/e0", (512,), 1.0)[None]
               + S.normal(seed, f"walk/{r}", (4, 512), 3.0).cumsum(0)).astype(np.float32))
    eps = dev(S.normal(seed, f"eps{r}", (16, 4, 8, 8), 1.0, np.float32))
    return hidden, noise, mot, eps


def _stream(P, seed):
    st = P.Stream(P.make_config((8, 8), [(s * s, C) for _, s, C in LAYERS]))
    w, ref, anchors, fixed = _inputs(seed)
    st.bank_init(w, ref, anchors, *fixed)
    st._inputs = (w, ref, anchors, fixed)
    return st


def _run(P, st, seed, r, stream):
    hidden, noise, mot, eps = _round_inputs(seed, r)
    out = torch.empty((4, 4, 8, 8), dtype=torch.float32, device="cuda")
    flags = torch.zeros(4, dtype=torch.uint8, device="cuda")
    lo = [torch.empty((16, s * s, C), dtype=torch.float16, device="cuda") for _, s, C in LAYERS]
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        st.round(noise, mot, hidden, eps, out, flags, lo, stream=stream)
    stream.synchronize()
    return host(out), host(flags), [host(t) for t in lo]


def test_export_import_continues_the_stream_bit_for_bit(P):
    seed = 3001
    stream = torch.cuda.Stream()
    a = _stream(P, seed)
    for r in range(1, 4):
        _run(P, a, seed, r, stream)
    snap = a.export_state(stream)
    assert a.state()["appends"] == 3 and a.state()["rounds"] == 3
    b = _stream(P, seed)
    b.import_state(snap, stream)
    assert b.state() == a.state()
    assert np.array_equal(b.motion_bank(), a.motion_bank())
    for r in range(4, 7):
        oa, fa, la = _run(P, a, seed, r, stream)
        ob, fb, lb = _run(P, b, seed, r, stream)
        assert np.array_equal(oa, ob) and np.array_equal(fa, fb), r
        for x, y in zip(la, lb):
            assert np.array_equal(x, y), r
    assert b.state() == a.state() and b.device_status() == 0
    a.close()
    b.close()


def test_import_refuses_mismatched_or_impossible_snapshots(P):
    seed = 3002
    stream = torch.cuda.Stream()
    a = _stream(P, seed)
    _run(P, a, seed, 1, stream)
    snap = a.export_state(stream)
    # another latent size: refused
    other = P.Stream(P.make_config((16, 16), [(s * s, C) for _, s, C in LAYERS]))
    w, ref, anchors, fixed = _inputs(seed)
    other.bank_init(w, ref, anchors, fixed[0], fixed[1],
                    dev(S.normal(seed, "rl16", (4, 16, 16), 1.0, np.float32)),
                    dev(S.normal(seed, "pe16", (12, 4, 16, 16), 1.0, np.float32)))
    with pytest.raises(P.PLError) as e:
        other.import_state(snap, stream)
    assert e.value.status == P.PL_EINVAL
    # a bank count past the capacity: refused, the target keeps its state
    b = _stream(P, seed)
    before = b.state()
    bad = snap.copy()
    hdr = 8 + 4 + 4 + 4 * 4 + 4 * 8          # header bytes
    bad[hdr + 5 * 4:hdr + 6 * 4] = np.frombuffer(np.int32(7).tobytes(), np.uint8)   # bank_count
    with pytest.raises(P.PLError) as e:
        b.import_state(bad, stream)
    assert e.value.status == P.PL_EINVAL and b.state() == before
    with pytest.raises(P.PLError):
        b.import_state(snap[:100], stream)
    for s in (a, b, other):
        s.close()


def test_profiled_round_matches_the_graph_round(P):
    seed = 3003
    stream = torch.cuda.Stream()
    a = _stream(P, seed)
    b = _stream(P, seed)
    b.set_profiling(True)
    with pytest.raises(P.PLError):
        b.layer_ms()                          # no profiled round yet
    for r in (1, 2):
        oa, fa, la = _run(P, a, seed, r, stream)
        ob, fb, lb = _run(P, b, seed, r, stream)
        assert np.array_equal(oa, ob) and np.array_equal(fa, fb)
        for x, y in zip(la, lb):
            assert np.array_equal(x, y)
        ms = b.layer_ms()
        assert len(ms) == len(LAYERS) and all(t > 0 for t in ms), ms
    b.set_profiling(False)
    with pytest.raises(P.PLError):
        b.layer_ms()
    with pytest.raises(P.PLError):
        b.round_kernels()                     # b has run no round from a capture
    # a ran from its captured graph: the same kernel count every round, at
    # least the reference attention, its projection and the motion sub-layer
    # per layer plus the ring, DDIM and bank-check kernels
    k = a.round_kernels()
    assert k >= 3 * len(LAYERS) + 4, k
    _run(P, a, seed, 3, stream)
    assert a.round_kernels() == k
    a.close()
    b.close()
