"""Several streams served by one context (cfg.sessions = S): every session
against its own oracle state machine, and the batch against S single-stream
contexts (same numbers bit for bit)."""
import numpy as np
import pytest

import oracle as O
import synthetic as S
from _gpu_util import (ATTN_MAX_ABS, ATTN_MEAN_ABS, DDIM_ABS, attn_errors, dev, host,
                       layer_weights_np, pack_weights, scaled_gates)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

# two levels: 8x8 tokens at C = 320 (head_dim 40, two S buffers per query
# tile) and 8x8 tokens at C = 1280 (head_dim 160, one S buffer)
LAYERS = [("d00", 8, 320), ("m", 8, 1280)]
H = W = 8


@pytest.fixture(scope="module")
def P():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import denoise_step_b200 as P
    return P


class Session:
    """Seeded inputs of one stream; the weights are the model's (shared)."""

    def __init__(self, seed, walk_sigma, weights, layers=LAYERS, hw=(H, W)):
        self.seed, self.w, self.layers, self.hw = seed, weights, layers, hw
        h, w = hw
        self.ref_feats = [S.bank_features(seed, n, 0, s * s, C) for n, s, C in layers]
        self.anchors = [[S.bank_features(seed, n, a, s * s, C) for n, s, C in layers]
                        for a in range(1, 4)]
        self.ref_latent = S.normal(seed, "ref_latent", (4, h, w), 1.0, np.float32)
        self.prefill_eps = S.normal(seed, "prefill_eps", (12, 4, h, w), 1.0, np.float32)
        self.ref_motion = S.normal(seed, "walk/e0", (512,), 1.0, np.float32)
        self.drive0 = S.normal(seed, "drive0", (512,), 1.0, np.float32)
        self.walk_sigma = walk_sigma
        self.e = self.ref_motion.astype(np.float64)
        self.orc = O.PyramidStream(self.ref_latent, self.prefill_eps, self.ref_motion,
                                   self.drive0, state_dtype=np.float32)

    def next_motion(self, r):
        steps = S.normal(self.seed, f"walk/step{r}", (4, 512), self.walk_sigma)
        out = np.empty((4, 512), np.float32)
        for j in range(4):
            self.e = self.e + steps[j]
            out[j] = self.e.astype(np.float32)
            self.e = out[j].astype(np.float64)
        return out

    def round_inputs(self, r):
        h, w = self.hw
        hidden = [S.layer_hidden(self.seed, n, r, 16, s * s, C) for n, s, C in self.layers]
        noise = S.normal(self.seed, f"noise{r}", (4, 4, h, w), 1.0, np.float32)
        eps = S.normal(self.seed, f"eps{r}", (16, 4, h, w), 1.0, np.float32)
        return hidden, noise, eps

    def kv_bank(self, li, n_entries):
        return [self.ref_feats[li]] + [self.anchors[a][li] for a in range(n_entries - 1)]


def _sessions(sigmas, layers=LAYERS, hw=(H, W)):
    base = S.SEEDS["tiny"]
    weights = [layer_weights_np(base, n, C) for n, _, C in layers]
    return [Session(base + 100 * (z + 1), sig, weights, layers, hw)
            for z, sig in enumerate(sigmas)]


def _ctx(P, sess):
    """One context serving `sess` (leading session dimension on every input)."""
    layers = sess[0].layers
    cfg = P.make_config(sess[0].hw, [(s * s, C) for _, s, C in layers], sessions=len(sess))
    st = P.Stream(cfg)
    pw = [pack_weights(w) for w in sess[0].w]
    stack = lambda xs: dev(np.stack(xs))
    ref = [stack([z.ref_feats[li] for z in sess]) for li in range(len(layers))]
    anc = [stack([z.anchors[a][li] for z in sess]) for a in range(3) for li in range(len(layers))]
    st.bank_init(pw, ref, anc, stack([z.ref_motion for z in sess]),
                 stack([z.drive0 for z in sess]), stack([z.ref_latent for z in sess]),
                 stack([z.prefill_eps for z in sess]))
    return st


def _run_round(st, sess, inputs, stream):
    Sn = len(sess)
    layers, (h, w) = sess[0].layers, sess[0].hw
    stack = lambda xs: dev(np.stack(xs))
    d_hidden = [stack([inp[0][li] for inp in inputs]) for li in range(len(layers))]
    d_noise = stack([inp[1] for inp in inputs])
    d_mot = stack([inp[3] for inp in inputs])
    d_eps = stack([inp[2] for inp in inputs])
    out = torch.empty((Sn, 4, 4, h, w), dtype=torch.float32, device="cuda")
    flags = torch.zeros((Sn, 4), dtype=torch.uint8, device="cuda")
    layer_out = [torch.empty((Sn, 16, s * s, C), dtype=torch.float16, device="cuda")
                 for _, s, C in layers]
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        st.round(d_noise, d_mot, d_hidden, d_eps, out, flags, layer_out, stream=stream)
    stream.synchronize()
    return host(out), host(flags), [host(t) for t in layer_out]


def test_sessions_match_their_oracles(P):
    # three streams with different walks: their banks grow at different rounds,
    # so one attention launch serves sessions with different KV-bank lengths
    sess = _sessions([3.0, 0.5, 3.0])
    st = _ctx(P, sess)
    stream = torch.cuda.Stream()
    mixed = False     # some round ran sessions with different KV-bank lengths together
    for r in range(1, 5):
        mixed |= len({z.orc.appends for z in sess}) > 1
        inputs = []
        for z in sess:
            hidden, noise, eps = z.round_inputs(r)
            inputs.append((hidden, noise, eps, z.next_motion(r)))
        out, flags, layer_out = _run_round(st, sess, inputs, stream)
        for zi, (z, (hidden, noise, eps, mot)) in enumerate(zip(sess, inputs)):
            orc = z.orc
            n_kv = 1 + orc.appends
            orc.append(noise, mot)
            bm = orc.batch_motion()
            for li, (_, side, C) in enumerate(LAYERS):
                for f in (0, 7, 15):
                    want = O.layer_forward_frame(hidden[li][f], z.w[li], z.kv_bank(li, n_kv),
                                                 O.motion_tokens(bm[f]), 8)
                    mx, mean, rel = attn_errors(layer_out[li][zi, f], want)
                    g = scaled_gates(want)
                    assert mx <= ATTN_MAX_ABS * g and mean <= ATTN_MEAN_ABS * g, (r, zi, li, f, mx)
                    assert rel < 2e-3, (r, zi, li, f, rel)
            want_x0 = orc.step_and_pop(eps)
            _, _, want_flags = orc.check_bank(mot)
            orc.rounds += 1
            assert np.max(np.abs(out[zi] - want_x0)) <= DDIM_ABS, (r, zi)
            assert list(flags[zi]) == want_flags, (r, zi)
            s = st.state(session=zi)
            assert s["bank_count"] == len(orc.bank) and s["appends"] == orc.appends, (r, zi)
            assert [s["slot_t"][(s["head"] + k) & 3] for k in range(3)] == orc.batch_timesteps()
            assert s["rounds"] == r and s["device_status"] == 0
    for zi, z in enumerate(sess):
        assert np.array_equal(st.motion_bank(session=zi), np.array(z.orc.bank, np.float32))
    # the walks did what they were chosen for: sessions 0 and 2 hit the cap in
    # round 1, session 1 (sigma 0.5) later, so some launch mixed bank lengths
    assert sess[0].orc.appends == 3 and sess[2].orc.appends == 3
    assert mixed
    st.close()


@pytest.mark.parametrize("geometry", ["8x8", "64x64"])
def test_batched_sessions_equal_single_streams(P, geometry):
    # at 64x64 the motion cross-attention runs folded, its per-frame GEMMs in
    # one launch per 16 frames (two launches for the batched pair)
    if geometry == "8x8":
        sess = _sessions([3.0, 0.5])
    else:
        sess = _sessions([3.0, 0.5], [("d00", 64, 320)], (64, 64))
    batched = _ctx(P, sess)
    singles = [_ctx(P, [z]) for z in sess]
    stream = torch.cuda.Stream()
    for r in range(1, 4):
        inputs = []
        for z in sess:
            hidden, noise, eps = z.round_inputs(r)
            inputs.append((hidden, noise, eps, z.next_motion(r)))
        out_b, flags_b, lo_b = _run_round(batched, sess, inputs, stream)
        for zi, (z, single) in enumerate(zip(sess, singles)):
            out_s, flags_s, lo_s = _run_round(single, [z], [inputs[zi]], stream)
            assert np.array_equal(out_b[zi], out_s[0]), (r, zi)
            assert np.array_equal(flags_b[zi], flags_s[0]), (r, zi)
            for li in range(len(sess[0].layers)):
                assert np.array_equal(lo_b[li][zi], lo_s[li][0]), (r, zi, li)
            assert batched.state(session=zi) == single.state(), (r, zi)
    batched.close()
    for s in singles:
        s.close()


def test_sessions_host_round_equals_device_round(P):
    # the host-buffer round with S = 3 (staging sets scaled by S, two sets
    # alternating) against the device round of an identical context; three
    # rounds enqueued before one synchronisation
    sess = _sessions([3.0, 0.5, 3.0])
    dev_ctx = _ctx(P, sess)
    host_ctx = _ctx(P, sess)
    stream = torch.cuda.Stream()
    rounds = []
    for r in range(1, 4):
        inputs = []
        for z in sess:
            hidden, noise, eps = z.round_inputs(r)
            inputs.append((hidden, noise, eps, z.next_motion(r)))
        rounds.append(inputs)
    want = [_run_round(dev_ctx, sess, inputs, stream)[0] for inputs in rounds]
    pin = lambda xs: torch.from_numpy(np.ascontiguousarray(np.stack(xs))).pin_memory()
    h_args, h_out = [], []
    for inputs in rounds:
        h_hidden = [pin([inp[0][li] for inp in inputs]) for li in range(len(LAYERS))]
        h_args.append((pin([inp[1] for inp in inputs]), pin([inp[3] for inp in inputs]), h_hidden,
                       pin([inp[2] for inp in inputs])))
        h_out.append(torch.full((len(sess), 4, 4, H, W), float("nan")).pin_memory())
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for (hn, hm, hh, he), ho in zip(h_args, h_out):
            host_ctx.round_host(hn, hm, hh, he, ho, stream=stream)
    stream.synchronize()
    for r, (w, ho) in enumerate(zip(want, h_out)):
        assert np.array_equal(ho.numpy(), w), r
    for zi in range(len(sess)):
        assert host_ctx.state(session=zi) == dev_ctx.state(session=zi), zi
    dev_ctx.close()
    host_ctx.close()
