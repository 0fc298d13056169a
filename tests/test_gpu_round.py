"""GPU parity of whole rounds (pl_stream_round) against the oracle's deque state machine."""
import numpy as np
import pytest

import oracle as O
import synthetic as S
from _gpu_util import (ATTN_MAX_ABS, ATTN_MEAN_ABS, DDIM_ABS, attn_errors, dev, host,
                       layer_weights_np, pack_weights, scaled_gates)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def P():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import denoise_step_b200 as P
    return P


class Case:
    """Seeded inputs of a stream: weights, bank features, prefill, per-round inputs."""

    def __init__(self, seed, layers, H, W, walk_sigma, n_anchor=3):
        self.seed, self.layers, self.H, self.W = seed, layers, H, W
        self.w = [layer_weights_np(seed, name, C) for name, _, C in layers]
        self.ref_feats = [S.bank_features(seed, name, 0, side * side, C) for name, side, C in layers]
        self.anchors = [[S.bank_features(seed, name, a, side * side, C) for name, side, C in layers]
                        for a in range(1, 1 + n_anchor)]
        self.ref_latent = S.normal(seed, "ref_latent", (4, H, W), 1.0, np.float32)
        self.prefill_eps = S.normal(seed, "prefill_eps", (12, 4, H, W), 1.0, np.float32)
        self.ref_motion = S.normal(seed, "walk/e0", (512,), 1.0, np.float32)
        self.walk_sigma = walk_sigma
        self.e = self.ref_motion.astype(np.float64)
        self.drive0 = None

    def next_motion(self, r):
        steps = S.normal(self.seed, f"walk/step{r}", (4, 512), self.walk_sigma)
        out = np.empty((4, 512), np.float32)
        for j in range(4):
            self.e = self.e + steps[j]
            out[j] = self.e.astype(np.float32)
            self.e = out[j].astype(np.float64)
        return out

    def round_inputs(self, r):
        H, W = self.H, self.W
        hidden = [S.layer_hidden(self.seed, name, r, 16, side * side, C)
                  for name, side, C in self.layers]
        noise = S.normal(self.seed, f"noise{r}", (4, 4, H, W), 1.0, np.float32)
        eps = S.normal(self.seed, f"eps{r}", (16, 4, H, W), 1.0, np.float32)
        return hidden, noise, eps


def _setup(P, case):
    layers = [(side * side, C) for _, side, C in case.layers]
    cfg = P.make_config((case.H, case.W), layers)
    st = P.Stream(cfg)
    pw = [pack_weights(w) for w in case.w]
    drive0 = S.normal(case.seed, "drive0", (512,), 1.0, np.float32)
    dev_anchor = [dev(a) for an in case.anchors for a in an]
    st.bank_init(pw, [dev(f) for f in case.ref_feats], dev_anchor, dev(case.ref_motion),
                 dev(drive0), dev(case.ref_latent), dev(case.prefill_eps))
    orc = O.PyramidStream(case.ref_latent, case.prefill_eps, case.ref_motion, drive0,
                          state_dtype=np.float32)
    return st, orc, pw


def _kv_bank(case, li, n_entries):
    return [case.ref_feats[li]] + [case.anchors[a][li] for a in range(n_entries - 1)]


@pytest.mark.parametrize("walk_sigma", [3.0, 0.5])
def test_tiny_rounds_match_oracle(P, walk_sigma):
    # 16 frames, one 8x8 level (C = 1280, head_dim 160), latents 16x4x8x8
    case = Case(S.SEEDS["tiny"], [("m", 8, 1280)], 8, 8, walk_sigma)
    st, orc, _ = _setup(P, case)
    saw_keep = False        # a check that found the bank close enough (no append, room left)
    stream = torch.cuda.Stream()
    out = torch.empty((4, 4, 8, 8), dtype=torch.float32, device="cuda")
    flags = torch.zeros(4, dtype=torch.uint8, device="cuda")
    layer_out = [torch.empty((16, 64, 1280), dtype=torch.float16, device="cuda")]
    for r in range(1, 6):
        hidden, noise, eps = case.round_inputs(r)
        mot = case.next_motion(r)
        d_hidden = [dev(h) for h in hidden]
        d_noise, d_mot, d_eps = dev(noise), dev(mot), dev(eps)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            st.round(d_noise, d_mot, d_hidden, d_eps, out, flags, layer_out, stream=stream)
        stream.synchronize()
        # oracle: append, layers on the batch, step + pop, bank check
        n_kv = 1 + orc.appends
        orc.append(noise, mot)
        bm = orc.batch_motion()
        got = host(layer_out[0])
        for f in range(16):
            want = O.layer_forward_frame(hidden[0][f], case.w[0], _kv_bank(case, 0, n_kv),
                                         O.motion_tokens(bm[f]), 8)
            mx, mean, rel = attn_errors(got[f], want)
            g = scaled_gates(want)
            assert mx <= ATTN_MAX_ABS * g and mean <= ATTN_MEAN_ABS * g, (r, f, mx, mean, rel, g)
            assert rel < 2e-3, (r, f, rel)
        want_x0 = orc.step_and_pop(eps)
        appends_before = orc.appends
        _, mind2, want_flags = orc.check_bank(mot)
        saw_keep |= any(f == 0 and d <= 289.0 for f, d in zip(want_flags, mind2)) and appends_before < 3
        orc.rounds += 1
        assert np.max(np.abs(host(out) - want_x0)) <= DDIM_ABS, r
        assert list(host(flags)) == want_flags, r
        s = st.state()
        assert s["bank_count"] == len(orc.bank) and s["appends"] == orc.appends
        assert [s["slot_t"][(s["head"] + k) & 3] for k in range(3)] == orc.batch_timesteps()
        assert s["rounds"] == r and s["device_status"] == 0
    if walk_sigma == 3.0:
        assert orc.appends == 3          # step norm ~68 >> 17: the cap is reached in round 1
    else:
        assert saw_keep                  # step norm ~11: some checks stay below the threshold
    assert np.array_equal(st.motion_bank(), np.array(orc.bank, np.float32))
    st.close()


def test_host_round_matches_device_round(P):
    # the host-buffer round (inputs copied on the context's copy stream into
    # two alternating staging sets, x0 frames copied back) gives the device
    # round's frames bit for bit, with four rounds enqueued back to back
    # before a single synchronisation
    case = Case(S.SEEDS["tiny"], [("m", 8, 1280)], 8, 8, 3.0)
    st_a, _, _ = _setup(P, case)
    st_b, _, _ = _setup(P, Case(S.SEEDS["tiny"], [("m", 8, 1280)], 8, 8, 3.0))
    stream = torch.cuda.Stream()
    ins = []
    for r in range(1, 5):
        hidden, noise, eps = case.round_inputs(r)
        ins.append((hidden, noise, case.next_motion(r), eps))
    want = []
    out = torch.empty((4, 4, 8, 8), dtype=torch.float32, device="cuda")
    for hidden, noise, mot, eps in ins:
        d_args = (dev(noise), dev(mot), [dev(h) for h in hidden], dev(eps))
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            st_a.round(*d_args, out, stream=stream)
        stream.synchronize()
        want.append(host(out).copy())
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    h_in = [([pin(h) for h in hidden], pin(noise), pin(mot), pin(eps))
            for hidden, noise, mot, eps in ins]
    h_out = [torch.full((4, 4, 8, 8), float("nan"), dtype=torch.float32).pin_memory() for _ in ins]
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for (hh, hn, hm, he), ho in zip(h_in, h_out):
            st_b.round_host(hn, hm, hh, he, ho, stream=stream)
    stream.synchronize()
    for r, (w, ho) in enumerate(zip(want, h_out)):
        assert np.array_equal(ho.numpy(), w), r
    assert st_a.state() == st_b.state()
    assert st_b.device_status() == 0
    st_a.close()
    st_b.close()


def test_full_geometry_rounds_spot_checked(P):
    # 16 reference-attention layers in the SD-UNet layout, bank x4 after round 1,
    # DDIM on 16x4x64x64, bank check; sampled rows of one layer per level. In
    # round 2 the round also returns the reference-attention sub-layer output
    # (Wo and Mq then applied separately), held to the plain attention gates;
    # rounds 1 and 3 run the folded Wo Mq projection
    case = Case(S.SEEDS["full"], list(S.LAYERS), 64, 64, 3.0)
    st, orc, _ = _setup(P, case)
    stream = torch.cuda.Stream()
    out = torch.empty((4, 4, 64, 64), dtype=torch.float32, device="cuda")
    flags = torch.zeros(4, dtype=torch.uint8, device="cuda")
    layer_out = [torch.empty((16, side * side, C), dtype=torch.float16, device="cuda")
                 for _, side, C in case.layers]
    attn_out = [torch.empty_like(t) for t in layer_out]
    check_layers = {0: "d00", 2: "d10", 4: "d20", 6: "m", 15: "u32"}
    rows_all = S.uniform_int(case.seed, "rows", 24, 4096)
    for r in range(1, 4):
        hidden, noise, eps = case.round_inputs(r)
        mot = case.next_motion(r)
        d_hidden = [dev(h) for h in hidden]
        d_noise, d_mot, d_eps = dev(noise), dev(mot), dev(eps)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            st.round(d_noise, d_mot, d_hidden, d_eps, out, flags, layer_out, stream=stream,
                     attn_out=attn_out if r == 2 else None)
        stream.synchronize()
        n_kv = 1 + orc.appends
        orc.append(noise, mot)
        bm = orc.batch_motion()
        for li in check_layers:
            _, side, C = case.layers[li]
            N = side * side
            rows = np.unique(rows_all % N)
            got = host(layer_out[li])
            got_a = host(attn_out[li]) if r == 2 else None
            for f in (0, 9):
                if got_a is not None:
                    want_a = O.ref_attention_frame(hidden[li][f], case.w[li],
                                                   _kv_bank(case, li, n_kv), 8, rows=rows)
                    mx, mean, rel = attn_errors(got_a[f][rows], want_a)
                    assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (r, li, f, mx, mean, rel)
                want = O.layer_forward_frame(hidden[li][f], case.w[li], _kv_bank(case, li, n_kv),
                                             O.motion_tokens(bm[f]), 8, rows=rows)
                mx, mean, rel = attn_errors(got[f][rows], want)
                g = scaled_gates(want)
                assert mx <= ATTN_MAX_ABS * g and mean <= ATTN_MEAN_ABS * g, (r, li, f, mx, mean, rel)
                assert rel < 2e-3, (r, li, f, rel)
        want_x0 = orc.step_and_pop(eps)
        _, _, want_flags = orc.check_bank(mot)
        assert np.max(np.abs(host(out) - want_x0)) <= DDIM_ABS, r
        assert list(host(flags)) == want_flags
        s = st.state()
        assert s["appends"] == orc.appends and s["device_status"] == 0
    assert orc.appends == 3
    st.close()


def _block2_logit_std(h, w, bank, motion, heads=8, rows=None):
    """Std of the second motion block's logits (fp64, oracle inputs; `rows`:
    those query rows only)."""
    tok = O.motion_tokens(motion)
    y1 = O.motion_xattn_frame(O.ref_attention_frame(h, w, bank, heads, rows=rows), tok, w, heads)
    q = y1 @ np.asarray(w["mq2"], np.float64)
    k = tok @ np.asarray(w["mk2"], np.float64)
    hd = q.shape[1] // heads
    s = [q[:, i * hd:(i + 1) * hd] @ k[:, i * hd:(i + 1) * hd].T / np.sqrt(hd) for i in range(heads)]
    return float(np.std(np.concatenate([x.ravel() for x in s])))


@pytest.mark.parametrize("sublayer", [False, True])
def test_two_motion_blocks_tiny_rounds(P, sublayer):
    # two motion cross-attention blocks per layer (own weights, same tokens,
    # block 2 queried by block 1's output), tiny geometry, 3 rounds; with
    # `sublayer` the round also returns the reference-attention output and
    # applies Wo, Mq, Mo, Mq2 separately, else their folded products. Block
    # 2's queries come from block 1's fp16 output, whose magnitude follows the
    # walking motion embedding, and its softmax multiplies that rounding by
    # the spread of its logits: the layer-output gates carry that factor
    # (kappa, as on the long stream); the sub-layer output has plain gates
    case = Case(S.SEEDS["tiny"] + 7, [("m", 8, 1280)], 8, 8, 3.0)
    case.w[0].update(S.motion_block_weights(case.seed, "m", 1280, 2, np.float16))
    cfg = P.make_config((8, 8), [(64, 1280)], motion_blocks=2)
    st = P.Stream(cfg)
    pw = [pack_weights(w) for w in case.w]
    drive0 = S.normal(case.seed, "drive0", (512,), 1.0, np.float32)
    st.bank_init(pw, [dev(f) for f in case.ref_feats], [dev(a) for an in case.anchors for a in an],
                 dev(case.ref_motion), dev(drive0), dev(case.ref_latent), dev(case.prefill_eps))
    orc = O.PyramidStream(case.ref_latent, case.prefill_eps, case.ref_motion, drive0,
                          state_dtype=np.float32)
    stream = torch.cuda.Stream()
    out = torch.empty((4, 4, 8, 8), dtype=torch.float32, device="cuda")
    flags = torch.zeros(4, dtype=torch.uint8, device="cuda")
    layer_out = [torch.empty((16, 64, 1280), dtype=torch.float16, device="cuda")]
    attn_out = [torch.empty_like(layer_out[0])] if sublayer else None
    for r in range(1, 4):
        hidden, noise, eps = case.round_inputs(r)
        mot = case.next_motion(r)
        d_in = ([dev(h) for h in hidden], dev(noise), dev(mot), dev(eps))
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            st.round(d_in[1], d_in[2], d_in[0], d_in[3], out, flags, layer_out, stream=stream,
                     attn_out=attn_out)
        stream.synchronize()
        n_kv = 1 + orc.appends
        orc.append(noise, mot)
        bm = orc.batch_motion()
        got = host(layer_out[0])
        for f in range(0, 16, 3):
            bank = _kv_bank(case, 0, n_kv)
            want = O.layer_forward_frame(hidden[0][f], case.w[0], bank, O.motion_tokens(bm[f]), 8,
                                         motion_blocks=2)
            mx, mean, rel = attn_errors(got[f], want)
            g = scaled_gates(want)
            kappa = max(1.0, _block2_logit_std(hidden[0][f], case.w[0], bank, bm[f]))
            assert mx <= ATTN_MAX_ABS * g * kappa and mean <= ATTN_MEAN_ABS * g * kappa, \
                (r, f, mx, mean, rel, g, kappa)
            assert rel < 2e-3 * kappa, (r, f, rel, kappa)
            if sublayer:
                want_a = O.ref_attention_frame(hidden[0][f], case.w[0], bank, 8)
                mx, mean, rel = attn_errors(host(attn_out[0])[f], want_a)
                assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (r, f, mx, mean, rel)
        want_x0 = orc.step_and_pop(eps)
        _, _, want_flags = orc.check_bank(mot)
        orc.rounds += 1
        assert np.max(np.abs(host(out) - want_x0)) <= DDIM_ABS, r
        assert list(host(flags)) == want_flags, r
    assert st.device_status() == 0
    st.close()


@pytest.mark.parametrize("sublayer", [False, True])
def test_two_motion_blocks_level64_folded(P, sublayer):
    # At 64x64 the round runs the motion cross-attention folded: per frame the
    # scores X W_qk (W_qk = Wq K^T / sqrt(hd), fp16) with the softmax over each
    # head's 32 tokens in the GEMM epilogue, then the block output P VM (VM =
    # V Mo per head). Two blocks, block 2 queried by block 1's fp16 output,
    # two rounds (bank x2 in round 2), sampled rows of frames 0 and 9, the
    # gates of the tiny two-block rounds; with `sublayer` Wo, Mq and Mq2 are
    # applied separately and the reference-attention output is checked too
    case = Case(S.SEEDS["tiny"] + 11, [("m", 64, 320)], 64, 64, 3.0)
    case.w[0].update(S.motion_block_weights(case.seed, "m", 320, 2, np.float16))
    cfg = P.make_config((64, 64), [(4096, 320)], motion_blocks=2)
    st = P.Stream(cfg)
    pw = [pack_weights(w) for w in case.w]
    drive0 = S.normal(case.seed, "drive0", (512,), 1.0, np.float32)
    st.bank_init(pw, [dev(f) for f in case.ref_feats], [dev(a) for an in case.anchors for a in an],
                 dev(case.ref_motion), dev(drive0), dev(case.ref_latent), dev(case.prefill_eps))
    orc = O.PyramidStream(case.ref_latent, case.prefill_eps, case.ref_motion, drive0,
                          state_dtype=np.float32)
    stream = torch.cuda.Stream()
    out = torch.empty((4, 4, 64, 64), dtype=torch.float32, device="cuda")
    flags = torch.zeros(4, dtype=torch.uint8, device="cuda")
    layer_out = [torch.empty((16, 4096, 320), dtype=torch.float16, device="cuda")]
    attn_out = [torch.empty_like(layer_out[0])] if sublayer else None
    rows = np.unique(S.uniform_int(case.seed, "rows", 24, 4096))
    for r in (1, 2):
        hidden, noise, eps = case.round_inputs(r)
        mot = case.next_motion(r)
        d_in = ([dev(h) for h in hidden], dev(noise), dev(mot), dev(eps))
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            st.round(d_in[1], d_in[2], d_in[0], d_in[3], out, flags, layer_out, stream=stream,
                     attn_out=attn_out)
        stream.synchronize()
        n_kv = 1 + orc.appends
        orc.append(noise, mot)
        bm = orc.batch_motion()
        got = host(layer_out[0])
        for f in (0, 9):
            bank = _kv_bank(case, 0, n_kv)
            want = O.layer_forward_frame(hidden[0][f], case.w[0], bank, O.motion_tokens(bm[f]), 8,
                                         rows=rows, motion_blocks=2)
            mx, mean, rel = attn_errors(got[f][rows], want)
            g = scaled_gates(want)
            kappa = max(1.0, _block2_logit_std(hidden[0][f], case.w[0], bank, bm[f], rows=rows))
            assert mx <= ATTN_MAX_ABS * g * kappa and mean <= ATTN_MEAN_ABS * g * kappa, \
                (r, f, mx, mean, rel, g, kappa)
            assert rel < 2e-3 * kappa, (r, f, rel, kappa)
            if sublayer:
                want_a = O.ref_attention_frame(hidden[0][f], case.w[0], bank, 8, rows=rows)
                mx, mean, rel = attn_errors(host(attn_out[0])[f][rows], want_a)
                assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (r, f, mx, mean, rel)
        want_x0 = orc.step_and_pop(eps)
        _, _, want_flags = orc.check_bank(mot)
        orc.rounds += 1
        assert np.max(np.abs(host(out) - want_x0)) <= DDIM_ABS, r
        assert list(host(flags)) == want_flags, r
    assert st.device_status() == 0
    st.close()
