"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test pins the oracle to something other than itself: constants printed
on the pages (tests/golden/), closed forms, invariants, special cases and
brute force on tiny inputs. CPU only.
"""
import math
import os

import numpy as np
import pytest

import oracle as O
import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "personalive_constants.txt")


def _golden():
    out = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = (s.strip() for s in line.split("=", 1))
                out[k] = v
    return out


# ---------------------------------------------------------------- constants

def test_constants_match_pages():
    g = _golden()
    assert int(g["temporal_adaptive_step"]) == O.TEMPORAL_ADAPTIVE_STEP
    assert int(g["temporal_window_size"]) == O.TEMPORAL_WINDOW_SIZE
    assert int(g["num_inference_steps"]) == O.NUM_INFERENCE_STEPS
    assert tuple(int(x) for x in g["timesteps"].split(",")) == O.TIMESTEPS
    assert int(g["step_length"]) == O.STEP_LENGTH
    assert int(g["batch_frames"]) == O.TEMPORAL_ADAPTIVE_STEP * O.TEMPORAL_WINDOW_SIZE
    assert int(g["drift_threshold"]) == O.DRIFT_THRESHOLD
    assert int(g["append_cap"]) == O.APPEND_CAP
    assert int(g["motion_dim"]) == O.MOTION_DIM
    assert int(g["motion_tokens"]) * int(g["motion_token_dim"]) == O.MOTION_DIM
    assert int(g["motion_token_dim"]) == O.MOTION_TOKEN_DIM
    assert int(g["motion_heads"]) == S.HEADS
    assert tuple(g["reference_layers"].split(",")) == tuple(n for n, _, _ in S.LAYERS)
    assert max(int(x) for x in g["bank_dims"].split(",")) == 1 + O.APPEND_CAP
    # the ladder: consecutive table entries differ by the step length
    assert all(a - b == O.STEP_LENGTH for a, b in zip(O.TIMESTEPS, O.TIMESTEPS[1:]))
    assert int(g["prefill_frames"]) == (O.TEMPORAL_ADAPTIVE_STEP - 1) * O.TEMPORAL_WINDOW_SIZE


# ---------------------------------------------------------------- schedule

def test_beta_endpoints_and_sqrt_linearity():
    b = O.betas()
    assert b.shape == (1000,)
    assert abs(b[0] - 0.00085) < 1e-15
    assert abs(b[-1] - 0.012) < 1e-15
    r = np.sqrt(b)
    # sqrt(beta) is an arithmetic progression: zero second differences
    assert np.max(np.abs(np.diff(r, 2))) < 1e-15
    assert np.all(np.diff(b) > 0)


def test_alphas_cumprod_recursion_and_log_route():
    b = O.betas()
    a = O.alphas_cumprod()
    assert abs(a[0] - (1 - b[0])) < 1e-16
    # ratio of consecutive products is the per-step survival 1 - beta
    assert np.max(np.abs(a[1:] / a[:-1] - (1 - b[1:]))) < 1e-14
    assert np.all(np.diff(a) < 0)
    # independent route through logarithms
    via_log = np.exp(np.cumsum(np.log1p(-b)))
    assert np.max(np.abs(via_log / a - 1)) < 1e-12
    assert O.alpha_bar(-333) == 1.0


# ---------------------------------------------------------------- DDIM

@pytest.mark.parametrize("t", [999, 666, 333, 0])
def test_x0_inverts_forward_noising(t):
    x0 = S.normal(7, "x0", (4, 8, 8))
    eps = S.normal(7, "eps", (4, 8, 8))
    xt = O.forward_noise(x0, eps, t)
    _, x0_hat = O.ddim_step(xt, eps, t)
    assert np.max(np.abs(x0_hat - x0)) < 1e-12


@pytest.mark.parametrize("t", [999, 666, 333])
def test_eta0_step_lands_on_forward_trajectory(t):
    # with the true epsilon, a deterministic DDIM step lands exactly on q(x_{t-333} | x0)
    x0 = S.normal(8, "x0", (4, 8, 8))
    eps = S.normal(8, "eps", (4, 8, 8))
    x_prev, _ = O.ddim_step(O.forward_noise(x0, eps, t), eps, t)
    assert np.max(np.abs(x_prev - O.forward_noise(x0, eps, t - 333))) < 1e-12


def test_t0_step_prev_equals_x0():
    x = S.normal(9, "x", (4, 8, 8))
    e = S.normal(9, "e", (4, 8, 8))
    x_prev, x0 = O.ddim_step(x, e, 0)
    assert np.array_equal(x_prev, x0)


def test_ddim_consistency_over_the_ladder():
    # constant epsilon per window: x0 predicted at t=999 equals the x0 popped at t=0
    x = S.normal(10, "x999", (4, 8, 8))
    e = S.normal(10, "e", (4, 8, 8))
    _, x0_first = O.ddim_step(x, e, 999)
    cur = x
    for t in (999, 666, 333):
        cur, _ = O.ddim_step(cur, e, t)
    _, x0_last = O.ddim_step(cur, e, 0)
    assert np.max(np.abs(x0_first - x0_last)) < 1e-12


# ---------------------------------------------------------------- stream state machine

def _stream(seed, H=8, W=8, dtype=np.float64):
    ref = S.normal(seed, "ref_latent", (4, H, W))
    pe = S.normal(seed, "prefill_eps", (12, 4, H, W))
    rm = S.normal(seed, "ref_motion", (512,))
    d0 = S.normal(seed, "drive0", (512,))
    return O.PyramidStream(ref, pe, rm, d0, state_dtype=dtype), ref, pe


def test_prefill_staircase_and_first_round_outputs_reference():
    st, ref, pe = _stream(11)
    assert st.batch_timesteps() == [0, 333, 666]
    # round 1 with the prefill noise as epsilon pops the oldest prefill window:
    # its x0 is the reference latent itself
    eps = np.zeros((16, 4, 8, 8))
    eps[0:12] = pe
    out, *_ = st.round(S.normal(11, "n", (4, 4, 8, 8)), S.normal(11, "m", (4, 512)), eps)
    assert np.max(np.abs(out - ref[None])) < 1e-12


def test_ladder_queue_and_output_order():
    # every window carries a marker x0 and a constant epsilon; the popped x0
    # identifies which driving frames come out in which round
    H = W = 4
    st, ref, pe = _stream(12, H, W)
    R = 12
    eps_of = {}          # window id -> its constant epsilon
    win_ids = ["pA", "pB", "pC"]
    for i, wid in enumerate(win_ids):
        eps_of[wid] = pe[4 * i:4 * i + 4]
    pops = []
    for r in range(1, R + 1):
        wid = f"d{r}"
        marker = np.zeros((4, 4, H, W))
        for j in range(4):
            marker[j] = 4 * (r - 1) + j + 100.0          # driving frame index + 100
        e = S.normal(12, f"e{r}", (4, 4, H, W))
        eps_of[wid] = e
        st.append(O.forward_noise(marker, e, 999), S.normal(12, f"m{r}", (4, 512)))
        win_ids.append(wid)
        assert st.batch_timesteps() == [0, 333, 666, 999]
        assert len(st.pile) == 4
        eps = np.concatenate([eps_of[w] for w in win_ids[-4:]], axis=0)
        out = st.step_and_pop(eps)
        pops.append(out)
        assert st.batch_timesteps() == [0, 333, 666]
        assert st.frames_in == 4 * r and st.frames_out == 4 * r
        win_ids = win_ids[-3:]
    # driving frame k is output at round k // 4 + 4 (1-indexed)
    for r in range(4, R + 1):
        for j in range(4):
            k = 4 * (r - 4) + j
            assert abs(pops[r - 1][j].mean() - (k + 100.0)) < 1e-9
            assert (k // 4) + 4 == r


def test_prefill_motion_ramp():
    a = S.normal(13, "a", (512,))
    b = S.normal(13, "b", (512,))
    m = O.prefill_motion(a, b)
    assert m.shape == (12, 512)
    assert np.array_equal(m[0], a)
    full = O.interpolate(a, b, 13)
    assert np.max(np.abs(full[-1] - b)) < 1e-12          # the dropped 13th point is drive0
    d = np.diff(full, axis=0)
    assert np.max(np.abs(d - (b - a) / 12)) < 1e-12       # equal spacing


# ---------------------------------------------------------------- motion bank

def test_threshold_edge_is_strict():
    bank = [np.zeros(512)]
    q = np.zeros(512)
    q[0] = 17.0
    _, d2, flags, _, n = O.bank_check(bank, [q], 0)
    assert d2 == [289.0] and flags == [0] and n == 0
    q2 = np.zeros(512, np.float32)
    q2[0] = np.nextafter(np.float32(17.0), np.float32(100.0))
    _, d2, flags, bank2, n = O.bank_check(bank, [q2], 0)
    assert d2[0] > 289.0 and flags == [1] and n == 1 and len(bank2) == 2


def test_appends_see_earlier_appends_and_cap():
    bank = [np.zeros(4)]
    qs = [np.array([20.0, 0, 0, 0]), np.array([21.0, 0, 0, 0]),
          np.array([0, 40.0, 0, 0]), np.array([0, 0, 60.0, 0]), np.array([0, 0, 0, 90.0])]
    amin, d2, flags, bank2, n = O.bank_check(bank, qs, 0)
    # q1 is within 1 of the just-appended q0, so it does not append
    assert flags == [1, 0, 1, 1, 0]
    assert amin[1] == 1 and d2[1] == 1.0
    assert n == 3 and len(bank2) == 4


def test_argmin_ties_lowest_index():
    bank = [np.array([1.0, 0]), np.array([-1.0, 0]), np.array([0, 1.0])]
    amin, d2, *_ = O.bank_check(bank, [np.zeros(2)], 0)
    assert amin == [0] and d2 == [1.0]


def test_long_walk_caps_at_three():
    # seeded Gaussian random walk of the 512-d embedding, step sigma 3
    st, *_ = _stream(14, 2, 2)
    e = S.normal(1004, "walk/e0", (512,))
    st.bank = [e.copy()]
    rounds = 300
    steps = S.normal(1004, "walk/steps", (rounds * 4, 512), 3.0)
    for r in range(rounds):
        qs = []
        for j in range(4):
            e = e + steps[4 * r + j]
            qs.append(e.copy())
        st.check_bank(qs)
        assert 1 <= len(st.bank) <= 4 and st.appends <= 3
    assert st.appends == 3


def test_small_walk_exercises_no_append_branch():
    e0 = S.normal(15, "e0", (512,))
    qs = [e0 + S.normal(15, f"s{i}", (512,), 0.5) for i in range(8)]
    _, d2, flags, _, n = O.bank_check([e0], qs[:1], 0)
    assert flags == [0] and d2[0] < 289.0


def test_pose_retrieve_brute_force():
    store = S.normal(16, "store", (64, 64))
    d = S.normal(16, "d", (64,))
    j = O.pose_retrieve(store, d)
    best = min(range(64), key=lambda i: sum((float(d[k]) - float(store[i, k])) ** 2 for k in range(64)))
    assert j == best


# ---------------------------------------------------------------- attention

def _brute_attention(q, k, v, heads):
    """Pure-Python loops: softmax(q k^T / sqrt(hd)) v per head."""
    Nq, C = len(q), len(q[0])
    hd = C // heads
    out = [[0.0] * C for _ in range(Nq)]
    for h in range(heads):
        c0 = h * hd
        for i in range(Nq):
            s = [sum(q[i][c0 + c] * k[j][c0 + c] for c in range(hd)) / math.sqrt(hd) for j in range(len(k))]
            m = max(s)
            w = [math.exp(x - m) for x in s]
            z = sum(w)
            for c in range(hd):
                out[i][c0 + c] = sum(w[j] * v[j][c0 + c] for j in range(len(k))) / z
    return np.array(out)


def test_two_key_closed_form():
    q = np.array([[0.3, -1.2, 0.7, 2.0]])
    k = np.array([[1.0, 0.5, -0.5, 0.25], [-0.75, 0.1, 1.5, -0.3]])
    v = np.array([[2.0, -1.0, 0.5, 3.0], [-4.0, 1.0, 0.0, 1.0]])
    s1 = float(q[0] @ k[0]) / 2.0
    s2 = float(q[0] @ k[1]) / 2.0
    sig = lambda x: 1.0 / (1.0 + math.exp(-x))
    want = sig(s1 - s2) * v[0] + sig(s2 - s1) * v[1]
    got = O.mha(q, k, v, heads=1)
    assert np.max(np.abs(got[0] - want)) < 1e-15


def test_mha_brute_force_tiny():
    q = S.normal(17, "q", (3, 8))
    k = S.normal(17, "k", (5, 8))
    v = S.normal(17, "v", (5, 8))
    assert np.max(np.abs(O.mha(q, k, v, 2) - _brute_attention(q.tolist(), k.tolist(), v.tolist(), 2))) < 1e-13


def _tiny_layer(seed, N=6, C=16, nb=2):
    w = S.layer_weights(seed, "t", C, np.float64)
    h = S.normal(seed, "h", (N, C))
    bank = [S.normal(seed, f"b{i}", (N, C)) for i in range(nb)]
    return h, w, bank


def test_ref_attention_brute_force_with_explicit_concat():
    h, w, bank = _tiny_layer(18)
    feats = np.concatenate([h] + bank)
    want = _brute_attention((h @ w["wq"]).tolist(), (feats @ w["wk"]).tolist(),
                            (feats @ w["wv"]).tolist(), 8) @ w["wo"]
    got = O.ref_attention_frame(h, w, bank, heads=8)
    assert np.max(np.abs(got - want)) < 1e-12


def test_bank_equal_to_own_keeps_weights():
    h, w, _ = _tiny_layer(19)
    a = O.ref_attention_frame(h, w, [], 8)
    b = O.ref_attention_frame(h, w, [h, h, h], 8)
    assert np.max(np.abs(a - b)) < 1e-12


def test_constant_values_and_zero_queries():
    h, w, bank = _tiny_layer(20)
    C = h.shape[1]
    # Wv reads only input column 0, which is 1 on every token: all value rows
    # equal vrow, so every output row is vrow Wo whatever the weights are
    vrow = S.normal(20, "vrow", (C,))
    w2 = dict(w)
    w2["wv"] = np.zeros((C, C))
    w2["wv"][0, :] = vrow
    h_c = h.copy()
    h_c[:, 0] = 1.0
    bank_c = [b.copy() for b in bank]
    for b in bank_c:
        b[:, 0] = 1.0
    got = O.ref_attention_frame(h_c, w2, bank_c, 8)
    assert np.max(np.abs(got - (vrow @ w2["wo"])[None])) < 1e-12
    # zero queries: uniform weights, output = mean of V over [own ; bank]
    w3 = dict(w)
    w3["wq"] = np.zeros((C, C))
    feats = np.concatenate([h] + bank)
    want = (feats @ w["wv"]).mean(axis=0) @ w["wo"]
    got = O.ref_attention_frame(h, w3, bank, 8)
    assert np.max(np.abs(got - want[None])) < 1e-12


def test_key_permutation_invariance_and_rows_subset():
    h, w, bank = _tiny_layer(21)
    a = O.ref_attention_frame(h, w, bank, 8)
    b = O.ref_attention_frame(h, w, bank[::-1], 8)
    assert np.max(np.abs(a - b)) < 1e-12
    rows = np.array([4, 1])
    c = O.ref_attention_frame(h, w, bank, 8, rows=rows)
    assert np.max(np.abs(c - a[rows])) < 1e-12


def test_segment_attention_matches_concat():
    q = S.normal(22, "q", (4, 16))
    segs = [S.normal(22, f"k{i}", (3, 16)) for i in range(3)]
    vals = [S.normal(22, f"v{i}", (3, 16)) for i in range(3)]
    want = _brute_attention(q.tolist(), np.concatenate(segs).tolist(), np.concatenate(vals).tolist(), 2)
    assert np.max(np.abs(O.segment_attention(q, segs, vals, 2) - want)) < 1e-13


# ---------------------------------------------------------------- motion

def test_motion_pe_structure():
    pe = O.motion_pe()
    assert pe.shape == (32, 16)
    assert np.array_equal(pe[0], np.tile([0.0, 1.0], 8))
    # each (sin, cos) pair lies on the unit circle
    assert np.max(np.abs((pe[:, 0::2] ** 2 + pe[:, 1::2] ** 2) - 1)) < 1e-15
    # the first pair has unit frequency, frequencies fall with the pair index
    p = np.arange(32)
    assert np.max(np.abs(pe[:, 0] - np.sin(p))) < 1e-15
    assert np.max(np.abs(pe[:, 1] - np.cos(p))) < 1e-15


def test_motion_pe_hand_values_at_later_pairs():
    # literal values of later pairs (golden file): an exponent i/d instead of
    # 2i/d, a swapped sin/cos or a shifted pair index fails here
    path = os.path.join(os.path.dirname(__file__), "golden", "motion_pe_values.txt")
    pe = O.motion_pe()
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 8
    for p, c, v in rows:
        assert abs(pe[int(p), int(c)] - float(v)) < 1e-14, (p, c)


def test_motion_pe_frequency_drops_a_decade_every_two_pairs():
    # pair i + 2 turns ten times slower than pair i (10000^(-2(i+2)/16) =
    # 10000^(-2i/16) / 10), so position 10p on pair i + 2 repeats position p
    # on pair i; with any other exponent the decade lands elsewhere
    pe = O.motion_pe()
    for p in (1, 2, 3):
        for i in range(6):
            assert abs(pe[10 * p, 2 * (i + 2)] - pe[p, 2 * i]) < 1e-12, (p, i)
            assert abs(pe[10 * p, 2 * (i + 2) + 1] - pe[p, 2 * i + 1]) < 1e-12, (p, i)


def test_motion_tokens_reshape_is_row_major():
    e = np.arange(512, dtype=np.float64)
    tok = O.motion_tokens(e) - O.motion_pe()
    assert np.array_equal(tok[3], np.arange(48, 64, dtype=np.float64))


def test_motion_xattn_identical_tokens():
    C = 32
    w = S.layer_weights(23, "mx", C, np.float64)
    x = S.normal(23, "x", (5, C))
    m = np.tile(S.normal(23, "m", (16,)), (32, 1))
    got = O.motion_xattn_frame(x, m, w, 8)
    want = (m[0] @ w["mv"]) @ w["mo"]
    assert np.max(np.abs(got - want[None])) < 1e-12


def test_two_motion_blocks_with_identical_tokens():
    # with 32 identical tokens each block returns the constant row (m Mv) Mo
    # whatever its queries, so the layer's output is block 2's constant row
    # (own weights, not block 1's) and block 1's queries do not matter
    C = 32
    w = S.layer_weights(24, "mx", C, np.float64)
    w.update(S.motion_block_weights(24, "mx", C, 2, np.float64))
    m = np.tile(S.normal(24, "m", (16,)), (32, 1))
    h = S.normal(24, "h", (6, C))
    bank = [S.normal(24, "b", (6, C))]
    got = O.layer_forward_frame(h, w, bank, m, 8, motion_blocks=2)
    want2 = (m[0] @ w["mv2"]) @ w["mo2"]
    want1 = (m[0] @ w["mv"]) @ w["mo"]
    assert np.max(np.abs(got - want2[None])) < 1e-12
    assert np.max(np.abs(want2 - want1)) > 1e-3          # the blocks' weights differ


def test_second_motion_block_takes_the_first_blocks_output():
    # identical tokens in block 1 make every row of its output the same, so
    # block 2 (varied tokens) must see identical query rows and return
    # identical rows; fed the reference-attention output instead (rows
    # differ) it would not
    C = 32
    w = S.layer_weights(25, "mx", C, np.float64)
    w.update(S.motion_block_weights(25, "mx", C, 2, np.float64))
    h = S.normal(25, "h", (6, C))
    bank = [S.normal(25, "b", (6, C))]
    a = O.ref_attention_frame(h, w, bank, 8)
    m1 = np.tile(S.normal(25, "m1", (16,)), (32, 1))
    m_var = S.normal(25, "mvar", (32, 16))
    y1 = O.motion_xattn_frame(a, m1, w, 8)
    assert np.max(np.abs(y1 - y1[0][None])) < 1e-12
    y2 = O.motion_xattn_frame(y1, m_var, w, 8, block=2)
    assert np.max(np.abs(y2 - y2[0][None])) < 1e-12
    assert np.max(np.abs(O.motion_xattn_frame(a, m_var, w, 8, block=2)[1:] -
                         O.motion_xattn_frame(a, m_var, w, 8, block=2)[0])) > 1e-3
    # motion_blocks = 1 is the single block of the round
    one = O.layer_forward_frame(h, w, bank, m_var, 8)
    assert np.array_equal(one, O.motion_xattn_frame(a, m_var, w, 8))


def test_motion_xattn_brute_force():
    C = 16
    w = S.layer_weights(24, "mx", C, np.float64)
    x = S.normal(24, "x", (3, C))
    m = S.normal(24, "m", (32, 16))
    want = _brute_attention((x @ w["mq"]).tolist(), (m @ w["mk"]).tolist(), (m @ w["mv"]).tolist(), 8) @ w["mo"]
    assert np.max(np.abs(O.motion_xattn_frame(x, m, w, 8) - want)) < 1e-12


# ------------------------------------------------------------------ PR-Sink cache ([LA])

def _block_kv(b, n=4, C=8):
    """Block b: every key the same (so attention weights are uniform over the
    attended tokens) and every value equal to b."""
    return np.ones((n, C)), np.full((n, C), float(b))


def test_pr_sink_cache_lifecycle():
    # pool of 2: the hand-derived contents after each block (ids of the blocks)
    cache = O.PRSinkCache(pool_capacity=2, heads=2)
    want = {  # t: (rolling oldest first, pool by slot)
        0: ([], []), 1: ([1], []), 2: ([1, 2], []), 3: ([1, 2, 3], []),
        4: ([2, 3, 4], [1]), 5: ([3, 4, 5], [1, 2]), 6: ([4, 5, 6], [3, 2]),
        7: ([5, 6, 7], [3, 4]),
    }
    for t in range(8):
        k, v = _block_kv(t)
        cache.step(np.ones((4, 8)), k, v, np.array([float(t)]))
        roll, pool = want[t]
        assert cache.sink[1][0, 0] == 0.0
        assert [int(r[1][0, 0]) for r in cache.rolling] == roll
        assert [int(p[1][0, 0]) for p in cache.pool] == pool
        assert cache.blocks == t + 1


def test_pr_sink_step_attends_own_sink_rolling_and_retrieved():
    # with uniform weights the output is the mean of the attended blocks' values
    cache = O.PRSinkCache(pool_capacity=2, heads=2)
    means = []
    for t in range(8):
        k, v = _block_kv(t)
        out, slot = cache.step(np.ones((4, 8)), k, v, np.array([float(t)]))
        means.append(float(out[0, 0]))
        # the pool first receives a block in the update of t = 4
        assert (slot is None) == (t <= 4)
    # t = 5: own 5, sink 0, rolling 2 3 4, pool {1} -> retrieved 1: mean 15 / 6
    assert abs(means[5] - 15 / 6) < 1e-12
    # t = 6: own 6, sink 0, rolling 3 4 5, pool {1, 2}, pose 6 nearest to 2's: (6+0+12+2)/6
    assert abs(means[6] - 20 / 6) < 1e-12
    # t = 1: own 1 + sink 0 only
    assert abs(means[1] - 0.5) < 1e-12
    assert abs(means[0] - 0.0) < 1e-12


def test_pr_sink_retrieval_nearest_pose_lowest_slot_on_ties():
    cache = O.PRSinkCache(pool_capacity=4, heads=1)
    poses = [np.array([0.0, 0.0]), np.array([5.0, 0.0]), np.array([1.0, 0.0]),
             np.array([-1.0, 0.0]), np.array([3.0, 3.0]), np.array([9.0, 9.0]),
             np.array([9.0, 8.0])]
    for t, ps in enumerate(poses):
        k, v = _block_kv(t)
        cache.step(np.ones((4, 8)), k, v, ps)
    # pool holds blocks 1, 2, 3 (poses (5,0), (1,0), (-1,0)) in slots 0, 1, 2
    assert [int(p[1][0, 0]) for p in cache.pool] == [1, 2, 3]
    _, _, slot = cache.parts(np.array([0.0, 0.0]))    # (1,0) and (-1,0) tie
    assert slot == 1
    _, _, slot = cache.parts(np.array([4.0, 0.0]))
    assert slot == 0


# ------------------------------------------------------------------ rotary code and the LPM window

def test_rope_hand_values_and_identity_at_zero():
    x = np.array([[1.0, 0.0]])
    assert np.allclose(O.rope(x, 1, heads=1), [[np.cos(1.0), np.sin(1.0)]], atol=1e-15)
    # head_dim 4, base 100: pair 1 turns by 100^(-1/2) = 0.1 rad per position
    y = O.rope(np.array([[0.0, 0.0, 0.0, 2.0]]), 3, heads=1, base=100.0)
    assert np.allclose(y, [[0.0, 0.0, -2.0 * np.sin(0.3), 2.0 * np.cos(0.3)]], atol=1e-15)
    z = S.normal(31, "rz", (1, 64))
    assert np.array_equal(O.rope(z, 0, heads=2), z)


def test_rope_keeps_pair_norms():
    x = S.normal(32, "rn", (7, 2 * 64))
    y = O.rope(x, 1000, heads=2)
    nx = np.hypot(x[:, 0::2], x[:, 1::2])
    ny = np.hypot(y[:, 0::2], y[:, 1::2])
    assert np.max(np.abs(nx - ny)) < 1e-12


def test_rope_attention_depends_only_on_relative_positions():
    heads, C = 2, 128
    q = S.normal(33, "q", (5, C))
    ks = [S.normal(33, f"k{i}", (L, C)) for i, L in enumerate((6, 9))]
    vs = [S.normal(33, f"v{i}", (L, C)) for i, L in enumerate((6, 9))]
    a = O.rope_attention(q, 20, ks, vs, [0, 6], heads)
    b = O.rope_attention(q, 20 + 777, ks, vs, [777, 6 + 777], heads)
    assert np.max(np.abs(a - b)) < 1e-10
    c = O.rope_attention(q, 21, ks, vs, [0, 6], heads)     # one position apart: differs
    assert np.max(np.abs(a - c)) > 1e-6


def test_lpm_window_lifecycle():
    R, L, heads, C = 3, 4, 1, 64
    cache = O.LPMCache(np.zeros((R, C)), np.zeros((R, C)), heads)
    want_q_pos0 = [R, R + L, R + 2 * L, R + 3 * L, R + 4 * L, R + 5 * L, R + 5 * L, R + 5 * L]
    for t in range(8):
        k = np.full((L, C), float(t))
        _, q_pos0 = cache.step(np.zeros((L, C)), k, k)
        assert q_pos0 == want_q_pos0[t]
    assert [int(k[0, 0]) for k, _ in cache.sinks] == [0, 1, 2]
    assert [int(k[0, 0]) for k, _ in cache.slide] == [6, 7]
    # chunk 7 sits right after the sinks' and chunk 6's tokens; the next step moves it
    parts, _ = cache.window()
    assert [(int(k[0, 0]) if len(k) == L else -1, p) for k, _, p in parts] == [
        (-1, 0), (0, R), (1, R + L), (2, R + 2 * L), (6, R + 3 * L), (7, R + 4 * L)]


# ------------------------------------------------------------------ pose path front ([PL] 三条条件通路)

def test_rotation_axes_and_orthogonality():
    assert np.array_equal(O.rotation(0, 0, 0), np.eye(3))
    ex, ey = np.array([1.0, 0, 0]), np.array([0, 1.0, 0])
    assert np.allclose(O.rotation(0, 0, 90) @ ex, [0, 1, 0], atol=1e-15)    # roll: x -> y
    assert np.allclose(O.rotation(90, 0, 0) @ ey, [0, 0, 1], atol=1e-15)    # pitch: y -> z
    assert np.allclose(O.rotation(0, 90, 0) @ ex, [0, 0, -1], atol=1e-15)   # yaw: x -> -z
    R = O.rotation(17.0, -33.0, 71.0)
    assert np.allclose(R @ R.T, np.eye(3), atol=1e-15) and abs(np.linalg.det(R) - 1) < 1e-14


def test_retarget_keeps_canonical_points_and_scale_halves_translation():
    c = S.normal(41, "canon", (21, 3))
    got = O.retarget(c, 1.7, (0, 0, 0, 0.2, -0.4, 3.0))
    assert np.allclose(got, 1.7 * c + [0.1, -0.2, 1.5], atol=1e-15)
    # rotation only enters through R: distances between points scale by 1.7
    r = O.retarget(c, 1.7, (10, 20, 30, 0, 0, 0))
    assert np.allclose(np.linalg.norm(r[3] - r[5]), 1.7 * np.linalg.norm(c[3] - c[5]), atol=1e-14)


def test_dot_image_disc_and_painter_order():
    col = np.array([[1, 0, 0], [0, 1, 0]], np.float32)
    # a dot on a pixel centre: radius 0.5 covers that pixel, radius 1 its 4 neighbours too
    img = O.dot_image(np.array([[3.5, 2.5]]), col[:1], 0.5, 6, 8)
    assert img[0].sum() == 1 and img[0, 2, 3] == 1
    img = O.dot_image(np.array([[3.5, 2.5]]), col[:1], 1.0, 6, 8)
    assert img[0].sum() == 5 and img[0, 1, 3] == 1 and img[0, 2, 4] == 1 and img[0, 1, 4] == 0
    # overlapping dots: the later one wins where both cover
    img = O.dot_image(np.array([[3.5, 2.5], [4.5, 2.5]]), col, 1.0, 6, 8)
    assert img[1, 2, 4] == 1 and img[0, 2, 4] == 0 and img[0, 2, 2] == 1


def test_dot_centres_corners_and_centre_on_a_wide_image():
    # orthographic map of [-1, 1] x [-1, 1] onto [0, W] x [0, H] with H != W,
    # so a swapped axis, a missing half-width or a half-pixel shift fails
    H, W = 48, 80
    kps = np.array([[-1.0, -1.0, 0.3], [1.0, 1.0, -0.2], [0.0, 0.0, 5.0], [1.0, -1.0, 0.0],
                    [-1.0, 1.0, 0.0], [0.5, -0.5, 0.0], [-0.25, 0.75, 0.0], [9.0, 9.0, 9.0]])
    got = O.dot_centres(kps, [0, 1, 2, 3, 4, 5, 6], H, W)
    want = np.array([[0.0, 0.0], [80.0, 48.0], [40.0, 24.0], [80.0, 0.0], [0.0, 48.0],
                     [60.0, 12.0], [30.0, 42.0]])
    assert np.array_equal(got, want)
    # the selection picks rows in the order given
    assert np.array_equal(O.dot_centres(kps, [2, 0], H, W), want[[2, 0]])


def test_prefill_keypoints_ramp():
    a, b = S.normal(42, "a", (7, 3)), S.normal(42, "b", (7, 3))
    k = O.prefill_keypoints(a, b)
    assert k.shape == (12, 7, 3) and np.array_equal(k[0], a)
    assert np.allclose(k[11] + (k[11] - k[10]), b, atol=1e-14)     # the dropped 13th point
