"""GPU parity of each kernel against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest

import oracle as O
import synthetic as S
from _gpu_util import (ATTN_MAX_ABS, ATTN_MEAN_ABS, DDIM_ABS, attn_errors, dev, host,
                       layer_weights_np, pack_weights)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def P():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import denoise_step_b200 as P
    return P


# ------------------------------------------------------------------ GEMM

@pytest.mark.parametrize("M,N,K", [(128, 160, 64), (300, 160, 320), (1000, 960, 320),
                                   (130, 48, 72), (257, 2560, 1280), (4096, 640, 320)])
def test_gemm_matches_fp64(P, M, N, K):
    a = S.normal(31, f"a{M}{N}{K}", (M, K), 1.0, np.float16)
    b = S.normal(31, f"b{M}{N}{K}", (K, N), 1.0 / np.sqrt(K), np.float16)
    got = host(P.gemm(dev(a), dev(b))).astype(np.float64)
    want = a.astype(np.float64) @ b.astype(np.float64)
    err = np.abs(got - want)
    # fp16 output rounding (2^-11 relative) plus fp32 accumulation
    assert np.all(err <= 1e-3 + 1e-3 * np.abs(want)), float(err.max())
    torch.cuda.synchronize()


# ------------------------------------------------------------------ attention core

@pytest.mark.parametrize("hd", [40, 64, 80, 128, 160])
def test_segment_attention_ragged_segments(P, hd):
    F, Nq, heads = 2, 200, 2
    Cc = heads * hd
    q = S.normal(41, f"q{hd}", (F, Nq, Cc), 1.0, np.float16)
    own_k = S.normal(41, f"ok{hd}", (F, Nq, Cc), 1.0, np.float16)
    own_v = S.normal(41, f"ov{hd}", (F, Nq, Cc), 1.0, np.float16)
    b_k = [S.normal(41, f"bk{hd}{i}", (L, Cc), 1.0, np.float16) for i, L in enumerate((77, 130))]
    b_v = [S.normal(41, f"bv{hd}{i}", (L, Cc), 1.0, np.float16) for i, L in enumerate((77, 130))]
    segs = [(dev(own_k), dev(own_v))] + [(dev(k), dev(v)) for k, v in zip(b_k, b_v)]
    got = host(P.segment_attention(dev(q), segs, heads, hd)).astype(np.float64)
    for f in range(F):
        want = O.segment_attention(q[f], [own_k[f]] + b_k, [own_v[f]] + b_v, heads)
        mx, mean, rel = attn_errors(got[f], want)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (mx, mean, rel)
        assert rel < 5e-3, rel


def test_segment_attention_peaky_scores(P):
    # large logits (q, k ~ N(0, 16)): near one-hot softmax, the max-subtraction path matters
    F, Nq, heads, hd = 1, 256, 2, 64
    Cc = heads * hd
    q = S.normal(42, "q", (F, Nq, Cc), 4.0, np.float16)
    k = S.normal(42, "k", (F, 384, Cc), 4.0, np.float16)
    v = S.normal(42, "v", (F, 384, Cc), 1.0, np.float16)
    got = host(P.segment_attention(dev(q), [(dev(k), dev(v))], heads, hd)).astype(np.float64)
    want = O.segment_attention(q[0], [k[0]], [v[0]], heads)
    mx, mean, rel = attn_errors(got[0], want)
    assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS and rel < 1e-2, (mx, mean, rel)


@pytest.mark.parametrize("hd", [40, 64])
@pytest.mark.parametrize("L", [1, 50, 80, 81, 161])
def test_segment_attention_few_key_tiles(P, hd, L):
    # one or two key tiles in all (a single key, a partial tile, exactly one
    # or two tiles, one key past a tile): the first tile's maximum starts the
    # running maximum and the last, mostly masked tile ends it
    F, Nq, heads = 2, 300, 2
    Cc = heads * hd
    q = S.normal(44, f"q{hd}{L}", (F, Nq, Cc), 1.0, np.float16)
    k = S.normal(44, f"k{hd}{L}", (F, L, Cc), 1.0, np.float16)
    v = S.normal(44, f"v{hd}{L}", (F, L, Cc), 1.0, np.float16)
    got = host(P.segment_attention(dev(q), [(dev(k), dev(v))], heads, hd)).astype(np.float64)
    for f in range(F):
        want = O.segment_attention(q[f], [k[f]], [v[f]], heads)
        mx, mean, rel = attn_errors(got[f], want)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (f, mx, mean, rel)


@pytest.mark.parametrize("hd", [40, 80, 128, 160])
@pytest.mark.parametrize("shape", ["ramp", "spikes"])
def test_segment_attention_growing_max(P, hd, shape):
    # the row maximum keeps growing along the keys, so later KV tiles overflow
    # the running maximum by far more than 2^8: "ramp" raises the key scale
    # from 0.25 to 8 (scores up to ~40 in log2 units), "spikes" puts keys 64x
    # larger into a few late tiles (scores past 128 in log2 units, beyond the
    # range of a plain exponent-field exp2)
    F, Nq, heads = 1, 160, 2
    Cc = heads * hd
    L = 700
    q = S.normal(43, f"q{hd}", (F, Nq, Cc), 1.0, np.float16)
    k = S.normal(43, f"k{hd}", (F, L, Cc), 1.0, np.float64)
    if shape == "ramp":
        k *= np.geomspace(0.25, 8.0, L)[None, :, None]
    else:
        k[:, 300::97, :] *= 64.0
    k = k.astype(np.float16)
    v = S.normal(43, f"v{hd}", (F, L, Cc), 1.0, np.float16)
    got = host(P.segment_attention(dev(q), [(dev(k), dev(v))], heads, hd)).astype(np.float64)
    want = O.segment_attention(q[0], [k[0]], [v[0]], heads)
    assert np.all(np.isfinite(got[0]))
    mx, mean, rel = attn_errors(got[0], want)
    assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS and rel < 1e-2, (mx, mean, rel)


# ------------------------------------------------------------------ reference attention layer

def _ref_case(seed, F, N, C, n_bank, scale=1.0):
    w = layer_weights_np(seed, "L", C)
    h = S.normal(seed, "hidden", (F, N, C), scale, np.float16)
    bank = [S.bank_features(seed, "L", b, N, C) for b in range(n_bank)]
    return w, h, bank


def test_ref_attention_tiny_config_full(P):
    # 16 frames, one 8x8 level, C = 1280, 8 heads (head_dim 160), bank x1 (KV 128)
    F, N, C, heads = 16, 64, 1280, 8
    w, h, bank = _ref_case(S.SEEDS["tiny"], F, N, C, 1)
    pw = pack_weights(w)
    got = host(P.ref_attention(dev(h), pw["w_qkv"], pw["w_o"], [dev(b) for b in bank], heads))
    for f in range(F):
        want = O.ref_attention_frame(h[f], w, bank, heads)
        mx, mean, rel = attn_errors(got[f], want)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (f, mx, mean, rel)


@pytest.mark.parametrize("n_bank", [1, 2, 3, 4])
def test_ref_attention_bank_counts(P, n_bank):
    F, N, C, heads = 2, 256, 640, 8
    w, h, bank = _ref_case(50 + n_bank, F, N, C, n_bank)
    pw = pack_weights(w)
    got = host(P.ref_attention(dev(h), pw["w_qkv"], pw["w_o"], [dev(b) for b in bank], heads))
    for f in range(F):
        want = O.ref_attention_frame(h[f], w, bank, heads)
        mx, mean, rel = attn_errors(got[f], want)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (f, mx, mean, rel)


def test_ref_attention_level64_sampled_rows(P):
    # 16 frames x 4096 tokens, C = 320, head_dim 40, bank x1 (KV 8192): sampled query rows
    F, N, C, heads = 16, 4096, 320, 8
    w, h, bank = _ref_case(S.SEEDS["level64"], F, N, C, 1)
    pw = pack_weights(w)
    got = host(P.ref_attention(dev(h), pw["w_qkv"], pw["w_o"], [dev(b) for b in bank], heads))
    rows = np.sort(S.uniform_int(S.SEEDS["level64"], "rows", 48, N))
    rows = np.unique(np.concatenate([rows, [0, N - 1]]))
    for f in (0, 7, 15):
        want = O.ref_attention_frame(h[f], w, bank, heads, rows=rows)
        mx, mean, rel = attn_errors(got[f][rows], want)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (f, mx, mean, rel)


# ------------------------------------------------------------------ motion cross-attention

@pytest.mark.parametrize("N,C", [(64, 1280), (256, 640), (1024, 320)])
def test_motion_xattn(P, N, C):
    F, heads = 16, 8
    w = layer_weights_np(60, "M", C)
    x = S.normal(60, f"x{N}", (F, N, C), 1.0, np.float16)
    e = S.normal(60, f"e{N}", (F, 512), 1.0, np.float32)
    pw = pack_weights(w)
    got = host(P.motion_xattn(dev(x), dev(e), pw["m_q"], pw["m_kv"], pw["m_o"], heads))
    for f in (0, 5, 15):
        want = O.motion_xattn_frame(x[f], O.motion_tokens(e[f]), w, heads)
        mx, mean, rel = attn_errors(got[f], want)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (f, mx, mean, rel)


# ------------------------------------------------------------------ motion bank

def _bank_run(P, bank_np, count, queries, thr, cap, capacity, flag=None):
    """One bank check on the device. `flag` (a list) receives, for the large
    path, whether the fp64 pass ran: the int32 16 bytes before the end of the
    workspace (0 = the fp32 screen settled every nearest entry)."""
    dim = bank_np.shape[1]
    bank = torch.zeros((capacity, dim), dtype=torch.float32, device="cuda")
    bank[:count] = dev(bank_np[:count])
    cnt = torch.tensor([count], dtype=torch.int32, device="cuda")
    app = torch.zeros(1, dtype=torch.int32, device="cuda")
    nq = len(queries)
    am = torch.full((nq,), -7, dtype=torch.int32, device="cuda")
    d2 = torch.zeros(nq, dtype=torch.float64, device="cuda")
    fl = torch.zeros(nq, dtype=torch.uint8, device="cuda")
    need = P.sz()
    P.check(P.lib.pl_motion_bank_check_workspace_bytes(capacity, dim, nq, P.C.byref(need)), "ws")
    ws = torch.full((max(need.value, 16),), 0x55, dtype=torch.uint8, device="cuda")
    P.motion_bank_check(bank, cnt, app, dev(np.asarray(queries, np.float32)), thr, cap, am, d2, fl,
                        workspace=ws if need.value > 0 else None)
    torch.cuda.synchronize()
    if flag is not None and need.value > 0:
        flag.append(int(ws[need.value - 16:need.value - 12].view(torch.int32).item()))
    return host(bank), int(cnt.item()), int(app.item()), host(am), host(d2), host(fl)


def test_bank_check_tiny_config_bit_exact(P):
    seed = S.SEEDS["tiny"]
    bank = S.normal(seed, "mbank", (8, 512), 2.0, np.float32)
    qs = S.normal(seed, "mq", (4, 512), 2.0, np.float32)
    gbank, cnt, app, am, d2, fl = _bank_run(P, bank, 8, qs, 17.0, 3, 12)
    w_am, w_d2, w_fl, w_bank, w_app = O.bank_check(list(bank), list(qs), 0)
    assert list(am) == w_am and list(fl) == w_fl and app == w_app and cnt == len(w_bank)
    assert np.max(np.abs(d2 - np.array(w_d2)) / np.array(w_d2)) < 1e-12
    assert np.array_equal(gbank[:cnt], np.array(w_bank, np.float32))


def test_bank_check_threshold_edge_and_cap(P):
    z = np.zeros((1, 512), np.float32)
    q = np.zeros((1, 512), np.float32)
    q[0, 0] = 17.0
    _, cnt, app, am, d2, fl = _bank_run(P, z, 1, q, 17.0, 3, 4)
    assert (cnt, app, int(fl[0]), float(d2[0])) == (1, 0, 0, 289.0)
    q[0, 0] = np.nextafter(np.float32(17.0), np.float32(100.0))
    _, cnt, app, am, d2, fl = _bank_run(P, z, 1, q, 17.0, 3, 4)
    assert (cnt, app, int(fl[0])) == (2, 1, 1)
    # five far-apart queries: only 3 appends
    qs = np.zeros((5, 512), np.float32)
    for i in range(5):
        qs[i, i] = 100.0 * (i + 1)
    _, cnt, app, am, d2, fl = _bank_run(P, z, 1, qs, 17.0, 3, 4)
    assert list(fl) == [1, 1, 1, 0, 0] and cnt == 4 and app == 3


@pytest.mark.parametrize("count,dim,nq", [(30000, 512, 6), (5000, 64, 40), (70, 128, 5),
                                          (50, 30, 6)])
def test_bank_check_large_banks_bit_exact(P, count, dim, nq):
    # banks past 32 entries or more than 32 queries: per-CTA minima over the
    # stored entries, then the in-order decisions over those minima and the
    # query-query distances. Queries: far ones (appended while the cap
    # allows), ones next to a stored entry (kept, argmin known), and ones next
    # to an earlier far query (their nearest entry is that query's appended
    # copy once it was appended)
    seed = 71
    bank = S.normal(seed, f"lb{count}/{dim}", (count, dim), 2.0, np.float32)
    far = S.normal(seed, f"lq{count}/{dim}", (nq, dim), 6.0, np.float32)
    pick = S.uniform_int(seed, f"lpick{count}", nq, count)
    jit = S.normal(seed, f"ljit{count}", (nq, dim), 0.05, np.float32)
    qs = far.copy()
    for k in range(nq):
        if k % 3 == 1:
            qs[k] = bank[pick[k]] + jit[k]
        elif k % 3 == 2 and k >= 2:
            qs[k] = qs[k - 2] + jit[k]
    flag = []
    gbank, cnt, app, am, d2, fl = _bank_run(P, bank, count, qs, 17.0, 3, count + 3, flag)
    w_am, w_d2, w_fl, w_bank, w_app = O.bank_check(list(bank), list(qs), 0)
    assert list(am) == w_am and list(fl) == w_fl and app == w_app and cnt == len(w_bank)
    assert np.max(np.abs(d2 - np.array(w_d2)) / np.maximum(np.array(w_d2), 1e-300)) < 1e-12
    assert np.array_equal(gbank[:cnt], np.array(w_bank, np.float32))
    assert w_fl[0] == 1 and w_am[2] == count        # query 2 finds query 0's appended copy
    # no near-tie among these: the fp32 screen decides alone where it takes the
    # rows (multiples of 4 floats up to 512), else the fp64 pass runs
    assert flag == [0 if dim % 4 == 0 and dim <= 512 else 1]


def test_bank_check_large_bank_ties_take_the_fp64_pass(P):
    # Exact duplicates among the stored entries tie in every precision, so the
    # fp32 screen cannot settle those queries' nearest entry and the fp64 pass
    # decides (lowest index on ties): query 0 sits next to entry 1234 (copied
    # to 3000), query 1 next to entry 77 (copied to 78 and 4000), query 2 is
    # far from everything (appended).
    seed = 73
    count, dim = 5000, 64
    bank = S.normal(seed, "tb", (count, dim), 2.0, np.float32)
    bank[3000] = bank[1234]
    bank[78] = bank[77]
    bank[4000] = bank[77]
    jit = S.normal(seed, "tj", (2, dim), 0.05, np.float32)
    far = S.normal(seed, "tf", (1, dim), 6.0, np.float32)
    qs = np.stack([bank[1234] + jit[0], bank[77] + jit[1], far[0]]).astype(np.float32)
    flag = []
    gbank, cnt, app, am, d2, fl = _bank_run(P, bank, count, qs, 17.0, 3, count + 3, flag)
    assert flag == [1]
    w_am, w_d2, w_fl, w_bank, w_app = O.bank_check(list(bank), list(qs), 0)
    assert w_am[:2] == [1234, 77] and w_fl == [0, 0, 1]
    assert list(am) == w_am and list(fl) == w_fl and app == w_app and cnt == len(w_bank)
    assert np.max(np.abs(d2 - np.array(w_d2)) / np.array(w_d2)) < 1e-12
    assert np.array_equal(gbank[:cnt], np.array(w_bank, np.float32))


def test_bank_check_large_path_single_entry(P):
    # a capacity past the one-CTA path with one stored entry: the screen has no
    # runner-up, its pick stands; every query is far, so the first three are
    # appended and later ones find those copies
    seed = 74
    bank = S.normal(seed, "sb", (1, 128), 2.0, np.float32)
    qs = S.normal(seed, "sq", (5, 128), 2.0, np.float32)
    flag = []
    gbank, cnt, app, am, d2, fl = _bank_run(P, bank, 1, qs, 17.0, 3, 40, flag)
    assert flag == [0]
    w_am, w_d2, w_fl, w_bank, w_app = O.bank_check(list(bank), list(qs), 0)
    assert list(am) == w_am and list(fl) == w_fl and app == w_app and cnt == len(w_bank)
    assert np.max(np.abs(d2 - np.array(w_d2)) / np.array(w_d2)) < 1e-12
    assert np.array_equal(gbank[:cnt], np.array(w_bank, np.float32))


def test_pose_retrieval_argmin(P):
    seed = S.SEEDS["sink"]
    store = S.normal(seed, "poses", (64, 64), 1.0, np.float32)
    d = S.normal(seed, "pose_q", (3, 64), 1.0, np.float32)
    _, cnt, app, am, d2, fl = _bank_run(P, store, 64, d, 0.0, 0, 64)
    assert cnt == 64 and app == 0 and not fl.any()
    assert list(am) == [O.pose_retrieve(store, d[i]) for i in range(3)]


# ------------------------------------------------------------------ pile, DDIM, prefill

def _stream_inputs(seed, H, W):
    ref = S.normal(seed, "ref_latent", (4, H, W), 1.0, np.float32)
    pe = S.normal(seed, "prefill_eps", (12, 4, H, W), 1.0, np.float32)
    rm = S.normal(seed, "ref_motion", (512,), 1.0, np.float32)
    d0 = S.normal(seed, "drive0", (512,), 1.0, np.float32)
    return ref, pe, rm, d0


def _ring_view(P, st, H, W):
    base = st.workspace.data_ptr()
    off = st.ring_latents() - base
    n = 16 * 4 * H * W
    return st.workspace[off:off + 4 * n].view(torch.float32).view(4, 4, 4, H, W)


@pytest.mark.parametrize("H,W", [(8, 8), (64, 64)])
def test_pile_ddim_prefill_and_state(P, H, W):
    seed = S.SEEDS["tiny"] if H == 8 else S.SEEDS["level64"]
    ref, pe, rm, d0 = _stream_inputs(seed, H, W)
    cfg = P.make_config((H, W), [])
    st = P.Stream(cfg)
    st.bank_init([], [], None, dev(rm), dev(d0), dev(ref), dev(pe))
    orc = O.PyramidStream(ref, pe, rm, d0, state_dtype=np.float32)
    s0 = st.state()
    assert s0["slot_t"] == [0, 333, 666, -1] and s0["head"] == 0 and s0["bank_count"] == 1
    ring = _ring_view(P, st, H, W)
    for w in range(3):
        assert np.max(np.abs(host(ring[w]) - orc.pile[w].x)) <= DDIM_ABS
    out = torch.empty((4, 4, H, W), dtype=torch.float32, device="cuda")
    for r in range(1, 7):
        noise = S.normal(seed, f"noise{r}", (4, 4, H, W), 1.0, np.float32)
        mot = S.normal(seed, f"motion{r}", (4, 512), 1.0, np.float32)
        eps = S.normal(seed, f"eps{r}", (16, 4, H, W), 1.0, np.float32)
        st.ring_push(dev(noise), dev(mot))
        st.ddim_step(dev(eps), out)
        st.bank_check(dev(mot))
        want, flags, _, _ = orc.round(noise, mot, eps)
        assert np.max(np.abs(host(out) - want)) <= DDIM_ABS, r
        s = st.state()
        logical = [s["slot_t"][(s["head"] + k) & 3] for k in range(4)]
        assert logical == orc.batch_timesteps() + [-1], (r, s)
        assert s["rounds"] == r and s["frames_in"] == 4 * r and s["frames_out"] == 4 * r
        assert s["bank_count"] == len(orc.bank) and s["appends"] == orc.appends
        assert s["device_status"] == 0
        ring = _ring_view(P, st, H, W)
        for k in range(3):
            slot = (s["head"] + k) & 3
            assert np.max(np.abs(host(ring[slot]) - orc.pile[k].x)) <= DDIM_ABS, (r, k)
    assert np.array_equal(st.motion_bank(), np.array(orc.bank, np.float32))
    st.close()


# ------------------------------------------------------------------ PR-Sink bounded attention

def test_pr_sink_attention_retrieves_and_attends(P):
    # 40 heads x head_dim 128; KV = query block + static sink + pose-retrieved block
    # (argmin over 64 stored 64-d pose descriptors) + 3 rolling blocks; ragged block length
    seed, n, heads, hd, n_pool = S.SEEDS["sink"], 1000, 40, 128, 64
    Cc = heads * hd
    g = lambda name, shape, std=1.0: S.normal(seed, name, shape, std, np.float16)
    q = g("q", (n, Cc))
    own = (g("k_own", (n, Cc)), g("v_own", (n, Cc)))
    sink = (g("k_sink", (n, Cc)), g("v_sink", (n, Cc)))
    roll = [(g(f"k_roll{r}", (n, Cc)), g(f"v_roll{r}", (n, Cc))) for r in range(3)]
    store = S.normal(seed, "poses", (n_pool, 64), 1.0, np.float32)
    pq = S.normal(seed, "pose_q", (64,), 1.0, np.float32)
    target = O.pose_retrieve(store, pq)
    # only the retrieved block carries full seeded values; the others are scaled
    # copies of a small base, so attending the wrong block changes the output
    base_k, base_v = g("pool_base_k", (n, Cc), 0.5), g("pool_base_v", (n, Cc), 0.5)
    pool_k = torch.empty((n_pool, n, Cc), dtype=torch.float16, device="cuda")
    pool_v = torch.empty_like(pool_k)
    for j in range(n_pool):
        pool_k[j] = dev(base_k) * (1.0 + j / n_pool)
        pool_v[j] = dev(base_v) * (1.0 - j / (2 * n_pool))
    tk, tv = g("pool_target_k", (n, Cc)), g("pool_target_v", (n, Cc))
    pool_k[target] = dev(tk)
    pool_v[target] = dev(tv)
    d2 = torch.zeros(1, dtype=torch.float64, device="cuda")
    out, ret = P.pr_sink_attention(dev(q), (dev(own[0]), dev(own[1])), (dev(sink[0]), dev(sink[1])),
                                   (pool_k, pool_v), dev(store), dev(pq),
                                   [(dev(k), dev(v)) for k, v in roll], heads, hd, retrieved_d2=d2)
    torch.cuda.synchronize()
    assert int(ret.item()) == target
    assert abs(float(d2.item()) - O.sq_dist(pq, store[target])) <= 1e-12 * O.sq_dist(pq, store[target])
    rows = np.unique(np.concatenate([S.uniform_int(seed, "rows", 40, n), [0, n - 1]]))
    want = O.segment_attention(q[rows], [own[0], sink[0], tk] + [k for k, _ in roll],
                               [own[1], sink[1], tv] + [v for _, v in roll], heads)
    mx, mean, rel = attn_errors(host(out)[rows], want)
    assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (mx, mean, rel)


# ------------------------------------------------------------------ nearest vector over a large store

@pytest.mark.parametrize("count,dim", [(200000, 64), (50001, 30)])
def test_nearest_large_store_bit_exact(P, count, dim):
    seed = S.SEEDS["sink"]
    store = S.normal(seed, f"store{count}", (count, dim), 1.0, np.float32)
    q = S.normal(seed, f"q{count}", (dim,), 1.0, np.float32)
    d2 = np.sum((store.astype(np.float64) - q.astype(np.float64)) ** 2, axis=1)
    j = int(np.argmin(d2))
    # plant an exact tie later in the store: the lowest index must win
    store[count - 3] = store[j]
    am, md = P.nearest(dev(store), dev(q))
    torch.cuda.synchronize()
    assert int(am.item()) == O.pose_retrieve(store, q) == j
    assert abs(float(md.item()) - O.sq_dist(q, store[j])) <= 1e-12 * O.sq_dist(q, store[j])
