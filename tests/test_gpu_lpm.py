"""Rotary attention over a pre-rotary KV cache (pl_rope_*, pl_lpm_*) against the oracle."""
import numpy as np
import pytest

import oracle as O
import synthetic as S
from _gpu_util import ATTN_MAX_ABS, ATTN_MEAN_ABS, attn_errors, dev, host

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def P():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import denoise_step_b200 as P
    return P


@pytest.mark.parametrize("head_dim", [64, 128])
def test_rope_table_matches_fp64(P, head_dim):
    positions = 5000
    tab = host(P.rope_table(positions, head_dim)).astype(np.float64)
    theta = 10000.0 ** (-2.0 * np.arange(head_dim // 2) / head_dim)
    ang = np.arange(positions, dtype=np.float64)[:, None] * theta[None, :]
    assert np.max(np.abs(tab[..., 0] - np.cos(ang))) <= 1e-7
    assert np.max(np.abs(tab[..., 1] - np.sin(ang))) <= 1e-7


@pytest.mark.parametrize("head_dim", [40, 64, 128])
def test_rope_attention_matches_oracle(P, head_dim):
    heads, n_q = 2, 200
    C = heads * head_dim
    seed = S.SEEDS["tiny"] + 7 * head_dim
    lens = (77, 130, 200)
    q = S.normal(seed, "q", (n_q, C), 1.0, np.float16)
    ks = [S.normal(seed, f"k{i}", (L, C), 1.0, np.float16) for i, L in enumerate(lens)]
    vs = [S.normal(seed, f"v{i}", (L, C), 1.0, np.float16) for i, L in enumerate(lens)]
    pos = [0, 77, 207]
    q_pos0 = 207
    tab = P.rope_table(1024, head_dim)
    got = host(P.rope_attention(dev(q), q_pos0, [(dev(k), dev(v)) for k, v in zip(ks, vs)], pos,
                                heads, head_dim, tab))
    want = O.rope_attention(q, q_pos0, ks, vs, pos, heads)
    mx, mean, rel = attn_errors(got, want)
    assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS and rel < 2e-3, (mx, mean, rel)
    # positions matter: the same data at other positions gives another result
    other = O.rope_attention(q, q_pos0 + 40, ks, vs, pos, heads)
    assert attn_errors(got, other)[0] > 20 * mx


@pytest.mark.parametrize("head_dim", [64, 128])
def test_lpm_cache_matches_oracle(P, head_dim):
    R, L, heads, T = 50, 96, 2, 8
    C = heads * head_dim
    seed = S.SEEDS["tiny"] + 11 * head_dim
    ref_k = S.normal(seed, "rk", (R, C), 1.0, np.float16)
    ref_v = S.normal(seed, "rv", (R, C), 1.0, np.float16)
    lpm = P.Lpm(R, L, heads, head_dim)
    rk, rv = lpm.ref_kv()
    rk.copy_(dev(ref_k))
    rv.copy_(dev(ref_v))
    orc = O.LPMCache(ref_k, ref_v, heads)
    stream = torch.cuda.Stream()
    for t in range(T):
        q = S.normal(seed, f"q{t}", (L, C), 1.0, np.float16)
        k = S.normal(seed, f"k{t}", (L, C), 1.0, np.float16)
        v = S.normal(seed, f"v{t}", (L, C), 1.0, np.float16)
        kd, vd = lpm.chunk_kv()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            kd.copy_(dev(k))
            vd.copy_(dev(v))
            out = lpm.step(dev(q), stream=stream)
        stream.synchronize()
        want, q_pos0 = orc.step(q, k, v)
        mx, mean, rel = attn_errors(host(out), want)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS and rel < 2e-3, (t, mx, mean, rel)
        st = lpm.state()
        assert st["last_q_pos0"] == q_pos0 and st["chunks"] == t + 1
        assert st["n_sink"] == len(orc.sinks) and st["n_slide"] == len(orc.slide)
    lpm.close()
