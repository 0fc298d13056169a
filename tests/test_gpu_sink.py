"""GPU PR-Sink cache (pl_sink_*) against the oracle's PRSinkCache, block by block."""
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
def test_sink_cache_matches_oracle(P, head_dim):
    n, heads, pool, dim, T = 200, 2, 3, 16, 14       # ragged block, small pool (it wraps)
    C = heads * head_dim
    seed = S.SEEDS["tiny"] + head_dim
    base = S.normal(seed, "poses", (4, dim), 1.0, np.float32)
    sink = P.Sink(n, heads, head_dim, pool, dim)
    orc = O.PRSinkCache(pool, heads)
    stream = torch.cuda.Stream()
    retrieved_seen = set()
    for t in range(T):
        q = S.normal(seed, f"q{t}", (n, C), 1.0, np.float16)
        k = S.normal(seed, f"k{t}", (n, C), 1.0, np.float16)
        v = S.normal(seed, f"v{t}", (n, C), 1.0, np.float16)
        # poses come back to four base poses, so the pool holds near matches
        pose = (base[t % 4] + 0.05 * S.normal(seed, f"pn{t}", (dim,), 1.0)).astype(np.float32)
        kd, vd = sink.block_kv()
        with torch.cuda.stream(stream):
            kd.copy_(dev(k))
            vd.copy_(dev(v))
            out = sink.step(dev(q), dev(pose), stream=stream)
        stream.synchronize()
        orc_pose_before = [p for _, _, p in orc.pool]      # the pool this block searches
        want, slot = orc.step(q, k, v, pose)
        mx, mean, rel = attn_errors(host(out), want)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS and rel < 2e-3, (t, mx, mean, rel)
        st = sink.state(stream)
        assert st["retrieved"] == (-1 if slot is None else slot), (t, st, slot)
        if slot is not None:
            retrieved_seen.add(slot)
            want_d2 = O.sq_dist(pose, orc_pose_before[slot])
            assert abs(st["retrieved_d2"] - want_d2) <= 1e-12 * max(1.0, want_d2), (t, st, want_d2)
        assert st["blocks"] == t + 1 and st["has_sink"] == 1
        assert st["n_roll"] == len(orc.rolling) and st["pool_count"] == len(orc.pool)
        assert st["device_status"] == 0
    assert len(retrieved_seen) >= 2          # retrieval moved between pool slots
    sink.close()


def test_sink_step_needs_the_block_kv(P):
    sink = P.Sink(64, 1, 64, 2, 8)
    q = torch.zeros((64, 64), dtype=torch.float16, device="cuda")
    pose = torch.zeros(8, dtype=torch.float32, device="cuda")
    with pytest.raises(P.PLError):
        sink.step(q, pose)                   # pl_sink_block_kv was not called
    sink.close()
