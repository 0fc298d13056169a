"""Device-side failure paths, exercised without faulting or hanging the GPU.

The attention kernel's mbarrier waits are bounded; when one runs out the
kernel raises its abort flag, every role leaves its loop, TMEM is freed and
the status word gets a timeout bit. A kernel handed a tensor-map box that is
not its key tile refuses to run. Both are planted through the test hook
pl_test_segment_attention_fault: in the first mode no K/V copy is ever
started (so nothing is in flight when the waits give up), in the second the
kernel returns before any copy. A normal launch right after each must still
match the oracle, which shows the context is intact.
"""
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


def _case(hd, L=300, Nq=260, heads=2, F=2):
    Cc = heads * hd
    q = S.normal(61, f"q{hd}", (F, Nq, Cc), 1.0, np.float16)
    k = S.normal(61, f"k{hd}", (F, L, Cc), 1.0, np.float16)
    v = S.normal(61, f"v{hd}", (F, L, Cc), 1.0, np.float16)
    return q, k, v, heads


def _check_normal_launch(P, q, k, v, heads, hd):
    got = host(P.segment_attention(dev(q), [(dev(k), dev(v))], heads, hd)).astype(np.float64)
    assert P.call_status() == P.PL_OK
    for f in range(q.shape[0]):
        want = O.segment_attention(q[f], [k[f]], [v[f]], heads)
        mx, mean, _ = attn_errors(got[f], want)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (f, mx, mean)


@pytest.mark.parametrize("hd", [40, 128, 160])
def test_wait_timeout_is_reported_and_the_gpu_keeps_working(P, hd):
    q, k, v, heads = _case(hd)
    assert P.call_status() == P.PL_OK          # clear anything earlier
    out = torch.full((q.shape[0], q.shape[1], heads * hd), 7.0, dtype=torch.float16, device="cuda")
    r = P.segment_attention_fault(dev(q), [(dev(k), dev(v))], heads, hd, P.PL_TEST_NO_KV,
                                  1000, out)   # 1 ms wait limit
    assert r == P.PL_OK
    assert P.call_status() == P.PL_ETIMEOUT
    assert P.call_status() == P.PL_OK          # read clears the word
    assert torch.all(out == 7.0).item()        # no row was written
    _check_normal_launch(P, q, k, v, heads, hd)


@pytest.mark.parametrize("hd", [40, 80])
def test_mismatched_box_is_refused_on_the_device(P, hd):
    q, k, v, heads = _case(hd)
    assert P.call_status() == P.PL_OK
    out = torch.full((q.shape[0], q.shape[1], heads * hd), 7.0, dtype=torch.float16, device="cuda")
    r = P.segment_attention_fault(dev(q), [(dev(k), dev(v))], heads, hd, P.PL_TEST_BAD_BOX,
                                  1000, out)
    assert r == P.PL_OK
    assert P.call_status() == P.PL_EDEVICE
    assert torch.all(out == 7.0).item()
    _check_normal_launch(P, q, k, v, heads, hd)


def test_fault_hook_validates_its_arguments(P):
    q, k, v, heads = _case(40)
    out = torch.empty((q.shape[0], q.shape[1], heads * 40), dtype=torch.float16, device="cuda")
    assert P.segment_attention_fault(dev(q), [(dev(k), dev(v))], heads, 40, 3, 1000, out) == P.PL_EINVAL
    assert P.segment_attention_fault(dev(q), [(dev(k), dev(v))], heads, 40, 1, 0, out) == P.PL_EINVAL
    assert P.call_status() == P.PL_OK
