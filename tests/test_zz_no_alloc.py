"""pl_ref_attention_noalloc: reference attention for callers that cannot allocate.

Such callers (an embedding host that owns all device memory, a real-time
thread that may not block in cudaMalloc) get the same result as
pl_ref_attention with the intermediates in the library's built-in scratch.
This file is collected last so that a run stopping at its first failure has
already run every other test.
"""
import ctypes as C

import numpy as np
import pytest

import synthetic as S
from _gpu_util import dev, host, layer_weights_np, pack_weights


def test_oversized_problem_is_rejected_before_device_work():
    import denoise_step_b200 as P
    # 16 frames x 4096 tokens x 320 channels needs ~168 MB of scratch: PL_ENOMEM, no GPU touched
    hp = (C.c_void_p * 1)(None)
    r = P.lib.pl_ref_attention_noalloc(None, None, None, hp, 1, 16, 4096, 320, 8, None, None)
    assert r == P.PL_ENOMEM
    need = C.c_size_t()
    assert P.lib.pl_ref_attention_workspace_bytes(16, 64, 1280, 1, C.byref(need)) == P.PL_OK
    assert need.value <= (32 << 20)


def test_scratch_limit_sits_between_the_two_largest_cases():
    import denoise_step_b200 as P
    # 3 frames of the 64x64/C320 layer: 15/16 of the scratch without a bank
    # entry (accepted below), 35/32 of it with one (rejected)
    need = C.c_size_t()
    assert P.lib.pl_ref_attention_workspace_bytes(3, 4096, 320, 0, C.byref(need)) == P.PL_OK
    assert need.value == 30 << 20 and need.value <= (32 << 20)
    assert P.lib.pl_ref_attention_workspace_bytes(3, 4096, 320, 1, C.byref(need)) == P.PL_OK
    assert need.value > (32 << 20)
    hp = (C.c_void_p * 1)(None)
    assert P.lib.pl_ref_attention_noalloc(None, None, None, hp, 1, 3, 4096, 320, 8, None,
                                          None) == P.PL_ENOMEM


# (frames, tokens, channels, bank entries): head_dim 160 with one and two bank
# entries, head_dim 80 with no bank entry, head_dim 40 filling 15/16 of the scratch
CASES = [(16, 64, 1280, 1), (16, 64, 1280, 2), (2, 256, 640, 0), (3, 4096, 320, 0)]


@pytest.mark.gpu
@pytest.mark.parametrize("F,N,Cc,nb", CASES)
def test_noalloc_matches_workspace_entry_on_two_calls(F, N, Cc, nb):
    # both entries run the same kernels on the same inputs, so the results
    # must agree bit for bit; two calls in a row with different inputs also
    # show that the shared array's previous contents do not leak into a call
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import denoise_step_b200 as P
    heads = 8
    for call, seed in enumerate((2001, 2002)):
        w = layer_weights_np(seed + 10 * nb, "L", Cc)
        pw = pack_weights(w)
        h = dev(S.normal(seed, f"hidden{F}{N}", (F, N, Cc), 1.0, np.float16))
        bank = [dev(S.bank_features(seed, "L", b, N, Cc)) for b in range(nb)]
        want = host(P.ref_attention(h, pw["w_qkv"], pw["w_o"], bank, heads))
        got = host(P.ref_attention_noalloc(h, pw["w_qkv"], pw["w_o"], bank, heads))
        torch.cuda.synchronize()
        assert np.array_equal(got, want), (call, float(np.abs(got.astype(np.float64) - want).max()))
        assert P.call_status() == P.PL_OK
