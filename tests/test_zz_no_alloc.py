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
from _gpu_util import ATTN_MAX_ABS, ATTN_MEAN_ABS, attn_errors, dev, host, layer_weights_np, pack_weights


def test_oversized_problem_is_rejected_before_device_work():
    import denoise_step_b200 as P
    # 16 frames x 4096 tokens x 320 channels needs ~168 MB of scratch: PL_ENOMEM, no GPU touched
    hp = (C.c_void_p * 1)(None)
    r = P.lib.pl_ref_attention_noalloc(None, None, None, hp, 1, 16, 4096, 320, 8, None, None)
    assert r == P.PL_ENOMEM
    need = C.c_size_t()
    assert P.lib.pl_ref_attention_workspace_bytes(16, 64, 1280, 1, C.byref(need)) == P.PL_OK
    assert need.value <= (32 << 20)


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_on_two_calls():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import denoise_step_b200 as P
    F, N, Cc, heads = 16, 64, 1280, 8
    for call, seed in enumerate((2001, 2002)):
        w = layer_weights_np(seed, "L", Cc)
        pw = pack_weights(w)
        h = dev(S.normal(seed, "hidden", (F, N, Cc), 1.0, np.float16))
        bank = [dev(S.bank_features(seed, "L", b, N, Cc)) for b in range(1 + call)]
        want = host(P.ref_attention(h, pw["w_qkv"], pw["w_o"], bank, heads))
        got = host(P.ref_attention_noalloc(h, pw["w_qkv"], pw["w_o"], bank, heads))
        torch.cuda.synchronize()
        mx, mean, _ = attn_errors(got, want)
        assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, (call, mx, mean)
