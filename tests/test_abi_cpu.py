"""The C-ABI library loads and exports every symbol include/pl.h declares, and
its host-side validation rejects bad arguments without touching a GPU."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "pl.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pl_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary_calls():
    names = _declared()
    for must in ("pl_bank_init", "pl_ref_attention", "pl_motion_xattn", "pl_pyramid_ddim_step",
                 "pl_motion_bank_check", "pl_stream_round"):
        assert must in names


def test_library_exports_every_declared_symbol():
    import denoise_step_b200 as P
    for name in _declared():
        assert hasattr(P.lib, name), name
        assert name in P.EXPORTED, name


def test_status_strings_and_abi():
    import denoise_step_b200 as P
    assert P.lib.pl_abi_version() == 3
    for s in range(8):
        assert P.lib.pl_status_string(s)
    assert P.lib.pl_status_string(99) == b"unknown status"


def test_host_validation_rejects_bad_arguments():
    import denoise_step_b200 as P
    L = P.lib
    assert L.pl_gemm_f16(None, 8, None, 8, None, 8, 8, 16, 8, None) == P.PL_EINVAL
    n = C.c_size_t()
    assert L.pl_ref_attention_workspace_bytes(0, 64, 1280, 1, C.byref(n)) == P.PL_EINVAL
    assert L.pl_ref_attention_workspace_bytes(16, 64, 1280, 5, C.byref(n)) == P.PL_EINVAL
    assert L.pl_ref_attention_workspace_bytes(16, 64, 1280, 1, C.byref(n)) == P.PL_OK
    # qkv 3*F*N*C + bank 2*N*C + o F*N*C halves, each region 256-byte aligned
    assert n.value >= 2 * (3 * 16 * 64 * 1280 + 2 * 64 * 1280 + 16 * 64 * 1280)
    seg = (P.KVSegment * 1)()
    assert L.pl_segment_attention(None, 8, 8, seg, 1, 1, 1, 1, 40, None, 8, 8, None) == P.PL_EINVAL
    assert L.pl_motion_bank_check(None, None, None, 4, 512, None, 1, 17.0, 3, None, None, None,
                                  None, 0, None) == P.PL_EINVAL
    # the one-CTA check needs no workspace; larger banks need per-CTA minima
    assert L.pl_motion_bank_check_workspace_bytes(32, 512, 32, C.byref(n)) == P.PL_OK
    assert n.value == 0
    assert L.pl_motion_bank_check_workspace_bytes(33, 512, 4, C.byref(n)) == P.PL_OK
    assert n.value >= 16 * 4
    assert L.pl_motion_bank_check_workspace_bytes(4, 512, 33, C.byref(n)) == P.PL_OK
    assert n.value >= 16 * 33
    assert L.pl_motion_bank_check_workspace_bytes(4, 512, 65, C.byref(n)) == P.PL_EINVAL
    assert L.pl_ctx_destroy(None) == P.PL_OK


def test_config_validation_and_workspace_size():
    import denoise_step_b200 as P
    import synthetic as S
    layers = [(side * side, c) for _, side, c in S.LAYERS]
    cfg = P.make_config((64, 64), layers)
    n = C.c_size_t()
    assert P.lib.pl_workspace_bytes(C.byref(cfg), C.byref(n)) == P.PL_OK
    assert n.value > 0
    bad = P.make_config((64, 64), [(4096, 320)], heads=7)
    assert P.lib.pl_workspace_bytes(C.byref(bad), C.byref(n)) == P.PL_EINVAL
    unsup = P.make_config((64, 64), [(4096, 96 * 8)], heads=8)        # head_dim 96
    assert P.lib.pl_workspace_bytes(C.byref(unsup), C.byref(n)) == P.PL_EUNSUPPORTED
    toomany = P.make_config((64, 64), [], append_cap=4)
    assert P.lib.pl_workspace_bytes(C.byref(toomany), C.byref(n)) == P.PL_EINVAL
    h = C.c_void_p()
    assert P.lib.pl_ctx_create(C.byref(cfg), None, 0, C.byref(h)) == P.PL_EINVAL
    assert P.lib.pl_ctx_create(C.byref(cfg), C.c_void_p(256), 16, C.byref(h)) == P.PL_ENOMEM


def test_sessions_scale_the_workspace():
    import denoise_step_b200 as P
    import synthetic as S
    layers = [(side * side, c) for _, side, c in S.LAYERS]
    n = C.c_size_t()
    sizes = {}
    for sess in (0, 1, 2, 4, 8):
        cfg = P.make_config((64, 64), layers, sessions=sess)
        assert P.lib.pl_workspace_bytes(C.byref(cfg), C.byref(n)) == P.PL_OK
        sizes[sess] = n.value
    assert sizes[0] == sizes[1]                        # 0 is read as one session
    # every buffer is per session except the folded [C][C] projections
    # (Wo Mq per layer, fp16), which all sessions share (256-byte rounding aside)
    shared = sum(2 * c * c for _, c in layers)
    assert abs(sizes[2] - 2 * sizes[1] + shared) < 64 * 256
    assert abs(sizes[8] - 8 * sizes[1] + 7 * shared) < 256 * 256
    for sess in (-1, 9):
        cfg = P.make_config((64, 64), layers, sessions=sess)
        assert P.lib.pl_workspace_bytes(C.byref(cfg), C.byref(n)) == P.PL_EINVAL


def test_second_motion_block_adds_its_buffers():
    import denoise_step_b200 as P
    import synthetic as S
    layers = [(side * side, c) for _, side, c in S.LAYERS]
    n1, n2 = C.c_size_t(), C.c_size_t()
    for blocks, n in ((1, n1), (2, n2)):
        cfg = P.make_config((64, 64), layers, motion_blocks=blocks)
        assert P.lib.pl_workspace_bytes(C.byref(cfg), C.byref(n)) == P.PL_OK
    # per layer: the block's motion K/V (fp32 [16][32][2C]) and Mo Mq2 (fp16 [C][C])
    extra = sum(4 * 16 * 32 * 2 * c + 2 * c * c for _, c in layers)
    assert abs(n2.value - n1.value - extra) < 64 * 256
    bad = P.make_config((64, 64), layers, motion_blocks=3)
    assert P.lib.pl_workspace_bytes(C.byref(bad), C.byref(n1)) == P.PL_EINVAL


def test_host_staging_size_and_validation():
    import denoise_step_b200 as P
    import synthetic as S
    layers = [(side * side, c) for _, side, c in S.LAYERS]
    n = C.c_size_t()
    cfg = P.make_config((64, 64), layers)
    assert P.lib.pl_host_staging_bytes(C.byref(cfg), C.byref(n)) == P.PL_OK
    # two sets of: noise 4 frames, motion 4 x 512, hidden 16 frames per layer
    # (fp16), eps 16 frames, x0 4 frames; each region 256-byte aligned
    fe = 4 * 64 * 64
    per_set = 4 * (4 * fe + 4 * 512 + 16 * fe + 4 * fe) + sum(2 * 16 * N * c for N, c in layers)
    assert 2 * per_set <= n.value < 2 * per_set + 2 * (4 + len(layers)) * 256
    n2 = C.c_size_t()
    cfg2 = P.make_config((64, 64), layers, sessions=2)
    assert P.lib.pl_host_staging_bytes(C.byref(cfg2), C.byref(n2)) == P.PL_OK
    assert abs(n2.value - 2 * n.value) < 2 * (4 + len(layers)) * 256
    bad = P.make_config((64, 64), [(4096, 320)], heads=7)
    assert P.lib.pl_host_staging_bytes(C.byref(bad), C.byref(n)) == P.PL_EINVAL
    assert P.lib.pl_host_staging_bytes(C.byref(cfg), None) == P.PL_EINVAL
    assert P.lib.pl_stream_round_host(None, None, 0, None, None, None, None, None,
                                      None) == P.PL_EINVAL


def test_large_bank_check_needs_its_workspace():
    import denoise_step_b200 as P
    L = P.lib
    fake = C.c_void_p(1 << 20)                 # never dereferenced: rejected on the host
    n = C.c_size_t()
    assert L.pl_motion_bank_check_workspace_bytes(100000, 512, 4, C.byref(n)) == P.PL_OK
    need = n.value
    args = (fake, fake, fake, 100000, 512, fake, 4, 17.0, 3, None, None, None)
    assert L.pl_motion_bank_check(*args, None, 0, None) == P.PL_EINVAL          # no workspace
    assert L.pl_motion_bank_check(*args, fake, need - 1, None) == P.PL_ENOMEM  # too small
    assert L.pl_motion_bank_check(*args, C.c_void_p((1 << 20) + 8), need,
                                  None) == P.PL_EINVAL                          # misaligned
    # queries x dim past the shared-memory budget of the multi-CTA pass
    assert L.pl_motion_bank_check_workspace_bytes(100000, 4096, 8, C.byref(n)) == P.PL_OK
    assert L.pl_motion_bank_check(fake, fake, fake, 100000, 4096, fake, 8, 17.0, 3, None, None,
                                  None, fake, n.value, None) == P.PL_EUNSUPPORTED


def test_state_and_profiling_calls_validate_their_arguments():
    import denoise_step_b200 as P
    n = C.c_size_t()
    assert P.lib.pl_state_bytes(None, C.byref(n)) == P.PL_EINVAL
    assert P.lib.pl_state_export(None, None, 0, None) == P.PL_EINVAL
    assert P.lib.pl_state_import(None, None, 0, None) == P.PL_EINVAL
    assert P.lib.pl_set_profiling(None, 1) == P.PL_EINVAL
    buf = (C.c_float * 4)()
    assert P.lib.pl_get_layer_ms(None, buf, 4) == P.PL_EINVAL
    k = C.c_int()
    assert P.lib.pl_round_kernel_count(None, C.byref(k)) == P.PL_EINVAL


def test_round_before_init_is_a_state_error():
    import denoise_step_b200 as P
    # a null context is rejected before any device work
    assert P.lib.pl_stream_round(None, None, None, None, None, None, None, None, None,
                                 None) == P.PL_EINVAL
    assert P.lib.pl_ring_push(None, None, None, None) == P.PL_EINVAL


def test_sink_validation():
    import denoise_step_b200 as P
    n = C.c_size_t()
    L = P.lib
    assert L.pl_sink_workspace_bytes(4096, 40, 128, 64, 64, C.byref(n)) == P.PL_OK
    # arena: pool + 5 blocks of K and V, each n * heads * head_dim fp16
    assert n.value >= 2 * 69 * 4096 * 5120 * 2
    assert L.pl_sink_workspace_bytes(4096, 40, 96, 64, 64, C.byref(n)) == P.PL_EUNSUPPORTED
    assert L.pl_sink_workspace_bytes(4096, 40, 128, 0, 64, C.byref(n)) == P.PL_EINVAL
    assert L.pl_sink_workspace_bytes(0, 40, 128, 64, 64, C.byref(n)) == P.PL_EINVAL
    assert L.pl_sink_workspace_bytes(64, 1, 64, 4097, 8, C.byref(n)) == P.PL_EINVAL
    h = C.c_void_p()
    assert L.pl_sink_create(64, 1, 64, 2, 8, None, 0, C.byref(h)) == P.PL_EINVAL
    assert L.pl_sink_create(64, 1, 64, 2, 8, C.c_void_p(256), 16, C.byref(h)) == P.PL_ENOMEM
    assert L.pl_sink_step(None, None, None, None, None) == P.PL_EINVAL


def test_rope_and_lpm_validation():
    import denoise_step_b200 as P
    n = C.c_size_t()
    L = P.lib
    assert L.pl_lpm_workspace_bytes(1024, 4096, 40, 128, C.byref(n)) == P.PL_OK
    # 6 chunk blocks of K and V, the reference's K and V, the rotated window, the queries, the table
    row = 40 * 128 * 2
    assert n.value >= (12 * 4096 + 2 * 1024 + (1024 + 6 * 4096) + 4096) * row
    assert L.pl_lpm_workspace_bytes(1024, 4096, 40, 96, C.byref(n)) == P.PL_EUNSUPPORTED
    assert L.pl_lpm_workspace_bytes(-1, 4096, 40, 128, C.byref(n)) == P.PL_EINVAL
    assert L.pl_lpm_workspace_bytes(0, 0, 40, 128, C.byref(n)) == P.PL_EINVAL
    h = C.c_void_p()
    assert L.pl_lpm_create(16, 64, 1, 64, 10000.0, None, 0, C.byref(h)) == P.PL_EINVAL
    assert L.pl_lpm_create(16, 64, 1, 64, 1.0, C.c_void_p(256), 1 << 40, C.byref(h)) == P.PL_EINVAL
    assert L.pl_rope_table(None, 10, 64, 10000.0, None) == P.PL_EINVAL
    assert L.pl_rope_table(C.c_void_p(256), 10, 63, 10000.0, None) == P.PL_EINVAL
    assert L.pl_rope_attention_workspace_bytes(0, 10, 1, 64, C.byref(n)) == P.PL_EINVAL


def test_round_host_binding_checks_host_tensors():
    # the binding refuses host tensors of the wrong size or type before any C
    # call (the C side copies fixed byte counts from the pointers it is given)
    import torch
    import denoise_step_b200 as P

    class Fake(P.Stream):
        def __init__(self, cfg):       # no device workspace, no context
            self.cfg = cfg
            self.handle = None
            self._staging = torch.empty(0, dtype=torch.uint8)

    cfg = P.make_config((8, 8), [(64, 320)])
    st = Fake(cfg)
    fe = 4 * 8 * 8
    ok = dict(h_noise=torch.zeros(4 * fe), h_motion=torch.zeros(4 * 512),
              h_hidden=[torch.zeros(16 * 64 * 320, dtype=torch.float16)],
              h_eps=torch.zeros(16 * fe), h_out_frames=torch.zeros(4 * fe))
    for key, bad in [("h_noise", torch.zeros(4 * fe - 1)),
                     ("h_eps", torch.zeros(16 * fe, dtype=torch.float64)),
                     ("h_hidden", [torch.zeros(16 * 64 * 320)]),
                     ("h_hidden", [])]:
        args = dict(ok, **{key: bad})
        with pytest.raises(ValueError):
            st.round_host(**args)
