"""denoise_step_b200: the streaming pyramid denoising round on B200 (sm_100a).

A thin ctypes binding over the C ABI in include/pl.h (libpl.so, built in-tree
by `python denoise_step_b200/build.py`). Every step of the round runs in the
library's CUDA kernels; this module only marshals arguments (torch tensors
supply device memory and streams). There is no CPU fallback: importing the
package without the built library raises.
"""
from __future__ import annotations

import ctypes as C
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libpl.so")

PL_OK, PL_EINVAL, PL_ESTATE, PL_ENOMEM, PL_ECUDA, PL_ETIMEOUT, PL_EDEVICE, PL_EUNSUPPORTED = range(8)
PL_TEST_NO_KV, PL_TEST_BAD_BOX = 1, 2
MAX_LAYERS = 16


class PLError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib.pl_status_string(status).decode()} (status {status})")


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python denoise_step_b200/build.py`")
lib = C.CDLL(LIB_PATH)

vp, i32, i64, f32, sz = C.c_void_p, C.c_int, C.c_int64, C.c_float, C.c_size_t


class KVSegment(C.Structure):
    _fields_ = [("k", vp), ("v", vp), ("len", i64), ("ld", i64), ("frame_stride", i64)]


class Config(C.Structure):
    _fields_ = [("latent_c", C.c_int32), ("latent_h", C.c_int32), ("latent_w", C.c_int32),
                ("n_layers", C.c_int32), ("layer_tokens", C.c_int32 * MAX_LAYERS),
                ("layer_channels", C.c_int32 * MAX_LAYERS), ("heads", C.c_int32),
                ("drift_threshold", C.c_float), ("append_cap", C.c_int32),
                ("sessions", C.c_int32), ("motion_blocks", C.c_int32)]


class SinkState(C.Structure):
    _fields_ = [("blocks", C.c_int64), ("has_sink", C.c_int32), ("n_roll", C.c_int32),
                ("pool_count", C.c_int32), ("retrieved", C.c_int32), ("retrieved_d2", C.c_double),
                ("device_status", C.c_uint32)]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


class LpmState(C.Structure):
    _fields_ = [("chunks", C.c_int64), ("n_sink", C.c_int32), ("n_slide", C.c_int32),
                ("last_q_pos0", C.c_int32)]

    def as_dict(self):
        return {k: getattr(self, k) for k, _ in self._fields_}


class LayerWeights(C.Structure):
    _fields_ = [("w_qkv", vp), ("w_o", vp), ("m_q", vp), ("m_kv", vp), ("m_o", vp),
                ("m2_q", vp), ("m2_kv", vp), ("m2_o", vp)]


class State(C.Structure):
    _fields_ = [("initialised", C.c_int32), ("head", C.c_int32), ("slot_t", C.c_int32 * 4),
                ("rounds", C.c_int64), ("frames_in", C.c_int64), ("frames_out", C.c_int64),
                ("bank_count", C.c_int32), ("appends", C.c_int32), ("device_status", C.c_uint32)]

    def as_dict(self):
        return {"initialised": self.initialised, "head": self.head, "slot_t": list(self.slot_t),
                "rounds": self.rounds, "frames_in": self.frames_in, "frames_out": self.frames_out,
                "bank_count": self.bank_count, "appends": self.appends,
                "device_status": self.device_status}


_SIGS = {
    "pl_status_string": (C.c_char_p, [i32]),
    "pl_abi_version": (i32, []),
    "pl_gemm_f16": (i32, [vp, i64, vp, i64, vp, i64, i32, i32, i32, vp]),
    "pl_segment_attention": (i32, [vp, i64, i64, C.POINTER(KVSegment), i32, i32, i32, i32, i32,
                                   vp, i64, i64, vp]),
    "pl_test_segment_attention_fault": (i32, [vp, i64, i64, C.POINTER(KVSegment), i32, i32, i32,
                                              i32, i32, vp, i64, i64, i32, C.c_uint32, vp]),
    "pl_get_call_status": (i32, [vp]),
    "pl_pr_sink_attention": (i32, [vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, i32, C.POINTER(vp),
                                   C.POINTER(vp), i32, i32, i32, i32, vp, vp, vp, vp]),
    "pl_ref_attention_workspace_bytes": (i32, [i32, i32, i32, i32, C.POINTER(sz)]),
    "pl_ref_attention": (i32, [vp, vp, vp, C.POINTER(vp), i32, i32, i32, i32, i32, vp, vp, sz, vp]),
    "pl_ref_attention_noalloc": (i32, [vp, vp, vp, C.POINTER(vp), i32, i32, i32, i32, i32, vp, vp]),
    "pl_motion_xattn_workspace_bytes": (i32, [i32, i32, i32, C.POINTER(sz)]),
    "pl_motion_xattn": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, vp, sz, vp]),
    "pl_motion_bank_check_workspace_bytes": (i32, [i32, i32, i32, C.POINTER(sz)]),
    "pl_motion_bank_check": (i32, [vp, vp, vp, i32, i32, vp, i32, f32, i32, vp, vp, vp, vp, sz,
                                   vp]),
    "pl_nearest_workspace_bytes": (i32, [i64, C.POINTER(sz)]),
    "pl_nearest": (i32, [vp, i64, i32, vp, vp, vp, vp, sz, vp]),
    "pl_workspace_bytes": (i32, [C.POINTER(Config), C.POINTER(sz)]),
    "pl_ctx_create": (i32, [C.POINTER(Config), vp, sz, C.POINTER(vp)]),
    "pl_ctx_destroy": (i32, [vp]),
    "pl_bank_init": (i32, [vp, C.POINTER(LayerWeights), C.POINTER(vp), C.POINTER(vp), vp, vp, vp,
                           vp, vp]),
    "pl_ring_push": (i32, [vp, vp, vp, vp]),
    "pl_pyramid_ddim_step": (i32, [vp, vp, vp, vp]),
    "pl_ctx_bank_check": (i32, [vp, vp, i32, vp, vp, vp, vp]),
    "pl_stream_round": (i32, [vp, vp, vp, C.POINTER(vp), vp, vp, vp, C.POINTER(vp),
                              C.POINTER(vp), vp]),
    "pl_host_staging_bytes": (i32, [C.POINTER(Config), C.POINTER(sz)]),
    "pl_stream_round_host": (i32, [vp, vp, sz, vp, vp, C.POINTER(vp), vp, vp, vp]),
    "pl_get_state": (i32, [vp, C.POINTER(State), vp]),
    "pl_get_session_state": (i32, [vp, i32, C.POINTER(State), vp]),
    "pl_get_motion_bank": (i32, [vp, vp, C.POINTER(C.c_int32), vp]),
    "pl_get_session_motion_bank": (i32, [vp, i32, vp, C.POINTER(C.c_int32), vp]),
    "pl_get_device_status": (i32, [vp, vp]),
    "pl_set_profiling": (i32, [vp, i32]),
    "pl_get_layer_ms": (i32, [vp, vp, i32]),
    "pl_round_kernel_count": (i32, [vp, vp]),
    "pl_state_bytes": (i32, [vp, C.POINTER(sz)]),
    "pl_state_export": (i32, [vp, vp, sz, vp]),
    "pl_state_import": (i32, [vp, vp, sz, vp]),
    "pl_ctx_ring_latents": (vp, [vp]),
    "pl_sink_workspace_bytes": (i32, [i32, i32, i32, i32, i32, C.POINTER(sz)]),
    "pl_sink_create": (i32, [i32, i32, i32, i32, i32, vp, sz, C.POINTER(vp)]),
    "pl_sink_destroy": (i32, [vp]),
    "pl_sink_block_kv": (i32, [vp, C.POINTER(vp), C.POINTER(vp)]),
    "pl_sink_step": (i32, [vp, vp, vp, vp, vp]),
    "pl_sink_get_state": (i32, [vp, C.POINTER(SinkState), vp]),
    "pl_rope_table": (i32, [vp, i32, i32, f32, vp]),
    "pl_rope_attention_workspace_bytes": (i32, [i32, i64, i32, i32, C.POINTER(sz)]),
    "pl_rope_attention": (i32, [vp, i64, i32, C.POINTER(KVSegment), C.POINTER(i64), i32, i32, i32,
                                i32, vp, i32, vp, i64, vp, sz, vp]),
    "pl_lpm_workspace_bytes": (i32, [i32, i32, i32, i32, C.POINTER(sz)]),
    "pl_lpm_create": (i32, [i32, i32, i32, i32, f32, vp, sz, C.POINTER(vp)]),
    "pl_lpm_destroy": (i32, [vp]),
    "pl_lpm_ref_kv": (i32, [vp, C.POINTER(vp), C.POINTER(vp)]),
    "pl_lpm_chunk_kv": (i32, [vp, C.POINTER(vp), C.POINTER(vp)]),
    "pl_lpm_step": (i32, [vp, vp, vp, vp]),
    "pl_lpm_get_state": (i32, [vp, C.POINTER(LpmState)]),
    "pl_pose_keypoints": (i32, [vp, f32, vp, i32, C.POINTER(i32), vp, vp]),
    "pl_pose_ramp": (i32, [vp, vp, i32, vp, vp]),
    "pl_pose_dots": (i32, [vp, i32, C.POINTER(f32), f32, i32, i32, vp, vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_SIGS)


def check(status: int, what: str) -> None:
    if status != PL_OK:
        raise PLError(status, what)


# --------------------------------------------------------------------------- helpers

def _ptr(t) -> int | None:
    return None if t is None else int(t.data_ptr())


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream) or None
    return int(getattr(stream, "cuda_stream", stream)) or None


def _ptr_array(ts):
    arr = (vp * len(ts))()
    for i, t in enumerate(ts):
        arr[i] = _ptr(t)
    return arr


def _contig(t, name):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


# --------------------------------------------------------------------------- primitives

def gemm(a, b, out=None, stream=None):
    """out[M,N] = a[M,K] @ b[K,N] (fp16, fp32 accumulate) on tcgen05."""
    import torch
    M, K = a.shape
    N = b.shape[1]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=a.device)
    check(lib.pl_gemm_f16(_ptr(a), a.stride(0), _ptr(b), b.stride(0), _ptr(out), out.stride(0),
                          M, N, K, _stream(stream)), "pl_gemm_f16")
    return out


def _segments(segments):
    segs = (KVSegment * len(segments))()
    for i, (k, v) in enumerate(segments):
        if k.dim() == 3:
            segs[i] = KVSegment(_ptr(k), _ptr(v), k.shape[1], k.stride(1), k.stride(0))
        else:
            segs[i] = KVSegment(_ptr(k), _ptr(v), k.shape[0], k.stride(0), 0)
    return segs


def call_status(stream=None) -> int:
    """Synchronise `stream` and read (and clear) the device status word of the
    context-free calls: PL_OK, PL_ETIMEOUT or PL_EDEVICE."""
    return lib.pl_get_call_status(_stream(stream))


def segment_attention_fault(q, segments, heads, head_dim, mode, wait_us, out, stream=None):
    """pl_test_segment_attention_fault: segment attention with a planted device-side
    failure (PL_TEST_NO_KV: the bounded waits run out; PL_TEST_BAD_BOX: the kernel
    refuses its box). Returns the launch status; read the outcome with call_status()."""
    F, Nq = q.shape[0], q.shape[1]
    segs = _segments(segments)
    return lib.pl_test_segment_attention_fault(_ptr(q), q.stride(1), q.stride(0), segs,
                                               len(segments), F, Nq, heads, head_dim, _ptr(out),
                                               out.stride(1), out.stride(0), int(mode),
                                               int(wait_us), _stream(stream))


def segment_attention(q, segments, heads, head_dim, out=None, stream=None):
    """Attention of q [F, Nq, ld] over KV segments (k, v, frame_shared) without concatenation.

    Each segment is (k, v) with k/v [F, L, ld] (per-frame) or [L, ld] (shared).
    """
    import torch
    F, Nq = q.shape[0], q.shape[1]
    segs = _segments(segments)
    if out is None:
        out = torch.empty((F, Nq, heads * head_dim), dtype=torch.float16, device=q.device)
    check(lib.pl_segment_attention(_ptr(q), q.stride(1), q.stride(0), segs, len(segments), F, Nq,
                                   heads, head_dim, _ptr(out), out.stride(1), out.stride(0),
                                   _stream(stream)), "pl_segment_attention")
    return out


def pr_sink_attention(q, own, sink, pool, pose_store, pose_query, rolling, heads, head_dim,
                      out=None, retrieved=None, retrieved_d2=None, stream=None):
    """PR-Sink block attention: own/sink (k, v) [n, ld]; pool (k, v) [n_pool, n, ld];
    rolling: list of (k, v) [n, ld]; pose_store [n_pool, d] fp32, pose_query [d] fp32."""
    import torch
    n = q.shape[0]
    if out is None:
        out = torch.empty_like(q)
    if retrieved is None:
        retrieved = torch.zeros(1, dtype=torch.int32, device=q.device)
    kr = _ptr_array([k for k, _ in rolling]) if rolling else None
    vr = _ptr_array([v for _, v in rolling]) if rolling else None
    check(lib.pl_pr_sink_attention(_ptr(q), _ptr(own[0]), _ptr(own[1]), _ptr(sink[0]), _ptr(sink[1]),
                                   _ptr(pool[0]), _ptr(pool[1]), pool[0].shape[0], _ptr(pose_store),
                                   _ptr(pose_query), pose_store.shape[1], kr, vr, len(rolling), n,
                                   heads, head_dim, _ptr(out), _ptr(retrieved), _ptr(retrieved_d2),
                                   _stream(stream)), "pl_pr_sink_attention")
    return out, retrieved


def ref_attention(hidden, w_qkv, w_o, bank_feats, heads, out=None, workspace=None, stream=None):
    """Reference attention layer: hidden [F,N,C], bank_feats list of [N,C]."""
    import torch
    F, N, Cc = hidden.shape
    nb = len(bank_feats)
    need = sz()
    check(lib.pl_ref_attention_workspace_bytes(F, N, Cc, nb, C.byref(need)), "workspace")
    if workspace is None:
        workspace = torch.empty(need.value, dtype=torch.uint8, device=hidden.device)
    if out is None:
        out = torch.empty_like(hidden)
    arr = _ptr_array(bank_feats) if nb else None
    check(lib.pl_ref_attention(_ptr(_contig(hidden, "hidden")), _ptr(w_qkv), _ptr(w_o), arr, nb, F,
                               N, Cc, heads, _ptr(out), _ptr(workspace), workspace.numel(),
                               _stream(stream)), "pl_ref_attention")
    return out


def ref_attention_noalloc(hidden, w_qkv, w_o, bank_feats, heads, out=None, stream=None):
    """ref_attention with the library's built-in scratch (no workspace argument)."""
    import torch
    F, N, Cc = hidden.shape
    nb = len(bank_feats)
    if out is None:
        out = torch.empty_like(hidden)
    arr = _ptr_array(bank_feats) if nb else None
    check(lib.pl_ref_attention_noalloc(_ptr(_contig(hidden, "hidden")), _ptr(w_qkv), _ptr(w_o),
                                       arr, nb, F, N, Cc, heads, _ptr(out), _stream(stream)),
          "pl_ref_attention_noalloc")
    return out


def motion_xattn(x, motion, m_q, m_kv, m_o, heads, out=None, workspace=None, stream=None):
    """Motion cross-attention: x [F,N,C] fp16, motion [F,512] fp32."""
    import torch
    F, N, Cc = x.shape
    need = sz()
    check(lib.pl_motion_xattn_workspace_bytes(F, N, Cc, C.byref(need)), "workspace")
    if workspace is None:
        workspace = torch.empty(need.value, dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty_like(x)
    check(lib.pl_motion_xattn(_ptr(_contig(x, "x")), _ptr(motion), _ptr(m_q), _ptr(m_kv),
                              _ptr(m_o), F, N, Cc, heads, _ptr(out), _ptr(workspace),
                              workspace.numel(), _stream(stream)), "pl_motion_xattn")
    return out


def motion_bank_check(bank, count, appends, queries, threshold, cap, argmin=None, min_d2=None,
                      appended=None, workspace=None, stream=None):
    """In-order bank check; bank [capacity, dim] fp32, count/appends int32 [1] (device state).
    Banks past 32 entries (or more than 32 queries) need a device workspace; it is
    allocated here when not given."""
    import torch
    cap_, dim = bank.shape
    nq = queries.shape[0]
    need = sz()
    check(lib.pl_motion_bank_check_workspace_bytes(cap_, dim, nq, C.byref(need)), "workspace")
    if workspace is None and need.value > 0:
        workspace = torch.empty(need.value, dtype=torch.uint8, device=bank.device)
    wb = workspace.numel() if workspace is not None else 0
    check(lib.pl_motion_bank_check(_ptr(bank), _ptr(count), _ptr(appends), cap_, dim,
                                   _ptr(queries), nq, float(threshold), int(cap), _ptr(argmin),
                                   _ptr(min_d2), _ptr(appended), _ptr(workspace), wb,
                                   _stream(stream)),
          "pl_motion_bank_check")


def nearest(store, query, argmin=None, min_d2=None, workspace=None, stream=None):
    """argmin_j ||query - store_j||^2 over a large fp32 store [count, dim] (one read)."""
    import torch
    count, dim = store.shape
    need = sz()
    check(lib.pl_nearest_workspace_bytes(count, C.byref(need)), "pl_nearest_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(need.value, dtype=torch.uint8, device=store.device)
    if argmin is None:
        argmin = torch.zeros(1, dtype=torch.int64, device=store.device)
    if min_d2 is None:
        min_d2 = torch.zeros(1, dtype=torch.float64, device=store.device)
    check(lib.pl_nearest(_ptr(_contig(store, "store")), count, dim, _ptr(query), _ptr(argmin),
                         _ptr(min_d2), _ptr(workspace), workspace.numel(), _stream(stream)),
          "pl_nearest")
    return argmin, min_d2


# --------------------------------------------------------------------------- stream context

def make_config(latent_hw=(64, 64), layers=(), heads=8, threshold=17.0, append_cap=3, latent_c=4,
                sessions=1, motion_blocks=1):
    """layers: sequence of (tokens N, channels C); sessions: streams served together;
    motion_blocks: motion cross-attention blocks per layer (1 or 2)."""
    cfg = Config()
    cfg.latent_c, (cfg.latent_h, cfg.latent_w) = latent_c, latent_hw
    cfg.n_layers = len(layers)
    for i, (n, c) in enumerate(layers):
        cfg.layer_tokens[i] = n
        cfg.layer_channels[i] = c
    cfg.heads = heads
    cfg.drift_threshold = threshold
    cfg.append_cap = append_cap
    cfg.sessions = sessions
    cfg.motion_blocks = motion_blocks
    return cfg


class Stream:
    """PersonaLive stream(s): the device-resident piles and reference banks.

    With cfg.sessions = S > 1 the context serves S independent streams in the
    same launches; every per-stream tensor argument then has a leading
    dimension S (session-major, contiguous)."""

    def __init__(self, cfg: Config, device="cuda"):
        import torch
        self.cfg = cfg
        need = sz()
        check(lib.pl_workspace_bytes(C.byref(cfg), C.byref(need)), "pl_workspace_bytes")
        self.workspace = torch.empty(need.value, dtype=torch.uint8, device=device)
        h = vp()
        check(lib.pl_ctx_create(C.byref(cfg), _ptr(self.workspace), need.value, C.byref(h)),
              "pl_ctx_create")
        self.handle = h
        self._keep = []

    def close(self):
        if self.handle:
            lib.pl_ctx_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def bank_init(self, weights, ref_feats, anchor_feats, ref_motion, drive0_motion, ref_latent,
                  prefill_eps, stream=None):
        """weights: list of dicts with w_qkv, w_o, m_q, m_kv, m_o (device fp16), and
        m2_q, m2_kv, m2_o for a second motion block."""
        L = self.cfg.n_layers
        wa = (LayerWeights * max(L, 1))()
        for i, w in enumerate(weights[:L]):
            wa[i] = LayerWeights(_ptr(w["w_qkv"]), _ptr(w["w_o"]), _ptr(w["m_q"]),
                                 _ptr(w["m_kv"]), _ptr(w["m_o"]), _ptr(w.get("m2_q")),
                                 _ptr(w.get("m2_kv")), _ptr(w.get("m2_o")))
        rf = _ptr_array(ref_feats) if L else None
        af = _ptr_array(anchor_feats) if anchor_feats else None
        self._keep = [weights, ref_feats, anchor_feats, ref_motion, drive0_motion, ref_latent,
                      prefill_eps]
        check(lib.pl_bank_init(self.handle, wa if L else None, rf, af, _ptr(ref_motion),
                               _ptr(drive0_motion), _ptr(ref_latent), _ptr(prefill_eps),
                               _stream(stream)), "pl_bank_init")

    def ring_push(self, new_noise, new_motion, stream=None):
        check(lib.pl_ring_push(self.handle, _ptr(new_noise), _ptr(new_motion), _stream(stream)),
              "pl_ring_push")

    def ddim_step(self, eps, out_x0, stream=None):
        check(lib.pl_pyramid_ddim_step(self.handle, _ptr(eps), _ptr(out_x0), _stream(stream)),
              "pl_pyramid_ddim_step")

    def bank_check(self, queries, argmin=None, min_d2=None, appended=None, stream=None):
        check(lib.pl_ctx_bank_check(self.handle, _ptr(queries), queries.shape[0], _ptr(argmin),
                                    _ptr(min_d2), _ptr(appended), _stream(stream)),
              "pl_ctx_bank_check")

    def round(self, new_noise, new_motion, hidden, eps, out_frames, appended=None,
              layer_out=None, stream=None, attn_out=None):
        """attn_out: optional per-layer buffers for the reference-attention sub-layer output."""
        L = self.cfg.n_layers
        hp = _ptr_array(hidden) if L else None
        lo = _ptr_array(layer_out) if layer_out is not None else None
        ao = _ptr_array(attn_out) if attn_out is not None else None
        check(lib.pl_stream_round(self.handle, _ptr(new_noise), _ptr(new_motion), hp, _ptr(eps),
                                  _ptr(out_frames), _ptr(appended), lo, ao, _stream(stream)),
              "pl_stream_round")

    def round_host(self, h_noise, h_motion, h_hidden, h_eps, h_out_frames, stream=None):
        """One round from pinned host tensors to a pinned host tensor (asynchronous:
        h_out_frames is valid once `stream` is synchronised). The device staging the
        C call needs is allocated on first use and kept with the stream."""
        import torch
        if getattr(self, "_staging", None) is None:
            need = sz()
            check(lib.pl_host_staging_bytes(C.byref(self.cfg), C.byref(need)),
                  "pl_host_staging_bytes")
            self._staging = torch.empty(need.value, dtype=torch.uint8,
                                        device=self.workspace.device)
        for t in [h_noise, h_motion, h_eps, h_out_frames, *h_hidden]:
            if t.is_cuda or not t.is_contiguous():
                raise ValueError("round_host takes contiguous host tensors")
        # the C call copies fixed byte counts from these pointers: check them here
        c = self.cfg
        S = max(c.sessions, 1)
        fe = c.latent_c * c.latent_h * c.latent_w
        want = [(h_noise, torch.float32, S * 4 * fe), (h_motion, torch.float32, S * 4 * 512),
                (h_eps, torch.float32, S * 16 * fe), (h_out_frames, torch.float32, S * 4 * fe)]
        if len(h_hidden) != c.n_layers:
            raise ValueError(f"round_host: {len(h_hidden)} hidden tensors for {c.n_layers} layers")
        want += [(h, torch.float16, S * 16 * c.layer_tokens[l] * c.layer_channels[l])
                 for l, h in enumerate(h_hidden)]
        for t, dt, n in want:
            if t.dtype != dt or t.numel() != n:
                raise ValueError(f"round_host: expected {dt} with {n} elements, got {t.dtype} "
                                 f"with {t.numel()}")
        hp = _ptr_array(h_hidden) if self.cfg.n_layers else None
        check(lib.pl_stream_round_host(self.handle, _ptr(self._staging), self._staging.numel(),
                                       _ptr(h_noise), _ptr(h_motion), hp, _ptr(h_eps),
                                       _ptr(h_out_frames), _stream(stream)),
              "pl_stream_round_host")

    def state(self, stream=None, session=0):
        s = State()
        check(lib.pl_get_session_state(self.handle, session, C.byref(s), _stream(stream)),
              "pl_get_session_state")
        return s.as_dict()

    def motion_bank(self, stream=None, session=0):
        import numpy as np
        buf = np.zeros((4, 512), dtype=np.float32)
        n = C.c_int32()
        check(lib.pl_get_session_motion_bank(self.handle, session, buf.ctypes.data, C.byref(n),
                                             _stream(stream)), "pl_get_session_motion_bank")
        return buf[: n.value].copy()

    def device_status(self, stream=None) -> int:
        return lib.pl_get_device_status(self.handle, _stream(stream))

    def set_profiling(self, on: bool = True):
        check(lib.pl_set_profiling(self.handle, 1 if on else 0), "pl_set_profiling")

    def layer_ms(self):
        """Per-layer times (ms) of the latest profiled round."""
        L = self.cfg.n_layers
        buf = (C.c_float * max(L, 1))()
        check(lib.pl_get_layer_ms(self.handle, buf, L), "pl_get_layer_ms")
        return [buf[i] for i in range(L)]

    def round_kernels(self) -> int:
        """Kernels one round launches, counted in the captured round graph."""
        n = i32()
        check(lib.pl_round_kernel_count(self.handle, C.byref(n)), "pl_round_kernel_count")
        return n.value

    def export_state(self, stream=None):
        """Snapshot of the streams' state as a numpy uint8 array (blocks)."""
        import numpy as np
        n = sz()
        check(lib.pl_state_bytes(self.handle, C.byref(n)), "pl_state_bytes")
        buf = np.zeros(n.value, dtype=np.uint8)
        check(lib.pl_state_export(self.handle, buf.ctypes.data, n.value, _stream(stream)),
              "pl_state_export")
        return buf

    def import_state(self, snapshot, stream=None):
        """Restore a snapshot taken by export_state (after bank_init; blocks)."""
        import numpy as np
        buf = np.ascontiguousarray(snapshot, dtype=np.uint8)
        check(lib.pl_state_import(self.handle, buf.ctypes.data, buf.size, _stream(stream)),
              "pl_state_import")

    def ring_latents(self):
        return lib.pl_ctx_ring_latents(self.handle)


class _DeviceArray:
    """A device buffer the library owns, shown to torch without a copy."""

    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3}


class Sink:
    """PR-Sink bounded KV cache of one block stream (pl_sink_*)."""

    def __init__(self, n, heads, head_dim, pool_capacity, pose_dim, device="cuda"):
        import torch
        self.n, self.heads, self.head_dim = n, heads, head_dim
        need = sz()
        check(lib.pl_sink_workspace_bytes(n, heads, head_dim, pool_capacity, pose_dim,
                                          C.byref(need)), "pl_sink_workspace_bytes")
        self.workspace = torch.empty(need.value, dtype=torch.uint8, device=device)
        h = vp()
        check(lib.pl_sink_create(n, heads, head_dim, pool_capacity, pose_dim,
                                 _ptr(self.workspace), need.value, C.byref(h)), "pl_sink_create")
        self.handle = h

    def close(self):
        if self.handle:
            lib.pl_sink_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def block_kv(self):
        """torch views [n, heads*head_dim] fp16 of where the next block's K and V go."""
        import torch
        k, v = vp(), vp()
        check(lib.pl_sink_block_kv(self.handle, C.byref(k), C.byref(v)), "pl_sink_block_kv")
        shape = (self.n, self.heads * self.head_dim)
        return (torch.as_tensor(_DeviceArray(k.value, shape, "<f2"), device="cuda"),
                torch.as_tensor(_DeviceArray(v.value, shape, "<f2"), device="cuda"))

    def step(self, q, pose, out=None, stream=None):
        import torch
        if out is None:
            out = torch.empty_like(q)
        check(lib.pl_sink_step(self.handle, _ptr(_contig(q, "q")), _ptr(pose), _ptr(out),
                               _stream(stream)), "pl_sink_step")
        return out

    def state(self, stream=None):
        s = SinkState()
        check(lib.pl_sink_get_state(self.handle, C.byref(s), _stream(stream)), "pl_sink_get_state")
        return s.as_dict()


def rope_table(positions, head_dim, base=10000.0, out=None, stream=None):
    """Device fp32 [positions, head_dim/2, 2] = (cos, sin)(pos * base^(-2i/head_dim))."""
    import torch
    if out is None:
        out = torch.empty((positions, head_dim // 2, 2), dtype=torch.float32, device="cuda")
    check(lib.pl_rope_table(_ptr(out), positions, head_dim, float(base), _stream(stream)),
          "pl_rope_table")
    return out


def rope_attention(q, q_pos0, segments, seg_pos0, heads, head_dim, table, out=None, stream=None):
    """Attention of un-rotated q [n, ld] over un-rotated (k, v) segments [len, ld], the
    rotary code applied (once per key) at the given window positions."""
    import torch
    segs = (KVSegment * len(segments))()
    pos = (i64 * len(segments))()
    for i, ((k, v), p0) in enumerate(zip(segments, seg_pos0)):
        segs[i] = KVSegment(_ptr(k), _ptr(v), k.shape[0], k.stride(0), 0)
        pos[i] = int(p0)
    if out is None:
        out = torch.empty_like(q)
    need = sz()
    keys = sum(k.shape[0] for k, _ in segments)
    check(lib.pl_rope_attention_workspace_bytes(q.shape[0], keys, heads, head_dim, C.byref(need)),
          "pl_rope_attention_workspace_bytes")
    ws = torch.empty(need.value, dtype=torch.uint8, device=q.device)
    check(lib.pl_rope_attention(_ptr(q), q.stride(0), int(q_pos0), segs, pos, len(segments),
                                q.shape[0], heads, head_dim, _ptr(table), table.shape[0],
                                _ptr(out), out.stride(0), _ptr(ws), need.value, _stream(stream)),
          "pl_rope_attention")
    return out


class Lpm:
    """LPM window cache: reference tokens + 3 sink chunks + 2 sliding chunks (pl_lpm_*)."""

    def __init__(self, ref_tokens, chunk_tokens, heads, head_dim, base=10000.0, device="cuda"):
        import torch
        self.ref_tokens, self.chunk_tokens = ref_tokens, chunk_tokens
        self.heads, self.head_dim = heads, head_dim
        need = sz()
        check(lib.pl_lpm_workspace_bytes(ref_tokens, chunk_tokens, heads, head_dim,
                                         C.byref(need)), "pl_lpm_workspace_bytes")
        self.workspace = torch.empty(need.value, dtype=torch.uint8, device=device)
        h = vp()
        check(lib.pl_lpm_create(ref_tokens, chunk_tokens, heads, head_dim, float(base),
                                _ptr(self.workspace), need.value, C.byref(h)), "pl_lpm_create")
        self.handle = h

    def close(self):
        if self.handle:
            lib.pl_lpm_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _views(self, fn, rows):
        import torch
        k, v = vp(), vp()
        check(fn(self.handle, C.byref(k), C.byref(v)), fn.__name__)
        shape = (rows, self.heads * self.head_dim)
        return (torch.as_tensor(_DeviceArray(k.value, shape, "<f2"), device="cuda"),
                torch.as_tensor(_DeviceArray(v.value, shape, "<f2"), device="cuda"))

    def ref_kv(self):
        return self._views(lib.pl_lpm_ref_kv, self.ref_tokens)

    def chunk_kv(self):
        return self._views(lib.pl_lpm_chunk_kv, self.chunk_tokens)

    def step(self, q, out=None, stream=None):
        import torch
        if out is None:
            out = torch.empty_like(q)
        check(lib.pl_lpm_step(self.handle, _ptr(_contig(q, "q")), _ptr(out), _stream(stream)),
              "pl_lpm_step")
        return out

    def state(self):
        s = LpmState()
        check(lib.pl_lpm_get_state(self.handle, C.byref(s)), "pl_lpm_get_state")
        return s.as_dict()


def pose_keypoints(canon, scale, poses, sel, out=None, stream=None):
    """Retargeted selected keypoints [frames, 7, 3] (fp64) of poses [frames, 6]."""
    import torch
    frames = poses.shape[0]
    if out is None:
        out = torch.empty((frames, 7, 3), dtype=torch.float64, device=poses.device)
    s = (i32 * 7)(*[int(x) for x in sel])
    check(lib.pl_pose_keypoints(_ptr(canon), float(scale), _ptr(_contig(poses, "poses")), frames,
                                s, _ptr(out), _stream(stream)), "pl_pose_keypoints")
    return out


def pose_ramp(kps_from, kps_to, frames=12, out=None, stream=None):
    import torch
    if out is None:
        out = torch.empty((frames, 7, 3), dtype=torch.float64, device=kps_from.device)
    check(lib.pl_pose_ramp(_ptr(kps_from), _ptr(kps_to), frames, _ptr(out), _stream(stream)),
          "pl_pose_ramp")
    return out


def pose_dots(kps, colours, radius, H, W, out=None, stream=None):
    """Dot images [frames, 3, H, W] fp32 of keypoints [frames, 7, 3]."""
    import numpy as np
    import torch
    frames = kps.shape[0]
    if out is None:
        out = torch.empty((frames, 3, H, W), dtype=torch.float32, device=kps.device)
    col = (f32 * 21)(*[float(x) for x in np.asarray(colours, np.float32).ravel()])
    check(lib.pl_pose_dots(_ptr(_contig(kps, "kps")), frames, col, float(radius), H, W, _ptr(out),
                           _stream(stream)), "pl_pose_dots")
    return out
