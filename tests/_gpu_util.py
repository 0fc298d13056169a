"""Helpers shared by the GPU parity tests (input upload, weight packing, error metrics)."""
import numpy as np

import synthetic as S


def dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None and t.dtype != dtype:
        t = t.to(dtype)
    return t.cuda()


def host(t):
    return t.detach().cpu().numpy()


def layer_weights_np(seed, name, C):
    """fp16 weights as numpy arrays (the exact values both sides use)."""
    return S.layer_weights(seed, name, C, np.float16)


def pack_weights(w):
    """Device tensors in the library's layout: w_qkv = [Wq|Wk|Wv], m_kv = [Mk|Mv]
    (and m2_* for a second motion block when w holds mq2, mk2, mv2, mo2)."""
    out = {
        "w_qkv": dev(np.concatenate([w["wq"], w["wk"], w["wv"]], axis=1)),
        "w_o": dev(w["wo"]),
        "m_q": dev(w["mq"]),
        "m_kv": dev(np.concatenate([w["mk"], w["mv"]], axis=1)),
        "m_o": dev(w["mo"]),
    }
    if "mq2" in w:
        out["m2_q"] = dev(w["mq2"])
        out["m2_kv"] = dev(np.concatenate([w["mk2"], w["mv2"]], axis=1))
        out["m2_o"] = dev(w["mo2"])
    return out


def attn_errors(got, want):
    d = np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64))
    rel = np.linalg.norm(d) / max(np.linalg.norm(want), 1e-30)
    return float(d.max()), float(d.mean()), float(rel)


def scaled_gates(want):
    """Scale of the attention gates for an output of RMS r: max(1, r).

    The absolute gates hold for outputs of unit scale or below (the reference
    attention's outputs have RMS ~ 0.02-0.4). The layer output after the motion
    cross-attention carries the motion embedding's magnitude, which a sigma = 3
    random walk raises to ~8 within two rounds; there the same gates apply to
    the output divided by its RMS.
    """
    r = float(np.sqrt(np.mean(np.square(np.asarray(want, np.float64)))))
    return max(1.0, r)


# tolerances of the floating-point paths
ATTN_MAX_ABS = 1e-2
ATTN_MEAN_ABS = 1e-3
DDIM_ABS = 1e-5
