"""Orders of evaluation the library uses where the pages define a module,
checked in fp64 against the oracle's definition (CPU only; no library code).

The round evaluates the motion cross-attention of a layer ([PL] 三条条件通路:
Q = x Mq, K = m Mk, V = m Mv, softmax(Q K^T / sqrt(hd)) V Mo over 8 heads)
per head as scores x (Mq_h K_h^T / sqrt(hd)) and output P_h (V_h Mo_h),
summed over the heads. In real arithmetic the two orders agree; here fp64
must agree to rounding, for one block and for a second block queried by the
first block's output.
"""
import numpy as np

import oracle as O
import synthetic as S


def _folded(x, tok, w, heads, sfx=""):
    mq, mk, mv, mo = (np.asarray(w[n + sfx], np.float64) for n in ("mq", "mk", "mv", "mo"))
    C = mq.shape[0]
    hd = C // heads
    k, v = tok @ mk, tok @ mv                      # [32, C]
    out = np.zeros((x.shape[0], C))
    for h in range(heads):
        sl = slice(h * hd, (h + 1) * hd)
        w_qk = mq[:, sl] @ k[:, sl].T / np.sqrt(hd)   # [C, 32]
        s = x @ w_qk
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        out += p @ (v[:, sl] @ mo[sl, :])           # P_h (V_h Mo_h)
    return out


def _close(got, want):
    err = np.max(np.abs(got - want))
    return err <= 1e-11 * max(1.0, float(np.max(np.abs(want)))), err


def test_folded_motion_cross_attention_equals_the_definition():
    seed = S.SEEDS["tiny"] + 5
    for C in (320, 640, 1280):
        w = S.layer_weights(seed, f"f{C}", C, np.float64)
        w.update(S.motion_block_weights(seed, f"f{C}", C, 2, np.float64))
        x = S.normal(seed, f"x{C}", (48, C), 1.0)
        tok = O.motion_tokens(S.normal(seed, f"e{C}", (512,), 3.0, np.float32))
        y1 = O.motion_xattn_frame(x, tok, w, 8)
        ok, err = _close(_folded(x, tok, w, 8), y1)
        assert ok, (C, err)
        y2 = O.motion_xattn_frame(y1, tok, w, 8, block=2)
        ok, err = _close(_folded(_folded(x, tok, w, 8), tok, w, 8, sfx="2"), y2)
        assert ok, (C, err)


def test_folded_order_catches_a_transposed_head_block():
    # the check has teeth: pairing head h's queries with head h+1's keys (a
    # plausible indexing slip in a fold) moves the output far past rounding
    seed = S.SEEDS["tiny"] + 6
    C = 320
    w = S.layer_weights(seed, "g", C, np.float64)
    x = S.normal(seed, "x", (16, C), 1.0)
    tok = O.motion_tokens(S.normal(seed, "e", (512,), 3.0, np.float32))
    want = O.motion_xattn_frame(x, tok, w, 8)
    bad = dict(w)
    mk = np.asarray(w["mk"], np.float64).copy()
    hd = C // 8
    mk[:, :hd], mk[:, hd:2 * hd] = mk[:, hd:2 * hd].copy(), mk[:, :hd].copy()
    bad["mk"] = mk
    ok, _ = _close(_folded(x, tok, bad, 8), want)
    assert not ok
