"""fp64 oracle of PersonaLive's streaming pyramid denoising round (CPU, numpy).

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
bench's CPU-baseline leg, never by the product path.

Sources (web pages; cited by page and section):
  [PL]  PersonaLive write-up (juhe.plus): sections "流式金字塔去噪" (streaming
        pyramid denoising), "首帧怎么办" (first frames / prefill),
        "抗身份漂移的补丁" (identity-drift guard), "三条条件通路" (three
        conditioning paths), "TensorRT 融合" (fused graph signature).
  [LA]  LiveAnimate (iitog.ru): PR-Sink paragraph (bounded KV cache of a
        static sink block, one pose-retrieved block and three rolling slots).
  [LPM] LPM 1.0 real-time digital actor write-up (sjmshsh.github.io):
        sections 7.3 "滑动窗口注意力" (3 sink chunks, 2 sliding chunks,
        reference tokens kept) and 7.4 "Pre-RoPE KV Cache" (cache K/V before
        the rotary code, rotate by the current window position).

Every function computes the plain definition in float64 with library matmuls
as the only primitive; nothing is blocked, fused or reordered.

Readings where the pages are silent (the plainest reading the rest supports):
  * beta schedule: SD "scaled linear", beta_start 0.00085, beta_end 0.012,
    1000 steps (the pages name DDIM with epsilon prediction and the SD VAE
    scale 0.18215 but print no schedule);
  * eta = 0, no clipping; alpha_bar_prev = 1 when t - 333 < 0 (unused: the
    t = 0 window is popped with its x0);
  * the hard-coded table {999, 666, 333, 0} governs over "trailing";
  * attention scale 1/sqrt(head_dim), no biases, no residual, no norm inside
    the op (the bank holds norm_hidden_states, already normalised);
  * KV order [own ; bank_0 ; ... ; bank_{n-1}] (softmax is order-invariant);
  * motion tokens: 512-d -> 32 x 16 row-major, plus interleaved sinusoidal
    PE (sin on even, cos on odd channels, base 10000);
  * motion cross-attention queries come from the reference-attention output
    of the same layer (the next sub-layer consumes the previous one's result);
  * bank check: Euclidean distance, "exceeds 17" = d > 17 (compared as
    d^2 > 289), each of the round's 4 new embeddings in order, lowest index
    wins ties, append only while fewer than 3 appends happened;
  * anchor k (k = 1..3) features are a caller-supplied stand-in for the
    Reference UNet re-run (weights absent);
  * latents are stored as float32 between rounds (each step computed in fp64,
    rounded once), unless `state_dtype=np.float64` is asked for.
"""
from __future__ import annotations

import math
from collections import deque

import numpy as np

# [PL] "流式金字塔去噪": the three config numbers and the hard-coded table.
TEMPORAL_ADAPTIVE_STEP = 4   # windows in the pile
TEMPORAL_WINDOW_SIZE = 4     # frames per window
NUM_INFERENCE_STEPS = 4
TIMESTEPS = (999, 666, 333, 0)
STEP_LENGTH = 333
# [PL] "抗身份漂移的补丁": threshold and append cap.
DRIFT_THRESHOLD = 17.0
APPEND_CAP = 3
# [PL] "三条条件通路": motion tokens.
MOTION_DIM, MOTION_TOKENS, MOTION_TOKEN_DIM = 512, 32, 16
# SD scaled-linear schedule (reading; the pages print none).
BETA_START, BETA_END, TRAIN_STEPS = 0.00085, 0.012, 1000


# ---------------------------------------------------------------------------
# Schedule and DDIM step
# ---------------------------------------------------------------------------

def betas() -> np.ndarray:
    """beta_i = (sqrt(0.00085) + i (sqrt(0.012) - sqrt(0.00085)) / 999)^2."""
    i = np.arange(TRAIN_STEPS, dtype=np.float64)
    a, b = math.sqrt(BETA_START), math.sqrt(BETA_END)
    return (a + i * (b - a) / (TRAIN_STEPS - 1)) ** 2


def alphas_cumprod() -> np.ndarray:
    """alpha_bar_t = prod_{i <= t} (1 - beta_i)."""
    return np.cumprod(1.0 - betas())


def alpha_bar(t: int) -> float:
    """alpha_bar at timestep t; 1.0 below zero (reading: unused by the pop)."""
    return 1.0 if t < 0 else float(alphas_cumprod()[t])


def ddim_step(x: np.ndarray, eps: np.ndarray, t: int, step: int = STEP_LENGTH):
    """One deterministic DDIM step (eta = 0) with epsilon prediction.

    [PL] "流式金字塔去噪": each window moves one level per round along
    {999, 666, 333, 0} with step length 333.
      x0     = (x_t - sqrt(1 - a_t) eps) / sqrt(a_t)
      x_prev = sqrt(a_prev) x0 + sqrt(1 - a_prev) eps,  a_prev = alpha_bar(t - step)
    Returns (x_prev, x0) in float64.
    """
    x = np.asarray(x, dtype=np.float64)
    eps = np.asarray(eps, dtype=np.float64)
    a_t = alpha_bar(t)
    a_p = alpha_bar(t - step)
    x0 = (x - math.sqrt(1.0 - a_t) * eps) / math.sqrt(a_t)
    x_prev = math.sqrt(a_p) * x0 + math.sqrt(1.0 - a_p) * eps
    return x_prev, x0


def forward_noise(x0: np.ndarray, eps: np.ndarray, t: int) -> np.ndarray:
    """q(x_t | x0) sample: sqrt(a_t) x0 + sqrt(1 - a_t) eps."""
    a_t = alpha_bar(t)
    return math.sqrt(a_t) * np.asarray(x0, np.float64) + math.sqrt(1.0 - a_t) * np.asarray(eps, np.float64)


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def softmax_rows(s: np.ndarray) -> np.ndarray:
    """Row softmax, max-subtracted (the value is the plain definition)."""
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    return p / p.sum(axis=-1, keepdims=True)


def mha(q: np.ndarray, k: np.ndarray, v: np.ndarray, heads: int) -> np.ndarray:
    """Multi-head scaled dot-product attention, no mask.

    q [Nq, C], k/v [Nk, C]; head h uses columns [h*hd, (h+1)*hd).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    C = q.shape[1]
    hd = C // heads
    out = np.empty((q.shape[0], v.shape[1]), dtype=np.float64)
    for h in range(heads):
        sl = slice(h * hd, (h + 1) * hd)
        p = softmax_rows(q[:, sl] @ k[:, sl].T / math.sqrt(hd))
        out[:, sl] = p @ v[:, sl]
    return out


def ref_attention_frame(h: np.ndarray, w: dict, bank: list, heads: int,
                        rows=None) -> np.ndarray:
    """Reference attention of one frame. [PL] "三条条件通路".

    The frame's queries attend over its own tokens concatenated with the
    reference KV bank (bank entries are norm_hidden_states of the Reference
    UNet, projected by this layer's Wk/Wv):
      K = [h ; bank_0 ; ... ] Wk,  V = [h ; bank_0 ; ...] Wv,
      out = softmax(Q K^T / sqrt(hd)) V Wo,  Q = h Wq.
    `rows` (optional index array) evaluates only those query rows.
    """
    h = np.asarray(h, np.float64)
    feats = np.concatenate([h] + [np.asarray(b, np.float64) for b in bank], axis=0)
    k = feats @ np.asarray(w["wk"], np.float64)
    v = feats @ np.asarray(w["wv"], np.float64)
    hq = h if rows is None else h[rows]
    q = hq @ np.asarray(w["wq"], np.float64)
    return mha(q, k, v, heads) @ np.asarray(w["wo"], np.float64)


def segment_attention(q: np.ndarray, segs_k: list, segs_v: list, heads: int) -> np.ndarray:
    """Attention over an explicit concatenation of already-projected K/V segments.

    q [Nq, C]; each segment [len_i, C]. Output [Nq, C] (no output projection).
    """
    k = np.concatenate([np.asarray(s, np.float64) for s in segs_k], axis=0)
    v = np.concatenate([np.asarray(s, np.float64) for s in segs_v], axis=0)
    return mha(q, k, v, heads)


# ---------------------------------------------------------------------------
# Motion tokens and motion cross-attention. [PL] "三条条件通路".
# ---------------------------------------------------------------------------

def motion_pe(n: int = MOTION_TOKENS, d: int = MOTION_TOKEN_DIM) -> np.ndarray:
    """Sinusoidal PE: PE[p, 2i] = sin(p / 10000^(2i/d)), PE[p, 2i+1] = cos(same)."""
    pe = np.zeros((n, d), dtype=np.float64)
    for p in range(n):
        for i in range(d // 2):
            ang = p / (10000.0 ** (2.0 * i / d))
            pe[p, 2 * i] = math.sin(ang)
            pe[p, 2 * i + 1] = math.cos(ang)
    return pe


def motion_tokens(e: np.ndarray) -> np.ndarray:
    """512-d expression embedding -> 32 tokens x 16 channels, plus PE."""
    e = np.asarray(e, np.float64).reshape(MOTION_TOKENS, MOTION_TOKEN_DIM)
    return e + motion_pe()


def motion_xattn_frame(x: np.ndarray, tokens: np.ndarray, w: dict, heads: int,
                       block: int = 1) -> np.ndarray:
    """Cross-attention of one frame's tokens to its 32 motion tokens.

    cross_attention_dim 16, 8 heads: Q = x Mq ([C,C]), K = m Mk, V = m Mv
    ([16, C]), out = softmax(Q K^T / sqrt(hd)) V Mo. Block 1 uses the
    weights mq, mk, mv, mo; block b > 1 uses mq<b>, mk<b>, mv<b>, mo<b>.
    """
    sfx = "" if block == 1 else str(block)
    x = np.asarray(x, np.float64)
    m = np.asarray(tokens, np.float64)
    q = x @ np.asarray(w["mq" + sfx], np.float64)
    k = m @ np.asarray(w["mk" + sfx], np.float64)
    v = m @ np.asarray(w["mv" + sfx], np.float64)
    return mha(q, k, v, heads) @ np.asarray(w["mo" + sfx], np.float64)


def layer_forward_frame(h, w, bank, tokens, heads, rows=None, motion_blocks=1):
    """One reference-attention layer followed by its motion cross-attention
    block(s). [PL] "三条条件通路" lists the motion module's attention blocks as
    [Spatial_Cross, Spatial_Cross]; with motion_blocks = 2 the second block
    (own weights, same 32 tokens) takes the first block's output as its
    queries, the way each sub-layer consumes the previous one's result."""
    a = ref_attention_frame(h, w, bank, heads, rows=rows)
    for b in range(1, motion_blocks + 1):
        a = motion_xattn_frame(a, tokens, w, heads, block=b)
    return a


# ---------------------------------------------------------------------------
# Motion bank (identity-drift guard). [PL] "抗身份漂移的补丁".
# ---------------------------------------------------------------------------

def sq_dist(a: np.ndarray, b: np.ndarray) -> float:
    """Squared Euclidean distance in float64 (sum in index order)."""
    d = np.asarray(a, np.float64) - np.asarray(b, np.float64)
    return float(np.dot(d, d))


def bank_check(bank: list, queries, appends: int, threshold: float = DRIFT_THRESHOLD,
               cap: int = APPEND_CAP):
    """Check each query in order against the bank; append while allowed.

    For each query q: d_j = ||q - bank_j||, j over the current bank (including
    entries appended earlier in the same call); j* = first index of the
    minimum; if d_{j*} > threshold (as d^2 > threshold^2) and appends < cap,
    append q. Returns (argmin list, min d^2 list, appended flags, new bank,
    new appends). The input list is not modified.
    """
    bank = [np.asarray(b, np.float64) for b in bank]
    amin, mind2, flags = [], [], []
    t2 = float(threshold) * float(threshold)
    for q in queries:
        q = np.asarray(q, np.float64)
        d2 = [sq_dist(q, b) for b in bank]
        j = int(np.argmin(d2))  # first occurrence on ties
        amin.append(j)
        mind2.append(d2[j])
        if d2[j] > t2 and appends < cap:
            bank.append(q.copy())
            appends += 1
            flags.append(1)
        else:
            flags.append(0)
    return amin, mind2, flags, bank, appends


def pose_retrieve(store: np.ndarray, desc: np.ndarray) -> int:
    """[LA] PR-Sink dynamic sink: index of the stored pose descriptor nearest to `desc`."""
    d2 = [sq_dist(desc, s) for s in np.asarray(store)]
    return int(np.argmin(d2))


class PRSinkCache:
    """[LA] PR-Sink: the bounded KV cache of one block stream.

    Parts (the page): the static sink (the first generated block, kept for
    good), one dynamic block retrieved from the history by pose, and a
    rolling buffer of three blocks. Readings where the page is silent: a
    block joins the cache after its own step (the first one as the sink, the
    others in the rolling buffer); the block a full rolling buffer pushes out
    enters the pose pool with its descriptor; a full pool replaces its oldest
    entry; retrieval is pose_retrieve over the pool in slot order and only
    happens once the pool holds something. Attention of a block: full
    (non-causal) over [own ; sink ; rolling oldest first ; retrieved].
    """

    ROLLING = 3

    def __init__(self, pool_capacity: int, heads: int):
        self.pool_capacity, self.heads = pool_capacity, heads
        self.sink = None            # (k, v)
        self.rolling = deque()      # (k, v, pose), oldest first
        self.pool = []              # (k, v, pose) per pool slot
        self.pool_oldest = 0        # slot a full pool replaces next
        self.blocks = 0

    def parts(self, pose):
        """The cache's K/V parts a block with this pose attends, and the retrieved slot."""
        ks, vs = [], []
        if self.sink is not None:
            ks.append(self.sink[0])
            vs.append(self.sink[1])
        for k, v, _ in self.rolling:
            ks.append(k)
            vs.append(v)
        slot = None
        if self.pool:
            slot = pose_retrieve(np.array([p for _, _, p in self.pool]), pose)
            ks.append(self.pool[slot][0])
            vs.append(self.pool[slot][1])
        return ks, vs, slot

    def step(self, q, k, v, pose):
        """Attention of block q (own K/V k, v) over the cache, then the cache update."""
        ks, vs, slot = self.parts(pose)
        out = segment_attention(q, [k] + ks, [v] + vs, self.heads)
        if self.sink is None:
            self.sink = (k, v)
        else:
            if len(self.rolling) == self.ROLLING:
                old = self.rolling.popleft()
                if len(self.pool) < self.pool_capacity:
                    self.pool.append(old)
                else:
                    self.pool[self.pool_oldest] = old
                    self.pool_oldest = (self.pool_oldest + 1) % self.pool_capacity
            self.rolling.append((k, v, np.asarray(pose)))
        self.blocks += 1
        return out, slot


# ---------------------------------------------------------------------------
# Pre-rotary KV cache with a sliding window. [LPM] sections 7.3
# "滑动窗口注意力" (sliding-window attention) and 7.4 "Pre-RoPE KV Cache".
# ---------------------------------------------------------------------------

def rope(x: np.ndarray, pos0: int, heads: int, base: float = 10000.0) -> np.ndarray:
    """Rotary code: in each head, the pair (2i, 2i+1) of row r turns by the
    angle (pos0 + r) * base^(-2i / head_dim). x [n, heads*head_dim]."""
    x = np.asarray(x, np.float64)
    n, C = x.shape
    hd = C // heads
    theta = base ** (-2.0 * np.arange(hd // 2) / hd)
    ang = (pos0 + np.arange(n, dtype=np.float64))[:, None] * theta[None, :]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    pairs = x.reshape(n, heads, hd // 2, 2)
    y0 = pairs[..., 0] * c - pairs[..., 1] * s
    y1 = pairs[..., 0] * s + pairs[..., 1] * c
    return np.stack([y0, y1], axis=-1).reshape(n, C)


def rope_attention(q, q_pos0, segs_k, segs_v, seg_pos0, heads, base=10000.0):
    """Attention after the rotary code: Q at q_pos0.., segment s at seg_pos0[s].."""
    ks = [rope(k, p, heads, base) for k, p in zip(segs_k, seg_pos0)]
    return segment_attention(rope(q, q_pos0, heads, base), ks, segs_v, heads)


class LPMCache:
    """[LPM] The window of a new chunk: the reference tokens (always kept),
    three fixed sink chunks and the two most recent chunks; K/V kept before
    the rotary code. Readings where the write-up is silent: the first three
    chunks become the sinks, later ones slide (a full window drops its
    oldest); positions follow the window's order [reference ; sinks ;
    sliding oldest first ; current], so a sliding chunk's position changes
    as it ages and its cached K is rotated afresh every step.
    """

    SINKS, SLIDE = 3, 2

    def __init__(self, ref_k, ref_v, heads, base=10000.0):
        self.ref = (ref_k, ref_v) if ref_k is not None and len(ref_k) else None
        self.heads, self.base = heads, base
        self.sinks = []
        self.slide = deque()
        self.chunks = 0

    def window(self):
        parts = ([self.ref] if self.ref is not None else []) + self.sinks + list(self.slide)
        pos, out = 0, []
        for k, v in parts:
            out.append((k, v, pos))
            pos += len(k)
        return out, pos

    def step(self, q, k, v):
        parts, q_pos0 = self.window()
        ks = [p[0] for p in parts] + [k]
        vs = [p[1] for p in parts] + [v]
        ps = [p[2] for p in parts] + [q_pos0]
        out = rope_attention(q, q_pos0, ks, vs, ps, self.heads, self.base)
        if len(self.sinks) < self.SINKS:
            self.sinks.append((k, v))
        else:
            if len(self.slide) == self.SLIDE:
                self.slide.popleft()
            self.slide.append((k, v))
        self.chunks += 1
        return out, q_pos0


# ---------------------------------------------------------------------------
# Prefill. [PL] "首帧怎么办".
# ---------------------------------------------------------------------------

def interpolate(a: np.ndarray, b: np.ndarray, num: int) -> np.ndarray:
    """`num` points of the straight line from a to b, both ends included."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    w = np.arange(num, dtype=np.float64) / (num - 1)
    return a[None, :] + w[:, None] * (b - a)[None, :]


def prefill_motion(ref_motion, drive0_motion, frames: int = 12) -> np.ndarray:
    """Motion of the 12 prefill frames: 13-point ramp ref -> drive0, last point dropped."""
    return interpolate(ref_motion, drive0_motion, frames + 1)[:-1]


# ---------------------------------------------------------------------------
# Pose path front. [PL] "三条条件通路" (pose as a residual): 21 implicit 3D
# keypoints with pitch / yaw / roll / translation / scale; retargeting keeps
# the reference's canonical keypoints and scale, takes only the driving
# rotation and half its translation; 7 of the 21 points are drawn as coloured
# dots. Readings where the page is silent (the plainest consistent one): angles in
# degrees, R = Rz(roll) Ry(yaw) Rx(pitch) acting on column vectors; keypoint
# = scale * R c + 0.5 t; the dot image is orthographic with x, y in [-1, 1]
# mapped to [0, W] x [0, H] (z dropped); a pixel (centre (x + 0.5, y + 0.5))
# takes the colour of the last of the 7 dots whose centre lies within the
# radius (d^2 <= r^2, fp64), black elsewhere; the prefill frames' keypoints
# are the 13-point ramp from the reference pose to the first driving pose,
# last point dropped (as the motion ramp).
# ---------------------------------------------------------------------------

def rotation(pitch: float, yaw: float, roll: float) -> np.ndarray:
    """R = Rz(roll) @ Ry(yaw) @ Rx(pitch), angles in degrees."""
    p, y, r = np.radians([pitch, yaw, roll])
    rx = np.array([[1, 0, 0], [0, np.cos(p), -np.sin(p)], [0, np.sin(p), np.cos(p)]])
    ry = np.array([[np.cos(y), 0, np.sin(y)], [0, 1, 0], [-np.sin(y), 0, np.cos(y)]])
    rz = np.array([[np.cos(r), -np.sin(r), 0], [np.sin(r), np.cos(r), 0], [0, 0, 1]])
    return rz @ ry @ rx


def retarget(canon: np.ndarray, scale: float, pose) -> np.ndarray:
    """Keypoints [21, 3] = scale * R(pose) c + 0.5 t: the reference's canonical
    points and scale, the driving frame's rotation, half its translation.
    pose = (pitch, yaw, roll, tx, ty, tz)."""
    pose = np.asarray(pose, np.float64)
    R = rotation(*pose[:3])
    return scale * (np.asarray(canon, np.float64) @ R.T) + 0.5 * pose[3:6][None, :]


def dot_centres(kps: np.ndarray, sel, H: int, W: int) -> np.ndarray:
    """Pixel coordinates [7, 2] (x, y) of the selected keypoints."""
    k = np.asarray(kps, np.float64)[list(sel)]
    return np.stack([(k[:, 0] + 1.0) * 0.5 * W, (k[:, 1] + 1.0) * 0.5 * H], axis=1)


def dot_image(centres: np.ndarray, colours: np.ndarray, radius: float, H: int, W: int):
    """[3, H, W] fp32: each pixel the colour of the last dot covering it."""
    img = np.zeros((3, H, W), np.float32)
    yy, xx = np.meshgrid(np.arange(H) + 0.5, np.arange(W) + 0.5, indexing="ij")
    for (cx, cy), col in zip(np.asarray(centres, np.float64), np.asarray(colours, np.float32)):
        inside = (xx - cx) ** 2 + (yy - cy) ** 2 <= float(radius) ** 2
        img[:, inside] = col[:, None]
    return img


def prefill_keypoints(kps_ref: np.ndarray, kps_drive0: np.ndarray, frames: int = 12):
    """Keypoints of the prefill frames: the 13-point ramp, last point dropped."""
    a = np.asarray(kps_ref, np.float64).ravel()
    b = np.asarray(kps_drive0, np.float64).ravel()
    return interpolate(a, b, frames + 1)[:-1].reshape(frames, *np.shape(kps_ref))


# ---------------------------------------------------------------------------
# The round's state machine (explicit deque). [PL] "流式金字塔去噪".
# ---------------------------------------------------------------------------

class Window:
    __slots__ = ("x", "t", "motion")

    def __init__(self, x, t, motion):
        self.x, self.t, self.motion = x, t, motion


class PyramidStream:
    """The latents pile as a deque of windows, oldest on the left.

    init (reference fusion): 3 prefill windows at t = 0, 333, 666 (oldest
    first), window w = forward-noised reference latent with its own noise;
    motion bank = [ref_motion], no appends yet.
    round: append the new window (pure noise, t = 999) on the right; the batch
    is the 4 windows oldest -> newest; each window takes one DDIM step with its
    epsilon; the leftmost window (t = 0) is popped and its x0 is the output;
    then the 4 new motion embeddings are checked against the bank.
    """

    def __init__(self, ref_latent, prefill_eps, ref_motion, drive0_motion,
                 state_dtype=np.float32):
        self.state_dtype = state_dtype
        self.pile: deque = deque()
        ref_latent = np.asarray(ref_latent, np.float64)        # [4, H, W]
        prefill_eps = np.asarray(prefill_eps, np.float64)      # [12, 4, H, W]
        mot = prefill_motion(ref_motion, drive0_motion, 3 * TEMPORAL_WINDOW_SIZE)
        for w, t in enumerate((0, 333, 666)):
            fr = slice(w * TEMPORAL_WINDOW_SIZE, (w + 1) * TEMPORAL_WINDOW_SIZE)
            x = forward_noise(ref_latent[None], prefill_eps[fr], t)
            self.pile.append(Window(x.astype(state_dtype), t, mot[fr].copy()))
        self.bank = [np.asarray(ref_motion, np.float64)]
        self.appends = 0
        self.rounds = 0
        self.frames_in = 0
        self.frames_out = 0

    def batch_timesteps(self):
        return [w.t for w in self.pile]

    def batch_motion(self) -> np.ndarray:
        """Motion embeddings of the 16 batch frames, oldest window first."""
        return np.concatenate([w.motion for w in self.pile], axis=0)

    def append(self, new_noise, new_motion):
        assert len(self.pile) == TEMPORAL_ADAPTIVE_STEP - 1
        self.pile.append(Window(np.asarray(new_noise, np.float64).astype(self.state_dtype),
                                TIMESTEPS[0], np.asarray(new_motion, np.float64).copy()))
        self.frames_in += TEMPORAL_WINDOW_SIZE

    def step_and_pop(self, eps):
        """DDIM step of every window with eps [16, 4, H, W]; pop the t=0 window's x0."""
        eps = np.asarray(eps, np.float64)
        assert len(self.pile) == TEMPORAL_ADAPTIVE_STEP
        out = None
        for w_idx, win in enumerate(self.pile):
            fr = slice(w_idx * TEMPORAL_WINDOW_SIZE, (w_idx + 1) * TEMPORAL_WINDOW_SIZE)
            x_prev, x0 = ddim_step(win.x, eps[fr], win.t)
            if win.t == 0:
                out = x0
            else:
                win.x = x_prev.astype(self.state_dtype)
                win.t -= STEP_LENGTH
        popped = self.pile.popleft()
        assert popped.t == 0
        self.frames_out += TEMPORAL_WINDOW_SIZE
        return out.astype(self.state_dtype)

    def check_bank(self, new_motion):
        amin, mind2, flags, self.bank, self.appends = bank_check(
            self.bank, new_motion, self.appends)
        return amin, mind2, flags

    def round(self, new_noise, new_motion, eps):
        """One full round (layers excluded): append, step, pop, bank check."""
        self.append(new_noise, new_motion)
        out = self.step_and_pop(eps)
        amin, mind2, flags = self.check_bank(new_motion)
        self.rounds += 1
        return out, flags, amin, mind2
