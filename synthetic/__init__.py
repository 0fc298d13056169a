"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

This module holds random-number generation and workload shapes only. It holds
none of the method's arithmetic (no schedule, no attention, no DDIM, no
distances), so that the oracle and the CUDA path stay independent.

Generator: counter-based SplitMix64 (Steele, Lea and Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014): the i-th 64-bit word of stream
`key` is mix64(key + (i + 1) * 0x9E3779B97F4A7C15). Two consecutive words give
two 53-bit uniforms u1 in (0, 1], u2 in [0, 1) and Box-Muller (Box and
Muller, 1958) turns them into two N(0, 1) deviates in fp64:
    z0 = sqrt(-2 ln u1) cos(2 pi u2),  z1 = sqrt(-2 ln u1) sin(2 pi u2).
Values are scaled by `std` in fp64 and rounded once to the requested dtype.
"""
from __future__ import annotations

import hashlib

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def stream_key(seed: int, name: str) -> int:
    """64-bit key of the named stream under a config seed (BLAKE2b of both)."""
    h = hashlib.blake2b(f"{seed}:{name}".encode(), digest_size=8).digest()
    return int.from_bytes(h, "little")


def _mix64(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def words(key: int, start: int, count: int) -> np.ndarray:
    """Words start..start+count-1 of the counter-based SplitMix64 stream `key`."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + idx * _GOLDEN
    return _mix64(z)


def normal(seed: int, name: str, shape, std: float = 1.0, dtype=np.float64) -> np.ndarray:
    """N(0, std^2) array of `shape`, rounded once to `dtype`."""
    n = int(np.prod(shape)) if len(shape) else 1
    pairs = (n + 1) // 2
    w = words(stream_key(seed, name), 0, 2 * pairs)
    u1 = ((w[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * (1.0 / 9007199254740992.0)
    u2 = (w[1::2] >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)
    r = np.sqrt(-2.0 * np.log(u1))
    z = np.empty(2 * pairs, dtype=np.float64)
    z[0::2] = r * np.cos(2.0 * np.pi * u2)
    z[1::2] = r * np.sin(2.0 * np.pi * u2)
    return (z[:n] * std).reshape(shape).astype(dtype)


def uniform_int(seed: int, name: str, count: int, high: int) -> np.ndarray:
    """`count` integers in [0, high) (top 53 bits of each word, scaled)."""
    w = words(stream_key(seed, name), 0, count)
    u = (w >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)
    return np.minimum((u * high).astype(np.int64), high - 1)


# ---------------------------------------------------------------------------
# Workload shapes (the pages' geometry: 512x512 frames, 64x64x4 latents,
# SD-UNet attention levels, 4 windows x 4 frames). Sizes only.
# ---------------------------------------------------------------------------

#: The 16 reference-attention layers of the SD UNet, in forward order, with
#: (latent side, channels). d0x/u3x at 64x64, d1x/u2x at 32x32, d2x/u1x at
#: 16x16, m at 8x8.
LAYERS = (
    ("d00", 64, 320), ("d01", 64, 320), ("d10", 32, 640), ("d11", 32, 640),
    ("d20", 16, 1280), ("d21", 16, 1280), ("m", 8, 1280),
    ("u10", 16, 1280), ("u11", 16, 1280), ("u12", 16, 1280),
    ("u20", 32, 640), ("u21", 32, 640), ("u22", 32, 640),
    ("u30", 64, 320), ("u31", 64, 320), ("u32", 64, 320),
)
HEADS = 8
WINDOWS = 4
FRAMES_PER_WINDOW = 4
BATCH_FRAMES = WINDOWS * FRAMES_PER_WINDOW
LATENT_C = 4
MOTION_DIM = 512
MOTION_TOKENS = 32
MOTION_TOKEN_DIM = 16

SEEDS = {"tiny": 1001, "level64": 1002, "full": 1003, "long": 1004, "sink": 1005}


def layer_weights(seed: int, layer: str, C: int, dtype=np.float16):
    """Per-layer projection weights, N(0, 1/fan_in), stored [in, out].

    Returns dict: wq, wk, wv, wo ([C, C]) of the reference attention and
    mq ([C, C]), mk, mv ([16, C]), mo ([C, C]) of the motion cross-attention.
    """
    s_c = 1.0 / np.sqrt(C)
    s_m = 1.0 / np.sqrt(MOTION_TOKEN_DIM)
    return {
        "wq": normal(seed, f"{layer}/wq", (C, C), s_c, dtype),
        "wk": normal(seed, f"{layer}/wk", (C, C), s_c, dtype),
        "wv": normal(seed, f"{layer}/wv", (C, C), s_c, dtype),
        "wo": normal(seed, f"{layer}/wo", (C, C), s_c, dtype),
        "mq": normal(seed, f"{layer}/mq", (C, C), s_c, dtype),
        "mk": normal(seed, f"{layer}/mk", (MOTION_TOKEN_DIM, C), s_m, dtype),
        "mv": normal(seed, f"{layer}/mv", (MOTION_TOKEN_DIM, C), s_m, dtype),
        "mo": normal(seed, f"{layer}/mo", (C, C), s_c, dtype),
    }


def motion_block_weights(seed: int, layer: str, C: int, block: int, dtype=np.float16):
    """Weights of motion cross-attention block `block` (2, ...) of a layer, as
    layer_weights draws block 1's: mq, mo [C, C] N(0, 1/C); mk, mv [16, C]
    N(0, 1/16). Keys carry the block number (mq2, mk2, ...)."""
    s_c = 1.0 / np.sqrt(C)
    s_m = 1.0 / np.sqrt(MOTION_TOKEN_DIM)
    b = int(block)
    return {
        f"mq{b}": normal(seed, f"{layer}/mq{b}", (C, C), s_c, dtype),
        f"mk{b}": normal(seed, f"{layer}/mk{b}", (MOTION_TOKEN_DIM, C), s_m, dtype),
        f"mv{b}": normal(seed, f"{layer}/mv{b}", (MOTION_TOKEN_DIM, C), s_m, dtype),
        f"mo{b}": normal(seed, f"{layer}/mo{b}", (C, C), s_c, dtype),
    }


def layer_hidden(seed: int, layer: str, round_idx: int, F: int, N: int, C: int,
                 scale: float = 1.0, dtype=np.float16):
    """Per-round `norm_hidden_states` stand-in, N(0, scale^2), [F, N, C]."""
    return normal(seed, f"{layer}/hidden/{round_idx}", (F, N, C), scale, dtype)


def bank_features(seed: int, layer: str, entry: int, N: int, C: int, dtype=np.float16):
    """Reference (entry 0) or anchor (entry 1..3) feature stand-in, [N, C]."""
    return normal(seed, f"{layer}/bank/{entry}", (N, C), 1.0, dtype)
