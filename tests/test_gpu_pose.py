"""Pose path front (pl_pose_*) against the oracle: keypoints, prefill ramp, dot images."""
import numpy as np
import pytest

import oracle as O
import synthetic as S
from _gpu_util import dev, host

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

SEL = [0, 3, 5, 8, 11, 15, 20]
COLOURS = np.array([[1, 0, 0], [0, 1, 0], [0, 0, 1], [1, 1, 0], [1, 0, 1], [0, 1, 1],
                    [0.5, 0.5, 0.5]], np.float32)


@pytest.fixture(scope="module")
def P():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import denoise_step_b200 as P
    return P


def _inputs(frames=4):
    seed = S.SEEDS["tiny"] + 500
    canon = S.normal(seed, "canon", (21, 3), 0.3, np.float32)
    poses = np.concatenate([S.normal(seed, "angles", (frames, 3), 15.0),
                            S.normal(seed, "trans", (frames, 3), 0.1)], axis=1).astype(np.float32)
    return canon, np.float32(0.9), poses


def test_pose_keypoints_and_ramp_match_oracle(P):
    canon, scale, poses = _inputs()
    got = host(P.pose_keypoints(dev(canon), scale, dev(poses), SEL))
    want = np.stack([O.retarget(canon, float(scale), p)[SEL] for p in poses])
    assert np.max(np.abs(got - want)) <= 1e-12
    ramp = host(P.pose_ramp(dev(want[0]), dev(want[1])))
    assert np.max(np.abs(ramp - O.prefill_keypoints(want[0], want[1]))) <= 1e-14


@pytest.mark.parametrize("H,W,radius", [(512, 512, 6.0), (200, 333, 2.5), (64, 64, 0.0)])
def test_pose_dots_match_oracle_bit_exact(P, H, W, radius):
    canon, scale, poses = _inputs()
    kps = np.stack([O.retarget(canon, float(scale), p)[SEL] for p in poses])
    # the splat on the oracle's own keypoints: every pixel decision identical
    got = host(P.pose_dots(dev(kps), COLOURS, radius, H, W))
    for f in range(len(kps)):
        want = O.dot_image(O.dot_centres(kps[f], range(7), H, W), COLOURS, radius, H, W)
        assert np.array_equal(got[f], want), (f, np.argwhere(got[f] != want)[:5])
    # the whole path from poses: only pixels on a dot's rim may differ (keypoints
    # agree to ~1e-16, the disc test to the last bit)
    kd = P.pose_keypoints(dev(canon), scale, dev(poses), SEL)
    full = host(P.pose_dots(kd, COLOURS, radius, H, W))
    for f in range(len(kps)):
        want = O.dot_image(O.dot_centres(kps[f], range(7), H, W), COLOURS, radius, H, W)
        bad = np.argwhere(np.any(full[f] != want, axis=0))
        cen = O.dot_centres(kps[f], range(7), H, W)
        for y, x in bad:
            margin = min(abs((x + 0.5 - cx) ** 2 + (y + 0.5 - cy) ** 2 - radius ** 2) for cx, cy in cen)
            assert margin < 1e-9, (f, y, x, margin)


def test_pose_dots_cover_something(P):
    canon, scale, poses = _inputs()
    img = host(P.pose_dots(P.pose_keypoints(dev(canon), scale, dev(poses), SEL), COLOURS, 6.0,
                           512, 512))
    assert (img.sum(axis=1) > 0).sum() > 100       # the dots land inside the frame
