"""The seeded input generator: deterministic, the documented shapes, and
OpenCV look-at cameras."""
import numpy as np

from scenes import SPECS, make_cameras, make_scene, make_target, look_at


def test_scenes_are_seeded_and_shaped():
    a = make_scene("student", n=5000)
    b = make_scene("student", n=5000)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])
        assert a[k].dtype == np.float32 and a[k].flags.c_contiguous
    assert a["means"].shape == (5000, 3) and a["quats"].shape == (5000, 4)
    assert a["opacity_logits"].shape == (5000,)
    assert np.all(np.abs(a["means"]) <= 5.0)
    assert abs(a["log_scales"].mean() - SPECS["student"].log_scale_mean) < 0.05
    c = make_scene("student", n=5000, seed=99)
    assert not np.array_equal(a["means"], c["means"])


def test_look_at_is_opencv():
    pos = np.array([3.0, -1.0, 2.0])
    V = look_at(pos).astype(np.float64)
    R, t = V[:3, :3], V[:3, 3]
    np.testing.assert_allclose(R @ R.T, np.eye(3), atol=1e-6)
    assert np.linalg.det(R) > 0
    np.testing.assert_allclose(R @ pos + t, 0, atol=1e-5)           # camera at the origin
    c = R @ np.zeros(3) + t
    assert c[2] > 0 and abs(c[0]) < 1e-5 and abs(c[1]) < 1e-5      # target straight ahead
    np.testing.assert_allclose(R[1] @ np.array([0, 1.0, 0]) > 0, True)  # +y down


def test_ring_cameras_and_target():
    cams = make_cameras("student")
    assert len(cams) == 60 and cams[0].width == 980 and cams[0].height == 545
    assert cams[0].tiles == 62 * 35 and cams[0].cx == 490.0
    t = make_target(980, 545)
    assert t.shape == (545, 980, 3) and 0 <= t.min() and t.max() < 1
