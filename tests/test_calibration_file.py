"""Calibration artefacts on disk (transform_rope_head_b200.calibration): bit-exact round trip,
resumption by adding accumulators, and the checks on shapes and metadata.  CPU only."""
import numpy as np
import pytest

from transform_rope_head_b200 import calibration as C


def _arrays(layers=3, d_h=128, seed=0):
    rng = np.random.default_rng(seed)
    P = d_h // 2
    m = rng.standard_normal((layers, 2, P, 6))
    m[..., 0] = rng.integers(1, 1 << 40, size=(layers, 2, P)).astype(np.float64)  # counts
    m[0, 0, 0, 1] = np.nextafter(1.0, 2.0)                                     # last-bit values
    m[0, 0, 0, 2] = 5e-324                                                      # subnormal
    phi = rng.uniform(-np.pi / 4, np.pi / 4, size=(layers, P)).astype(np.float32)
    return m, phi


def test_round_trip_is_bit_exact(tmp_path):
    m, phi = _arrays()
    path = str(tmp_path / "cal.npz")
    C.save(path, m, phi, d_h=128, theta=5e5, estimator="k_only", layers=["l0", "l1", "l2"],
           extra={"tokens": 262144})
    got = C.load(path)
    assert got["moments"].tobytes() == m.tobytes()
    assert got["phi"].tobytes() == phi.tobytes()
    assert (got["d_h"], got["theta"], got["rope_style"], got["estimator"]) == (128, 5e5, "half", "k_only")
    assert got["layers"] == ["l0", "l1", "l2"] and got["extra"] == {"tokens": 262144}


def test_single_layer_arrays_and_resumption(tmp_path):
    """One layer's [2][P][6] and [P] are saved as one-layer stacks; resuming a calibration is
    adding the next batches' accumulators to the loaded ones (the sums are raw, uncentred)."""
    m, phi = _arrays(layers=1, d_h=64, seed=1)
    path = str(tmp_path / "one.npz")
    C.save(path, m[0], phi[0], d_h=64, theta=5e5)
    got = C.load(path)
    assert got["moments"].shape == (1, 2, 32, 6) and got["layers"] == ["0"]
    more, _ = _arrays(layers=1, d_h=64, seed=2)
    resumed = got["moments"][0] + more[0]
    np.testing.assert_array_equal(resumed, m[0] + more[0])


def test_torch_tensors_are_accepted(tmp_path):
    torch = pytest.importorskip("torch")
    m, phi = _arrays(layers=2, d_h=64, seed=3)
    path = str(tmp_path / "t.npz")
    C.save(path, torch.from_numpy(m), torch.from_numpy(phi), d_h=64, theta=1e6)
    assert C.load(path)["moments"].tobytes() == m.tobytes()


@pytest.mark.parametrize("bad", [
    dict(d_h=96), dict(d_h=64), dict(estimator="median"), dict(rope_style="neox"),
    dict(layers=["only one"]),
])
def test_rejects_mismatched_shapes_and_metadata(tmp_path, bad):
    m, phi = _arrays(layers=2, d_h=128, seed=4)
    kw = dict(d_h=128, theta=5e5)
    kw.update(bad)
    with pytest.raises(ValueError):
        C.save(str(tmp_path / "x.npz"), m, phi, **kw)


def test_rejects_wrong_dtypes_and_foreign_files(tmp_path):
    m, phi = _arrays(layers=1, d_h=64, seed=5)
    with pytest.raises(TypeError):
        C.save(str(tmp_path / "x.npz"), m.astype(np.float32), phi, d_h=64, theta=5e5)
    with pytest.raises(TypeError):
        C.save(str(tmp_path / "x.npz"), m, phi.astype(np.float64), d_h=64, theta=5e5)
    other = str(tmp_path / "other.npz")
    np.savez(other, moments=m, phi=phi, meta=np.frombuffer(b'{"format": "x"}', np.uint8))
    with pytest.raises(ValueError):
        C.load(other)
