"""Pins of the counter-based gradient streams (workloads.counter_rng).

Philox4x32-10 against the known-answer vectors published with the
generator's definition (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers:
As Easy as 1, 2, 3", SC 2011; the Random123 library's known-answer tests):
counter / key all zero, all ones, and the hexadecimal digits of pi. The
float32 Box-Muller steps against float64 numpy functions, and the stream's
moments against the standard normal."""
import numpy as np
import pytest

from workloads import counter_rng as R


@pytest.mark.parametrize("ctr,key,out", [
    ([0, 0, 0, 0], [0, 0], [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]),
    ([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2, [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]),
    ([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344], [0xA4093822, 0x299F31D0],
     [0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]),
])
def test_philox4x32_10_known_answers(ctr, key, out):
    got = R.philox4x32_10(np.array([ctr], np.uint32), np.array([key], np.uint32))[0]
    assert [int(v) for v in got] == out


def test_ln_and_sincos_are_accurate_float32():
    u = np.concatenate([np.linspace(2.0 ** -24, 1, 200001), [2.0 ** -24, 0.5, 1.0]]).astype(np.float32)
    ref = np.log(u.astype(np.float64))
    got = R.ln_f32(u).astype(np.float64)
    assert np.all(np.abs(got - ref) <= 2e-7 * np.maximum(1.0, np.abs(ref)))
    assert R.ln_f32(np.float32(1.0)) == 0.0  # u1 = 1 gives radius 0 exactly
    r = np.linspace(0, 1, 100001, endpoint=False).astype(np.float32)
    for q in range(4):
        c, s = R.sincos_quadrant(np.full(r.shape, q), r)
        th = (q + r.astype(np.float64)) * np.pi / 2
        assert np.max(np.abs(c - np.cos(th))) < 3e-7
        assert np.max(np.abs(s - np.sin(th))) < 3e-7


def test_stream_moments_and_tails():
    z = R.gaussian_entries(7, 3, 11, 2, 2_000_000).astype(np.float64)
    assert abs(z.mean()) < 4 * (1 / np.sqrt(z.size))
    assert abs(z.var() - 1) < 4e-3
    assert abs(np.mean(z ** 4) - 3) < 3e-2
    # P(|z| > 3) of the standard normal is 0.0027
    assert abs(np.mean(np.abs(z) > 3) - 0.0027) < 3e-4
    assert np.max(np.abs(z)) <= np.sqrt(-2 * np.log(2.0 ** -24)) + 1e-3  # the radius bound of u1 >= 2^-24


def test_stream_is_a_function_of_its_coordinates():
    a = R.gaussian_entries(0, 1, 2, 3, 1001)
    b = R.gaussian_entries(0, 1, 2, 3, 4000)
    np.testing.assert_array_equal(a, b[:1001])  # entries do not depend on the matrix size
    for other in (R.gaussian_entries(0, 2, 2, 3, 1001), R.gaussian_entries(0, 1, 3, 3, 1001),
                  R.gaussian_entries(0, 1, 2, 4, 1001)):  # another worker, matrix or step
        assert np.mean(a == other) < 0.01
    # seed_base + worker is the key: (seed 1, worker 0) is (seed 0, worker 1)
    np.testing.assert_array_equal(R.gaussian_entries(1, 0, 2, 3, 64), R.gaussian_entries(0, 1, 2, 3, 64))
    np.testing.assert_array_equal(R.gaussian_entries(0, 1, 2, 3, 64, sigma=0.5),
                                  (a[:64] * np.float32(0.5)).astype(np.float32))


def test_entry_layout_in_groups_of_four():
    """Entry 4g + j is the j-th Gaussian of counter g (two Box-Muller pairs)."""
    x = R.philox4x32_10(np.array([[5, 0, 9, 0]], np.uint32), np.array([[4, 6]], np.uint32))[0]
    z0, z1 = R.box_muller(x[0:1], x[1:2])
    z2, z3 = R.box_muller(x[2:3], x[3:4])
    got = R.gaussian_entries(0, 4, 6, 9, 24)[20:24]
    np.testing.assert_array_equal(got, np.array([z0[0], z1[0], z2[0], z3[0]], np.float32))
