"""The seeded input generator: the Python and C halves agree, and both follow
the published SplitMix64 definition (its reference outputs for seed 0) and
IEEE round-to-nearest-even for bf16.  The generator holds none of the
method's arithmetic; these checks only keep the inputs of every test and of
the benchmark what their recipes say."""
import ctypes

import numpy as np

import synth

SPLITMIX64_SEED0 = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def _c():
    lib = synth._L()
    u64 = ctypes.c_uint64
    lib.synth_mix64.restype = u64
    lib.synth_mix64.argtypes = [u64]
    lib.synth_draw.restype = u64
    lib.synth_draw.argtypes = [u64, u64]
    lib.synth_normal.restype = ctypes.c_double
    lib.synth_normal.argtypes = [u64, u64]
    lib.synth_to_bf16.restype = ctypes.c_uint16
    lib.synth_to_bf16.argtypes = [ctypes.c_double]
    return lib


def test_splitmix64_reference_outputs():
    # the generator's stream for key 0 is SplitMix64 seeded with 0
    assert [synth.draw(0, i) for i in range(3)] == SPLITMIX64_SEED0
    assert [_c().synth_draw(0, i) for i in range(3)] == SPLITMIX64_SEED0


def test_python_and_c_draws_agree():
    lib = _c()
    rng = np.random.default_rng(3)
    for key in [0, 1, 0xFFFFFFFFFFFFFFFF] + [int(x) for x in rng.integers(0, 2**63, 20)]:
        for i in [0, 1, 2, 1000, 2**40 + 7]:
            assert synth.draw(key, i) == lib.synth_draw(key, i)
        assert synth.mix64(key) == lib.synth_mix64(key)


def test_bf16_rounding_is_nearest_even_in_both_halves():
    lib = _c()
    cases = {
        1.0: 0x3F80,
        1.0 + 2.0 ** -8: 0x3F80,          # halfway between 1 and 1 + 2^-7: to even (down)
        1.0 + 3 * 2.0 ** -8: 0x3F82,      # halfway between 1 + 2^-7 and 1 + 2^-6: to even (up)
        1.0 + 2.0 ** -8 + 2.0 ** -20: 0x3F81,  # just above halfway: up
        -2.0: 0xC000,
        0.0: 0x0000,
    }
    for x, bits in cases.items():
        assert int(synth.to_bf16(np.array([x]))[0]) == bits, x
        assert lib.synth_to_bf16(x) == bits, x
    rng = np.random.default_rng(4)
    xs = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-6, 6, 2000),
                         synth.bf16_to_f64(rng.integers(0, 0x7F7F, 500).astype(np.uint16)) * (1 + 2.0 ** -8)])
    py = synth.to_bf16(xs)
    c = np.array([lib.synth_to_bf16(float(x)) for x in xs], dtype=np.uint16)
    assert np.array_equal(py, c)


def test_box_muller_normals_are_standard():
    lib = _c()
    key = synth.tensor_key(9, 9)
    z = np.array([lib.synth_normal(key, i) for i in range(40000)])
    assert abs(z.mean()) < 0.03 and abs(z.std() - 1.0) < 0.03
    # the same draws through the bf16 fill, rounded: identical to rounding them here
    got = synth.normal_bf16(key, (100, 40))
    assert np.array_equal(got.reshape(-1), synth.to_bf16(z[:4000]))
