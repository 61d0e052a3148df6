"""The oracle against its pins, and proof that the pins catch planted mistakes.

The mutation tests copy the oracle's C source, plant one plausible mistake
(a swapped bit order, a transposed index, a dropped term...), compile the copy
into a temporary library on the CPU and require at least one pin to fail.
"""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
from tests import oracle_pins

ORACLE_SRC = os.path.join(os.path.dirname(oracle.__file__), "eva_oracle.c")


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle)


class _Mutant:
    """The oracle module's functions bound to a different compiled library."""

    def __init__(self, libpath):
        self._path = libpath

    def __getattr__(self, name):
        fn = getattr(oracle, name)

        def call(*a, **k):
            saved = oracle._lib
            try:
                oracle._lib = None
                real_build = oracle.build
                oracle.build = lambda force=False: self._path
                try:
                    return fn(*a, **k)
                finally:
                    oracle.build = real_build
            finally:
                oracle._lib = saved
        return call


MUTATIONS = {
    "sign_bit_msb_first": ("((byte >> (k % 8)) & 1)", "((byte >> (7 - k % 8)) & 1)"),
    "sign_polarity": ("? 1.0 : -1.0;\n}", "? -1.0 : 1.0;\n}"),
    "subvector_strided": ("int c = index_of(d, wi, o, k / d->d);", "int c = index_of(d, wi, o, k % (d->K / d->d));"),
    "nibble_order_swapped": ("return (byte >> (4 * (j & 1))) & 15;", "return (byte >> (4 * (1 - (j & 1)))) & 15;"),
    "nibble_byte_strided": ("(size_t)(J / 2) + (size_t)(j / 2)];", "(size_t)(J / 2) + (size_t)(j % (J / 2))];"),
    "centroid_component_reversed": ("(size_t)(k % d->d)]", "(size_t)(d->d - 1 - k % d->d)]"),
    "codebook_group_modulo": ("return d->codebook_rows ? o / d->codebook_rows : 0;",
                              "return d->codebook_rows ? o % (d->N / d->codebook_rows) : 0;"),
    "alpha_group_shifted": ("(size_t)(k / d->residual_group)]",
                            "(size_t)((k / d->residual_group + 1) % ngroups)]"),
    "residual_dropped": ("wrow[k] += a * sign_of(d, signs, o, k);", "(void)a;"),
    "hadamard_sign_dropped": ("xout[k] = (double)hsign[k] * acc * inv;", "xout[k] = acc * inv;"),
    "hadamard_unnormalised": ("double inv = 1.0 / sqrt((double)b);", "double inv = 1.0;"),
    "hadamard_transposed_block": ("acc += block_entry(b, q, p) * xb[q];",
                                  "acc += block_entry(b, (q + 1) % b, p) * xb[q];"),
    "paley_not_transposed": ("acc += block_entry(b, q, p) * xb[q];", "acc += block_entry(b, p, q) * xb[q];"),
    "paley_chi_flipped": ("return r == 1 ? 1 : -1;", "return r == 1 ? -1 : 1;"),
    "paley_wrong_modulus": ("z[1] = (z[1] + z[3]) % 3; z[0] = (z[0] + z[3]) % 3;",
                            "z[1] = (z[1] + z[3]) % 3; z[0] = (z[0] + 2 * z[3]) % 3;"),
    "paley_kronecker_swapped": ("return paley28(p / m, q / m) * sylvester(p % m, q % m);",
                                "return paley28(p % 28, q % 28) * sylvester(p / 28, q / 28);"),
    "paley_border_sign": ("if (j == 0) return -1.0;", "if (j == 0) return 1.0;"),
    "f16_exponent_bias": ("expo - 25)", "expo - 24)"),
    "f16_subnormal_scale": ("ldexp((double)mant, -24)", "ldexp((double)mant, -25)"),
    "alpha_not_mean": ("num += v * s;", "num += v * v;"),
    "kmeans_tie_to_last": ("if (c == 0 || dist < best_d) {", "if (c == 0 || dist <= best_d) {"),
    "kmeans_component_dropped": ("            for (int t = 0; t < d; ++t) {\n                const float diff",
                                 "            for (int t = 1; t < d; ++t) {\n                const float diff"),
    "kmeans_mean_off_by_one": ("/ (double)cnt[gc])", "/ (double)(cnt[gc] + 1))"),
    "kmeans_empty_zeroed": (": old_cent[(size_t)gc * d + t];", ": 0.f;"),
    "kmeans_codebook_modulo": ("const int64_t g = vecs_per_cb ? m / vecs_per_cb : 0;\n        const float *cb",
                               "const int64_t g = vecs_per_cb ? m % 2 : 0;\n        const float *cb"),
    "residual_zero_negative": ("if (r >= 0.f)", "if (r > 0.f)"),
    "residual_msb_first": ("(uint8_t)(1u << (k % 8))", "(uint8_t)(1u << (7 - k % 8))"),
    "residual_alpha_rms": ("acc += fabs((double)r);", "acc += (double)r * (double)r;"),
    "residual_codebook_modulo": ("const int g = codebook_rows ? o / codebook_rows : 0;\n        for (int q",
                                 "const int g = codebook_rows ? o % (N / codebook_rows) : 0;\n        for (int q"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path):
    src = open(ORACLE_SRC).read()
    old, new = MUTATIONS[name]
    assert src.count(old) >= 1, f"mutation anchor missing: {old!r}"
    mutated = src.replace(old, new)
    csrc = tmp_path / "mutant.c"
    csrc.write_text(mutated)
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o", str(lib),
                    str(csrc), "-lm"], check=True)
    m = _Mutant(str(lib))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(m)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught mutation {name}"


def test_oracle_rejects_bad_arguments():
    wc = np.zeros((256, 4), np.float16)
    wi = np.zeros((4, 3), np.uint8)
    with pytest.raises(ValueError):
        oracle.linear(wc, wi, np.zeros((1, 13), np.float16))          # K != J*d
    with pytest.raises(ValueError):
        oracle.linear(wc[:8], np.full((4, 3), 9, np.uint8), np.zeros((1, 12), np.float16))  # index >= 2^n
    with pytest.raises(ValueError):
        oracle.linear(wc, np.zeros((4, 64), np.uint8), np.zeros((1, 256), np.float16),
                      residual_group=128)                              # residual without signs


def test_oracle_threads_do_not_change_result():
    rng = np.random.default_rng(0)
    wc = rng.normal(0, 0.02, size=(256, 4)).astype(np.float16)
    wi = rng.integers(0, 256, size=(300, 64)).astype(np.uint8)
    x = rng.normal(size=(2, 256)).astype(np.float16)
    assert np.array_equal(oracle.linear(wc, wi, x, nthreads=1), oracle.linear(wc, wi, x, nthreads=4))


def test_page5_bit_budget():
    """The 3.125-bit format: 2 bits of index + 1 sign bit + 16/128 bits of alpha
    per weight (3-bit SRAM-lookup article, Gemma-2-9B result); 16/3.125 = 5.12;
    a shared 256-entry codebook makes 256/N of the dense fp16 multiplies
    (92.9% fewer at N = 3584, the article's ~93%)."""
    from vector_quantized_weight_b200 import synth
    for shape in synth.CONFIGS["gemma_3bit"].layers:
        lay = synth.make_layer(shape, 1)
        bits = 8 * (lay.wi.nbytes + lay.signs.nbytes + lay.alpha.nbytes) / (shape.N * shape.K)
        assert bits == 3.125
    assert 16 / 3.125 == 5.12
    assert abs((1 - 256 / 3584) - 0.929) < 5e-4
