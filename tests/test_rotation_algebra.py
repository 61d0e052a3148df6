"""The algebra the batched paths' rotation rests on, checked against the
oracle's rotation (the randomized Hadamard of the 3-bit SRAM-lookup article,
quantize() steps, and its order-K Paley variant).

- Sylvester block b > 256 (the dequantize kernel's on-chip rotation): with
  H_b = H_{b/256} (x) H_256, slice a of a block is
  sum_sb (-1)^popc(sb & a) H_256 x_sb, the sub-block transforms combined with
  signs instead of further butterfly stages.
- Paley block b = 28 m (the standalone input-rotation kernel): the two
  Kronecker factors commute, so mixing the 28 sub-blocks with H28 first and
  running the m-point transform on each mixture afterwards gives x~.
"""
import numpy as np
import pytest
from scipy.linalg import hadamard as sylvester

import oracle


def _popc(v: int) -> int:
    return bin(v).count("1")


@pytest.mark.parametrize("b", [512, 1024, 2048, 4096])
def test_sylvester_block_as_signed_sum_of_256_transforms(b):
    rng = np.random.default_rng(b)
    K = 2 * b
    x = rng.integers(-8, 9, size=(3, K)).astype(np.float16)
    hs = (rng.integers(0, 2, size=K) * 2 - 1).astype(np.int8)
    ref = oracle.hadamard(x, hs, b)
    h256 = sylvester(256).astype(np.float64)
    got = np.empty_like(ref)
    xd = x.astype(np.float64)
    for blk in range(K // b):
        base = blk * b
        t = [xd[:, base + 256 * sb: base + 256 * (sb + 1)] @ h256.T for sb in range(b // 256)]
        for a in range(b // 256):
            acc = sum((-1.0) ** _popc(sb & a) * t[sb] for sb in range(b // 256))
            k = slice(base + 256 * a, base + 256 * (a + 1))
            got[:, k] = hs[k] * acc / np.sqrt(b)
    assert np.allclose(got, ref, rtol=0, atol=1e-9)


@pytest.mark.parametrize("m", [64, 128])
def test_paley_block_mixing_before_the_transform(m):
    b = 28 * m
    ones = np.ones(b, np.int8)
    # Columns a' m of the oracle's rotation (unit inputs, no signs) hold H28:
    # entry (a m, a' m) is H28[a'][a] times H_m[0][0] = 1.
    units = np.zeros((28, b), np.float16)
    units[np.arange(28), np.arange(28) * m] = 1.0
    cols = oracle.hadamard(units, ones, b) * np.sqrt(b)      # cols[a'] = R[:, a' m]
    h28t = np.round(cols[:, ::m].T)                          # h28t[a][a'] = H28[a'][a]
    assert np.allclose(cols[:, ::m].T, h28t, rtol=0, atol=1e-9)
    assert np.array_equal(h28t @ h28t.T, 28 * np.eye(28))   # a Hadamard matrix of order 28
    hm = sylvester(m).astype(np.float64)
    rng = np.random.default_rng(m)
    x = rng.integers(-8, 9, size=b).astype(np.float16)
    ref = oracle.hadamard(x[None, :], ones, b)[0] * np.sqrt(b)
    z = h28t @ x.astype(np.float64).reshape(28, m)           # z[a][c] = sum_a' H28[a'][a] x[a' m + c]
    got = (z @ hm.T).reshape(b)                              # m-point transform of each mixture
    assert np.allclose(got, ref, rtol=0, atol=1e-8)
