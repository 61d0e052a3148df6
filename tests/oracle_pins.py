"""Pins for the double-precision oracle: checks against facts that do not come
from the oracle itself (hand-worked examples, library routines, closed forms,
invariants, factorisation of a dense matrix).

Each pin takes the oracle module (or a stand-in with the same functions, as
the mutation tests use) and raises AssertionError when it is violated.
"""
from __future__ import annotations

import json
import os

import numpy as np
import scipy.linalg

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- fixtures

def pin_golden_vq(orc):
    g = _golden("vq_lookup_handworked.json")
    wc = np.zeros((256, 4), np.float16)
    for c, v in g["centroids"].items():
        wc[int(c)] = v
    wi = np.array(g["wi"], np.uint8)
    x = np.array(g["x"], np.float16)[None]
    y = orc.linear(wc, wi, x)
    assert np.array_equal(y[0], np.array(g["y"], np.float64)), (y, g["y"])
    yl, _ = orc.lookup_form(wc, wi, x)
    assert np.array_equal(yl[0], np.array(g["y"], np.float64)), (yl, g["y"])


def pin_golden_residual(orc):
    g = _golden("sign_residual_handworked.json")
    K, N = g["K"], g["N"]
    wc = np.zeros((256, 4), np.float16)
    wi = np.zeros((N, K // 4), np.uint8)
    signs = np.repeat(np.array(g["sign_byte_per_row"], np.uint8)[:, None], K // 8, axis=1)
    alpha = np.array(g["alpha"], np.float16)
    k = np.arange(K)
    x = ((k % 8 + 1) * np.where(k < 128, 1, 2)).astype(np.float16)[None]
    y = orc.linear(wc, wi, x, signs=signs, alpha=alpha, residual_group=128)
    assert np.array_equal(y[0], np.array(g["y"], np.float64)), (y, g["y"])


def pin_golden_hadamard(orc):
    g = _golden("hadamard_handworked.json")
    x = np.array(g["x"], np.float16)[None]
    s = np.array(g["s"], np.int8)
    xr = orc.hadamard(x, s, g["b"])
    assert np.array_equal(xr[0], np.array(g["x_rot"], np.float64)), xr


# ------------------------------------------------------ library routines

def pin_f16_decode(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = orc.f16_to_f64(bits)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def pin_hadamard_scipy(orc, seed=1):
    rng = np.random.default_rng(seed)
    for b, nblk in ((4, 3), (64, 2), (512, 3)):
        K = b * nblk
        x = rng.normal(size=(2, K)).astype(np.float16)
        s = (rng.integers(0, 2, K) * 2 - 1).astype(np.int8)
        H = scipy.linalg.hadamard(b).astype(np.float64)
        ref = np.empty((2, K))
        for blk in range(nblk):
            sl = slice(blk * b, (blk + 1) * b)
            ref[:, sl] = (x[:, sl].astype(np.float64) @ H.T) / np.sqrt(b) * s[sl]
        got = orc.hadamard(x, s, b)
        assert np.allclose(got, ref, rtol=0, atol=1e-12 * np.abs(ref).max()), (b, np.abs(got - ref).max())


def pin_factorisation(orc, seed=2):
    """Start from a dense integer W whose rows are built from a small pool of
    4-vectors, factor it with numpy.unique into (codebook, indices), and
    require the oracle to reproduce W @ x exactly.  Unused codebook slots
    hold junk so a wrong index reads a wrong value."""
    rng = np.random.default_rng(seed)
    for N, K, rows_per_cb in ((24, 64, 0), (32, 48, 8)):
        J = K // 4
        pool = rng.integers(-3, 4, size=(40, 4))
        W = pool[rng.integers(0, 40, size=(N, J))].reshape(N, K)
        G = N // rows_per_cb if rows_per_cb else 1
        rows = rows_per_cb or N
        wc = rng.integers(-9, 10, size=(G, 256, 4)).astype(np.float16)   # junk everywhere
        wi = np.zeros((N, J), np.uint8)
        for g in range(G):
            sub = W[g * rows:(g + 1) * rows].reshape(rows * J, 4)
            uniq, inv = np.unique(sub, axis=0, return_inverse=True)
            perm = rng.permutation(256)[:len(uniq)]            # scatter entries
            wc[g, perm] = uniq
            wi[g * rows:(g + 1) * rows] = perm[inv.reshape(-1)].reshape(rows, J)
        x = rng.integers(-5, 6, size=(3, K))
        y = orc.linear(wc, wi, x.astype(np.float16), codebook_rows=rows_per_cb)
        ref = (W @ x.T).T
        assert np.array_equal(y, ref.astype(np.float64)), (N, K, np.abs(y - ref).max())


def pin_factorisation_residual(orc, seed=3):
    """W = WC[WI] + alpha * sigma with sigma packed by numpy.packbits
    (little bit order); dyadic values keep every sum exact."""
    rng = np.random.default_rng(seed)
    N, K = 8, 384
    J = K // 4
    pool = rng.integers(-2, 3, size=(30, 4))
    Wvq = pool[rng.integers(0, 30, size=(N, J))].reshape(N, K).astype(np.float64)
    uniq, inv = np.unique(Wvq.reshape(N * J, 4), axis=0, return_inverse=True)
    wc = rng.integers(-9, 10, size=(256, 4)).astype(np.float16)
    wc[:len(uniq)] = uniq
    wi = inv.reshape(N, J).astype(np.uint8)
    sigma_bits = rng.integers(0, 2, size=(N, K)).astype(np.uint8)
    signs = np.packbits(sigma_bits, axis=1, bitorder="little")
    alpha = rng.choice([0.125, 0.25, 0.5, -0.25, 2.0], size=(N, K // 128)).astype(np.float16)
    W = Wvq + np.repeat(alpha.astype(np.float64), 128, axis=1) * (2.0 * sigma_bits - 1.0)
    x = rng.integers(-4, 5, size=(2, K))
    y = orc.linear(wc, wi, x.astype(np.float16), signs=signs, alpha=alpha, residual_group=128)
    assert np.array_equal(y, (W @ x.T).T), np.abs(y - (W @ x.T).T).max()


def pin_rotation_composite(orc, seed=4):
    """y = W (Q^T x) with Q^T x formed from scipy's Hadamard matrix."""
    rng = np.random.default_rng(seed)
    N, K, b = 6, 384, 128
    J = K // 4
    wc = rng.integers(-3, 4, size=(256, 4)).astype(np.float16)
    wi = rng.integers(0, 256, size=(N, J)).astype(np.uint8)
    W = wc.astype(np.float64)[wi].reshape(N, K)
    s = (rng.integers(0, 2, K) * 2 - 1).astype(np.int8)
    x = rng.normal(size=(2, K)).astype(np.float16)
    H = scipy.linalg.hadamard(b).astype(np.float64)
    xr = np.concatenate([(x[:, i:i + b].astype(np.float64) @ H.T) / np.sqrt(b) for i in range(0, K, b)], 1) * s
    ref = (W @ xr.T).T
    y = orc.linear(wc, wi, x, hsign=s, hadamard_block=b)
    assert np.allclose(y, ref, rtol=0, atol=1e-11 * np.abs(ref).max()), np.abs(y - ref).max()


# ------------------------------------------------------ special cases

def pin_unit_centroids(orc, seed=5):
    """Centroid c = (c//4 + 1) * e_(c mod 4): y[o] = sum_j (c//4+1) x[4j + c mod 4],
    formed by numpy gathering, no dequantisation."""
    rng = np.random.default_rng(seed)
    N, K = 16, 128
    J = K // 4
    c = np.arange(256)
    wc = np.zeros((256, 4), np.float16)
    wc[c, c % 4] = c // 4 + 1
    wi = rng.integers(0, 256, size=(N, J)).astype(np.uint8)
    x = rng.integers(-8, 9, size=(1, K)).astype(np.float16)
    idx = 4 * np.arange(J)[None, :] + (wi % 4)
    ref = ((wi // 4 + 1) * x[0].astype(np.float64)[idx]).sum(axis=1)
    y = orc.linear(wc, wi, x)
    assert np.array_equal(y[0], ref)


def pin_all_equal_indices(orc):
    N, K = 5, 64
    wc = np.zeros((256, 4), np.float16)
    wc[77] = 1.0
    wi = np.full((N, K // 4), 77, np.uint8)
    x = (np.arange(K) - 20).astype(np.float16)[None]
    y = orc.linear(wc, wi, x)
    assert np.array_equal(y[0], np.full(N, float(np.sum(np.arange(K) - 20))))


def pin_group_scaling(orc, seed=6):
    """Codebook g = (g+1) * base: row o's output scales by g(o)+1, so the
    row-to-codebook map o -> o // rows is pinned."""
    rng = np.random.default_rng(seed)
    rows, G, K = 4, 5, 64
    N = rows * G
    base = rng.integers(-4, 5, size=(256, 4))
    wc = np.stack([(g + 1) * base for g in range(G)]).astype(np.float16)
    wi = rng.integers(0, 256, size=(N, K // 4)).astype(np.uint8)
    x = rng.integers(-3, 4, size=(2, K)).astype(np.float16)
    y1 = orc.linear(base.astype(np.float16), wi, x)
    yg = orc.linear(wc, wi, x, codebook_rows=rows)
    scale = (np.arange(N) // rows + 1).astype(np.float64)
    assert np.array_equal(yg, y1 * scale[None, :])


def pin_residual_popcount(orc, seed=7):
    """WC = 0 and x = 1: y[o] = sum_q alpha[o][q] (2 popcount(q's bits) - 128),
    popcounts from numpy.unpackbits."""
    rng = np.random.default_rng(seed)
    N, K = 12, 512
    wc = np.zeros((256, 4), np.float16)
    wi = rng.integers(0, 256, size=(N, K // 4)).astype(np.uint8)
    signs = rng.integers(0, 256, size=(N, K // 8)).astype(np.uint8)
    alpha = rng.choice([0.25, 0.5, 1.0, 2.0, -0.5], size=(N, K // 128)).astype(np.float16)
    x = np.ones((1, K), np.float16)
    pc = np.unpackbits(signs, axis=1).reshape(N, K // 128, 128).sum(axis=2)
    ref = (alpha.astype(np.float64) * (2.0 * pc - 128)).sum(axis=1)
    y = orc.linear(wc, wi, x, signs=signs, alpha=alpha, residual_group=128)
    assert np.array_equal(y[0], ref)


def pin_residual_unit_inputs(orc, seed=8):
    """x = e_k: y[o] = alpha[o][k // 128] * sigma[o][k], sigma from
    numpy.unpackbits(bitorder='little')."""
    rng = np.random.default_rng(seed)
    N, K = 6, 256
    wc = np.zeros((256, 4), np.float16)
    wi = rng.integers(0, 256, size=(N, K // 4)).astype(np.uint8)
    signs = rng.integers(0, 256, size=(N, K // 8)).astype(np.uint8)
    alpha = rng.choice([0.25, 0.5, 1.0, 3.0], size=(N, K // 128)).astype(np.float16)
    sigma = 2.0 * np.unpackbits(signs, axis=1, bitorder="little") - 1.0
    ks = [0, 1, 7, 8, 127, 128, 200, 255]
    x = np.zeros((len(ks), K), np.float16)
    x[np.arange(len(ks)), ks] = 1.0
    y = orc.linear(wc, wi, x, signs=signs, alpha=alpha, residual_group=128)
    for t, k in enumerate(ks):
        assert np.array_equal(y[t], alpha[:, k // 128].astype(np.float64) * sigma[:, k]), k


def pin_hadamard_orthogonal(orc, seed=9):
    """Columns x~(e_i) form Q^T; Q^T Q = I and the rotation keeps norms."""
    rng = np.random.default_rng(seed)
    b, K = 32, 96
    s = (rng.integers(0, 2, K) * 2 - 1).astype(np.int8)
    E = np.eye(K, dtype=np.float16)
    QT = orc.hadamard(E, s, b).T
    assert np.allclose(QT @ QT.T, np.eye(K), atol=1e-12)
    x = rng.normal(size=(3, K)).astype(np.float16)
    xr = orc.hadamard(x, s, b)
    assert np.allclose(np.linalg.norm(xr, axis=1), np.linalg.norm(x.astype(np.float64), axis=1), rtol=1e-12)
    e0 = np.zeros((1, K), np.float16)
    e0[0, 0] = 1
    r0 = orc.hadamard(e0, s, b)[0]
    ref = np.zeros(K)
    ref[:b] = s[:b] / np.sqrt(b)
    assert np.allclose(r0, ref, atol=1e-15)


# ------------------------------------------------------ invariants

def pin_lookup_identity(orc, seed=10):
    """The output-codebook form equals the dequantised product (double)."""
    rng = np.random.default_rng(seed)
    cases = [dict(N=16, K=64), dict(N=16, K=256, codebook_rows=8),
             dict(N=8, K=256, residual_group=128, hadamard_block=64)]
    for c in cases:
        N, K = c["N"], c["K"]
        G = N // c.get("codebook_rows", N) if c.get("codebook_rows") else 1
        wc = rng.normal(0, 0.02, size=(G, 256, 4)).astype(np.float16)
        wi = rng.integers(0, 256, size=(N, K // 4)).astype(np.uint8)
        kw = dict(codebook_rows=c.get("codebook_rows", 0))
        if c.get("residual_group"):
            kw.update(signs=rng.integers(0, 256, size=(N, K // 8)).astype(np.uint8),
                      alpha=rng.uniform(0.001, 0.01, size=(N, K // 128)).astype(np.float16),
                      residual_group=128)
        if c.get("hadamard_block"):
            kw.update(hsign=(rng.integers(0, 2, K) * 2 - 1).astype(np.int8),
                      hadamard_block=c["hadamard_block"])
        x = rng.normal(size=(3, K)).astype(np.float16)
        y = orc.linear(wc, wi, x, **kw)
        yl, absy = orc.lookup_form(wc, wi, x, **kw)
        assert np.all(np.abs(y - yl) <= 1e-12 * absy + 1e-300), np.abs(y - yl).max()


def pin_batch_rows(orc, seed=11):
    """A batch of B tokens gives the B single-token results."""
    rng = np.random.default_rng(seed)
    N, K = 10, 128
    wc = rng.normal(0, 0.02, size=(256, 4)).astype(np.float16)
    wi = rng.integers(0, 256, size=(N, K // 4)).astype(np.uint8)
    x = rng.normal(size=(4, K)).astype(np.float16)
    y = orc.linear(wc, wi, x)
    for t in range(4):
        assert np.array_equal(y[t], orc.linear(wc, wi, x[t:t + 1])[0])


def pin_optimal_alpha(orc, seed=12):
    """Closed form mean|r|, and any other alpha gives a larger residual."""
    rng = np.random.default_rng(seed)
    r = rng.normal(size=(5, 256))
    a = orc.optimal_alpha(r, 128)
    ref = np.abs(r).reshape(5, 2, 128).mean(axis=2)
    assert np.allclose(a, ref, rtol=1e-14)
    s = np.where(r >= 0, 1.0, -1.0)
    loss = lambda al: ((r - np.repeat(al, 128, axis=1) * s) ** 2).sum()
    base = loss(a)
    for eps in (1e-3, -1e-3, 0.05):
        assert loss(a + eps) > base


# ------------------------------------------------------------- quantizer

def pin_kmeans_assign_scipy(orc, seed=13):
    """Nearest-centroid indices against scipy.cluster.vq.vq, one shared and two
    per-group codebooks; a duplicated centroid never wins over its first copy."""
    import scipy.cluster.vq
    rng = np.random.default_rng(seed)
    v = rng.normal(size=(6000, 4)).astype(np.float32)
    c = rng.normal(size=(64, 4)).astype(np.float32)
    ref, _ = scipy.cluster.vq.vq(v, c)
    assert np.array_equal(orc.kmeans_assign(v, c), ref)
    c2 = rng.normal(size=(2, 64, 4)).astype(np.float32)
    got = orc.kmeans_assign(v, c2, vecs_per_cb=3000)
    assert np.array_equal(got[:3000], scipy.cluster.vq.vq(v[:3000], c2[0])[0])
    assert np.array_equal(got[3000:], scipy.cluster.vq.vq(v[3000:], c2[1])[0])
    cd = np.concatenate([c, c[:8]])                # centroids 64..71 repeat 0..7
    assert orc.kmeans_assign(v, cd).max() < 64


def pin_kmeans_sklearn(orc, seed=14):
    """Lloyd iterations from the same start agree with scikit-learn's KMeans on
    well-separated blobs (labels exactly, centroids to float rounding)."""
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(seed)
    centres = rng.uniform(-8, 8, size=(24, 4))
    lab = rng.integers(0, 24, size=4000)
    v = (centres[lab] + rng.normal(0, 0.6, size=(4000, 4))).astype(np.float32)
    init = (centres + rng.normal(0, 0.8, size=centres.shape)).astype(np.float32)
    cent = init[None]
    for _ in range(6):
        idx = orc.kmeans_assign(v, cent)
        cent, counts = orc.kmeans_update(v, idx, cent)
    assert counts.min() > 0
    km = KMeans(n_clusters=24, init=init, n_init=1, max_iter=6, tol=0.0, algorithm="lloyd").fit(v)
    assert np.allclose(cent[0], km.cluster_centers_, rtol=1e-5, atol=1e-5)
    assert np.array_equal(orc.kmeans_assign(v, cent), km.predict(v))


def pin_quantize_exact_recovery(orc, seed=15):
    """A weight that IS a codebook reconstruction (fp16-exact, well-separated
    centroids) comes back exactly: same codebook and pointers, zero residual
    (every sign bit set: a zero residual counts as +1) and zero alpha.  A
    centroid no vector is near keeps its start value."""
    rng = np.random.default_rng(seed)
    ncent, N, K = 16, 32, 256
    wc_true = (rng.integers(-6, 7, size=(ncent, 4)) * 0.25).astype(np.float16)
    wc_true[:, 0] = np.arange(ncent) * 0.5          # rows distinct, far apart
    wi_true = rng.integers(0, ncent - 1, size=(N, K // 4)).astype(np.uint8)   # last centroid unused
    w = wc_true[wi_true].reshape(N, K)
    init = wc_true.astype(np.float32) + rng.uniform(-0.05, 0.05, size=wc_true.shape).astype(np.float32)
    init[-1] = [100, 100, 100, 100]
    wc, wi, signs, alpha, _ = orc.quantize(w, init, iters=3)
    assert np.array_equal(wc[0, :-1], wc_true[:-1])
    assert np.array_equal(wc[0, -1].astype(np.float32), init[-1])
    assert np.array_equal(wi, wi_true)
    assert np.all(signs == 0xFF) and np.all(alpha == 0)


def pin_quantize_rotation(orc, seed=16):
    """W_rot = W Q pairs with x~ = Q^T x: W_rot x~ = W x (Q orthogonal)."""
    rng = np.random.default_rng(seed)
    N, K, b = 8, 1024, 256
    w = rng.normal(0, 0.5, size=(N, K)).astype(np.float16)
    hs = rng.choice([-1, 1], size=K).astype(np.int8)
    x = rng.normal(size=(1, K)).astype(np.float16)
    init = rng.normal(0, 0.5, size=(256, 4)).astype(np.float32)
    *_, wrot = orc.quantize(w, init, iters=1, hsign=hs, hadamard_block=b)
    lhs = wrot.astype(np.float64) @ orc.hadamard(x, hs, b)[0]
    rhs = w.astype(np.float64) @ x[0].astype(np.float64)
    assert np.allclose(lhs, rhs, rtol=1e-5, atol=1e-4), np.abs(lhs - rhs).max()


def pin_residual_identity(orc, seed=17):
    """Per group, with alpha = mean|r| and the packed signs of r (bits decoded
    by numpy, LSB first): ||r - alpha s||^2 = ||r||^2 - G alpha^2, which holds
    only when s . r = sum |r|; also for per-group codebooks."""
    rng = np.random.default_rng(seed)
    N, K, G = 32, 512, 128
    wrot = rng.normal(0, 0.05, size=(N, K)).astype(np.float32)
    for cbr in (0, 16):
        ncb = N // cbr if cbr else 1
        wc = rng.normal(0, 0.05, size=(ncb, 256, 4)).astype(np.float16)
        wi = rng.integers(0, 256, size=(N, K // 4)).astype(np.uint8)
        signs, alpha = orc.residual(wrot, wc, wi, codebook_rows=cbr, group=G)
        g = (np.arange(N) // cbr) if cbr else np.zeros(N, int)
        rec = wc.astype(np.float64)[g[:, None], wi].reshape(N, K)
        r = wrot.astype(np.float64) - rec
        s = np.unpackbits(signs, axis=1, bitorder="little").astype(np.float64) * 2 - 1
        a = np.repeat(alpha, G, axis=1)
        lhs = ((r - a * s) ** 2).reshape(N, K // G, G).sum(axis=2)
        rhs = (r ** 2).reshape(N, K // G, G).sum(axis=2) - G * alpha ** 2
        assert np.allclose(lhs, rhs, rtol=1e-6, atol=1e-12), np.abs(lhs - rhs).max()
        assert np.all(alpha >= 0)


# ------------------------------------------------- order-K (Paley) rotation

def _rotation_matrix(orc, b):
    """M = H_b / sqrt(b), read off the oracle's rotation of unit vectors:
    rotating e_j gives H_b^T e_j / sqrt(b) = row j of M."""
    eye = np.eye(b, dtype=np.float16)
    return orc.hadamard(eye, np.ones(b, np.int8), b)


def _gf27_squares():
    """Nonzero squares of GF(27) = GF(3)[t] / (t^3 + 2t + 2), by enumeration;
    element c0 + 3 c1 + 9 c2 is c0 + c1 t + c2 t^2."""
    def mul(a, b):
        x = [(a // 3 ** i) % 3 for i in range(3)]
        y = [(b // 3 ** i) % 3 for i in range(3)]
        z = np.convolve(x, y) % 3                       # degree <= 4
        for d in (4, 3):                                # t^3 = -2t - 2 = t + 1 (mod 3)
            c, z[d] = z[d], 0
            z[d - 3] = (z[d - 3] + c) % 3
            z[d - 2] = (z[d - 2] + c) % 3
        return int(z[0] + 3 * z[1] + 9 * z[2])
    return {mul(a, a) for a in range(1, 27)}


def pin_paley_hadamard(orc):
    """Order 28: entries +-1, H H^T = 28 I, skew (H + H^T = 2 I); the interior
    is the quadratic character of GF(27) (squares found by enumeration)."""
    H = np.rint(_rotation_matrix(orc, 28) * np.sqrt(28)).astype(int)
    assert set(np.unique(H)) == {-1, 1}
    assert np.array_equal(H @ H.T, 28 * np.eye(28, dtype=int))
    assert np.array_equal(H + H.T, 2 * np.eye(28, dtype=int))
    assert np.all(H[0] == 1) and np.all(H[1:, 0] == -1)
    sq = _gf27_squares()
    assert len(sq) == 13
    def sub(a, b):
        return sum((((a // 3 ** i) - (b // 3 ** i)) % 3) * 3 ** i for i in range(3))
    for i in range(1, 28):
        for j in range(1, 28):
            if i != j:
                assert H[i, j] == (1 if sub(i - 1, j - 1) in sq else -1), (i, j)


def pin_paley_kronecker(orc):
    """H_56 = H_28 (x) H_2 and H_224 = H_28 (x) H_8 (scipy's Sylvester
    matrices), orthonormal after scaling."""
    H28 = _rotation_matrix(orc, 28) * np.sqrt(28)
    for m in (2, 8):
        M = _rotation_matrix(orc, 28 * m)
        ref = np.kron(H28, scipy.linalg.hadamard(m)) / np.sqrt(28 * m)
        assert np.allclose(M, ref, atol=1e-12)
        assert np.allclose(M @ M.T, np.eye(28 * m), atol=1e-12)


def pin_paley_rotation_pairs(orc, seed=18):
    """With a Paley block the weight rotation W_rot = W Q and the input
    rotation x~ = Q^T x still pair up: W_rot x~ = W x."""
    rng = np.random.default_rng(seed)
    N, K, b = 4, 1792, 1792
    w = rng.normal(0, 0.5, size=(N, K)).astype(np.float16)
    hs = rng.choice([-1, 1], size=K).astype(np.int8)
    x = rng.normal(size=(1, K)).astype(np.float16)
    init = rng.normal(0, 0.5, size=(16, 4)).astype(np.float32)
    *_, wrot = orc.quantize(w, init, iters=0, hsign=hs, hadamard_block=b)
    lhs = wrot.astype(np.float64) @ orc.hadamard(x, hs, b)[0]
    rhs = w.astype(np.float64) @ x[0].astype(np.float64)
    assert np.allclose(lhs, rhs, rtol=1e-5, atol=1e-4), np.abs(lhs - rhs).max()


# ------------------------------------------------- 4-bit (16-centroid) indices

def pin_factorisation_4bit(orc, seed=19):
    """16 centroids, indices packed two per byte (the even sub-vector in the
    low nibble): a dense integer weight rebuilt from its codebook and packed
    by plain integer arithmetic gives W x exactly, in both oracle forms, with
    one shared codebook and with one per 8 rows; and a byte 0x21 holds the
    indices (1, 2) in sub-vector order."""
    rng = np.random.default_rng(seed)
    N, K = 16, 64
    for cbr in (0, 8):
        G = N // cbr if cbr else 1
        wc = rng.integers(-3, 4, size=(G, 16, 4)).astype(np.float16)
        idx = rng.integers(0, 16, size=(N, K // 4))
        g = (np.arange(N) // cbr) if cbr else np.zeros(N, int)
        W = wc.astype(np.float64)[g[:, None], idx].reshape(N, K)
        packed = (idx[:, 0::2] + 16 * idx[:, 1::2]).astype(np.uint8)
        x = rng.integers(-3, 4, size=(2, K)).astype(np.float16)
        ref = x.astype(np.float64) @ W.T
        assert np.array_equal(orc.linear(wc, packed, x, codebook_rows=cbr, index_bits=4), ref)
        yl, _ = orc.lookup_form(wc, packed, x, codebook_rows=cbr, index_bits=4)
        assert np.array_equal(yl, ref)
    wc = np.zeros((16, 4), np.float16)
    wc[1] = [1, 0, 0, 0]
    wc[2] = [0, 0, 0, 10]
    x = np.arange(1, 9, dtype=np.float16)[None]          # K = 8: two sub-vectors
    y = orc.linear(wc, np.array([[0x21]], np.uint8), x, index_bits=4)
    assert y[0, 0] == 1 * 1 + 10 * 8                     # sub-vector 0 -> centroid 1, 1 -> 2


ALL_PINS = [
    pin_golden_vq, pin_golden_residual, pin_golden_hadamard, pin_f16_decode,
    pin_hadamard_scipy, pin_factorisation, pin_factorisation_residual, pin_rotation_composite,
    pin_unit_centroids, pin_all_equal_indices, pin_group_scaling, pin_residual_popcount,
    pin_residual_unit_inputs, pin_hadamard_orthogonal, pin_lookup_identity, pin_batch_rows,
    pin_optimal_alpha, pin_kmeans_assign_scipy, pin_kmeans_sklearn, pin_quantize_exact_recovery,
    pin_quantize_rotation, pin_residual_identity, pin_paley_hadamard, pin_paley_kronecker,
    pin_paley_rotation_pairs, pin_factorisation_4bit,
]
