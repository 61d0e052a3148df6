"""Double-precision CPU oracle for the VQ decode linear (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls it.

The arithmetic lives in ``eva_oracle.c`` (plain C, double); this module only
compiles it with gcc and marshals numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "eva_oracle.c")
_LIB = os.path.join(_HERE, "libeva_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile eva_oracle.c into libeva_oracle.so next to it (gcc, -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


class _Desc(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int), ("K", ctypes.c_int), ("d", ctypes.c_int),
                ("ncent", ctypes.c_int), ("index_bits", ctypes.c_int), ("codebook_rows", ctypes.c_int),
                ("residual_group", ctypes.c_int), ("hadamard_block", ctypes.c_int)]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        lib.vq_oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.vq_oracle_f16_to_f64.restype = ctypes.c_double
        lib.vq_oracle_f16_array_to_f64.argtypes = [P, ctypes.c_int64, P]
        lib.vq_oracle_f16_array_to_f64.restype = None
        lib.vq_oracle_hadamard.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
        lib.vq_oracle_hadamard.restype = ctypes.c_int
        lib.vq_oracle_linear.argtypes = [ctypes.POINTER(_Desc), P, P, P, P, P, P,
                                         ctypes.c_int, P, ctypes.c_int]
        lib.vq_oracle_linear.restype = ctypes.c_int
        lib.vq_oracle_lookup_form.argtypes = [ctypes.POINTER(_Desc), P, P, P, P, P, P,
                                              ctypes.c_int, P, P]
        lib.vq_oracle_lookup_form.restype = ctypes.c_int
        lib.vq_oracle_optimal_alpha.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
        lib.vq_oracle_optimal_alpha.restype = ctypes.c_int
        I64 = ctypes.c_int64
        lib.vq_oracle_kmeans_assign.argtypes = [P, I64, ctypes.c_int, P, ctypes.c_int, I64, P]
        lib.vq_oracle_kmeans_assign.restype = ctypes.c_int
        lib.vq_oracle_kmeans_update.argtypes = [P, I64, ctypes.c_int, P, ctypes.c_int, I64, P, P, P]
        lib.vq_oracle_kmeans_update.restype = ctypes.c_int
        lib.vq_oracle_residual.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, ctypes.c_int,
                                           P, ctypes.c_int, ctypes.c_int, P, P]
        lib.vq_oracle_residual.restype = ctypes.c_int
        lib.vq_oracle_max_threads.argtypes = []
        lib.vq_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c16(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float16).view(np.uint16)


def f16_to_f64(h) -> np.ndarray:
    """Decode fp16 values (array of float16 or uint16 bit patterns) into float64."""
    h = np.ascontiguousarray(h)
    bits = h.view(np.uint16) if h.dtype == np.float16 else h.astype(np.uint16)
    bits = np.ascontiguousarray(bits)
    out = np.empty(bits.shape, np.float64)
    _load().vq_oracle_f16_array_to_f64(_ptr(bits), bits.size, _ptr(out))
    return out


def hadamard(x, hsign, b: int) -> np.ndarray:
    """x~ = hsign * (H_b x) / sqrt(b) per block; x fp16 [B][K] -> float64 [B][K]."""
    x16 = _c16(np.atleast_2d(x))
    B, K = x16.shape
    hs = None if hsign is None else np.ascontiguousarray(hsign, dtype=np.int8)
    out = np.empty((B, K), np.float64)
    rc = _load().vq_oracle_hadamard(_ptr(x16), _ptr(hs), B, K, int(b), _ptr(out))
    if rc:
        raise ValueError(f"vq_oracle_hadamard: {rc}")
    return out


def _desc(N, K, d, ncent, codebook_rows, residual_group, hadamard_block, index_bits=8):
    return _Desc(int(N), int(K), int(d), int(ncent), int(index_bits), int(codebook_rows),
                 int(residual_group), int(hadamard_block))


def _prep(wc, wi, signs, alpha, hsign, x, codebook_rows, residual_group, hadamard_block, index_bits=8):
    wc16 = _c16(wc)
    if wc16.ndim == 2:
        wc16 = wc16[None]
    G, ncent, d = wc16.shape
    wi8 = np.ascontiguousarray(wi, dtype=np.uint8)
    N, J = wi8.shape
    if index_bits == 4:            # two indices per byte
        J *= 2
    x16 = _c16(np.atleast_2d(x))
    B, K = x16.shape
    if J * d != K:
        raise ValueError("WI width times d must equal K")
    if (N // codebook_rows if codebook_rows else 1) != G:
        raise ValueError("codebook count does not match codebook_rows")
    sg = None if signs is None else np.ascontiguousarray(signs, dtype=np.uint8)
    al = _c16(alpha)
    hs = None if hsign is None else np.ascontiguousarray(hsign, dtype=np.int8)
    desc = _desc(N, K, d, ncent, codebook_rows, residual_group, hadamard_block, index_bits)
    return desc, wc16, wi8, sg, al, hs, x16, B, N


def linear(wc, wi, x, *, signs=None, alpha=None, hsign=None, codebook_rows=0,
           residual_group=0, hadamard_block=0, nthreads=1, index_bits=8) -> np.ndarray:
    """y [B][N] float64: the dequantised-weight product (the plain definition).
    index_bits = 4: wi is packed two indices per byte ([N][K/8])."""
    desc, wc16, wi8, sg, al, hs, x16, B, N = _prep(
        wc, wi, signs, alpha, hsign, x, codebook_rows, residual_group, hadamard_block, index_bits)
    y = np.empty((B, N), np.float64)
    rc = _load().vq_oracle_linear(ctypes.byref(desc), _ptr(wc16), _ptr(wi8), _ptr(sg), _ptr(al),
                                  _ptr(hs), _ptr(x16), B, _ptr(y), int(nthreads))
    if rc:
        raise ValueError(f"vq_oracle_linear: {rc}")
    return y


def lookup_form(wc, wi, x, *, signs=None, alpha=None, hsign=None, codebook_rows=0,
                residual_group=0, hadamard_block=0, index_bits=8):
    """(y, sum|W x~|) [B][N] float64 via the output-codebook two-step form."""
    desc, wc16, wi8, sg, al, hs, x16, B, N = _prep(
        wc, wi, signs, alpha, hsign, x, codebook_rows, residual_group, hadamard_block, index_bits)
    y = np.empty((B, N), np.float64)
    absy = np.empty((B, N), np.float64)
    rc = _load().vq_oracle_lookup_form(ctypes.byref(desc), _ptr(wc16), _ptr(wi8), _ptr(sg),
                                       _ptr(al), _ptr(hs), _ptr(x16), B, _ptr(y), _ptr(absy))
    if rc:
        raise ValueError(f"vq_oracle_lookup_form: {rc}")
    return y, absy


def optimal_alpha(r, group: int) -> np.ndarray:
    """argmin_alpha ||r - alpha sign(r)||^2 per row and group of `group` columns."""
    r = np.ascontiguousarray(r, dtype=np.float64)
    rows, cols = r.shape
    out = np.empty((rows, cols // group), np.float64)
    rc = _load().vq_oracle_optimal_alpha(_ptr(r), rows, cols, int(group), _ptr(out))
    if rc:
        raise ValueError(f"vq_oracle_optimal_alpha: {rc}")
    return out


def max_threads() -> int:
    return int(_load().vq_oracle_max_threads())


def layer_linear(layer, x, nthreads=1) -> np.ndarray:
    """Oracle output for a synth.LayerData and activations x."""
    s = layer.shape
    return linear(layer.wc, layer.wi, x, signs=layer.signs, alpha=layer.alpha, hsign=layer.hsign,
                  codebook_rows=s.codebook_rows, residual_group=s.residual_group,
                  hadamard_block=s.hadamard_block, nthreads=nthreads, index_bits=s.index_bits)


# ------------------------------------------------------------------ quantizer

def kmeans_assign(v, centroids, vecs_per_cb: int = 0) -> np.ndarray:
    """Nearest centroid (fp32 squared distance, first minimum) of each vector.
    v: [M][d] float32; centroids: [G][ncent][d] (or [ncent][d]) float32 -> int32 [M]."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    c = np.ascontiguousarray(centroids, dtype=np.float32)
    if c.ndim == 2:
        c = c[None]
    M, d = v.shape
    out = np.empty(M, np.int32)
    rc = _load().vq_oracle_kmeans_assign(_ptr(v), M, d, _ptr(c), c.shape[1], int(vecs_per_cb), _ptr(out))
    if rc:
        raise ValueError(f"vq_oracle_kmeans_assign: {rc}")
    return out


def kmeans_update(v, idx, centroids, vecs_per_cb: int = 0):
    """(new centroids float32 [G][ncent][d], counts int64 [G][ncent]): cluster means in double."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    c = np.ascontiguousarray(centroids, dtype=np.float32)
    if c.ndim == 2:
        c = c[None]
    M, d = v.shape
    new = np.empty_like(c)
    counts = np.empty(c.shape[:2], np.int64)
    rc = _load().vq_oracle_kmeans_update(_ptr(v), M, d, _ptr(idx), c.shape[1], int(vecs_per_cb), _ptr(c),
                                         _ptr(new), _ptr(counts))
    if rc:
        raise ValueError(f"vq_oracle_kmeans_update: {rc}")
    return new, counts


def residual(wrot, wc, wi, *, codebook_rows: int = 0, group: int = 128):
    """(packed signs u8 [N][K/8], alpha float64 [N][K/group]) of wrot - wc[wi]."""
    wrot = np.ascontiguousarray(wrot, dtype=np.float32)
    wc16 = _c16(wc)
    if wc16.ndim == 2:
        wc16 = wc16[None]
    _, ncent, d = wc16.shape
    wi8 = np.ascontiguousarray(wi, dtype=np.uint8)
    N, K = wrot.shape
    signs = np.empty((N, K // 8), np.uint8)
    alpha = np.empty((N, K // group), np.float64)
    rc = _load().vq_oracle_residual(_ptr(wrot), N, K, d, _ptr(wc16), ncent, _ptr(wi8), int(codebook_rows),
                                    int(group), _ptr(signs), _ptr(alpha))
    if rc:
        raise ValueError(f"vq_oracle_residual: {rc}")
    return signs, alpha


def quantize(w, init_centroids, iters: int, *, hsign=None, hadamard_block: int = 0, codebook_rows: int = 0,
             group: int = 128, d: int = 4, init_index=None):
    """The 3-bit article's quantize() pipeline, step by step (plain K-means):
    1. W_rot = W Q (rows rotated like x~, dense per-block product, then fp32);
    2. blocks of d along each row; 3. `iters` Lloyd iterations from
    init_centroids [G][ncent][d]; the codebook is stored in fp16 and the
    pointers are the nearest fp16 centroids; 4.-7. residual, signs (packed),
    alpha = mean |r| per group (rounded to fp16).
    Returns (wc fp16 [G][ncent][d], wi u8 [N][K/d], signs u8 [N][K/8], alpha fp16 [N][K/group],
    wrot float32 [N][K])."""
    w16 = np.ascontiguousarray(w, dtype=np.float16)
    N, K = w16.shape
    if hadamard_block:
        wrot = hadamard(w16, hsign, hadamard_block).astype(np.float32)
    else:
        wrot = f16_to_f64(w16).astype(np.float32)
    v = wrot.reshape(N * (K // d), d)
    vecs_per_cb = codebook_rows * (K // d) if codebook_rows else 0
    if init_index is not None:      # starting centroids = chosen blocks of each codebook's rows
        ii = np.asarray(init_index, dtype=np.int64)
        per = vecs_per_cb or v.shape[0]
        cent = np.stack([v[g * per + ii[g]] for g in range(ii.shape[0])]).astype(np.float32)
    else:
        cent = np.ascontiguousarray(init_centroids, dtype=np.float32)
    if cent.ndim == 2:
        cent = cent[None]
    for _ in range(int(iters)):
        idx = kmeans_assign(v, cent, vecs_per_cb)
        cent, _counts = kmeans_update(v, idx, cent, vecs_per_cb)
    wc = cent.astype(np.float16)
    idx = kmeans_assign(v, wc.astype(np.float32), vecs_per_cb)
    wi = idx.astype(np.uint8).reshape(N, K // d)
    signs, alpha = residual(wrot, wc, wi, codebook_rows=codebook_rows, group=group)
    return wc, wi, signs, alpha.astype(np.float16), wrot
