"""Shared helpers of the GPU parity tests: run a layer through the C ABI and
compute the oracle on all rows or on a sample of rows."""
from __future__ import annotations

import numpy as np

import oracle

# Spec tolerance: per batch row, max_o |y - y*| / max_o |y*| <= 2e-3
# (fp32 accumulation against the fp64 oracle; norm-relative because the
# per-element relative error is unbounded where y* crosses zero).
TOL = 2e-3


def sub_layer_oracle(layer, x, rows, nthreads=8):
    """Oracle outputs for the given output rows only: the rows' indices,
    signs and alpha, each row with its own codebook (codebook_rows = 1)."""
    s = layer.shape
    rows = np.asarray(rows)
    wi = layer.wi[rows]
    if s.codebook_rows:
        wc = layer.wc[rows // s.codebook_rows]
        cbr = 1
    else:
        wc = layer.wc
        cbr = 0
    signs = None if layer.signs is None else layer.signs[rows]
    alpha = None if layer.alpha is None else layer.alpha[rows]
    return oracle.linear(wc, wi, x, signs=signs, alpha=alpha, hsign=layer.hsign, codebook_rows=cbr,
                         residual_group=s.residual_group, hadamard_block=s.hadamard_block,
                         nthreads=nthreads, index_bits=s.index_bits)


def sample_rows(N, codebook_rows=0, n=256, seed=0):
    rng = np.random.default_rng(seed)
    picks = set(range(min(32, N))) | set(range(max(0, N - 32), N))
    if codebook_rows:
        for b in range(codebook_rows, N, codebook_rows * max(1, N // codebook_rows // 8)):
            picks |= {b - 1, b}
    picks |= set(rng.integers(0, N, size=min(n, N)).tolist())
    return np.array(sorted(p for p in picks if 0 <= p < N))


def norm_rel_err(y, ref):
    """Per batch row: max |y - ref| / max |ref|."""
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.maximum(np.abs(ref).max(axis=1), 1e-30)
    return np.abs(y - ref).max(axis=1) / den


def run_gpu(layer, x, *, out_dtype="float16", path=0, max_batch=None, independent=False):
    """One call through the C ABI; independent=True takes the EVA_RUN_INDEPENDENT
    launch (its own grid) that the benchmark times."""
    import torch
    from vector_quantized_weight_b200 import eva_vq
    B = x.shape[0]
    lin = eva_vq.from_layer(layer, max_batch=max_batch or B, out_dtype=out_dtype, path=path)
    xt = torch.from_numpy(x).cuda()
    y = lin(xt, independent=independent)
    torch.cuda.synchronize()
    out = y.float().cpu().numpy().astype(np.float64)
    # no bounded device wait gave up (and, in the bounds-checked build, no
    # access fell outside its buffer)
    assert eva_vq.eva_vq_sync_status(lin.handle) == eva_vq.EVA_OK
    lin.close()
    return out
