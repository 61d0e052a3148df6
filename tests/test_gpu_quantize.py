"""The offline quantizer on the GPU (eva_vq_quantize and its K-means and
residual steps) against the oracle, through the C ABI.

Decisions (nearest centroid, sign bits) are bit-exact: both sides take them
in fp32 with the same summation order.  Centroid means (double sums, one
rounding to fp32) agree to a float ulp, alpha (double sums, fp16) to an fp16
ulp.  The whole pipeline is checked step against step on the GPU's own
intermediate values (rotated rows, centroids), plus properties that hold at
any size: the K-means objective falls, the residual lowers the error, and the
quantized layer runs through the lookup path like any other layer.
"""
import time

import numpy as np
import pytest

import oracle
from tests.conftest import cuda_available
from tests.gpu_helpers import TOL, norm_rel_err
from vector_quantized_weight_b200 import synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


def _cuda(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _stream():
    from vector_quantized_weight_b200 import eva_vq
    return eva_vq._stream_handle(None)


@pytest.mark.parametrize("M,ncent,vpc", [(200_000, 256, 0), (65_536, 256, 16_384), (5_003, 16, 0),
                                          (40_000, 64, 10_000)])
def test_kmeans_assign_bit_exact(M, ncent, vpc):
    import torch
    from vector_quantized_weight_b200 import eva_vq
    rng = np.random.default_rng(M + ncent)
    G = (M + vpc - 1) // vpc if vpc else 1
    v = rng.normal(0, 0.05, size=(M, 4)).astype(np.float32)
    c = rng.normal(0, 0.05, size=(G, ncent, 4)).astype(np.float32)
    c[:, ncent // 2:ncent // 2 + 4] = c[:, :4]                  # duplicated centroids: first copy wins
    k = min(64, ncent)
    v[:k] = c[0, :k]                                            # exact hits (distance 0)
    ref = oracle.kmeans_assign(v, c, vpc)
    vt, ct = _cuda(v), _cuda(c)
    idx = torch.empty(M, dtype=torch.int32, device="cuda")
    eva_vq.eva_vq_kmeans_assign(vt.data_ptr(), M, 4, ct.data_ptr(), ncent, vpc, idx.data_ptr(), _stream())
    assert np.array_equal(idx.cpu().numpy(), ref)


@pytest.mark.parametrize("M,ncent,vpc", [(300_000, 256, 0), (65_536, 256, 8_192), (1_000, 256, 0)])
def test_kmeans_update_matches_oracle(M, ncent, vpc):
    import torch
    from vector_quantized_weight_b200 import eva_vq
    rng = np.random.default_rng(M)
    G = (M + vpc - 1) // vpc if vpc else 1
    v = rng.normal(0, 0.05, size=(M, 4)).astype(np.float32)
    c = rng.normal(0, 0.05, size=(G, ncent, 4)).astype(np.float32)
    idx = oracle.kmeans_assign(v, c, vpc)            # M = 1000 leaves clusters empty
    ref, ref_counts = oracle.kmeans_update(v, idx, c, vpc)
    new = torch.empty((G, ncent, 4), dtype=torch.float32, device="cuda")
    counts = torch.empty((G, ncent), dtype=torch.int64, device="cuda")
    vt, it, ct = _cuda(v), _cuda(idx), _cuda(c)
    eva_vq.eva_vq_kmeans_update(vt.data_ptr(), M, 4, it.data_ptr(), ncent, vpc, ct.data_ptr(), new.data_ptr(),
                                counts.data_ptr(), _stream())
    got = new.cpu().numpy()
    assert np.array_equal(counts.cpu().numpy(), ref_counts)
    assert np.allclose(got, ref, rtol=2e-7, atol=1e-12)
    assert np.mean(got == ref) > 0.999
    empty = ref_counts == 0
    assert np.array_equal(got[empty], c[empty])       # empty clusters keep their centroid


@pytest.mark.parametrize("N,K,cbr,group", [(64, 512, 0, 128), (256, 1024, 128, 128), (48, 96, 16, 32),
                                           (3584, 3584, 0, 128)])
def test_residual_bit_exact(N, K, cbr, group):
    import torch
    from vector_quantized_weight_b200 import eva_vq
    rng = np.random.default_rng(N + K)
    G = N // cbr if cbr else 1
    wrot = rng.normal(0, 0.02, size=(N, K)).astype(np.float32)
    wc = rng.normal(0, 0.02, size=(G, 256, 4)).astype(np.float16)
    wi = rng.integers(0, 256, size=(N, K // 4)).astype(np.uint8)
    wrot[0, :8] = wc[0, wi[0, :2]].reshape(8).astype(np.float32)   # zero residuals count as +1
    signs_ref, alpha_ref = oracle.residual(wrot, wc, wi, codebook_rows=cbr, group=group)
    signs = torch.empty((N, K // 8), dtype=torch.uint8, device="cuda")
    alpha = torch.empty((N, K // group), dtype=torch.float16, device="cuda")
    wt, ct, it = _cuda(wrot), _cuda(wc), _cuda(wi)
    eva_vq.eva_vq_residual(wt.data_ptr(), N, K, ct.data_ptr(), 256, it.data_ptr(), cbr, group, signs.data_ptr(),
                           alpha.data_ptr(), _stream())
    assert np.array_equal(signs.cpu().numpy(), signs_ref)
    assert signs.cpu().numpy()[0, 0] == 0xFF
    got = alpha.cpu().numpy().view(np.uint16).astype(np.int64)
    ref = alpha_ref.astype(np.float16).view(np.uint16).astype(np.int64)
    assert np.abs(got - ref).max() <= 1                 # one fp16 ulp at most
    assert np.mean(got == ref) > 0.999


def _run_quantize(w, hsign, b, cbr, iters, init_index, index_bits=8, residual_group=128):
    import torch
    from vector_quantized_weight_b200 import eva_vq
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    out = eva_vq.quantize(_cuda(w), _cuda(init_index), iters, hsign=None if hsign is None else _cuda(hsign),
                          hadamard_block=b, codebook_rows=cbr, residual_group=residual_group,
                          index_bits=index_bits, keep_wrot=True, keep_centroids=True)
    dt = time.perf_counter() - t0
    return {k: t.cpu().numpy() for k, t in out.items()}, dt


@pytest.mark.parametrize("N,K,b,cbr,iters", [
    (256, 512, 0, 0, 4),              # no rotation, one codebook
    (512, 1024, 256, 128, 3),         # rotation, one codebook per 128 rows
    (3584, 3584, 512, 0, 6),          # Gemma-2-9B-shaped 3.125-bit layer
    (64, 1792, 1792, 0, 3),           # order-K rotation with a Paley factor
])
def test_quantize_pipeline(N, K, b, cbr, iters):
    import torch
    from vector_quantized_weight_b200 import eva_vq
    seed = N + K + b
    w = synth.make_dense_weight(N, K, seed)
    hs = synth.make_hsign(K, seed) if b else None
    J, G = K // 4, (N // cbr if cbr else 1)
    vpc = cbr * J if cbr else 0
    init = synth.kmeans_init_index(vpc or N * J, G, 256, seed)
    out, dt = _run_quantize(w, hs, b, cbr, iters, init)
    print(f"quantize {N}x{K} b={b} cbr={cbr} iters={iters}: {dt * 1e3:.1f} ms")
    wrot = out["wrot"]
    # 1. rotated rows (fp32 fast transform) against the dense double product
    ref_rot = oracle.hadamard(w, hs, b) if b else oracle.f16_to_f64(w)
    assert np.abs(wrot - ref_rot).max() <= 1e-6 * np.abs(ref_rot).max()
    v = wrot.reshape(N * J, 4)
    # 2.-3. the stored codebook is the fp16 rounding of the final centroids, and
    # the pointers are the nearest fp16 centroids, bit-exactly
    assert np.array_equal(out["wc"], out["centroids"].astype(np.float16))
    assert np.array_equal(out["wi"].reshape(-1), oracle.kmeans_assign(v, out["wc"].astype(np.float32), vpc))
    # one more iteration on the GPU = one oracle step from the GPU's centroids
    out2, _ = _run_quantize(w, hs, b, cbr, iters + 1, init)
    assert np.array_equal(out2["wrot"], wrot)
    step, _ = oracle.kmeans_update(v, oracle.kmeans_assign(v, out["centroids"], vpc), out["centroids"], vpc)
    assert np.allclose(out2["centroids"], step, rtol=1e-5, atol=1e-9)
    # the objective falls from the starting centroids
    per = vpc or N * J
    start = np.stack([v[g * per + init[g]] for g in range(G)])
    cb_of = np.arange(N * J) // per

    def mse(c):
        return float(np.mean((v - c[cb_of, oracle.kmeans_assign(v, c, vpc)]) ** 2))
    assert mse(out["centroids"]) < mse(start)
    # 4.-7. signs bit-exact, alpha within an fp16 ulp of the oracle's
    signs_ref, alpha_ref = oracle.residual(wrot, out["wc"], out["wi"], codebook_rows=cbr, group=128)
    assert np.array_equal(out["signs"], signs_ref)
    d16 = np.abs(out["alpha"].view(np.uint16).astype(np.int64) -
                 alpha_ref.astype(np.float16).view(np.uint16).astype(np.int64))
    assert d16.max() <= 1
    # the quantized layer through the lookup path, against the oracle and the dense weight
    x = synth.make_x(K, 2, seed)
    lin = eva_vq.VQLinear(_cuda(out["wc"]), _cuda(out["wi"]), signs=_cuda(out["signs"]), alpha=_cuda(out["alpha"]),
                          hsign=None if hs is None else _cuda(hs), codebook_rows=cbr, residual_group=128,
                          hadamard_block=b, max_batch=2)
    y = lin(_cuda(x)).float().cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    lin.close()
    yq = oracle.linear(out["wc"], out["wi"], x, signs=out["signs"], alpha=out["alpha"], hsign=hs,
                       codebook_rows=cbr, residual_group=128, hadamard_block=b)
    assert np.all(norm_rel_err(y, yq) <= TOL)
    y_dense = x.astype(np.float64) @ w.astype(np.float64).T
    y_vq = oracle.linear(out["wc"], out["wi"], x, hsign=hs, codebook_rows=cbr, hadamard_block=b)
    e_res, e_vq = norm_rel_err(yq, y_dense).max(), norm_rel_err(y_vq, y_dense).max()
    print(f"  error vs dense: VQ only {e_vq:.3f}, with sign residual {e_res:.3f}")
    assert e_res < e_vq < 0.6


def test_quantize_rejects_out_of_range_start():
    from vector_quantized_weight_b200 import eva_vq
    w = synth.make_dense_weight(64, 256, 1)
    init = synth.kmeans_init_index(64 * 64, 1, 256, 1)
    init[0, 5] = 64 * 64                               # one past the last block
    with pytest.raises(eva_vq.EvaError) as ei:
        _run_quantize(w, None, 0, 0, 2, init)
    assert ei.value.status == eva_vq.EVA_ERR_INVALID_ARG


def test_quantize_four_bit_packed():
    """index_bits = 4: 16 centroids per codebook, the pointers packed two per
    byte (the layout the layer takes); unpacked they are the oracle's nearest
    fp16 centroids, the residual follows them, and the quantized layer (one
    codebook per 128 rows, rotation, sign residual) runs through the lookup
    path against the oracle."""
    import torch
    from vector_quantized_weight_b200 import eva_vq
    N, K, b, cbr, iters = 512, 1024, 256, 128, 3
    seed = 4242
    w = synth.make_dense_weight(N, K, seed)
    hs = synth.make_hsign(K, seed)
    J, G = K // 4, N // cbr
    vpc = cbr * J
    init = synth.kmeans_init_index(vpc, G, 16, seed)
    out, _ = _run_quantize(w, hs, b, cbr, iters, init, index_bits=4)
    assert out["wi"].shape == (N, K // 8)
    idx = np.stack([out["wi"] & 15, out["wi"] >> 4], axis=-1).reshape(N, J)
    v = out["wrot"].reshape(N * J, 4)
    assert np.array_equal(idx.reshape(-1), oracle.kmeans_assign(v, out["wc"].astype(np.float32), vpc))
    signs_ref, _ = oracle.residual(out["wrot"], out["wc"], idx.astype(np.uint8), codebook_rows=cbr, group=128)
    assert np.array_equal(out["signs"], signs_ref)
    x = synth.make_x(K, 3, seed)
    lin = eva_vq.VQLinear(_cuda(out["wc"]), _cuda(out["wi"]), signs=_cuda(out["signs"]), alpha=_cuda(out["alpha"]),
                          hsign=_cuda(hs), codebook_rows=cbr, residual_group=128, hadamard_block=b, max_batch=3,
                          index_bits=4)
    y = lin(_cuda(x)).float().cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    lin.close()
    yq = oracle.linear(out["wc"], out["wi"], x, signs=out["signs"], alpha=out["alpha"], hsign=hs, codebook_rows=cbr,
                       residual_group=128, hadamard_block=b, index_bits=4)
    assert np.all(norm_rel_err(y, yq) <= TOL)
