"""CUDA path against the double-precision oracle, through the C ABI.

Every configuration of the decode workloads (tiny, Llama-2-7B layer and
block at batch 1/4/16, Gemma-2-9B-shaped 3.125-bit layers, Llama-2-70B-shaped
layers with one codebook per 128 rows at batch 1/8/32) runs at full size in
both launch configurations: the plain call and the independent call (its
own grid); every output row is compared with the oracle (fp64, OpenMP over
rows on all host cores).  Indices are checked bit-exactly,
integer-valued problems exactly, everything else within the norm-relative
tolerance TOL.
"""
import os

import numpy as np
import pytest

import oracle
from tests.conftest import cuda_available
from tests.gpu_helpers import TOL, norm_rel_err, run_gpu

NTHREADS = os.cpu_count() or 8
from vector_quantized_weight_b200 import synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


def _layers_and_batches():
    out = []
    for key, cfg in synth.CONFIGS.items():
        for li, shape in enumerate(cfg.layers):
            for B in cfg.batches:
                out.append(pytest.param(key, li, B, id=f"{key}-{shape.name}-B{B}"))
    return out


@pytest.mark.parametrize("key,li,B", _layers_and_batches())
def test_config_parity(key, li, B):
    cfg = synth.CONFIGS[key]
    shape = cfg.layers[li]
    seed = synth.layer_seed(cfg.index, li)
    layer = synth.make_layer(shape, seed)
    x = synth.make_x(shape.K, B, seed)
    ref = oracle.layer_linear(layer, x, nthreads=NTHREADS)       # every output row
    for independent in (False, True):
        y = run_gpu(layer, x, independent=independent)
        err = norm_rel_err(y, ref)
        assert np.all(err <= TOL), (independent, err.max(), TOL)


@pytest.mark.parametrize("N,K,pattern", [
    (256, 512, "random"), (4096, 4096, "random"), (100, 300, "ramp"), (17, 260, "rowcol"),
    (11008, 4096, "a5"), (4096, 11008, "ones"), (48, 1024, "zeros"), (3584, 14336, "random"),
])
def test_index_roundtrip_bit_exact(N, K, pattern):
    import torch
    from vector_quantized_weight_b200 import eva_vq
    wi = synth.adversarial_wi(N, K // 4, pattern, seed=N + K)
    wc = torch.zeros((1, 256, 4), dtype=torch.float16, device="cuda")
    lin = eva_vq.VQLinear(wc, torch.from_numpy(wi).cuda())
    back = lin.unpack_indices().cpu().numpy()
    torch.cuda.synchronize()
    lin.close()
    assert np.array_equal(back, wi)


@pytest.mark.parametrize("B", [1, 2, 3, 4, 8, 9, 16, 17])
@pytest.mark.parametrize("N,K,cbr", [(256, 512, 0), (128, 1024, 16), (40, 264, 0)])
def test_integer_inputs_exact(N, K, cbr, B):
    """Small-integer codebooks and inputs: every product and sum is exact in
    fp16 / fp32, so the GPU must reproduce the oracle exactly (B >= 3, or
    B >= 2 with per-group codebooks, takes the dequantize path, smaller B the
    lookup path)."""
    rng = np.random.default_rng(N + K + B)
    G = N // cbr if cbr else 1
    layer = synth.LayerData(synth.LayerShape("int", N, K, codebook_rows=cbr),
                            rng.integers(-2, 3, size=(G, 256, 4)).astype(np.float16),
                            rng.integers(0, 256, size=(N, K // 4)).astype(np.uint8), None, None, None)
    x = rng.integers(-3, 4, size=(B, K)).astype(np.float16)
    y = run_gpu(layer, x, out_dtype="float32")
    ref = oracle.layer_linear(layer, x)
    assert np.array_equal(y, ref)


@pytest.mark.parametrize("N,K,B,cbr,resid,had", [
    (17, 260, 1, 0, 0, 0),          # ragged rows and a partial last K-slice
    (100, 132, 2, 0, 0, 0),
    (33, 384, 3, 0, 128, 0),        # odd batch, residual without rotation
    (64, 640, 1, 0, 128, 128),      # rotation block 128, residual
    (272, 1024, 5, 16, 0, 0),       # 17 codebooks of 16 rows, odd batch
    (3584, 3584, 1, 0, 128, 512),   # Gemma block structure
    (8, 8192, 64, 0, 0, 0),         # maximum batch
    (64, 1792, 3, 0, 128, 1792),    # order-28 Paley (x) Sylvester 64 rotation, token pairs
    (32, 7168, 2, 0, 128, 7168),    # Paley (x) Sylvester 256: partial sums per warp
    (48, 3584, 1, 0, 0, 1792),      # two Paley blocks, no residual
])
def test_edge_cases(N, K, B, cbr, resid, had):
    shape = synth.LayerShape("edge", N, K, codebook_rows=cbr, residual_group=resid, hadamard_block=had)
    layer = synth.make_layer(shape, 1234 + N, alpha_signed=True)
    x = synth.make_x(K, B, 99)
    for dt in ("float16", "float32"):
        y = run_gpu(layer, x, out_dtype=dt)
        ref = oracle.layer_linear(layer, x, nthreads=8)
        err = norm_rel_err(y, ref)
        assert np.all(err <= TOL), (dt, err.max())


def test_residual_only_changes_with_signs():
    """Flipping every sign bit of one row changes only that row, by
    -2 * sum_q alpha_q sum_k sigma_k x~_k (twice its residual)."""
    shape = synth.LayerShape("flip", 64, 512, residual_group=128)
    layer = synth.make_layer(shape, 77)
    x = synth.make_x(512, 1, 5)
    y0 = run_gpu(layer, x, out_dtype="float32")
    layer.signs[5] ^= 0xFF
    y1 = run_gpu(layer, x, out_dtype="float32")
    diff = np.abs(y1 - y0)[0]
    assert diff[5] > 0 and np.all(np.delete(diff, 5) == 0)


def test_deterministic_and_host_path():
    import torch
    from vector_quantized_weight_b200 import eva_vq
    shape = synth.CONFIGS["llama7b_layer"].layers[0]
    layer = synth.make_layer(shape, 5)
    x = synth.make_x(shape.K, 1, 5)
    lin = eva_vq.from_layer(layer, max_batch=1)
    xt = torch.from_numpy(x).cuda()
    y1 = lin(xt).cpu()
    y2 = lin(xt).cpu()
    assert torch.equal(y1, y2)
    xh = torch.from_numpy(x).pin_memory()
    yh = torch.empty((1, shape.N), dtype=torch.float16).pin_memory()
    lin.run_host(xh, yh)
    assert torch.equal(yh, y1)
    assert eva_vq.eva_vq_sync_status(lin.handle) == eva_vq.EVA_OK
    lin.close()


def test_run_rejects_bad_arguments():
    import ctypes
    import torch
    from vector_quantized_weight_b200 import eva_vq
    shape = synth.LayerShape("err", 64, 256)
    layer = synth.make_layer(shape, 3)
    lin = eva_vq.from_layer(layer, max_batch=2)
    lib = eva_vq.load()
    x = torch.zeros((4, 256), dtype=torch.float16, device="cuda")
    y = torch.zeros((4, 64), dtype=torch.float16, device="cuda")
    h = lin.handle
    assert lib.eva_vq_linear_run(h, x.data_ptr(), 0, y.data_ptr(), None) == eva_vq.EVA_ERR_INVALID_ARG
    assert lib.eva_vq_linear_run(h, x.data_ptr(), 3, y.data_ptr(), None) == eva_vq.EVA_ERR_INVALID_ARG
    assert lib.eva_vq_linear_run(h, x.data_ptr() + 2, 1, y.data_ptr(), None) == eva_vq.EVA_ERR_INVALID_ARG
    assert lib.eva_vq_linear_run(h, None, 1, y.data_ptr(), None) == eva_vq.EVA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    lin.close()


@pytest.mark.parametrize("key,li,B", [("llama7b_layer", 0, 1), ("llama7b_layer", 0, 2), ("llama7b_block", 4, 1),
                                      ("llama7b_block", 6, 1), ("llama7b_block", 6, 4), ("gemma_3bit", 0, 1),
                                      ("gemma_3bit", 1, 1), ("gemma_3bit_rotK", 0, 1), ("gemma_3bit_rotK", 0, 2),
                                      ("llama70b", 0, 1), ("llama70b", 0, 8), ("llama7b_layer_4bit", 0, 1)])
def test_independent_flag_matches_plain_run(key, li, B):
    """EVA_RUN_INDEPENDENT relaxes ordering and takes its own grid (fewer,
    longer CTAs and smaller clusters, so another fp32 summation order over
    the K-slices): back-to-back calls on one handle (distinct y) each match
    the oracle on every row and the plain call within the tolerance, and
    repeat bitwise."""
    import torch
    from vector_quantized_weight_b200 import eva_vq
    cfg = synth.CONFIGS[key]
    shape = cfg.layers[li]
    layer = synth.make_layer(shape, 31)
    lin = eva_vq.from_layer(layer, max_batch=B)
    xs_np = [synth.make_x(shape.K, B, 40 + i) for i in range(3)]
    xs = [torch.from_numpy(x).cuda() for x in xs_np]
    ref = [lin(x).clone() for x in xs]
    plain_grid = lin.info().grid
    outs = [lin(x, independent=True).clone() for x in xs]      # back to back, same handle
    again = [lin(x, independent=True) for x in xs]
    torch.cuda.synchronize()
    assert 0 < lin.info().grid <= plain_grid                   # never more CTAs than the plain call
    for x, a, b, c in zip(xs_np, ref, outs, again):
        assert torch.equal(b, c)
        yi = b.float().cpu().numpy().astype(np.float64)
        assert np.all(norm_rel_err(yi, a.float().cpu().numpy()) <= TOL)
        assert np.all(norm_rel_err(yi, oracle.layer_linear(layer, x, nthreads=NTHREADS)) <= TOL)
    lib = eva_vq.load()
    y = torch.empty_like(ref[0])
    assert lib.eva_vq_linear_run_ex(lin.handle, xs[0].data_ptr(), B, y.data_ptr(), None, 2) == \
        eva_vq.EVA_ERR_INVALID_ARG
    lin.close()


@pytest.mark.parametrize("key,li,B", [("llama7b_layer", 0, 1), ("llama7b_layer", 0, 2), ("llama7b_block", 4, 4),
                                      ("llama70b", 0, 8), ("tiny", 0, 1)])
def test_both_paths_match_the_oracle(key, li, B):
    """The lookup path and the dequantize path each meet the tolerance at any
    batch size; the handle reports which one ran."""
    import torch
    from vector_quantized_weight_b200 import eva_vq
    cfg = synth.CONFIGS[key]
    shape = cfg.layers[li]
    seed = synth.layer_seed(cfg.index, li)
    layer = synth.make_layer(shape, seed)
    x = synth.make_x(shape.K, B, seed)
    ref = oracle.layer_linear(layer, x, nthreads=NTHREADS)
    for path in (eva_vq.EVA_PATH_OC_LOOKUP, eva_vq.EVA_PATH_DEQUANT_MMA):
        lin = eva_vq.from_layer(layer, max_batch=B, path=path)
        y = lin(torch.from_numpy(x).cuda()).float().cpu().numpy()
        torch.cuda.synchronize()
        assert lin.info().path == path
        assert eva_vq.eva_vq_sync_status(lin.handle) == eva_vq.EVA_OK
        lin.close()
        err = norm_rel_err(y, ref)
        assert np.all(err <= TOL), (path, err.max())


@pytest.mark.parametrize("N,K,cbr,B", [(8192, 8192, 128, 20), (4096, 4096, 0, 24), (8192, 8192, 128, 1),
                                       (2064, 8192, 16, 9)])
def test_dequant_path_large_layers(N, K, cbr, B):
    """Layers whose index units do not all fit in shared memory next to the
    rest of the dequantize kernel's footprint: the units past the staged ones
    stream from global memory.  Two passes of 16 tokens, one token, and a
    ragged row count with 16-row codebooks: every row against the oracle, and
    a second call bitwise equal."""
    import torch
    from vector_quantized_weight_b200 import eva_vq
    shape = synth.LayerShape("ring", N, K, codebook_rows=cbr)
    layer = synth.make_layer(shape, 900 + B)
    x = synth.make_x(K, B, 901 + B)
    lin = eva_vq.from_layer(layer, max_batch=B, path=eva_vq.EVA_PATH_DEQUANT_MMA)
    y = lin(torch.from_numpy(x).cuda())
    again = lin(torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    assert lin.info().path == eva_vq.EVA_PATH_DEQUANT_MMA
    assert eva_vq.eva_vq_sync_status(lin.handle) == eva_vq.EVA_OK
    assert torch.equal(y, again)
    lin.close()
    err = norm_rel_err(y.float().cpu().numpy(), oracle.layer_linear(layer, x, nthreads=NTHREADS))
    assert np.all(err <= TOL), err.max()


@pytest.mark.parametrize("N,K,cbr", [(4096, 4096, 0), (1040, 2048, 0), (2048, 4096, 128)])
def test_dequant_path_ragged_batches(N, K, cbr):
    """The dequantize path at batch sizes that leave token groups partly empty
    (5, 9, 13 tokens) and a second pass partly empty (31): every row against
    the oracle, for one-slice CTAs (4096 x 4096), several slices per CTA and a
    ragged row count, and per-group codebooks."""
    import torch
    from vector_quantized_weight_b200 import eva_vq
    shape = synth.LayerShape("rag", N, K, codebook_rows=cbr)
    layer = synth.make_layer(shape, 4100 + N)
    lin = eva_vq.from_layer(layer, max_batch=31, path=eva_vq.EVA_PATH_DEQUANT_MMA)
    for B in (5, 9, 13, 31):
        x = synth.make_x(K, B, 4200 + B)
        y = lin(torch.from_numpy(x).cuda()).float().cpu().numpy()
        torch.cuda.synchronize()
        assert lin.info().path == eva_vq.EVA_PATH_DEQUANT_MMA
        err = norm_rel_err(y, oracle.layer_linear(layer, x, nthreads=NTHREADS))
        assert np.all(err <= TOL), (B, err.max())
    assert eva_vq.eva_vq_sync_status(lin.handle) == eva_vq.EVA_OK
    lin.close()


@pytest.mark.parametrize("shape,Bs", [
    (synth.LayerShape("gemma", 3584, 3584, residual_group=128, hadamard_block=512), (4, 9)),
    (synth.LayerShape("gemma_down", 3584, 14336, residual_group=128, hadamard_block=2048), (3,)),
    (synth.LayerShape("gemma_rotK", 3584, 3584, residual_group=128, hadamard_block=3584), (2, 16)),
    (synth.LayerShape("resid_only", 384, 1024, residual_group=128), (5, 17)),
    (synth.LayerShape("ragged", 200, 1152, residual_group=128, hadamard_block=64), (6,)),
    (synth.LayerShape("rot_only", 136, 520, hadamard_block=8), (3, 11)),
    (synth.LayerShape("syl4096", 256, 8192, residual_group=128, hadamard_block=4096), (3, 12)),
    (synth.LayerShape("syl1024", 512, 4096, residual_group=128, hadamard_block=1024), (5, 13)),
    (synth.LayerShape("syl256", 128, 768, hadamard_block=256), (4,)),
])
def test_dequant_path_with_residual_and_rotation(shape, Bs):
    """The dequantize path carries the 1-bit sign residual (signed alpha
    included) and the rotated input: Sylvester blocks of 64 to 4096 rotated
    on chip with the residual where a CTA takes one slice, through the
    rotation kernel otherwise, without the residual (8, 256) and for an
    order-K Paley block; K ranges ending mid-slice; every row against the
    oracle, the status word clean."""
    import torch
    from vector_quantized_weight_b200 import eva_vq
    layer = synth.make_layer(shape, 7100 + shape.N, alpha_signed=True)
    lin = eva_vq.from_layer(layer, max_batch=max(Bs), path=eva_vq.EVA_PATH_DEQUANT_MMA)
    for B in Bs:
        x = synth.make_x(shape.K, B, 7200 + B)
        y = lin(torch.from_numpy(x).cuda()).float().cpu().numpy()
        torch.cuda.synchronize()
        assert lin.info().path == eva_vq.EVA_PATH_DEQUANT_MMA
        err = norm_rel_err(y, oracle.layer_linear(layer, x, nthreads=NTHREADS))
        assert np.all(err <= TOL), (shape.name, B, err.max())
    assert eva_vq.eva_vq_sync_status(lin.handle) == eva_vq.EVA_OK
    lin.close()


def test_dequant_path_rejects_residual_with_group_codebooks():
    from vector_quantized_weight_b200 import eva_vq
    shape = synth.LayerShape("r", 256, 512, residual_group=128, codebook_rows=128)
    layer = synth.make_layer(shape, 1)
    with pytest.raises(eva_vq.EvaError) as ei:
        eva_vq.from_layer(layer, max_batch=8, path=eva_vq.EVA_PATH_DEQUANT_MMA)
    assert ei.value.status == eva_vq.EVA_ERR_UNSUPPORTED


def test_host_buffer_call_graph_and_pageable():
    """eva_vq_linear_run_host with page-locked buffers (read and written in
    place by the kernels for small x, else one replayed graph whose copy
    addresses follow new buffers) and with pageable ones: all equal to the
    device-buffer call."""
    import torch
    from vector_quantized_weight_b200 import eva_vq
    shape = synth.CONFIGS["llama7b_layer"].layers[0]
    layer = synth.make_layer(shape, 8)
    lin = eva_vq.from_layer(layer, max_batch=16)
    for B in (1, 16, 4, 16, 1):       # x of 8 and 32 KB: mapped host memory; 128 KB: the graph
        for i in range(3):
            x = synth.make_x(shape.K, B, 100 * B + i)
            ref = lin(torch.from_numpy(x).cuda()).cpu()
            xh = torch.from_numpy(x).pin_memory()
            yh = torch.empty((B, shape.N), dtype=torch.float16).pin_memory()
            lin.run_host(xh, yh)
            assert torch.equal(yh, ref)
            yp = torch.empty((B, shape.N), dtype=torch.float16)
            lin.run_host(torch.from_numpy(x), yp)
            assert torch.equal(yp, ref)
    lin.close()


@pytest.mark.parametrize("N,K,B,resid,cbr,had", [
    (4096, 4096, 1, 0, 0, 0), (256, 512, 2, 0, 0, 0), (100, 264, 3, 0, 0, 0), (64, 512, 1, 128, 0, 0),
    (48, 1024, 5, 128, 0, 0), (4096, 4096, 4, 0, 0, 0),
    (8192, 8192, 1, 0, 128, 0), (1024, 2048, 3, 0, 128, 0), (272, 1024, 2, 0, 16, 0),   # per-group codebooks
    (3584, 3584, 1, 128, 0, 512), (512, 1024, 2, 128, 0, 1024),                          # rotation + residual
    (3584, 3584, 1, 128, 0, 3584), (128, 1792, 3, 128, 128, 1792),                       # Paley blocks
])
def test_four_bit_indices(N, K, B, resid, cbr, had):
    """16-centroid codebooks with indices packed two per byte (shared or per
    group of rows, with or without rotation and sign residual): against the
    oracle (which reads the packed bytes itself) on every row, in both launch
    configurations, and the index round trip is bit-exact."""
    import torch
    from vector_quantized_weight_b200 import eva_vq
    shape = synth.LayerShape("idx4", N, K, residual_group=resid, index_bits=4, codebook_rows=cbr,
                             hadamard_block=had)
    layer = synth.make_layer(shape, N + K + B, alpha_signed=bool(resid))
    x = synth.make_x(K, B, 7)
    ref = oracle.layer_linear(layer, x, nthreads=NTHREADS)
    for independent in (False, True):
        y = run_gpu(layer, x, independent=independent)
        assert np.all(norm_rel_err(y, ref) <= TOL), independent
    lin = eva_vq.from_layer(layer, max_batch=B)
    back = lin.unpack_indices().cpu().numpy()
    torch.cuda.synchronize()
    lin.close()
    assert np.array_equal(back, layer.wi)


def test_four_bit_integer_exact():
    rng = np.random.default_rng(11)
    N, K = 128, 512
    wc = rng.integers(-2, 3, size=(1, 16, 4)).astype(np.float16)
    idx = rng.integers(0, 16, size=(N, K // 4))
    layer = synth.LayerData(synth.LayerShape("int4", N, K, index_bits=4), wc, synth.pack_nibbles(idx), None,
                            None, None)
    for B in (1, 2, 3):
        x = rng.integers(-3, 4, size=(B, K)).astype(np.float16)
        y = run_gpu(layer, x, out_dtype="float32")
        assert np.array_equal(y, oracle.layer_linear(layer, x))


@pytest.mark.parametrize("B", [1, 2, 4, 16])
def test_grouped_call_matches_separate_calls(B):
    """eva_vq_linear_run_group: one launch for layers of one shape and format
    (the lookup kernel at one or two tokens, the dequantize kernel from four
    on; bitwise equal to separate calls with the same flag, plain or
    independent, also with the residual), separate launches for a mixed
    group."""
    import torch
    from vector_quantized_weight_b200 import eva_vq
    for shape in (synth.LayerShape("g", 4096, 4096), synth.LayerShape("gr", 512, 1024, residual_group=128)):
        lins = [eva_vq.from_layer(synth.make_layer(shape, 50 + i), max_batch=B) for i in range(3)]
        xs = [torch.from_numpy(synth.make_x(shape.K, B, 60 + i)).cuda() for i in range(3)]
        for indep in (False, True):
            ref = [lin(x, independent=indep).clone() for lin, x in zip(lins, xs)]
            outs = eva_vq.run_group(lins, xs, independent=indep)
            torch.cuda.synchronize()
            if shape.name == "g":
                assert lins[0].info().path == (eva_vq.EVA_PATH_DEQUANT_MMA if B >= 3 else eva_vq.EVA_PATH_OC_LOOKUP)
            for a, b in zip(ref, outs):
                assert torch.equal(a, b)
        for lin in lins:
            assert eva_vq.eva_vq_sync_status(lin.handle) == eva_vq.EVA_OK
            lin.close()
    mixed = [synth.LayerShape("m1", 256, 512), synth.LayerShape("m2", 128, 1024, codebook_rows=16),
             synth.LayerShape("m3", 64, 512, residual_group=128, hadamard_block=128)]
    lins = [eva_vq.from_layer(synth.make_layer(sh, 70), max_batch=B) for sh in mixed]
    xs = [torch.from_numpy(synth.make_x(sh.K, B, 71)).cuda() for sh in mixed]
    ref = [lin(x).clone() for lin, x in zip(lins, xs)]
    outs = eva_vq.run_group(lins, xs)
    torch.cuda.synchronize()
    for a, b in zip(ref, outs):
        assert torch.equal(a, b)
    for lin in lins:
        lin.close()
