"""The large-batch path on the fifth-generation tensor cores (tcgen05.mma,
weights rebuilt from the codebook into tensor memory, fp32 accumulation in
tensor memory) against the double-precision oracle, on every output row:
shared and per-128-row codebooks, the Gemma-shaped 3.125-bit layers (sign
residual and Hadamard rotation, Sylvester and Paley blocks), ragged batches
(the MMA's N is the batch padded to 16) and the split-K cluster reduction."""
import os

import numpy as np
import pytest

import oracle
from tests.conftest import cuda_available
from tests.gpu_helpers import TOL, norm_rel_err
from vector_quantized_weight_b200 import synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]

NTHREADS = os.cpu_count() or 8


def _run(layer, x, path, out_dtype="float16", independent=False):
    import torch
    from vector_quantized_weight_b200 import eva_vq
    B = x.shape[0]
    lin = eva_vq.from_layer(layer, max_batch=B, out_dtype=out_dtype, path=path)
    y = lin(torch.from_numpy(x).cuda(), independent=independent).float().cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    info = lin.info()
    assert eva_vq.eva_vq_sync_status(lin.handle) == eva_vq.EVA_OK
    lin.close()
    return y, info


@pytest.mark.parametrize("shape,B", [
    (synth.LayerShape("tiny", 256, 512), 4),
    (synth.LayerShape("l7b", 4096, 4096), 4),
    (synth.LayerShape("l7b", 4096, 4096), 16),
    (synth.LayerShape("l7b", 4096, 4096), 64),
    (synth.LayerShape("l7b_gate", 11008, 4096), 16),
    (synth.LayerShape("l7b_down", 4096, 11008), 16),
    (synth.LayerShape("ragged", 200, 1088), 9),
    (synth.LayerShape("ragged", 1000, 2048), 33),
    (synth.LayerShape("l70b", 8192, 8192, codebook_rows=128), 8),
    (synth.LayerShape("l70b", 8192, 8192, codebook_rows=128), 32),
    (synth.LayerShape("cb256", 512, 1024, codebook_rows=256), 5),
    (synth.LayerShape("gemma", 3584, 3584, residual_group=128, hadamard_block=512), 4),
    (synth.LayerShape("gemma_up", 14336, 3584, residual_group=128, hadamard_block=512), 4),
    (synth.LayerShape("gemma_down", 3584, 14336, residual_group=128, hadamard_block=2048), 4),
    (synth.LayerShape("gemma_rotK", 3584, 3584, residual_group=128, hadamard_block=3584), 4),
    (synth.LayerShape("resid_only", 384, 1024, residual_group=128), 7),
])
def test_tcgen05_path_matches_the_oracle(shape, B):
    from vector_quantized_weight_b200 import eva_vq
    layer = synth.make_layer(shape, 5000 + shape.N + B, alpha_signed=bool(shape.residual_group))
    x = synth.make_x(shape.K, B, 17 + B)
    ref = oracle.layer_linear(layer, x, nthreads=NTHREADS)
    for independent in (False, True):
        y, info = _run(layer, x, eva_vq.EVA_PATH_TCGEN05, independent=independent)
        assert info.path == eva_vq.EVA_PATH_TCGEN05
        err = norm_rel_err(y, ref)
        assert np.all(err <= TOL), (independent, err.max())


def test_tcgen05_integer_inputs_exact():
    """Small-integer codebooks and inputs: every product and partial sum is
    exact in fp16 / fp32, so the tensor-core path reproduces the oracle exactly."""
    from vector_quantized_weight_b200 import eva_vq
    rng = np.random.default_rng(3)
    for N, K, cbr, B in ((256, 1024, 0, 16), (384, 2048, 128, 7)):
        G = N // cbr if cbr else 1
        layer = synth.LayerData(synth.LayerShape("int", N, K, codebook_rows=cbr),
                                rng.integers(-2, 3, size=(G, 256, 4)).astype(np.float16),
                                rng.integers(0, 256, size=(N, K // 4)).astype(np.uint8), None, None, None)
        x = rng.integers(-3, 4, size=(B, K)).astype(np.float16)
        y, _ = _run(layer, x, eva_vq.EVA_PATH_TCGEN05, out_dtype="float32")
        assert np.array_equal(y, oracle.layer_linear(layer, x))


def test_auto_path_by_batch():
    """AUTO: lookups below three tokens (two with per-group codebooks); from
    there on the warp-level dequantize path, the tcgen05 path past 32 tokens
    with one shared codebook -- 3.125-bit layers (rotation, residual)
    included."""
    from vector_quantized_weight_b200 import eva_vq
    plain = synth.LayerShape("l7b", 4096, 4096)
    gemma = synth.LayerShape("gemma", 3584, 3584, residual_group=128, hadamard_block=512)
    for shape, cases in ((plain, ((1, eva_vq.EVA_PATH_OC_LOOKUP), (2, eva_vq.EVA_PATH_OC_LOOKUP),
                                  (3, eva_vq.EVA_PATH_DEQUANT_MMA), (16, eva_vq.EVA_PATH_DEQUANT_MMA),
                                  (32, eva_vq.EVA_PATH_DEQUANT_MMA), (33, eva_vq.EVA_PATH_TCGEN05),
                                  (64, eva_vq.EVA_PATH_TCGEN05))),
                         (gemma, ((1, eva_vq.EVA_PATH_OC_LOOKUP), (2, eva_vq.EVA_PATH_OC_LOOKUP),
                                  (3, eva_vq.EVA_PATH_DEQUANT_MMA), (16, eva_vq.EVA_PATH_DEQUANT_MMA),
                                  (32, eva_vq.EVA_PATH_DEQUANT_MMA), (33, eva_vq.EVA_PATH_TCGEN05))),
                         (synth.LayerShape("l70b", 8192, 8192, codebook_rows=128),
                          ((1, eva_vq.EVA_PATH_OC_LOOKUP), (2, eva_vq.EVA_PATH_DEQUANT_MMA),
                           (8, eva_vq.EVA_PATH_DEQUANT_MMA), (32, eva_vq.EVA_PATH_DEQUANT_MMA)))):
        layer = synth.make_layer(shape, 8)
        for B, path in cases:
            x = synth.make_x(shape.K, B, 9)
            _, info = _run(layer, x, eva_vq.EVA_PATH_AUTO)
            assert info.path == path, (shape.name, B, info.path)


def test_tcgen05_rejects_layers_it_cannot_take():
    from vector_quantized_weight_b200 import eva_vq
    for shape in (synth.LayerShape("k_not_64", 256, 520), synth.LayerShape("cb16", 256, 512, codebook_rows=16),
                  synth.LayerShape("idx4", 256, 512, index_bits=4)):
        with pytest.raises(eva_vq.EvaError) as ei:
            eva_vq.from_layer(synth.make_layer(shape, 1), max_batch=8, path=eva_vq.EVA_PATH_TCGEN05)
        assert ei.value.status == eva_vq.EVA_ERR_UNSUPPORTED


def test_row_block_copy_only_where_the_path_can_run():
    """A handle keeps the tcgen05 path's row-block copy of the indices only
    where that path can run: AUTO with max_batch past 32 and one shared
    codebook (4096 x 4096: about 4 MB more than at 32), never for per-group
    codebooks, whose batches the warp-level path takes."""
    import torch
    from vector_quantized_weight_b200 import eva_vq

    def footprint(shape, **kw):
        layer = synth.make_layer(shape, 12)
        wc = torch.from_numpy(layer.wc).cuda()
        wi = torch.from_numpy(layer.wi).cuda()
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        lin = eva_vq.VQLinear(wc, wi, codebook_rows=shape.codebook_rows, **kw)
        torch.cuda.synchronize()
        used = free0 - torch.cuda.mem_get_info()[0]
        lin.close()
        torch.cuda.synchronize()
        return used

    plain = synth.LayerShape("l7b", 4096, 4096)
    copy = plain.N * plain.K // 4
    assert footprint(plain, max_batch=33) - footprint(plain, max_batch=32) >= 0.9 * copy
    grouped = synth.LayerShape("l70b_part", 4096, 4096, codebook_rows=128)
    assert footprint(grouped, max_batch=64) - footprint(grouped, max_batch=32) < 0.75 * copy
