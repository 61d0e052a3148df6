"""eva_vq_linear_run_noalloc: the allocation-free call, for callers that must
not touch the device allocator (for example while a whole decode step is
being captured into a CUDA graph, where cudaMalloc would fail or break the
capture).  Its only scratch -- the rotated input of a 3.125-bit layer --
comes from the library's static device array instead of the handle.

This file is collected last on purpose: the first call on a device looks up
the static array's address, and the test must pass both in a fresh process
and after every other test has run.
"""
import numpy as np
import pytest

from tests.conftest import cuda_available
from tests.gpu_helpers import TOL, norm_rel_err
from vector_quantized_weight_b200 import synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


@pytest.mark.parametrize("shape,B", [
    (synth.LayerShape("rot_3bit", 3584, 3584, residual_group=128, hadamard_block=512), 1),
    (synth.LayerShape("rot_pair", 512, 2048, residual_group=128, hadamard_block=2048), 3),
    (synth.LayerShape("plain_2bit", 4096, 4096), 1),
    (synth.LayerShape("rot_paley", 256, 3584, residual_group=128, hadamard_block=3584), 1),
])
def test_noalloc_run_matches_regular_run(shape, B):
    import torch
    from vector_quantized_weight_b200 import eva_vq
    layer = synth.make_layer(shape, 909)
    lin = eva_vq.from_layer(layer, max_batch=B)
    x = torch.from_numpy(synth.make_x(shape.K, B, 910)).cuda()
    ref = lin(x).float().cpu().numpy()
    stream = eva_vq._stream_handle(None)
    outs = []
    for _ in range(2):   # two calls in a row share (and overwrite) the static scratch
        y = torch.empty((B, shape.N), dtype=torch.float16, device="cuda")
        eva_vq.eva_vq_linear_run_noalloc(lin.handle, x.data_ptr(), B, y.data_ptr(), stream)
        outs.append(y)
    torch.cuda.synchronize()
    for y in outs:
        got = y.float().cpu().numpy()
        assert np.all(norm_rel_err(got, ref) <= TOL)
        assert np.array_equal(got, ref)     # same kernels, same order of sums
    lin.close()


@pytest.mark.parametrize("shape,B", [
    (synth.LayerShape("rot_3bit", 3584, 3584, residual_group=128, hadamard_block=512), 4),
    (synth.LayerShape("rot_paley", 256, 3584, residual_group=128, hadamard_block=3584), 2),
])
def test_noalloc_dequantize_path_with_rotation(shape, B):
    """The dequantize path of a rotated layer: a Sylvester block rotated on
    chip (one kernel), a Paley block through the rotation kernel into the
    static scratch (two; the lookup path fuses those); bitwise equal to the
    regular call either way."""
    import torch
    from vector_quantized_weight_b200 import eva_vq
    layer = synth.make_layer(shape, 911)
    lin = eva_vq.from_layer(layer, max_batch=B, path=eva_vq.EVA_PATH_DEQUANT_MMA)
    x = torch.from_numpy(synth.make_x(shape.K, B, 912)).cuda()
    ref = lin(x).clone()
    y = torch.empty((B, shape.N), dtype=torch.float16, device="cuda")
    eva_vq.eva_vq_linear_run_noalloc(lin.handle, x.data_ptr(), B, y.data_ptr(), eva_vq._stream_handle(None))
    torch.cuda.synchronize()
    assert lin.info().path == eva_vq.EVA_PATH_DEQUANT_MMA
    assert lin.info().kernels_per_run == (2 if shape.name == "rot_paley" else 1)
    assert torch.equal(y, ref)
    lin.close()


def test_noalloc_rejects_requests_beyond_the_static_scratch():
    import torch
    from vector_quantized_weight_b200 import eva_vq
    shape = synth.LayerShape("big_rot", 64, 16384, residual_group=128, hadamard_block=2048)
    layer = synth.make_layer(shape, 3)
    lin = eva_vq.from_layer(layer, max_batch=64)
    B = 64                                   # 64 * 16384 * 4 bytes: exactly the 4 MiB limit
    x = torch.zeros((B + 1, shape.K), dtype=torch.float16, device="cuda")
    y = torch.empty((B, shape.N), dtype=torch.float16, device="cuda")
    lib = eva_vq.load()
    assert lib.eva_vq_linear_run_noalloc(lin.handle, x.data_ptr(), B, y.data_ptr(), None) == eva_vq.EVA_OK
    torch.cuda.synchronize()
    lin.close()
    shape2 = synth.LayerShape("bigger_rot", 64, 20480, residual_group=128, hadamard_block=2048)
    lin2 = eva_vq.from_layer(synth.make_layer(shape2, 4), max_batch=64)
    x2 = torch.zeros((64, shape2.K), dtype=torch.float16, device="cuda")
    rc = lib.eva_vq_linear_run_noalloc(lin2.handle, x2.data_ptr(), 64, y.data_ptr(), None)
    assert rc == eva_vq.EVA_ERR_SCRATCH_TOO_SMALL
    assert "static scratch" in eva_vq.eva_vq_status_string(rc)
    torch.cuda.synchronize()
    lin2.close()
