"""Failure detection on the GPU without a fault, a trap or a hang.

The only spin-wait in the kernels is the bounded wait of a waiting call for
the bulk copy that stages its first index units in shared memory.  The test
hook eva_vq_debug_inject_wait_timeout makes the next such call issue neither
the copy nor its arrival on the mbarrier -- nothing is in flight and the
barrier cannot complete -- with a short round limit, so the wait runs out:
every CTA records the give-up in the handle's status word, still joins its
cluster barriers and exits.  The host then reads EVA_ERR_DEVICE_TIMEOUT, and
the context stays usable: a fresh handle matches the oracle.
"""
import numpy as np
import pytest

import oracle
from tests.conftest import cuda_available
from tests.gpu_helpers import TOL, norm_rel_err
from vector_quantized_weight_b200 import synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not cuda_available(), reason="needs a CUDA device")]


@pytest.mark.parametrize("shape", [
    synth.LayerShape("l7b_4096x4096", 4096, 4096),
    synth.LayerShape("gemma_3584x3584", 3584, 3584, residual_group=128, hadamard_block=512),
])
def test_bounded_wait_gives_up_and_reports_timeout(shape):
    import torch
    from vector_quantized_weight_b200 import eva_vq
    layer = synth.make_layer(shape, 4242)
    x_np = synth.make_x(shape.K, 1, 4243)
    x = torch.from_numpy(x_np).cuda()
    lin = eva_vq.from_layer(layer, max_batch=1)
    assert lin.info().staged_units > 0       # a plain call of this layer stages index units
    assert eva_vq.eva_vq_sync_status(lin.handle) == eva_vq.EVA_OK
    eva_vq.eva_vq_debug_inject_wait_timeout(lin.handle, 1024)
    lin(x)                                   # a plain (waiting) call: it stages index units
    torch.cuda.synchronize()
    assert eva_vq.eva_vq_sync_status(lin.handle) == eva_vq.EVA_ERR_DEVICE_TIMEOUT
    # the hook is one-shot: the next call copies its units again (the word stays set)
    y_again = lin(x)
    torch.cuda.synchronize()
    assert eva_vq.eva_vq_sync_status(lin.handle) == eva_vq.EVA_ERR_DEVICE_TIMEOUT
    lin.close()

    ref = oracle.layer_linear(layer, x_np, nthreads=8)
    assert np.all(norm_rel_err(y_again.float().cpu().numpy(), ref) <= TOL)
    fresh = eva_vq.from_layer(layer, max_batch=1)
    y = fresh(x).float().cpu().numpy()
    torch.cuda.synchronize()
    assert eva_vq.eva_vq_sync_status(fresh.handle) == eva_vq.EVA_OK
    assert np.all(norm_rel_err(y, ref) <= TOL)
    fresh.close()


def test_inject_rejects_bad_round_counts():
    import torch
    from vector_quantized_weight_b200 import eva_vq
    lin = eva_vq.from_layer(synth.make_layer(synth.LayerShape("s", 256, 512), 1), max_batch=1)
    lib = eva_vq.load()
    for bad in (0, -1, (1 << 20) + 1):
        assert lib.eva_vq_debug_inject_wait_timeout(lin.handle, bad) == eva_vq.EVA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    lin.close()


def test_bounded_wait_gives_up_on_the_dequantize_path():
    """The warp-level dequantize path (three tokens and more) stages its index
    units the same way: the hook makes its wait run out too."""
    import torch
    from vector_quantized_weight_b200 import eva_vq
    shape = synth.LayerShape("l7b_4096x4096", 4096, 4096)
    layer = synth.make_layer(shape, 4244)
    x_np = synth.make_x(shape.K, 4, 4245)
    x = torch.from_numpy(x_np).cuda()
    lin = eva_vq.from_layer(layer, max_batch=4)
    eva_vq.eva_vq_debug_inject_wait_timeout(lin.handle, 1024)
    lin(x)
    torch.cuda.synchronize()
    assert lin.info().path == eva_vq.EVA_PATH_DEQUANT_MMA
    assert eva_vq.eva_vq_sync_status(lin.handle) == eva_vq.EVA_ERR_DEVICE_TIMEOUT
    lin.close()
    fresh = eva_vq.from_layer(layer, max_batch=4)
    y = fresh(x).float().cpu().numpy()
    torch.cuda.synchronize()
    assert eva_vq.eva_vq_sync_status(fresh.handle) == eva_vq.EVA_OK
    assert np.all(norm_rel_err(y, oracle.layer_linear(layer, x_np, nthreads=8)) <= TOL)
    fresh.close()
