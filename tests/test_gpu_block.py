"""A whole Llama-2-7B-shaped decoder block of 2-bit layers on the GPU, with
the dependencies of a decode step: q, k and v in one grouped launch reading
the block input; o reading q's output (standing in for the attention
output); gate and up in one grouped launch reading o's output; down reading
gate's output (standing in for act(gate) * up).  Each launch waits for the one
before it on the stream.  Every layer's output is compared, on every row,
with the oracle fed the GPU's own fp16 input of that layer.
"""
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


@pytest.mark.parametrize("B", [1, 4, 16])
def test_decoder_block_chain_matches_the_oracle(B):
    import torch
    from vector_quantized_weight_b200 import eva_vq
    cfg = synth.CONFIGS["llama7b_block"]
    datas = [synth.make_layer(sh, synth.layer_seed(cfg.index, li)) for li, sh in enumerate(cfg.layers)]
    lins = [eva_vq.from_layer(d, max_batch=B) for d in datas]
    x = torch.from_numpy(synth.make_x(4096, B, 77)).cuda()
    ys = [torch.empty((B, d.shape.N), dtype=torch.float16, device="cuda") for d in datas]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        eva_vq.run_group(lins[0:3], [x] * 3, ys[0:3], stream=s)     # q, k, v
        lins[3](ys[0], out=ys[3], stream=s)                          # o <- q
        eva_vq.run_group(lins[4:6], [ys[3]] * 2, ys[4:6], stream=s)  # gate, up <- o
        lins[6](ys[4], out=ys[6], stream=s)                          # down <- gate
    s.synchronize()
    inputs = [x, x, x, ys[0], ys[3], ys[3], ys[4]]
    for li, (d, xin, y) in enumerate(zip(datas, inputs, ys)):
        xin_np = xin.cpu().numpy()
        assert np.all(np.isfinite(xin_np.astype(np.float32)))
        ref = oracle.layer_linear(d, xin_np, nthreads=NTHREADS)
        err = norm_rel_err(y.float().cpu().numpy(), ref)
        assert np.all(err <= TOL), (cfg.layers[li].name, err.max())
    for lin in lins:
        assert eva_vq.eva_vq_sync_status(lin.handle) == eva_vq.EVA_OK
        lin.close()
