"""A decode step captured in a CUDA graph (after one eager call, which sets
up the kernels' attributes) replays to exactly the eager outputs: the
persistent kernels' work counters and split tickets reset themselves, and
the programmatic launches become graph edges."""
import numpy as np
import pytest
import torch

import qsa_harness as H
from sparse_attention_decode_compress_b200 import QSADecodeStep, api
from workloads.qsa_inputs import WORKLOADS, make_batch

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda_and_cleanup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name,lens,S", [("b32_32k", [9000, 12345, 4099], 2),
                                         ("mtp_verify", [16384 + 3, 9001], 2),
                                         ("mixed_fp8", [4096, 11111], 4)])
def test_graph_replay_matches_eager(name, lens, S):
    b = make_batch(WORKLOADS[name], "cuda", ctx_lens=lens, seed=6)
    w = b.w
    step, cache = H.run_gpu(b, S, keep_scores=False)  # eager call (also sets the kernels up)
    want = (step.o.clone(), step.lse.clone(), step.sel.clone())
    inputs = H.step_inputs(b)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(inputs[0], inputs[1], inputs[2], b.q_idx, b.q, b.ctx_lens, inputs[3],
             stream=torch.cuda.current_stream())
    for _ in range(3):
        step.o.zero_()
        g.replay()
        torch.cuda.synchronize()
        st, flags = api.qsa_get_device_error()
        assert st == 0, (st, flags)
        assert torch.equal(step.sel, want[2])
        np.testing.assert_array_equal(step.o.cpu().numpy(), want[0].cpu().numpy())
        np.testing.assert_array_equal(step.lse.cpu().numpy(), want[1].cpu().numpy())
    del g
