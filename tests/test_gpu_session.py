"""GPU tests of the decode session (qsa_session_*): steps from pinned host
buffers give exactly the outputs of the same step run call by call on
device buffers (which the parity tests check against the oracle), and one
request is checked against the oracle directly."""
import numpy as np
import pytest
import torch

import qsa_harness as H
from sparse_attention_decode_compress_b200 import QSASession, api
from workloads.qsa_inputs import WORKLOADS, make_batch

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda_and_cleanup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _host_inputs(b):
    pos0, cu, k_new, n_sel = H.step_inputs(b)
    pin = lambda t: None if t is None else t.cpu().pin_memory()
    return dict(pos0=pin(pos0), cu_new=pin(cu), k_new=pin(k_new), q_idx=pin(b.q_idx), q=pin(b.q),
                ctx_lens=pin(b.ctx_lens), n_sel=pin(n_sel))


CASES = [("b32_32k", [9000, 12345, 4099], 2), ("mtp_verify", [16384 + 3, 9001, 12002, 4100], 2),
         ("mixed_fp8", [4096, 11111, 30007], 4), ("tiny", None, 1)]


@pytest.mark.parametrize("name,lens,S", CASES)
def test_session_steps_match_device_path(name, lens, S):
    b = make_batch(WORKLOADS[name], "cuda", ctx_lens=lens, seed=9)
    w = b.w
    step, cache = H.run_gpu(b, S, keep_scores=False)
    want_o, want_lse = step.o.cpu().numpy(), step.lse.cpu().numpy()
    H.check_request(b, step, cache, 0, S)
    q_dtype = torch.float32 if b.q.dtype == torch.float32 else torch.bfloat16
    sess = QSASession(cache, w.batch, w.T, w.Hq, w.topk, S, H.max_blocks_of(b), w.batch * w.T,
                      step.sm_scale, q_dtype=q_dtype)
    h = _host_inputs(b)
    outs = [(torch.empty(step.o.shape).pin_memory(), torch.empty(step.lse.shape).pin_memory())
            for _ in range(3)]
    for o, lse in outs:  # three steps in flight: both slots and a reuse
        sess.step(h["pos0"], h["cu_new"], h["k_new"], h["q_idx"], h["q"], h["ctx_lens"], h["n_sel"],
                  o, lse)
    sess.synchronize()
    st, flags = api.qsa_get_device_error()
    assert st == 0, (st, flags)
    for o, lse in outs:
        np.testing.assert_array_equal(o.numpy(), want_o)
        np.testing.assert_array_equal(lse.numpy(), want_lse)
    sess.close()


def test_session_rejects_bad_arguments():
    b = make_batch(WORKLOADS["b32_32k"], "cuda", ctx_lens=[5000, 6000], seed=2)
    w = b.w
    step, cache = H.run_gpu(b, 2, keep_scores=False)
    sess = QSASession(cache, w.batch, w.T, w.Hq, w.topk, 2, H.max_blocks_of(b), 1, step.sm_scale)
    h = _host_inputs(b)
    o = torch.empty(step.o.shape).pin_memory()
    lse = torch.empty(step.lse.shape).pin_memory()
    with pytest.raises(api.QSAError):  # 2 new tokens > max_new_tokens = 1
        sess.step(h["pos0"], h["cu_new"], h["k_new"], h["q_idx"], h["q"], h["ctx_lens"], None, o, lse)
    with pytest.raises(ValueError):  # device tensor where a host one is expected
        sess.step(h["pos0"].cuda(), h["cu_new"], h["k_new"], h["q_idx"], h["q"], h["ctx_lens"],
                  None, o, lse)
    sess.synchronize()
    sess.close()
