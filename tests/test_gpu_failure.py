"""Failure reporting on the GPU, with no GPU fault.

The tensor-core kernels wait on mbarriers, and every such wait is bounded: a
wait that runs out sets bit 0 of the caller's status word, and the kernel
runs to its end and releases its tensor memory instead of hanging.  A
correct run never hits the limit, so pa_selftest_wait_timeout makes one wait
run out on purpose, with nothing else in flight (one CTA holding tensor
memory, an mbarrier nothing arrives at), and the host reads the bit through
the same pa_workspace_status every attention call's caller uses.  The other
injected failure is a CUDA error raised on the host: a call that must
synchronize, made inside a stream capture, where synchronizing is not
allowed, returns PA_ERR_CUDA.  After each, normal calls on the same device
still give the oracle's results.
"""
import pytest
import torch

import paged_kv_attention_token_b200 as pa
import workloads as W
from tests.parity import assert_parity
from tests.test_gpu_parity import gpu_rows, oracle_subset, run_step

pytestmark = pytest.mark.gpu


def _tiny_step_matches_oracle(what):
    lay = W.layout("tiny_mixed")
    b = W.make_batch(lay, device="cuda", q_gain=8.0)
    _, _, out, _ = run_step(b)      # asserts a zero status word itself
    tok, want = oracle_subset(b, range(lay.num_seqs))
    assert_parity(gpu_rows(out, tok), want, what)


def test_bounded_wait_runs_out_and_is_reported(cuda_lib):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert pa.workspace_status(ws) == 0
    pa.selftest_wait_timeout(ws, 100_000)          # ~50 us at B200 clocks
    assert pa.workspace_status(ws) == 1
    pa.selftest_wait_timeout(ws, 1000)
    assert pa.workspace_status(ws) == 1            # bits accumulate, never clear by themselves
    plan = pa.Plan([0, 1], [1], pa.Dims(1, 1, 8, 1, 64, 4, 1, 16))
    pa.workspace_reset(ws, plan)
    assert pa.workspace_status(ws) == 0
    # the device is fine: a normal step on it matches the oracle
    _tiny_step_matches_oracle("after a bounded wait ran out")


def test_cuda_error_inside_stream_capture_is_returned(cuda_lib):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        g.capture_begin()
        try:
            # reading the status word synchronizes the stream: not allowed
            # while it is being captured, so the CUDA call fails
            with pytest.raises(pa.PaError) as e:
                pa.workspace_status(ws, stream=s)
            assert e.value.status == pa.PA_ERR_CUDA
        finally:
            try:
                g.capture_end()
            except RuntimeError:
                pass                                # the failed call invalidated the capture
    torch.cuda.synchronize()
    assert pa.workspace_status(ws) == 0
    _tiny_step_matches_oracle("after a CUDA error in a capture")
