"""The bounded-wait timeout path of both decode kernels, run on purpose.

Every wait of a decode kernel on a barrier gives up after a time limit: the
CTA stops, lets the TMA copies and MMAs it has already issued finish, frees
its tensor memory and reports MLA_ERR_DEVICE_TIMEOUT through device_status.
Nothing traps, so the CUDA context stays usable.  These tests lower the limit
to 1 microsecond (mla_set_wait_limit_ns): no wait for a copy from HBM or an
MMA can complete in that time, so the decode times out part-way through its
pipeline.  They check the reported status and that the next call, at the
default limit, matches the oracle.  No GPU fault, trap or hang is involved.
"""
import pytest
import torch

from mla_paged_latent_decode_b200 import binding, synth
from parity import full_parity, run_cuda

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("h_q,num_workers", [(16, None), (128, None), (128, 3)])
def test_timeout_is_reported_and_the_context_stays_usable(cuda_device, h_q, num_workers):
    # 16 heads: single-CTA kernel; 128 heads: CTA pairs (3 workers: split pieces)
    w = synth.custom_workload(3, 1, h_q, [700, 64, 1300])
    inp = synth.make_inputs(w, seed=41)
    prev = binding.set_wait_limit_ns(1000)
    try:
        res = run_cuda(inp, cuda_device, num_workers)
    finally:
        assert binding.set_wait_limit_ns(0) == 1000
    assert res["status"] == binding.MLA_ERR_DEVICE_TIMEOUT
    assert prev == 2_000_000_000
    # the default limit is back, and the next calls are exact again
    full_parity(inp, cuda_device, num_workers)
    full_parity(synth.make_inputs("tiny", seed=0), cuda_device)
    torch.cuda.synchronize(cuda_device)

