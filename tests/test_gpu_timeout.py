"""The bounded-wait timeout path of both decode kernels, run on purpose.

Every wait of a decode kernel gives up after a time limit: the CTA stops, lets
the TMA copies and MMAs it has already issued finish, frees its tensor memory
and reports MLA_ERR_DEVICE_TIMEOUT through device_status.  Nothing traps, so
the CUDA context stays usable.

These tests make one wait run out: through the test hook
mla_debug_set_stall_flag, the PV-issuing thread of every CTA waits before its
first PV for a device word that nothing sets, with the limit lowered to 50
microseconds (mla_set_wait_limit_ns).  At that point the CTA's page copies and
QK^T MMAs are in flight.  The tests check the reported status and that the
next calls, at the default limit, match the oracle.  No GPU fault, trap or
endless wait is involved: every wait, the hook's included, is bounded.
"""
import pytest
import torch

from mla_paged_latent_decode_b200 import binding, synth
from parity import full_parity, run_cuda

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("h_q,num_workers", [(16, None), (128, None), (128, 3), (16, 2)])
def test_timeout_is_reported_and_the_context_stays_usable(cuda_device, h_q, num_workers):
    # 16 heads: single-CTA kernel; 128 heads: CTA pairs; few workers: several
    # pages and pieces per CTA, so more copies are in flight at the stall
    w = synth.custom_workload(3, 1, h_q, [700, 64, 1300])
    inp = synth.make_inputs(w, seed=41)
    never = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    prev = binding.set_wait_limit_ns(50_000)
    binding.debug_set_stall_flag(never)
    try:
        res = run_cuda(inp, cuda_device, num_workers)
    finally:
        binding.debug_set_stall_flag(None)
        assert binding.set_wait_limit_ns(0) == 50_000
    assert prev == 2_000_000_000
    assert res["status"] == binding.MLA_ERR_DEVICE_TIMEOUT
    # the hook is off and the default limit is back: the next calls are exact
    full_parity(inp, cuda_device, num_workers)
    full_parity(synth.make_inputs("tiny", seed=0), cuda_device)
    torch.cuda.synchronize(cuda_device)


def test_stall_flag_that_is_set_does_not_stop_the_decode(cuda_device):
    # the hook's wait ends as soon as the word is non-zero: same results as without it
    w = synth.custom_workload(2, 2, 128, [300, 900], causal=True)
    inp = synth.make_inputs(w, seed=42)
    go = torch.ones(1, dtype=torch.int32, device=cuda_device)
    binding.debug_set_stall_flag(go)
    try:
        full_parity(inp, cuda_device)
    finally:
        binding.debug_set_stall_flag(None)
