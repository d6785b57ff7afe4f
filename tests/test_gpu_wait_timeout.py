"""The give-up path of the bounded waits, run on the GPU on purpose.

Every wait inside the library's tensor-core kernels is bounded: after a fixed
number of polls it raises the CTA's abort flag, records status bit 2 and
returns after freeing its TMEM, so that a wait that could never end (a copy
that never lands) leaves the GPU usable.  msa_selftest_wait_timeout runs that
exit with a short poll limit on an mbarrier that nothing arrives on, with no
copy or MMA in flight; these tests check that it returns, reports, and that the
library still computes correctly afterwards in the same process.
"""
import pytest
import torch

from block_sparse_gqa_04_b200 import msa
from block_sparse_gqa_04_b200.workload import Workload, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit", [1, 64, 4096, 1 << 14])
def test_bounded_wait_gives_up_and_reports(limit):
    status, gave_up = msa.selftest_wait_timeout(limit)
    assert status == 2          # kStatusWaitTimeout, and nothing else
    assert gave_up == 3         # the spinning MMA-style thread + two sleeping warps


def test_library_still_correct_after_a_timeout():
    msa.selftest_wait_timeout(4096)
    w = Workload("after_timeout", 1, 640, 640, 0, 32, 2, 128, 128, 128, 4, "bf16", 1)
    x = make_inputs(w, seed=3, device="cuda")
    a = msa.forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], top_k=w.top_k,
                    check_device_status=True)
    msa.selftest_wait_timeout(64)
    b = msa.forward(x["q"], x["k"], x["v"], x["q_idx"], x["k_idx"], top_k=w.top_k,
                    check_device_status=True)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_limit_is_checked_on_the_host():
    with pytest.raises(msa.MsaError):
        msa.selftest_wait_timeout(0)
    with pytest.raises(msa.MsaError):
        msa.selftest_wait_timeout((1 << 24) + 1)
