"""Failure detection on the device, without a fault: a kernel's bounded wait
that nothing satisfies expires after a short limit, records its site and
returns; nsa_sync_status reports NSA_ERR_DEVICE_TIMEOUT once, and the same
CUDA context then runs the operator to parity."""
import pytest
import torch

from helpers import check_forward
from sparse_attention_long_phi_b200 import inputs as I

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_the_context_stays_usable():
    from sparse_attention_long_phi_b200 import nsa
    nsa.sync_status()                                  # nothing pending
    nsa.check_timeout_path(1_000_000)                  # 1 ms limit
    with pytest.raises(nsa.NsaError) as e:
        nsa.sync_status()
    assert e.value.code == 5                           # NSA_ERR_DEVICE_TIMEOUT
    nsa.sync_status()                                  # the word was cleared
    torch.cuda.synchronize()
    check_forward(dict(I.WORKLOADS["tiny_fwd_T1024"], seed=6000))
    nsa.sync_status()


def test_limit_outside_the_range_is_rejected_on_the_host():
    from sparse_attention_long_phi_b200 import nsa
    for bad in (0, 3_000_000_000):
        with pytest.raises(nsa.NsaError) as e:
            nsa.check_timeout_path(bad)
        assert e.value.code == 1
