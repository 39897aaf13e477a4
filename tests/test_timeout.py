"""The bounded-wait give-up path of the tensor-core kernel, exercised without a hang.

The test hook makes every CTA's MMA thread wait on a barrier nothing arrives on, with a
short bound. The kernel must record the event, stop its other roles, drain its own copies,
free tensor memory and return; the host then reads WOQ_ETIMEOUT, and the context stays
usable: the next launch, with the hook off, is correct.
"""

import pytest

import oracle
import weight_only_bit_qgemv_b200 as woq
from weight_only_bit_qgemv_b200 import _lib, workloads
from tests.gpu_util import BF16_TOL, fro_rel, packed_from_weight

pytestmark = pytest.mark.gpu


def test_stuck_wait_reports_timeout_and_context_survives():
    W = workloads.weight(512, 1024, seed=8)
    w, p, s = packed_from_weight(W, 4)
    X = workloads.activations(256, 1024, seed=9)
    Xd = X.cuda()
    assert woq.device_status(clear=True) == _lib.WOQ_OK
    L = _lib.lib()
    try:
        L.woq_debug_set_wait_limit(-200000)   # ~0.1 ms stuck wait per CTA
        woq.qgemm(Xd, w, path="bf16_tc")
        assert woq.device_status(clear=True) == _lib.WOQ_ETIMEOUT
    finally:
        L.woq_debug_set_wait_limit(0)
    assert woq.device_status(clear=True) == _lib.WOQ_OK
    Y = woq.qgemm(Xd, w, path="bf16_tc").cpu().numpy()
    assert fro_rel(Y, oracle.qgemv_ref(X.numpy(), p, s, 4)) <= BF16_TOL
    assert woq.device_status(clear=True) == _lib.WOQ_OK
