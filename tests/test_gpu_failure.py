"""Failure detection on the GPU without a fault: a bounded device wait that nothing completes
gives up after its limit, the host reads NQ_ERR_TIMEOUT from nq_sync_status, the status is
cleared, and the context still computes the hot path correctly."""
import numpy as np
import pytest

import oracle
from rank_binary_factorized_b200 import synth
from tests.gpu_util import check_tolerance, download_bf16_bits, need_gpu, nq, upload_bf16, upload_projection

pytestmark = pytest.mark.gpu

NQ_ERR_TIMEOUT = 7


def test_bounded_wait_times_out_and_the_context_survives():
    need_gpu()
    mod = nq()
    mod.selftest_bounded_wait(20000)  # 20 ms
    with pytest.raises(mod.NQError) as exc:
        mod.sync_status()
    assert exc.value.status == NQ_ERR_TIMEOUT
    mod.sync_status()  # the error word was cleared
    p = synth.make_workload("tiny")[0]
    xb = synth.make_input("tiny", p.d_in, 1)
    for fn in ("lrb_matvec", "lrb_matmul"):
        y = getattr(mod, fn)(upload_projection(p), upload_bf16(xb))
        mod.sync_status()
        ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb)
        check_tolerance(download_bf16_bits(y), ref, S, "after the timeout, " + fn)
