"""The failure path of every pipelined kernel: a bounded mbarrier wait that runs out raises the
device error word and returns. A kernel whose wait can never be satisfied (nothing arrives on its
barrier) must end by itself, qgemm_sync_check must report the timeout once, and the context must
stay usable for ordinary calls."""
import pytest

import gemv_w4a16_w8a8_b200 as qg
from gpu_cases import W4Case, assert_fp16_close

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_the_context_survives():
    qg.qgemm_sync_check()                       # start from a clear error word
    qg.qgemm_selftest_bounded_wait(20000)       # gives up after 20 ms
    with pytest.raises(qg.QGemmError) as e:
        qg.qgemm_sync_check()
    assert e.value.status == qg.QG_ERR_DEVICE_TIMEOUT
    qg.qgemm_sync_check()                       # reported once, then cleared
    case = W4Case(8, 256, 1024, 128, 1, seed=5)
    assert_fp16_close(case.run(), case.ref_full(), "after a timed-out wait")
    qg.qgemm_sync_check()
