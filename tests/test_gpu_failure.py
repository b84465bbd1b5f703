"""Failure detection on the GPU without a fault: a bounded device-side wait
that nothing satisfies gives up, the kernel returns, the host reads
TG_ERR_TIMEOUT, and the context stays usable."""
import numpy as np
import pytest

import oracle
from gpu_util import assert_bitexact, run_gpu
from tiled_dense_gemm_fp16_b200 import inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    import torch
    import tiled_dense_gemm_fp16_b200 as tg
    torch.cuda.init()
    st, _ = tg.device_status()          # clear any earlier word
    assert st == tg.Status.OK
    assert tg.wait_timeout_selftest(2_000_000) == tg.Status.OK      # 2 ms budget
    st, word = tg.device_status()
    assert st == tg.Status.TIMEOUT and (word & 0xFF) == 0xEE, hex(word)
    st, word = tg.device_status()       # the word was cleared
    assert st == tg.Status.OK and word == 0
    A, B = inputs.operands(130, 264, 72, "int", seed=1)
    got, guards = run_gpu(A, B)
    assert guards
    assert_bitexact(got, oracle.gemm_relu_f16(A, B), "after timeout")
