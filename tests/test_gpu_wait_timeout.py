"""Failure detection on the GPU without a GPU fault: a bounded wait that runs out.

Every wait inside the library's kernels gives up after a time limit, sets
PKV_STATUS_WAIT_TIMEOUT and lets the kernel return.  pkv_selftest_wait_timeout
makes that happen on purpose -- one warp waits, through the same helper, on an
mbarrier nothing completes, with nothing in flight -- and the host reads the
status bit.  A decode afterwards shows the context is still usable.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import paged_kv_cache_450_b200 as pk
from paged_kv_cache_450_b200 import _lib
from paged_kv_cache_450_b200 import workloads as W
from step_helpers import assert_close, oracle_step, tol_for

DEV = "cuda:0"


@pytest.mark.gpu
def test_bounded_wait_gives_up_reports_and_the_context_stays_usable():
    lib = _lib.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream)
    pk.device_status(clear=True)
    gave_up = torch.zeros(1, dtype=torch.int32, device=DEV)
    t0 = time.perf_counter()
    assert lib.pkv_selftest_wait_timeout(50_000, gave_up.data_ptr(), stream) == 0   # 50 us
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert int(gave_up.item()) == 1
    assert pk.device_status(clear=True) == pk.STATUS_WAIT_TIMEOUT
    # the next launches run normally
    w = W.make_decode_workload(W.LLAMA7B.with_(num_seqs=4, num_q_heads=8, num_kv_heads=8, new_tokens=False),
                               seed=41, device=DEV)
    out = pk.paged_attention_decode(w.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens, w.scale,
                                    partition_tokens=64, validate=True)
    torch.cuda.synchronize()
    _, _, ref = oracle_step(w)
    assert_close(out.float().cpu().numpy().astype(np.float64), ref, *tol_for(w), what="decode after the timeout")
    assert pk.device_status(clear=True) == 0


def test_selftest_argument_errors_without_a_device():
    lib = _lib.load()
    assert lib.pkv_selftest_wait_timeout(0, ctypes.c_void_p(16), None) == -7          # PKV_ERR_BAD_SHAPE
    assert lib.pkv_selftest_wait_timeout(200_000_000, ctypes.c_void_p(16), None) == -7
    assert lib.pkv_selftest_wait_timeout(1000, None, None) == -1                       # PKV_ERR_NULL_POINTER
