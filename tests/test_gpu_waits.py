"""Bounded waits of the bulk-copy ring kernel.  A test setting makes every stage wait for
16 bytes more than its copies deliver, so no stage ever fills: the kernel must give up
after the (shortened) limit, report ROPE3D_ETIMEOUT through the tables' status word,
leave the GPU usable, and the next normal launch must be correct.  No fault is caused:
every copy lands; only the wait runs out."""
import numpy as np
import pytest
import torch

import oracle
from gpu_support import Case, assert_close, kernel_path, oracle_rows, to_device, to_f64
from rotary_position_encoding_b200 import rope3d, workloads as wl

pytestmark = pytest.mark.gpu


PATHS = [rope3d.ROPE3D_PATH_TMA]


@pytest.mark.parametrize("path", PATHS)
def test_status_is_ok_after_normal_launches(path):
    w = wl.chunk_480p()
    case = Case(w)
    q, k, v = (to_device(x, w.dtype) for x in wl.chunk_inputs(w, 0))
    with kernel_path(path):
        case.run(q, k, v, w.chunks[0])
    assert rope3d.rope3d_check_device_status(case.tables) == rope3d.ROPE3D_OK


@pytest.mark.parametrize("path", PATHS)
def test_wait_that_never_fills_times_out_and_reports(path):
    w = wl.chunk_480p()
    case = Case(w)
    q, k, v = (to_device(x, w.dtype) for x in wl.chunk_inputs(w, 0))
    chunk = w.chunks[0]
    rope3d.rope3d_testing_set_waits(20_000_000, 16)  # 20 ms, 16 bytes never delivered
    try:
        with kernel_path(path):
            case.run(q, k, v, chunk)
        status = rope3d.rope3d_check_device_status(case.tables)
    finally:
        rope3d.rope3d_testing_set_waits(0, 0)
    assert status == rope3d.ROPE3D_ETIMEOUT
    # the word was cleared by the read, the context still works, and a normal launch is right
    assert rope3d.rope3d_check_device_status(case.tables) == rope3d.ROPE3D_OK
    with kernel_path(path):
        q_out = case.run(q, k, v, chunk)
    assert rope3d.rope3d_check_device_status(case.tables) == rope3d.ROPE3D_OK
    raw = wl.chunk_inputs(w, 0)
    got = to_f64(q_out)
    for (b, r, q_ref, k_ref, v_ref, pos) in oracle_rows(w, case, *raw, chunk,
                                                        [(0, 0), (0, 2345), (0, 4679)], 0):
        assert_close(got[b, r], q_ref, "bf16", f"row {r} after a timed-out launch")
