"""The checked build of the library (-DROPE3D_DEVICE_CHECKS, librope3d_checked.so).

Its step kernels test every cache row, table row and sequence-parallel destination row
they derive against the call's extents and record a miss in the status word instead of
touching memory.  For valid arguments the host checks make a miss unreachable, so on
every workload here the checked build must report ROPE3D_OK and write exactly what the
plain build writes.  The firing path is exercised with the testing hook that makes the
row check withhold the last cache rows: those rows lie inside the caller's buffers, so
no access ever leaves them."""
import contextlib

import numpy as np
import pytest
import torch

from gpu_support import to_device
from rotary_position_encoding_b200 import build as native_build
from rotary_position_encoding_b200 import rope3d, workloads as wl

pytestmark = pytest.mark.gpu


@contextlib.contextmanager
def library(path):
    saved = rope3d._lib
    rope3d._lib = rope3d.load_library(path)
    try:
        yield rope3d._lib
    finally:
        rope3d._lib = saved


def _checked_path():
    if native_build.stale(native_build.CHECKED_LIBRARY):
        native_build.build_all()
    return native_build.CHECKED_LIBRARY


def _run_chunks(w, chunks, path, trig, cache_dtype="same", sp=0):
    """Run the given chunk calls of workload w through the current library; return every
    output tensor and the device status."""
    wq_np, wk_np = wl.norm_weights(w.seed, w.dim)
    wq, wk = torch.from_numpy(wq_np).cuda(), torch.from_numpy(wk_np).cuda()
    tables = rope3d.rope3d_tables_init(max_t=21, max_h=w.H, max_w=w.W)
    rope3d.rope3d_testing_force_path(path)
    outs = []
    try:
        D = wl.HEAD_DIM
        if sp:
            hl = w.N // sp
            n = w.tokens_per_chunk
            q_d = [torch.zeros((w.B, n, hl, D), dtype=torch.bfloat16, device="cuda")
                   for _ in range(sp)]
            k_d = [torch.zeros((w.B, w.cache_tokens, hl, D), dtype=torch.bfloat16,
                               device="cuda") for _ in range(sp)]
            v_d = [torch.zeros_like(k_d[0]) for _ in range(sp)]
            for ci in chunks:
                c = w.chunks[ci]
                q, k, v = (to_device(x, w.dtype) for x in wl.chunk_inputs(w, ci))
                for a, b in wl.slices(n, sp):
                    rope3d.rope3d_qk_norm_rope_append_sp(
                        q[:, a:b].contiguous(), k[:, a:b].contiguous(), v[:, a:b].contiguous(),
                        a, b, c.frame_offset, w.T, w.H, w.W, wq, wk, w.eps, q_d, k_d, v_d,
                        c.slot, tables, trig, q_row0=0)
            outs = q_d + k_d + v_d
        else:
            fp8 = cache_dtype == "fp8"
            shape = (w.B, w.cache_tokens, w.N, D)
            kc = torch.zeros(shape, dtype=torch.uint8 if fp8 else torch.bfloat16, device="cuda")
            vc = torch.zeros_like(kc)
            ks = torch.zeros(shape[:3], device="cuda") if fp8 else None
            vs = torch.zeros(shape[:3], device="cuda") if fp8 else None
            for ci in chunks:
                c = w.chunks[ci]
                q, k, v = (to_device(x, w.dtype) for x in wl.chunk_inputs(w, ci))
                qo = torch.full_like(q, 3.0)
                rope3d.rope3d_qk_norm_rope_append_ex(
                    q, k, v, qo, c.token_begin, c.token_end, c.frame_offset, w.T, w.H, w.W, wq,
                    wk, w.eps, kc, vc, c.slot, tables, trig, k_scale=ks, v_scale=vs)
                outs.append(qo)
            outs += [kc, vc] + ([ks, vs] if fp8 else [])
        torch.cuda.synchronize()
        status = rope3d.rope3d_check_device_status(tables)
    finally:
        rope3d.rope3d_testing_force_path(rope3d.ROPE3D_PATH_AUTO)
        tables.close()
    return outs, status


def _bits(t):
    return t.contiguous().view(torch.uint8).cpu().numpy()


@pytest.mark.parametrize("path", [rope3d.ROPE3D_PATH_REGISTERS, rope3d.ROPE3D_PATH_TMA])
@pytest.mark.parametrize("trig", [rope3d.ROPE3D_TRIG_TABLE, rope3d.ROPE3D_TRIG_ONTHEFLY])
def test_checked_build_reports_ok_and_matches_plain_build(path, trig):
    w = wl.chunk_480p()
    chunks = (0, 6)  # start frames 0 and 18: the table's first and last frames
    if path == rope3d.ROPE3D_PATH_TMA:
        w = wl.chunk_720p()
        w.chunks = w.chunks[:2]
        chunks = (0, 1)
    plain, st_plain = _run_chunks(w, chunks, path, trig)
    with library(_checked_path()):
        checked, st_checked = _run_chunks(w, chunks, path, trig)
    assert st_plain == rope3d.ROPE3D_OK
    assert st_checked == rope3d.ROPE3D_OK
    for a, b in zip(plain, checked):
        assert np.array_equal(_bits(a), _bits(b))


def test_checked_build_fp8_cache_and_sp_scatter():
    w = wl.chunk_480p()
    for kw in ({"cache_dtype": "fp8"}, {"sp": 4}):
        plain, st_plain = _run_chunks(w, (3,), rope3d.ROPE3D_PATH_AUTO,
                                      rope3d.ROPE3D_TRIG_TABLE, **kw)
        with library(_checked_path()):
            checked, st_checked = _run_chunks(w, (3,), rope3d.ROPE3D_PATH_AUTO,
                                              rope3d.ROPE3D_TRIG_TABLE, **kw)
        assert (st_plain, st_checked) == (rope3d.ROPE3D_OK, rope3d.ROPE3D_OK), kw
        for a, b in zip(plain, checked):
            assert np.array_equal(_bits(a), _bits(b)), kw


@pytest.mark.parametrize("path", [rope3d.ROPE3D_PATH_REGISTERS, rope3d.ROPE3D_PATH_TMA])
def test_checked_build_withholds_rows_beyond_the_check_bound(path):
    """With the row check told to accept cache rows below C - 100 only, the launch writing
    the cache's last rows skips exactly those token rows (q_out, K and V untouched) and
    the status reads ROPE3D_EINDEX; every other row is the plain build's."""
    w = wl.chunk_720p() if path == rope3d.ROPE3D_PATH_TMA else wl.chunk_480p()
    last = len(w.chunks) - 1
    w.chunks = [w.chunks[last]]  # start frame 18: cache rows C - n .. C - 1
    plain, _ = _run_chunks(w, (0,), path, rope3d.ROPE3D_TRIG_TABLE)
    with library(_checked_path()):
        rope3d.rope3d_testing_shrink_checked_cache(100)
        try:
            checked, status = _run_chunks(w, (0,), path, rope3d.ROPE3D_TRIG_TABLE)
        finally:
            rope3d.rope3d_testing_shrink_checked_cache(0)
        # the hook is reset: a rerun reports OK
        again, status2 = _run_chunks(w, (0,), path, rope3d.ROPE3D_TRIG_TABLE)
    assert status == rope3d.ROPE3D_EINDEX
    assert status2 == rope3d.ROPE3D_OK
    n = w.tokens_per_chunk
    qo_p, kc_p, vc_p = plain
    qo_c, kc_c, vc_c = checked
    cut = w.cache_tokens - 100  # cache rows >= cut belong to the chunk's last 100 tokens
    r0 = n - 100
    assert torch.equal(qo_c[:, :r0].view(torch.int16), qo_p[:, :r0].view(torch.int16))
    assert bool((qo_c[:, r0:].float() == 3.0).all())
    assert torch.equal(kc_c[:, :cut].view(torch.int16), kc_p[:, :cut].view(torch.int16))
    assert torch.equal(vc_c[:, :cut].view(torch.int16), vc_p[:, :cut].view(torch.int16))
    assert not bool(kc_c[:, cut:].any()) and not bool(vc_c[:, cut:].any())
    for a, b in zip(plain, again):
        assert np.array_equal(_bits(a), _bits(b))
