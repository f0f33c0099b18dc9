"""The no-allocation entry point against the ordinary one.

rope3d_qk_norm_rope_append_noalloc is for callers that cannot call cudaMalloc -- for
example a host framework that owns all device memory through its own allocator, or a
process whose caching allocator already holds the free memory -- and so cannot build a
rope3d_tables object (its init allocates the cos/sin tables and a status word).  The
variant keeps those in a fixed device array inside the library instead.  These tests
call it through the C ABI on two calls in a row (two chunks with different start frames,
so the second call must replace the first call's table rows) and compare every output
with rope3d_qk_norm_rope_append on tables built from the same configuration, within the
bf16 tolerance of the other tests (the two are in fact bit-identical).  The file is named
to be collected last and passes alone in a fresh process as well as after the others."""
import ctypes

import numpy as np
import pytest
import torch

from gpu_support import assert_close, kernel_path, to_device, to_f64
from rotary_position_encoding_b200 import rope3d, workloads as wl

pytestmark = pytest.mark.gpu


def _call_noalloc(lib, q, k, v, qo, chunk, w, wq, wk, kc, vc, trig):
    return lib.rope3d_qk_norm_rope_append_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), qo.data_ptr(), w.B, w.N, wl.HEAD_DIM,
        rope3d.ROPE3D_BF16, chunk.token_begin, chunk.token_end, chunk.frame_offset, w.T, w.H,
        w.W, wq.data_ptr(), wk.data_ptr(), ctypes.c_float(w.eps), kc.data_ptr(), vc.data_ptr(),
        w.cache_tokens, chunk.slot, 22, 21, 21, ctypes.c_double(10000.0),
        rope3d.ROPE3D_SCHEDULE_PER_AXIS, trig, torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("trig", [rope3d.ROPE3D_TRIG_TABLE, rope3d.ROPE3D_TRIG_ONTHEFLY])
def test_noalloc_matches_existing_entry_point_on_two_calls(trig):
    lib = rope3d.load_library()
    w = wl.chunk_480p()
    wq_np, wk_np = wl.norm_weights(w.seed, w.dim)
    wq, wk = torch.from_numpy(wq_np).cuda(), torch.from_numpy(wk_np).cuda()
    shape = (w.B, w.cache_tokens, w.N, wl.HEAD_DIM)
    kc_ref = torch.zeros(shape, dtype=torch.bfloat16, device="cuda")
    vc_ref = torch.zeros_like(kc_ref)
    kc_new = torch.zeros_like(kc_ref)
    vc_new = torch.zeros_like(kc_ref)
    tables = rope3d.rope3d_tables_init(max_t=21, max_h=w.H, max_w=w.W)
    for ci in (2, 5):  # start frames 6 and 15: the second call needs other table rows
        chunk = w.chunks[ci]
        q, k, v = (to_device(x, w.dtype) for x in wl.chunk_inputs(w, ci))
        q_ref = torch.empty_like(q)
        rope3d.rope3d_qk_norm_rope_append(q, k, v, q_ref, chunk.token_begin, chunk.token_end,
                                          chunk.frame_offset, w.T, w.H, w.W, wq, wk, w.eps,
                                          kc_ref, vc_ref, chunk.slot, tables, trig)
        q_new = torch.full_like(q, 9.0)
        rc = _call_noalloc(lib, q, k, v, q_new, chunk, w, wq, wk, kc_new, vc_new, trig)
        assert rc == rope3d.ROPE3D_OK, rope3d.rope3d_last_error()
        torch.cuda.synchronize()
        assert_close(to_f64(q_new), to_f64(q_ref), "bf16", f"q_out, call for chunk {ci}")
        assert_close(to_f64(kc_new), to_f64(kc_ref), "bf16", f"k_cache after chunk {ci}")
        assert torch.equal(vc_new.view(torch.int16), vc_ref.view(torch.int16))
        assert torch.equal(q_new.view(torch.int16), q_ref.view(torch.int16))
    tables.close()


def test_noalloc_rejects_tables_beyond_its_scratch():
    lib = rope3d.load_library()
    # 21 frames of a 45 x 80 grid need 21*22 + 45*21 + 80*21 = 3087 entries: fits.  The
    # range [0, 4) of a 400 x 400 grid touches frame 0 only, and needs 1*22 + 2*400*21 =
    # 16822 entries (frames touched * n_t + H * n_h + W * n_w): more than the 8192 it holds
    w = wl.chunk_480p()
    T, H, W = 3, 400, 400
    q = torch.zeros((1, 4, 2, wl.HEAD_DIM), dtype=torch.bfloat16, device="cuda")
    qo = torch.full_like(q, 7.0)
    kc = torch.full((1, 8, 2, wl.HEAD_DIM), 5.0, dtype=torch.bfloat16, device="cuda")
    vc = torch.full_like(kc, 5.0)
    wq = torch.ones(2 * wl.HEAD_DIM, device="cuda")
    chunk = wl.Chunk(frame_offset=0, slot=0, token_begin=0, token_end=4)
    w.B, w.N, w.T, w.H, w.W, w.cache_tokens = 1, 2, T, H, W, 8
    rc = _call_noalloc(lib, q, q, q, qo, chunk, w, wq, wq, kc, vc, rope3d.ROPE3D_TRIG_TABLE)
    assert rc == rope3d.ROPE3D_ERANGE
    assert "8192" in rope3d.rope3d_last_error()
    torch.cuda.synchronize()
    assert bool((qo.float() == 7.0).all()) and bool((kc.float() == 5.0).all())
    # the same call computing cos/sin on the fly needs no table rows and runs
    rc = _call_noalloc(lib, q, q, q, qo, chunk, w, wq, wq, kc, vc, rope3d.ROPE3D_TRIG_ONTHEFLY)
    assert rc == rope3d.ROPE3D_OK, rope3d.rope3d_last_error()
    torch.cuda.synchronize()
    assert bool((qo.float() == 0.0).all())


def test_noalloc_wrapper_checks_tensors_before_the_call():
    """The Python wrapper checks shapes and dtypes as the ordinary wrapper does: the C ABI
    sees only pointers and sizes, so a short q or a cache of another dtype would otherwise
    make the kernel read or write past the end of a tensor."""
    q = torch.zeros((1, 4, 2, wl.HEAD_DIM), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((1, 8, 2, wl.HEAD_DIM), dtype=torch.bfloat16, device="cuda")
    wq = torch.ones(2 * wl.HEAD_DIM, device="cuda")
    args = dict(frame_offset=0, T=1, H=2, W=4, q_norm_w=wq, k_norm_w=wq, eps=1e-6, slot=0)
    with pytest.raises(ValueError):  # the range holds 5 rows, q holds 4
        rope3d.rope3d_qk_norm_rope_append_noalloc(q, q, q, q.clone(), token_begin=0,
                                                  token_end=5, k_cache=kc, v_cache=kc.clone(),
                                                  **args)
    with pytest.raises(TypeError):  # fp32 caches with bf16 q
        rope3d.rope3d_qk_norm_rope_append_noalloc(q, q, q, q.clone(), token_begin=0,
                                                  token_end=4, k_cache=kc.float(),
                                                  v_cache=kc.float(), **args)
    with pytest.raises(ValueError):  # weights of the wrong length
        rope3d.rope3d_qk_norm_rope_append_noalloc(q, q, q, q.clone(), token_begin=0,
                                                  token_end=4, k_cache=kc, v_cache=kc.clone(),
                                                  **dict(args, q_norm_w=wq[:8]))


def test_noalloc_status_reports_a_wait_that_timed_out():
    """The status word of the no-allocation entry point: a bounded wait of the ring kernel
    that never fills (a test setting makes every stage wait for 16 bytes its copies never
    deliver; every copy lands, only the wait runs out) is reported by
    rope3d_noalloc_check_status; the read clears it, and the next call is bit-identical to
    the ordinary entry point."""
    w = wl.chunk_480p()
    wq_np, wk_np = wl.norm_weights(w.seed, w.dim)
    wq, wk = torch.from_numpy(wq_np).cuda(), torch.from_numpy(wk_np).cuda()
    shape = (w.B, w.cache_tokens, w.N, wl.HEAD_DIM)
    kc, vc = (torch.zeros(shape, dtype=torch.bfloat16, device="cuda") for _ in range(2))
    chunk = w.chunks[1]
    q, k, v = (to_device(x, w.dtype) for x in wl.chunk_inputs(w, 1))
    q_new = torch.empty_like(q)
    args = dict(frame_offset=chunk.frame_offset, T=w.T, H=w.H, W=w.W, q_norm_w=wq,
                k_norm_w=wk, eps=w.eps, slot=chunk.slot)
    assert rope3d.rope3d_noalloc_check_status() == rope3d.ROPE3D_OK
    rope3d.rope3d_testing_set_waits(20_000_000, 16)  # 20 ms, 16 bytes never delivered
    try:
        with kernel_path(rope3d.ROPE3D_PATH_TMA):
            rope3d.rope3d_qk_norm_rope_append_noalloc(
                q, k, v, q_new, chunk.token_begin, chunk.token_end, k_cache=kc, v_cache=vc,
                **args)
        status = rope3d.rope3d_noalloc_check_status()
    finally:
        rope3d.rope3d_testing_set_waits(0, 0)
    assert status == rope3d.ROPE3D_ETIMEOUT
    assert rope3d.rope3d_noalloc_check_status() == rope3d.ROPE3D_OK  # cleared by the read
    with kernel_path(rope3d.ROPE3D_PATH_TMA):
        rope3d.rope3d_qk_norm_rope_append_noalloc(
            q, k, v, q_new, chunk.token_begin, chunk.token_end, k_cache=kc, v_cache=vc, **args)
    assert rope3d.rope3d_noalloc_check_status() == rope3d.ROPE3D_OK
    tables = rope3d.rope3d_tables_init(max_t=21, max_h=w.H, max_w=w.W)
    kr, vr = (torch.zeros_like(kc) for _ in range(2))
    q_ref = torch.empty_like(q)
    rope3d.rope3d_qk_norm_rope_append(q, k, v, q_ref, chunk.token_begin, chunk.token_end,
                                      chunk.frame_offset, w.T, w.H, w.W, wq, wk, w.eps, kr, vr,
                                      chunk.slot, tables)
    torch.cuda.synchronize()
    assert torch.equal(q_new.view(torch.int16), q_ref.view(torch.int16))
    assert torch.equal(kc.view(torch.int16), kr.view(torch.int16))
    assert torch.equal(vc.view(torch.int16), vr.view(torch.int16))
    tables.close()
