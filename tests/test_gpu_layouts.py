"""Layout variants of the CUDA path against the fp64 oracle: the rotate_half pairing
(pair j = elements j and j + 64 of a head) -- with the head-wide schedule and a 16/24/24
split this is the M-RoPE layout that "Accelerating Video Generation Inference with
Sequential-Parallel 3D Positional Encoding Using a Global Time Index" (Section 3.3.1)
sets beside Wan2.1's complex form -- and the head-major KV cache [B][N][C][D]."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gpu_support import PATHS, assert_close, kernel_path, to_bits, to_device, to_f64, torch_dtype
from rotary_position_encoding_b200 import rope3d, workloads as wl

pytestmark = pytest.mark.gpu

D = wl.HEAD_DIM
HALF, ADJ = rope3d.ROPE3D_PAIRING_HALF, rope3d.ROPE3D_PAIRING_ADJACENT
TOKEN, HEAD = rope3d.ROPE3D_CACHE_TOKEN_MAJOR, rope3d.ROPE3D_CACHE_HEAD_MAJOR
MROPE = dict(n_t=16, n_h=24, n_w=24, schedule=1)   # M-RoPE split, head-wide schedule
WAN = dict(n_t=22, n_h=21, n_w=21, schedule=0)


def _cache(w, layout):
    shape = (w.B, w.cache_tokens, w.N, D) if layout == TOKEN else (w.B, w.N, w.cache_tokens, D)
    return (torch.zeros(shape, dtype=torch_dtype(w.dtype), device="cuda"),
            torch.zeros(shape, dtype=torch_dtype(w.dtype), device="cuda"))


def _run(w, dev, chunk, tables, wq, wk, kc, vc, pairing, layout, trig=rope3d.ROPE3D_TRIG_TABLE,
         tb=None, te=None):
    q, k, v = dev
    qo = torch.empty_like(q)
    rope3d.rope3d_qk_norm_rope_append_ex(
        q, k, v, qo, chunk.token_begin if tb is None else tb,
        chunk.token_end if te is None else te, chunk.frame_offset, w.T, w.H, w.W, wq, wk,
        w.eps, kc, vc, chunk.slot, tables, trig, pairing, layout)
    return qo


def _tables(w, freq, max_t):
    return rope3d.rope3d_tables_init(n_t=freq["n_t"], n_h=freq["n_h"], n_w=freq["n_w"],
                                     max_t=max_t, max_h=w.H, max_w=w.W,
                                     schedule=freq["schedule"])


@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("trig", [rope3d.ROPE3D_TRIG_TABLE, rope3d.ROPE3D_TRIG_ONTHEFLY])
@pytest.mark.parametrize("layout", [TOKEN, HEAD])
def test_mrope_480p_chunk_every_element(path, trig, layout):
    w = wl.chunk_480p()
    chunk = w.chunks[4]  # start frame 12
    raw = wl.chunk_inputs(w, 4)
    dev = [to_device(x, w.dtype) for x in raw]
    wq_np, wk_np = wl.norm_weights(w.seed, w.dim)
    wq, wk = torch.from_numpy(wq_np).cuda(), torch.from_numpy(wk_np).cuda()
    tables = _tables(w, MROPE, 21)
    kc, vc = _cache(w, layout)
    with kernel_path(PATHS[path]):
        qo = _run(w, dev, chunk, tables, wq, wk, kc, vc, HALF, layout, trig)
    torch.cuda.synchronize()
    f64 = [wl.to_f64(x, w.dtype) for x in raw]
    shape = (w.B, w.cache_tokens, w.N, D) if layout == TOKEN else (w.B, w.N, w.cache_tokens, D)
    kr, vr = np.zeros(shape), np.zeros(shape)
    ref_q = oracle.default().qk_norm_rope_append_layout(
        *f64, chunk.token_begin, chunk.token_end, chunk.frame_offset, w.T, w.H, w.W,
        wq_np.astype(np.float64), wk_np.astype(np.float64), w.eps, kr, vr, chunk.slot,
        HALF, layout, **MROPE)
    assert_close(to_f64(qo), ref_q, "bf16", "q_out")
    rows = np.arange(chunk.slot, chunk.slot + chunk.token_end)
    if layout == TOKEN:
        assert_close(to_f64(kc[:, rows]), kr[:, rows], "bf16", "k_cache")
        assert np.array_equal(to_f64(vc[:, rows]), vr[:, rows])
    else:
        assert_close(to_f64(kc[:, :, rows]), kr[:, :, rows], "bf16", "k_cache (head-major)")
        assert np.array_equal(to_f64(vc[:, :, rows]), vr[:, :, rows])


@pytest.mark.parametrize("dtype,N", [("f32", 2), ("f32", 3), ("bf16", 1), ("bf16", 5),
                                     ("bf16", 40), ("bf16", 128)])
@pytest.mark.parametrize("pairing", [ADJ, HALF])
@pytest.mark.parametrize("layout", [TOKEN, HEAD])
def test_variants_small_every_element(dtype, N, pairing, layout):
    T, H, W, s, C, slot, B = 2, 3, 5, 4, 64, 50, 2
    n = T * H * W
    rng = np.random.default_rng(300 + N)
    raw = [wl.normal_tensor(rng, (B, n, N, D), dtype) for _ in range(3)]
    wq_np = rng.uniform(0.5, 1.5, N * D).astype(np.float32)
    wk_np = rng.uniform(0.5, 1.5, N * D).astype(np.float32)
    dev = [to_device(x, dtype) for x in raw]
    shape = (B, C, N, D) if layout == TOKEN else (B, N, C, D)
    kc = torch.full(shape, 2.0, dtype=torch_dtype(dtype), device="cuda")
    vc = torch.full(shape, -2.0, dtype=torch_dtype(dtype), device="cuda")
    tables = rope3d.rope3d_tables_init(max_t=6, max_h=H, max_w=W)
    qo = torch.empty_like(dev[0])
    rope3d.rope3d_qk_norm_rope_append_ex(dev[0], dev[1], dev[2], qo, 0, n, s, T, H, W,
                                         torch.from_numpy(wq_np).cuda(),
                                         torch.from_numpy(wk_np).cuda(), 1e-6, kc, vc, slot,
                                         tables, rope3d.ROPE3D_TRIG_TABLE, pairing, layout)
    torch.cuda.synchronize()
    f64 = [wl.to_f64(x, dtype) for x in raw]
    kr, vr = np.full(shape, 2.0), np.full(shape, -2.0)
    ref_q = oracle.default().qk_norm_rope_append_layout(
        *f64, 0, n, s, T, H, W, wq_np.astype(np.float64), wk_np.astype(np.float64), 1e-6, kr,
        vr, slot, pairing, layout)
    assert_close(to_f64(qo), ref_q, dtype, "q_out")
    assert_close(to_f64(kc), kr, dtype, "k_cache (written and untouched rows)")
    assert np.array_equal(to_f64(vc), vr)


@pytest.mark.slow
@pytest.mark.parametrize("path", sorted(PATHS))
def test_half_pairing_720p_sampled_rows(path):
    w = wl.chunk_720p()
    chunk = w.chunks[6]
    raw = wl.chunk_inputs(w, 6)
    dev = [to_device(x, w.dtype) for x in raw]
    wq_np, wk_np = wl.norm_weights(w.seed, w.dim)
    tables = _tables(w, WAN, 21)
    kc, vc = _cache(w, HEAD)
    with kernel_path(PATHS[path]):
        qo = _run(w, dev, chunk, tables, torch.from_numpy(wq_np).cuda(),
                  torch.from_numpy(wk_np).cuda(), kc, vc, HALF, HEAD)
    torch.cuda.synchronize()
    orc = oracle.default()
    sample = sorted(set(np.random.default_rng(7).integers(0, 10800, 40).tolist()) | {0, 10799})
    got_q = to_f64(qo[0, sample])
    for si, r in enumerate(sample):
        q64, k64, v64 = (wl.to_f64(x[0, r], w.dtype) for x in raw)
        eq, ek, ev, pos = orc.token_pairing(q64, k64, v64, r, chunk.frame_offset, w.T, w.H, w.W,
                                            wq_np.astype(np.float64), wk_np.astype(np.float64),
                                            w.eps, chunk.slot, w.cache_tokens, HALF, **WAN)
        assert_close(got_q[si], eq, "bf16", f"q row {r}")
        assert_close(to_f64(kc[0, :, pos[3]]), ek, "bf16", f"k row {r} (head-major)")
        assert np.array_equal(to_bits(vc[0, :, pos[3]]), raw[2][0, r])


@pytest.mark.slow
def test_half_head_major_slices_bit_identical_and_layouts_transpose():
    w = wl.full_480p()
    n = w.tokens_per_chunk
    chunk = w.chunks[0]
    raw = wl.chunk_inputs(w, 0)
    dev = [to_device(x, w.dtype) for x in raw]
    wq_np, wk_np = wl.norm_weights(w.seed, w.dim)
    wq, wk = torch.from_numpy(wq_np).cuda(), torch.from_numpy(wk_np).cuda()
    tables = _tables(w, MROPE, 21)
    kc_w, vc_w = _cache(w, HEAD)
    q_w = _run(w, dev, chunk, tables, wq, wk, kc_w, vc_w, HALF, HEAD)
    kc_s, vc_s = _cache(w, HEAD)
    q_s = torch.empty_like(q_w)
    for (a, e) in wl.slices(n, 8):
        sub = [x[:, a:e].contiguous() for x in dev]
        q_s[:, a:e] = _run(w, sub, chunk, tables, wq, wk, kc_s, vc_s, HALF, HEAD, tb=a, te=e)
    kc_t, vc_t = _cache(w, TOKEN)
    q_t = _run(w, dev, chunk, tables, wq, wk, kc_t, vc_t, HALF, TOKEN)
    torch.cuda.synchronize()
    i16 = torch.int16
    assert torch.equal(q_w.view(i16), q_s.view(i16))
    assert torch.equal(kc_w.view(i16), kc_s.view(i16)) and torch.equal(vc_w.view(i16), vc_s.view(i16))
    assert torch.equal(q_w.view(i16), q_t.view(i16))
    assert torch.equal(kc_w.view(i16), kc_t.transpose(1, 2).contiguous().view(i16))
    assert torch.equal(vc_w.view(i16), vc_t.transpose(1, 2).contiguous().view(i16))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("trig", [rope3d.ROPE3D_TRIG_TABLE, rope3d.ROPE3D_TRIG_ONTHEFLY])
def test_apply_half_pairing(dtype, trig):
    T, H, W, s = 3, 30, 52, 9
    tb, te = 100, 1777
    rng = np.random.default_rng(13)
    raw = wl.normal_tensor(rng, (2, te - tb, 3, D), dtype)
    x = to_device(raw, dtype)
    tables = rope3d.rope3d_tables_init(n_t=16, n_h=24, n_w=24, max_t=12, max_h=H, max_w=W,
                                       schedule=1)
    out = torch.empty_like(x)
    rope3d.rope3d_apply_ex(x, out, tb, te, s, T, H, W, tables, trig, HALF)
    torch.cuda.synchronize()
    ref = oracle.default().apply_pairing(wl.to_f64(raw, dtype), tb, te, s, T, H, W, HALF,
                                         **MROPE)
    assert_close(to_f64(out), ref, dtype, "apply (half pairing)")


def test_invalid_options_rejected():
    lib = rope3d.load_library()
    w = wl.tiny()
    dev = [to_device(x, w.dtype) for x in wl.chunk_inputs(w, 0)]
    qo = torch.full_like(dev[0], 4.0)
    kc = torch.zeros((1, 144, 2, D), device="cuda")
    wq = torch.ones(256, device="cuda")
    tables = rope3d.rope3d_tables_init(max_t=6, max_h=4, max_w=6)
    reserved_set = rope3d.rope3d_options()
    reserved_set.reserved[1] = 1
    for opts in (rope3d.rope3d_options(2, 0), rope3d.rope3d_options(0, 5),
                 rope3d.rope3d_options(0, 0, 7), rope3d.rope3d_options(0, 0, 0, 1),
                 reserved_set):
        rc = lib.rope3d_qk_norm_rope_append_ex(
            dev[0].data_ptr(), dev[1].data_ptr(), dev[2].data_ptr(), qo.data_ptr(), 1, 2, D,
            rope3d.ROPE3D_F32, 0, 72, 0, 3, 4, 6, wq.data_ptr(), wq.data_ptr(), 1e-6,
            kc.data_ptr(), kc.data_ptr() + kc.numel() * 4 // 2, 72, 0, tables.handle, 0,
            ctypes.byref(opts), torch.cuda.current_stream().cuda_stream)
        assert rc == rope3d.ROPE3D_EINVAL, rope3d.rope3d_last_error()
    # the rotation alone takes no cache layout
    rc = lib.rope3d_apply_ex(dev[0].data_ptr(), qo.data_ptr(), 1, 2, D, rope3d.ROPE3D_F32, 0, 72,
                             0, 3, 4, 6, tables.handle, 0,
                             ctypes.byref(rope3d.rope3d_options(0, HEAD)),
                             torch.cuda.current_stream().cuda_stream)
    assert rc == rope3d.ROPE3D_EINVAL
    torch.cuda.synchronize()
    assert bool((qo == 4.0).all())
