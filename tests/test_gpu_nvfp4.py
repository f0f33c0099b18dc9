"""Quantize-on-append NVFP4 KV cache on the GPU against the oracle.

Each block of 16 elements of a head holds E2M1 codes under one E4M3 block scale and the
tensor's fp32 scale g.  V is quantized from its exact input values, so its codes and block
scales must match the oracle bit for bit.  K is quantized from its fp32 value after RMSNorm
and RoPE; the GPU's fp32 K and the oracle's fp64 K rounded to fp32 can differ in the last
bits, so a K block scale may differ where amax / (6 g) sits at an E4M3 rounding midpoint,
and a K code may differ where x r sits at an E2M1 rounding midpoint.  Every other code must
match, and every dequantized K value must lie within half an E2M1 step (times the block
scale and g) of the oracle's K, or within the saturation distance where the block's
largest value exceeds 6 steps."""
import numpy as np
import pytest
import torch

import oracle
from gpu_support import PATHS, assert_close, kernel_path, to_device, to_f64
from rotary_position_encoding_b200 import rope3d, workloads as wl

pytestmark = pytest.mark.gpu

D = wl.HEAD_DIM
TOKEN, HEAD = rope3d.ROPE3D_CACHE_TOKEN_MAJOR, rope3d.ROPE3D_CACHE_HEAD_MAJOR
ADJ, HALF = rope3d.ROPE3D_PAIRING_ADJACENT, rope3d.ROPE3D_PAIRING_HALF
_ORC = oracle.default()
E4M3 = np.array([_ORC.e4m3_value(c) for c in range(256)])
E2M1 = np.array([_ORC.e2m1_value(c) for c in range(16)])


def _alloc(w, layout):
    heads = (w.B, w.cache_tokens, w.N) if layout == TOKEN else (w.B, w.N, w.cache_tokens)
    dev = [torch.zeros(heads + (D // 2,), dtype=torch.uint8, device="cuda") for _ in range(2)]
    sc = [torch.zeros(heads + (D // 16,), dtype=torch.uint8, device="cuda") for _ in range(2)]
    return dev, sc


def _run_gpu(w, dev_in, chunk, tables, wq, wk, caches, scales, pairing, layout, kg, vg,
             tb=None, te=None):
    q, k, v = dev_in
    qo = torch.empty_like(q)
    rope3d.rope3d_qk_norm_rope_append_ex(
        q, k, v, qo, chunk.token_begin if tb is None else tb, chunk.token_end if te is None else te,
        chunk.frame_offset, w.T, w.H, w.W, wq, wk, w.eps, caches[0], caches[1], chunk.slot,
        tables, rope3d.ROPE3D_TRIG_TABLE, pairing, layout, k_scale=scales[0], v_scale=scales[1],
        k_global=kg, v_global=vg)
    return qo


def _oracle(w, raw, chunk, wq_np, wk_np, pairing, layout, heads, kg, vg):
    f64 = [wl.to_f64(x, w.dtype) for x in raw]
    codes = [np.zeros(heads + (D // 2,), dtype=np.uint8) for _ in range(2)]
    sc = [np.zeros(heads + (D // 16,), dtype=np.uint8) for _ in range(2)]
    kf = np.zeros(heads + (D,))
    vf = np.zeros(heads + (D,))
    args = (chunk.token_begin, chunk.token_end, chunk.frame_offset, w.T, w.H, w.W,
            wq_np.astype(np.float64), wk_np.astype(np.float64), w.eps)
    q_ref = _ORC.qk_norm_rope_append_nvfp4(*f64, *args, codes[0], codes[1], sc[0], sc[1],
                                           chunk.slot, kg or 1.0, vg or 1.0, pairing, layout)
    _ORC.qk_norm_rope_append_layout(*f64, *args, kf, vf, chunk.slot, pairing, layout)
    return q_ref, codes, sc, kf


def _nibbles(codes):
    return np.stack([codes & 15, codes >> 4], axis=-1).reshape(codes.shape[:-1] + (-1,))


def _check_k(codes, scales, ref_codes, ref_scales, ref_k, g):
    """codes [..., 64], scales [..., 8] (GPU and oracle) of the written rows; ref_k the
    oracle's fp64 K [..., 128]."""
    nib, ref_nib = _nibbles(codes), _nibbles(ref_codes)
    kb = ref_k.reshape(ref_k.shape[:-1] + (8, 16))
    amax = np.max(np.abs(kb.astype(np.float32).astype(np.float64)), axis=-1)
    sf = amax / np.float32(6.0 * g)
    diff = scales != ref_scales
    if diff.any():  # only where amax / (6 g) sits at an E4M3 rounding midpoint
        mid = (E4M3[scales[diff]] + E4M3[ref_scales[diff]]) / 2
        assert np.all(np.abs(sf[diff] - mid) <= 1e-5 * mid), "K block scales differ off a midpoint"
    sv = np.where(diff, E4M3[ref_scales], E4M3[scales]) * g  # both sides: the oracle's scale
    nb = nib.reshape(kb.shape)
    rb = ref_nib.reshape(kb.shape)
    same = ~diff[..., None] & np.ones(kb.shape, dtype=bool)
    mism = same & (nb != rb)
    if mism.any():
        x = np.abs(kb / np.where(sv > 0, sv, 1.0)[..., None])[mism]
        mid = (np.abs(E2M1[nb[mism]]) + np.abs(E2M1[rb[mism]])) / 2
        assert np.all(np.abs(x - mid) <= 1e-5 * np.maximum(x, 1.0)), \
            f"{int(mism.sum())} K codes differ away from an E2M1 midpoint"
    # dequantized GPU K against the oracle's K, with the GPU's own block scales
    s_gpu = E4M3[scales] * g
    deq = E2M1[nb] * s_gpu[..., None]
    y = np.abs(kb) / np.where(s_gpu > 0, s_gpu, np.inf)[..., None]
    step = np.where(y < 2, 0.5, np.where(y < 4, 1.0, 2.0))
    bound = np.where(y <= 6, 0.5 * step, y - 6) * s_gpu[..., None]
    bound = bound + 1e-5 * np.maximum(y, 1.0) * s_gpu[..., None] + 1e-6 * np.abs(kb)
    zero_scale = (s_gpu == 0)[..., None] & np.ones(kb.shape, dtype=bool)
    assert np.all((np.abs(deq - kb) <= bound) | zero_scale), "dequantized K outside the bound"
    # a zero block scale means amax / (6 g) rounded below half the smallest E4M3 step
    assert np.all(np.abs(kb[zero_scale]) <= 6 * g * 2.0 ** -10 * (1 + 1e-5)), "tiny block"


def _written(layout, rows):
    return (slice(None), rows) if layout == TOKEN else (slice(None), slice(None), rows)


@pytest.mark.parametrize("layout", [TOKEN, HEAD])
@pytest.mark.parametrize("pairing", [ADJ, HALF])
@pytest.mark.parametrize("kg,vg", [(0.0, 0.0), (0.4, 3.0)])
def test_nvfp4_cache_480p_chunk(layout, pairing, kg, vg):
    w = wl.chunk_480p()
    chunk = w.chunks[3]
    raw = wl.chunk_inputs(w, 3)
    dev_in = [to_device(x, w.dtype) for x in raw]
    wq_np, wk_np = wl.norm_weights(w.seed, w.dim)
    tables = rope3d.rope3d_tables_init(max_t=21, max_h=w.H, max_w=w.W)
    caches, scales = _alloc(w, layout)
    qo = _run_gpu(w, dev_in, chunk, tables, torch.from_numpy(wq_np).cuda(),
                  torch.from_numpy(wk_np).cuda(), caches, scales, pairing, layout, kg, vg)
    torch.cuda.synchronize()
    assert rope3d.rope3d_testing_last_path() == rope3d.ROPE3D_PATH_REGISTERS
    heads = tuple(caches[0].shape[:3])
    q_ref, ref_codes, ref_sc, ref_k = _oracle(w, raw, chunk, wq_np, wk_np, pairing, layout,
                                              heads, kg, vg)
    assert_close(to_f64(qo), q_ref, "bf16", "q_out")
    rows = np.arange(chunk.slot, chunk.slot + chunk.token_end)
    sel = _written(layout, rows)
    assert np.array_equal(caches[1].cpu().numpy(), ref_codes[1]), "V codes"
    assert np.array_equal(scales[1].cpu().numpy(), ref_sc[1]), "V block scales"
    _check_k(caches[0].cpu().numpy()[sel], scales[0].cpu().numpy()[sel], ref_codes[0][sel],
             ref_sc[0][sel], ref_k[sel], kg or 1.0)
    other = np.ones(w.cache_tokens, dtype=bool)
    other[rows] = False
    osel = _written(layout, other)
    assert not caches[0].cpu().numpy()[osel].any() and not scales[0].cpu().numpy()[osel].any()


@pytest.mark.parametrize("dtype,N", [("f32", 2), ("f32", 3), ("bf16", 1), ("bf16", 5),
                                     ("bf16", 40)])
@pytest.mark.parametrize("pairing", [ADJ, HALF])
def test_nvfp4_cache_small_shapes(dtype, N, pairing):
    w = wl.Workload("small", B=2, T=2, H=3, W=5, N=N, dtype=dtype, cache_tokens=64, seed=450 + N,
                    chunks=[wl.Chunk(4, 50, 0, 30)])
    chunk = w.chunks[0]
    rng = np.random.default_rng(w.seed)
    raw = [wl.normal_tensor(rng, (w.B, 30, N, D), dtype) for _ in range(3)]
    wq_np = rng.uniform(0.5, 1.5, N * D).astype(np.float32)
    wk_np = rng.uniform(0.5, 1.5, N * D).astype(np.float32)
    dev_in = [to_device(x, dtype) for x in raw]
    tables = rope3d.rope3d_tables_init(max_t=6, max_h=w.H, max_w=w.W)
    for layout in (TOKEN, HEAD):
        caches, scales = _alloc(w, layout)
        qo = _run_gpu(w, dev_in, chunk, tables, torch.from_numpy(wq_np).cuda(),
                      torch.from_numpy(wk_np).cuda(), caches, scales, pairing, layout, 0.7, 1.3)
        torch.cuda.synchronize()
        heads = tuple(caches[0].shape[:3])
        q_ref, ref_codes, ref_sc, ref_k = _oracle(w, raw, chunk, wq_np, wk_np, pairing, layout,
                                                  heads, 0.7, 1.3)
        assert_close(to_f64(qo), q_ref, dtype, "q_out")
        assert np.array_equal(caches[1].cpu().numpy(), ref_codes[1])
        assert np.array_equal(scales[1].cpu().numpy(), ref_sc[1])
        rows = np.array([(chunk.slot + i) % w.cache_tokens for i in range(30)])
        sel = _written(layout, rows)
        _check_k(caches[0].cpu().numpy()[sel], scales[0].cpu().numpy()[sel], ref_codes[0][sel],
                 ref_sc[0][sel], ref_k[sel], 0.7)


def test_nvfp4_extreme_blocks_v_bit_exact():
    """V blocks that are all zero, hold one huge value among tiny ones, sit below the
    smallest E4M3 scale, or saturate the block scale: codes and scales match the oracle."""
    w = wl.Workload("edge", B=1, T=1, H=2, W=4, N=2, dtype="bf16", cache_tokens=8, seed=9,
                    chunks=[wl.Chunk(0, 0, 0, 8)])
    chunk = w.chunks[0]
    rng = np.random.default_rng(9)
    x = rng.standard_normal((1, 8, 2, D)).astype(np.float32)
    x[0, 0, 0, :16] = 0.0
    x[0, 1, 0, :16] = 1e-4
    x[0, 1, 0, 3] = 3000.0
    x[0, 2, 1, 16:32] *= 1e-6
    x[0, 3, 1, 32:48] *= 1e4
    x[0, 4, 0, 48:64] = -0.0
    raw = [wl.normal_tensor(rng, x.shape, "bf16"), wl.normal_tensor(rng, x.shape, "bf16"),
           wl.f32_to_bf16_bits(x)]
    dev_in = [to_device(a, "bf16") for a in raw]
    wq_np = np.ones(2 * D, dtype=np.float32)
    tables = rope3d.rope3d_tables_init(max_t=1, max_h=2, max_w=4)
    caches, scales = _alloc(w, TOKEN)
    wq = torch.from_numpy(wq_np).cuda()
    _run_gpu(w, dev_in, chunk, tables, wq, wq, caches, scales, ADJ, TOKEN, 0.0, 0.0)
    torch.cuda.synchronize()
    _, ref_codes, ref_sc, _ = _oracle(w, raw, chunk, wq_np, wq_np, ADJ, TOKEN,
                                      tuple(caches[0].shape[:3]), 0.0, 0.0)
    assert np.array_equal(caches[1].cpu().numpy(), ref_codes[1])
    assert np.array_equal(scales[1].cpu().numpy(), ref_sc[1])


@pytest.mark.slow
def test_nvfp4_slices_bit_identical_to_whole():
    w = wl.full_480p()
    n = w.tokens_per_chunk
    chunk = w.chunks[0]
    raw = wl.chunk_inputs(w, 0)
    dev_in = [to_device(x, w.dtype) for x in raw]
    wq_np, wk_np = wl.norm_weights(w.seed, w.dim)
    wq, wk = torch.from_numpy(wq_np).cuda(), torch.from_numpy(wk_np).cuda()
    tables = rope3d.rope3d_tables_init(max_t=21, max_h=w.H, max_w=w.W)
    c_w, s_w = _alloc(w, HEAD)
    q_w = _run_gpu(w, dev_in, chunk, tables, wq, wk, c_w, s_w, ADJ, HEAD, 0.5, 2.0)
    c_s, s_s = _alloc(w, HEAD)
    q_s = torch.empty_like(q_w)
    for (a, e) in wl.slices(n, 8):
        sub = [x[:, a:e].contiguous() for x in dev_in]
        q_s[:, a:e] = _run_gpu(w, sub, chunk, tables, wq, wk, c_s, s_s, ADJ, HEAD, 0.5, 2.0,
                               tb=a, te=e)
    torch.cuda.synchronize()
    assert torch.equal(q_w.view(torch.int16), q_s.view(torch.int16))
    for a, b in zip(c_w + s_w, c_s + s_s):
        assert torch.equal(a, b)


def test_nvfp4_option_errors():
    import ctypes
    w = wl.tiny()
    dev_in = [to_device(x, w.dtype) for x in wl.chunk_inputs(w, 0)]
    tables = rope3d.rope3d_tables_init(max_t=6, max_h=4, max_w=6)
    caches = [torch.zeros((1, 144, 2, D // 2), dtype=torch.uint8, device="cuda")
              for _ in range(2)]
    sc = [torch.zeros((1, 144, 2, D // 16), dtype=torch.uint8, device="cuda") for _ in range(2)]
    qo = torch.empty_like(dev_in[0])
    wq = torch.ones(256, device="cuda")

    def status(**kw):
        with pytest.raises(rope3d.Rope3dError) as e:
            rope3d.rope3d_qk_norm_rope_append_ex(*dev_in, qo, 0, 72, 0, 3, 4, 6, wq, wq, 1e-6,
                                                 caches[0], caches[1], 0, tables, **kw)
        return e.value.status

    assert status(k_scale=sc[0], v_scale=sc[0]) == rope3d.ROPE3D_EOVERLAP
    assert status(k_scale=sc[0], v_scale=sc[1], k_global=-1.0) == rope3d.ROPE3D_EINVAL
    assert status(k_scale=sc[0], v_scale=sc[1], v_global=float("nan")) == rope3d.ROPE3D_EINVAL
    assert status(k_scale=sc[0], v_scale=sc[1], k_global=float("inf")) == rope3d.ROPE3D_EINVAL
    with kernel_path(PATHS["tma"]):  # the ring kernel has no NVFP4 form
        assert status(k_scale=sc[0], v_scale=sc[1]) == rope3d.ROPE3D_EINVAL
    # the C entry point directly: a misaligned block-scale array, a global scale without
    # an NVFP4 cache
    lib = rope3d.load_library()
    opts = rope3d.rope3d_options(0, TOKEN, rope3d.ROPE3D_CACHE_NVFP4, 0, sc[0].data_ptr() + 4,
                                 sc[1].data_ptr())
    args = (dev_in[0].data_ptr(), dev_in[1].data_ptr(), dev_in[2].data_ptr(), qo.data_ptr(), 1, 2,
            D, rope3d.ROPE3D_F32, 0, 72, 0, 3, 4, 6, wq.data_ptr(), wq.data_ptr(), 1e-6,
            caches[0].data_ptr(), caches[1].data_ptr(), 144, 0, tables.handle, 0)
    assert lib.rope3d_qk_norm_rope_append_ex(*args, ctypes.byref(opts), None) == rope3d.ROPE3D_EALIGN
    opts = rope3d.rope3d_options(0, TOKEN, rope3d.ROPE3D_CACHE_SAME)
    opts.nvfp4_k_global = 2.0
    assert lib.rope3d_qk_norm_rope_append_ex(*args, ctypes.byref(opts), None) == rope3d.ROPE3D_EINVAL
    torch.cuda.synchronize()
