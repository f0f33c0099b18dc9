"""Quantize-on-append FP8 E4M3 KV cache on the GPU against the oracle.

Scales are powers of two, so the scaling is exact.  V is quantized from its exact input
values, so its codes and scales must match the oracle bit for bit.  K is quantized from its
fp32 value after RMSNorm and RoPE: the GPU's fp32 K and the oracle's fp64 K (rounded to
fp32) can differ in the last bits, so a K scale may differ where the head's amax sits at
a power-of-two boundary and a K code may differ where x / scale sits at a rounding
midpoint; every other code must match, and every dequantized K value must lie within half
an E4M3 step of the oracle's K."""
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
E4M3 = np.array([oracle.default().e4m3_value(c) for c in range(256)])


def _alloc(w, layout):
    shape = (w.B, w.cache_tokens, w.N, D) if layout == TOKEN else (w.B, w.N, w.cache_tokens, D)
    sshape = shape[:3]
    dev = [torch.zeros(shape, dtype=torch.uint8, device="cuda") for _ in range(2)]
    sc = [torch.zeros(sshape, dtype=torch.float32, device="cuda") for _ in range(2)]
    host = ([np.zeros(shape, dtype=np.uint8) for _ in range(2)],
            [np.zeros(sshape, dtype=np.float32) for _ in range(2)])
    return dev, sc, host


def _run_gpu(w, dev_in, chunk, tables, wq, wk, caches, scales, pairing, layout, tb=None, te=None):
    q, k, v = dev_in
    qo = torch.empty_like(q)
    rope3d.rope3d_qk_norm_rope_append_ex(
        q, k, v, qo, chunk.token_begin if tb is None else tb, chunk.token_end if te is None else te,
        chunk.frame_offset, w.T, w.H, w.W, wq, wk, w.eps, caches[0], caches[1], chunk.slot,
        tables, rope3d.ROPE3D_TRIG_TABLE, pairing, layout, k_scale=scales[0], v_scale=scales[1])
    return qo


def _check_k(codes, scales, ref_codes, ref_scales, ref_k, rows_sel):
    """K codes equal except at rounding midpoints; dequantized K within half a step."""
    codes, ref_codes, ref_k = codes[rows_sel], ref_codes[rows_sel], ref_k[rows_sel]
    scales, ref_scales = scales[rows_sel], ref_scales[rows_sel]
    same_scale = scales == ref_scales
    if not same_scale.all():  # only where amax sits at a power-of-two boundary of 448
        r = ref_k.reshape(ref_k.shape[:-1] + (-1,))
        amax = np.max(np.abs(r), axis=-1)[~same_scale]
        edge = 448.0 * np.minimum(scales, ref_scales)[~same_scale]
        assert np.all(np.abs(amax - edge) <= 1e-6 * edge), "K scales differ away from an edge"
        keep = same_scale[..., None] & np.ones(codes.shape, dtype=bool)
        codes, ref_codes, ref_k = codes * keep, ref_codes * keep, ref_k * keep
        scales = np.where(same_scale, scales, ref_scales)
    ratio = ref_k / ref_scales[..., None].astype(np.float64)
    mism = codes != ref_codes
    if mism.any():
        a = np.abs(ratio[mism])
        lo = np.array([E4M3[c & 0x7F] for c in ref_codes[mism]])
        other = np.array([E4M3[c & 0x7F] for c in codes[mism]])
        mid = (lo + other) / 2
        # fp32 rounding of K differs between the two sides by ~1e-7 of the row's terms;
        # a small output can come from cancelling terms, so the allowance is absolute
        # below 1 (in units of the scale) and relative above
        assert np.all(np.abs(a - mid) <= 1e-5 * np.maximum(a, 1.0)), \
            f"{int(mism.sum())} K codes differ away from a rounding midpoint"
        assert np.all(np.abs((codes[mism] & 0x7F).astype(int) - (ref_codes[mism] & 0x7F)) == 1)
    deq = E4M3[codes] * scales[..., None].astype(np.float64)
    y = np.abs(ratio)
    step = np.where(y >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(y, 2.0 ** -6))) - 3),
                    2.0 ** -9)
    # half a step, plus the same fp32 allowance as for a midpoint decision above
    bound = (0.5 * step + 1e-5 * np.maximum(y, 1.0)) * scales[..., None] + 1e-6 * np.abs(ref_k)
    assert np.all(np.abs(deq - ref_k) <= bound), "dequantized K outside half an E4M3 step"


def _oracle_fp8(w, raw, chunk, wq_np, wk_np, pairing, layout, shape, tb=None, te=None):
    f64 = [wl.to_f64(x, w.dtype) for x in raw]
    codes = [np.zeros(shape, dtype=np.uint8) for _ in range(2)]
    sc = [np.zeros(shape[:3], dtype=np.float32) for _ in range(2)]
    kf = np.zeros(shape)
    vf = np.zeros(shape)
    orc = oracle.default()
    tb = chunk.token_begin if tb is None else tb
    te = chunk.token_end if te is None else te
    q_ref = orc.qk_norm_rope_append_fp8(*f64, tb, te, chunk.frame_offset, w.T, w.H, w.W,
                                        wq_np.astype(np.float64), wk_np.astype(np.float64), w.eps,
                                        codes[0], codes[1], sc[0], sc[1], chunk.slot, pairing,
                                        layout)
    orc.qk_norm_rope_append_layout(*f64, tb, te, chunk.frame_offset, w.T, w.H, w.W,
                                   wq_np.astype(np.float64), wk_np.astype(np.float64), w.eps, kf,
                                   vf, chunk.slot, pairing, layout)
    return q_ref, codes, sc, kf


@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("layout", [TOKEN, HEAD])
@pytest.mark.parametrize("pairing", [ADJ, HALF])
def test_fp8_cache_480p_chunk(path, layout, pairing):
    w = wl.chunk_480p()
    chunk = w.chunks[3]
    raw = wl.chunk_inputs(w, 3)
    dev_in = [to_device(x, w.dtype) for x in raw]
    wq_np, wk_np = wl.norm_weights(w.seed, w.dim)
    tables = rope3d.rope3d_tables_init(max_t=21, max_h=w.H, max_w=w.W)
    caches, scales, _ = _alloc(w, layout)
    with kernel_path(PATHS[path]):
        qo = _run_gpu(w, dev_in, chunk, tables, torch.from_numpy(wq_np).cuda(),
                      torch.from_numpy(wk_np).cuda(), caches, scales, pairing, layout)
    torch.cuda.synchronize()
    shape = tuple(caches[0].shape)
    q_ref, ref_codes, ref_sc, ref_k = _oracle_fp8(w, raw, chunk, wq_np, wk_np, pairing, layout,
                                                   shape)
    assert_close(to_f64(qo), q_ref, "bf16", "q_out")
    rows = np.arange(chunk.slot, chunk.slot + chunk.token_end)
    sel = (slice(None), rows) if layout == TOKEN else (slice(None), slice(None), rows)
    got_vc, got_vs = caches[1].cpu().numpy(), scales[1].cpu().numpy()
    assert np.array_equal(got_vc, ref_codes[1]), "V codes"
    assert np.array_equal(got_vs, ref_sc[1]), "V scales"
    _check_k(caches[0].cpu().numpy(), scales[0].cpu().numpy(), ref_codes[0], ref_sc[0], ref_k,
             sel)
    # untouched rows stay zero
    other = np.ones(w.cache_tokens, dtype=bool)
    other[rows] = False
    osel = (slice(None), other) if layout == TOKEN else (slice(None), slice(None), other)
    assert not caches[0].cpu().numpy()[osel].any() and not scales[0].cpu().numpy()[osel].any()


@pytest.mark.parametrize("dtype,N", [("f32", 2), ("f32", 3), ("bf16", 1), ("bf16", 5),
                                     ("bf16", 40)])
@pytest.mark.parametrize("pairing", [ADJ, HALF])
def test_fp8_cache_small_shapes(dtype, N, pairing):
    w = wl.Workload("small", B=2, T=2, H=3, W=5, N=N, dtype=dtype, cache_tokens=64, seed=400 + N,
                    chunks=[wl.Chunk(4, 50, 0, 30)])
    chunk = w.chunks[0]
    rng = np.random.default_rng(w.seed)
    raw = [wl.normal_tensor(rng, (w.B, 30, N, D), dtype) for _ in range(3)]
    wq_np = rng.uniform(0.5, 1.5, N * D).astype(np.float32)
    wk_np = rng.uniform(0.5, 1.5, N * D).astype(np.float32)
    dev_in = [to_device(x, dtype) for x in raw]
    tables = rope3d.rope3d_tables_init(max_t=6, max_h=w.H, max_w=w.W)
    for layout in (TOKEN, HEAD):
        caches, scales, _ = _alloc(w, layout)
        qo = _run_gpu(w, dev_in, chunk, tables, torch.from_numpy(wq_np).cuda(),
                      torch.from_numpy(wk_np).cuda(), caches, scales, pairing, layout)
        torch.cuda.synchronize()
        q_ref, ref_codes, ref_sc, ref_k = _oracle_fp8(w, raw, chunk, wq_np, wk_np, pairing,
                                                       layout, tuple(caches[0].shape))
        assert_close(to_f64(qo), q_ref, dtype, "q_out")
        assert np.array_equal(caches[1].cpu().numpy(), ref_codes[1])
        assert np.array_equal(scales[1].cpu().numpy(), ref_sc[1])
        rows = np.array([(chunk.slot + i) % w.cache_tokens for i in range(30)])
        sel = (slice(None), rows) if layout == TOKEN else (slice(None), slice(None), rows)
        _check_k(caches[0].cpu().numpy(), scales[0].cpu().numpy(), ref_codes[0], ref_sc[0],
                 ref_k, sel)


@pytest.mark.slow
def test_fp8_slices_bit_identical_to_whole():
    w = wl.full_480p()
    n = w.tokens_per_chunk
    chunk = w.chunks[0]
    raw = wl.chunk_inputs(w, 0)
    dev_in = [to_device(x, w.dtype) for x in raw]
    wq_np, wk_np = wl.norm_weights(w.seed, w.dim)
    wq, wk = torch.from_numpy(wq_np).cuda(), torch.from_numpy(wk_np).cuda()
    tables = rope3d.rope3d_tables_init(max_t=21, max_h=w.H, max_w=w.W)
    c_w, s_w, _ = _alloc(w, HEAD)
    q_w = _run_gpu(w, dev_in, chunk, tables, wq, wk, c_w, s_w, ADJ, HEAD)
    c_s, s_s, _ = _alloc(w, HEAD)
    q_s = torch.empty_like(q_w)
    for (a, e) in wl.slices(n, 8):
        sub = [x[:, a:e].contiguous() for x in dev_in]
        q_s[:, a:e] = _run_gpu(w, sub, chunk, tables, wq, wk, c_s, s_s, ADJ, HEAD, tb=a, te=e)
    torch.cuda.synchronize()
    assert torch.equal(q_w.view(torch.int16), q_s.view(torch.int16))
    for a, b in zip(c_w + s_w, c_s + s_s):
        assert torch.equal(a, b)


def test_fp8_option_errors():
    w = wl.tiny()
    dev_in = [to_device(x, w.dtype) for x in wl.chunk_inputs(w, 0)]
    tables = rope3d.rope3d_tables_init(max_t=6, max_h=4, max_w=6)
    caches = [torch.zeros((1, 144, 2, D), dtype=torch.uint8, device="cuda") for _ in range(2)]
    sc = torch.zeros((1, 144, 2), dtype=torch.float32, device="cuda")
    qo = torch.empty_like(dev_in[0])
    wq = torch.ones(256, device="cuda")
    with pytest.raises(rope3d.Rope3dError) as e:  # k_scale and v_scale are the same array
        rope3d.rope3d_qk_norm_rope_append_ex(*dev_in, qo, 0, 72, 0, 3, 4, 6, wq, wq, 1e-6,
                                             caches[0], caches[1], 0, tables, k_scale=sc,
                                             v_scale=sc)
    assert e.value.status == rope3d.ROPE3D_EOVERLAP
    with pytest.raises(ValueError):
        rope3d.rope3d_qk_norm_rope_append_ex(*dev_in, qo, 0, 72, 0, 3, 4, 6, wq, wq, 1e-6,
                                             caches[0], caches[1], 0, tables, k_scale=sc)
