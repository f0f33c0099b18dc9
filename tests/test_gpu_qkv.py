"""The QKV projection on the tensor cores (rope3d_qkv_project) and the projection-fed step
(rope3d_qkv_norm_rope_append) against the fp64 oracle.

"Accelerating Video Generation Inference with Sequential-Parallel 3D Positional Encoding
Using a Global Time Index", Algorithm 1/3 step 1 (q, k, v <- QKV(x)) and Section 3.4.1
item 3 (the projection fused with the rotary step).  The projection accumulates in fp32
and rounds once to bf16; the oracle accumulates in fp64.  A projected value may therefore
sit one bf16 step away from the oracle's rounding where the exact value is near a rounding
midpoint: the bound per element is one bf16 step of |ref| plus the fp32 accumulation error
(2^-20 of sum |x_i w_i| + |b|).  With an even head count the projection's epilogue does
the normalisation and rotation itself, on the fp32 projections: it is checked with the
step's bf16 tolerance against the oracle's step on the unrounded fp64 projections, and its
slices bit for bit against the whole.  With an odd head count the projection hands bf16
q and k to the step: checked against the oracle's step on the rounded projections, and bit
for bit against the plain step run on the GPU projection's outputs."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gpu_support import assert_close, to_device, to_f64
from rotary_position_encoding_b200 import rope3d, workloads as wl

pytestmark = pytest.mark.gpu

D = wl.HEAD_DIM
TOKEN, HEAD = rope3d.ROPE3D_CACHE_TOKEN_MAJOR, rope3d.ROPE3D_CACHE_HEAD_MAJOR


def _bf16(a):
    return to_device(a, "bf16")


def _projection_bound(x64, w64, b, ref):
    s = np.abs(x64) @ np.abs(w64).T + (0 if b is None else np.abs(b.astype(np.float64)))
    return 2.0 ** -8 * np.abs(ref) + 2.0 ** -20 * s + 1e-30


def _check_projection(x_bits, w_bits, b, outs, rows=None):
    """outs: the q, k, v outputs ([..., N, 128] with M rows in all); rows: the token rows to
    check (all if None)."""
    K = x_bits.shape[-1]
    x64 = wl.bf16_bits_to_f64(x_bits).reshape(-1, K)
    w64 = wl.bf16_bits_to_f64(w_bits)
    got = np.concatenate([to_f64(o).reshape(x64.shape[0], -1) for o in outs], axis=-1)
    if rows is not None:
        x64, got = x64[rows], got[rows]
    ref = np.concatenate(oracle.default().qkv_project(x64, w64, b), axis=-1)
    bound = _projection_bound(x64, w64, b, ref)
    err = np.abs(got - ref)
    assert np.all(err <= bound), f"{int((err > bound).sum())} projected values out of bound"


@pytest.fixture(params=[1, 2], ids=["cta1", "pair"])
def gemm_form(request):
    """Both forms of the projection kernel: one CTA per tile, or a 2-CTA pair."""
    rope3d.rope3d_testing_gemm_cta_group(request.param)
    yield request.param
    rope3d.rope3d_testing_gemm_cta_group(0)


@pytest.mark.parametrize("M,K,N,bias", [(200, 128, 2, True), (130, 256, 5, False),
                                        (1, 64, 1, True), (384, 1536, 12, True),
                                        (700, 512, 4, True)])
def test_projection_small(M, K, N, bias, gemm_form):
    rng = np.random.default_rng(M + K + N)
    x_bits = wl.f32_to_bf16_bits(rng.standard_normal((M, K), dtype=np.float32))
    w_bits = wl.f32_to_bf16_bits(rng.standard_normal((3 * N * D, K), dtype=np.float32)
                                 / np.float32(np.sqrt(K)))
    b = rng.standard_normal(3 * N * D).astype(np.float32) if bias else None
    outs = [torch.full((M, N, D), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    rope3d.rope3d_qkv_project(_bf16(x_bits), _bf16(w_bits),
                              None if b is None else torch.from_numpy(b).cuda(), *outs)
    torch.cuda.synchronize()
    _check_projection(x_bits, w_bits, b, outs)


def _fused_case(dtype_layout, B=2, N=4, K=256, T=2, H=3, W=5, s=4, C=64, slot=50, seed=11):
    rng = np.random.default_rng(seed)
    L = T * H * W
    x_bits = wl.f32_to_bf16_bits(rng.standard_normal((B, L, K), dtype=np.float32))
    # projections about N(0, 9): the RMSNorm scales them by about 1/3
    w_bits = wl.f32_to_bf16_bits(rng.standard_normal((3 * N * D, K), dtype=np.float32)
                                 * np.float32(3.0 / np.sqrt(K)))
    b = (rng.standard_normal(3 * N * D) * 0.1).astype(np.float32)
    wq = rng.uniform(0.5, 1.5, N * D).astype(np.float32)
    wk = rng.uniform(0.5, 1.5, N * D).astype(np.float32)
    return dict(B=B, N=N, K=K, T=T, H=H, W=W, s=s, C=C, slot=slot, L=L, x=x_bits, w=w_bits,
                b=b, wq=wq, wk=wk, layout=dtype_layout)


def _workspace(B, n_tok, N):
    nbytes = rope3d.rope3d_qkv_workspace_bytes(B, n_tok, N)
    return torch.zeros(nbytes, dtype=torch.uint8, device="cuda")


def _run_fused(c, tables, tb, te, ws=None):
    cshape = ((c["B"], c["C"], c["N"], D) if c["layout"] == TOKEN
              else (c["B"], c["N"], c["C"], D))
    kc = torch.full(cshape, 2.0, dtype=torch.bfloat16, device="cuda")
    vc = torch.full(cshape, -2.0, dtype=torch.bfloat16, device="cuda")
    x = _bf16(c["x"][:, tb:te].copy())
    qo = torch.empty((c["B"], te - tb, c["N"], D), dtype=torch.bfloat16, device="cuda")
    ws = _workspace(c["B"], te - tb, c["N"]) if ws is None else ws
    rope3d.rope3d_qkv_norm_rope_append(
        x, _bf16(c["w"]), torch.from_numpy(c["b"]).cuda(), qo, ws, tb, te, c["s"], c["T"],
        c["H"], c["W"], torch.from_numpy(c["wq"]).cuda(), torch.from_numpy(c["wk"]).cuda(), 1e-6,
        kc, vc, c["slot"], tables, cache_layout=c["layout"])
    return qo, ws, kc, vc


@pytest.mark.parametrize("layout", [TOKEN, HEAD])
@pytest.mark.parametrize("N", [4, 5])
@pytest.mark.parametrize("trig", [rope3d.ROPE3D_TRIG_TABLE, rope3d.ROPE3D_TRIG_ONTHEFLY])
def test_fused_small_against_oracle(layout, N, trig, gemm_form):
    c = _fused_case(layout, N=N)
    tables = rope3d.rope3d_tables_init(max_t=c["s"] + c["T"], max_h=c["H"], max_w=c["W"])
    cshape = ((c["B"], c["C"], N, D) if layout == TOKEN else (c["B"], N, c["C"], D))
    kc = torch.full(cshape, 2.0, dtype=torch.bfloat16, device="cuda")
    vc = torch.full(cshape, -2.0, dtype=torch.bfloat16, device="cuda")
    qo = torch.empty((c["B"], c["L"], N, D), dtype=torch.bfloat16, device="cuda")
    ws = _workspace(c["B"], c["L"], N)
    rope3d.rope3d_qkv_norm_rope_append(
        _bf16(c["x"]), _bf16(c["w"]), torch.from_numpy(c["b"]).cuda(), qo, ws, 0, c["L"],
        c["s"], c["T"], c["H"], c["W"], torch.from_numpy(c["wq"]).cuda(),
        torch.from_numpy(c["wk"]).cuda(), 1e-6, kc, vc, c["slot"], tables, trig, layout)
    torch.cuda.synchronize()
    fused = (N * D) % 256 == 0
    x64 = wl.bf16_bits_to_f64(c["x"])
    w64 = wl.bf16_bits_to_f64(c["w"])
    shape = (c["B"], c["C"], c["N"], D) if layout == TOKEN else (c["B"], c["N"], c["C"], D)
    kr, vr = np.full(shape, 2.0), np.full(shape, -2.0)
    orc = oracle.default()
    q_ref = orc.qkv_norm_rope_append(x64, w64, c["b"], c["N"], 0, c["L"], c["s"], c["T"], c["H"],
                                     c["W"], c["wq"].astype(np.float64),
                                     c["wk"].astype(np.float64), 1e-6, kr, vr, c["slot"],
                                     round_bf16=not fused, cache_layout=layout)
    assert_close(to_f64(qo), q_ref, "bf16", "q_out")
    assert_close(to_f64(kc), kr, "bf16", "k_cache (written and untouched rows)")
    # V: the exact projection within the projection bound (one bf16 step plus the fp32
    # accumulation error); rows the range does not map to keep their fill
    N, dim = c["N"], c["N"] * D
    _, _, v_exact = orc.qkv_project(x64, w64, c["b"])
    s_abs = np.abs(x64) @ np.abs(w64[2 * dim:]).T + np.abs(c["b"][2 * dim:].astype(np.float64))
    got_v = to_f64(vc)
    rows = (c["slot"] + np.arange(c["L"])) % c["C"]
    for bb in range(c["B"]):
        g = got_v[bb, rows] if layout == TOKEN else got_v[bb][:, rows].transpose(1, 0, 2)
        ref = v_exact[bb].reshape(c["L"], N, D)
        bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -19 * s_abs[bb].reshape(c["L"], N, D)
        assert np.all(np.abs(g.reshape(ref.shape) - ref) <= bound), "V cache rows"
    other = np.setdiff1d(np.arange(c["C"]), rows)
    untouched = got_v[:, other] if layout == TOKEN else got_v[:, :, other]
    assert np.all(untouched == -2.0), "V cache rows outside the range"


@pytest.mark.parametrize("layout", [TOKEN, HEAD])
@pytest.mark.parametrize("N", [12, 5])
def test_fused_against_projection_then_step(layout, N, gemm_form):
    """Against rope3d_qkv_project followed by the plain step on its outputs: V cache rows
    bit-identical always; q and K bit-identical for odd head counts (the same two passes)
    and within the bf16 tolerance of each other for even ones (the epilogue normalises the
    fp32 projections and rounds twice); slices of the range bit-identical to the whole."""
    c = _fused_case(layout, B=1, N=N, K=512, T=3, H=6, W=10, s=6, C=200, slot=170, seed=12)
    tables = rope3d.rope3d_tables_init(max_t=c["s"] + c["T"], max_h=c["H"], max_w=c["W"])
    qo, _, kc, vc = _run_fused(c, tables, 0, c["L"])
    x = _bf16(c["x"])
    outs = [torch.empty((1, c["L"], c["N"], D), dtype=torch.bfloat16, device="cuda")
            for _ in range(3)]
    rope3d.rope3d_qkv_project(x, _bf16(c["w"]), torch.from_numpy(c["b"]).cuda(), *outs)
    kc2, vc2 = torch.full_like(kc, 2.0), torch.full_like(vc, -2.0)
    qo2 = torch.empty_like(qo)
    rope3d.rope3d_qk_norm_rope_append_ex(*outs, qo2, 0, c["L"], c["s"], c["T"], c["H"], c["W"],
                                         torch.from_numpy(c["wq"]).cuda(),
                                         torch.from_numpy(c["wk"]).cuda(), 1e-6, kc2, vc2,
                                         c["slot"], tables, cache_layout=layout)
    torch.cuda.synchronize()
    assert torch.equal(vc.view(torch.int16), vc2.view(torch.int16))
    if (N * D) % 256:
        assert torch.equal(qo.view(torch.int16), qo2.view(torch.int16))
        assert torch.equal(kc.view(torch.int16), kc2.view(torch.int16))
    else:
        a, b = to_f64(qo), to_f64(qo2)
        assert np.all(np.abs(a - b) <= 1.6e-2 + 8e-3 * np.abs(b)), "q: fused against two passes"
        a, b = to_f64(kc), to_f64(kc2)
        assert np.all(np.abs(a - b) <= 1.6e-2 + 8e-3 * np.abs(b)), "K: fused against two passes"
    # slices of the range give the same caches and q rows
    qs = torch.empty_like(qo)
    kc3, vc3 = torch.full_like(kc, 2.0), torch.full_like(vc, -2.0)
    for a, e in ((0, 77), (77, 100), (100, c["L"])):
        q_a, _, k_a, v_a = _run_fused(c, tables, a, e)
        qs[:, a:e] = q_a
        rows = torch.from_numpy((c["slot"] + np.arange(a, e)) % c["C"]).cuda()
        if layout == TOKEN:
            kc3[:, rows], vc3[:, rows] = k_a[:, rows], v_a[:, rows]
        else:
            kc3[:, :, rows], vc3[:, :, rows] = k_a[:, :, rows], v_a[:, :, rows]
    torch.cuda.synchronize()
    assert torch.equal(qs.view(torch.int16), qo.view(torch.int16))
    assert torch.equal(kc3.view(torch.int16), kc.view(torch.int16))
    assert torch.equal(vc3.view(torch.int16), vc.view(torch.int16))


@pytest.mark.slow
def test_720p_chunk_sampled_rows(gemm_form):
    """The Wan-14B-shaped 720P chunk: 10800 tokens of 5120 features, 40 heads; sampled
    rows of the projection and of the step against the oracle."""
    w = wl.chunk_720p()
    K = w.dim
    chunk = w.chunks[2]
    x_bits = wl.hidden_states(w, 2, K)
    w_bits, b = wl.projection_weights(w.seed, w.dim, K)
    wq, wk = wl.norm_weights(w.seed, w.dim)
    tables = rope3d.rope3d_tables_init(max_t=21, max_h=w.H, max_w=w.W)
    x = _bf16(x_bits)
    wt = _bf16(w_bits)
    bt = torch.from_numpy(b).cuda()
    outs = [torch.empty((1, 10800, w.N, D), dtype=torch.bfloat16, device="cuda")
            for _ in range(3)]
    rope3d.rope3d_qkv_project(x, wt, bt, *outs)
    kc = torch.zeros((1, w.cache_tokens, w.N, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    qo = torch.empty_like(outs[0])
    ws = _workspace(1, 10800, w.N)
    rope3d.rope3d_qkv_norm_rope_append(x, wt, bt, qo, ws, 0, 10800, chunk.frame_offset, w.T,
                                       w.H, w.W, torch.from_numpy(wq).cuda(),
                                       torch.from_numpy(wk).cuda(), w.eps, kc, vc, chunk.slot,
                                       tables)
    torch.cuda.synchronize()
    rows = sorted(set(np.random.default_rng(5).integers(0, 10800, 24).tolist()) | {0, 10799})
    _check_projection(x_bits, w_bits, b, outs, rows=rows)
    orc = oracle.default()
    x64 = wl.bf16_bits_to_f64(x_bits)[0, rows]
    q, k, v = orc.qkv_project(x64, wl.bf16_bits_to_f64(w_bits), b)  # fp32-fed epilogue
    for j, i in enumerate(rows):
        eq, ek, ev, pos = orc.token(q[j].reshape(w.N, D), k[j].reshape(w.N, D),
                                    v[j].reshape(w.N, D), i, chunk.frame_offset, w.T, w.H, w.W,
                                    wq.astype(np.float64), wk.astype(np.float64), w.eps,
                                    chunk.slot, w.cache_tokens)
        assert_close(to_f64(qo[0, i]), eq, "bf16", f"q row {i}")
        assert_close(to_f64(kc[0, pos[3]]), ek, "bf16", f"K row {i}")
        # the V row is the projection's bf16 output, already checked against the bound
        assert torch.equal(vc[0, pos[3]].view(torch.int16), outs[2][0, i].view(torch.int16))


def test_argument_errors():
    c = _fused_case(TOKEN)
    tables = rope3d.rope3d_tables_init(max_t=c["s"] + c["T"], max_h=c["H"], max_w=c["W"])
    lib = rope3d.load_library()
    x = _bf16(c["x"])
    w = _bf16(c["w"])
    outs = [torch.empty((c["B"] * c["L"], c["N"], D), dtype=torch.bfloat16, device="cuda")
            for _ in range(3)]
    M = c["B"] * c["L"]
    P = lambda t: t.data_ptr()  # noqa: E731
    assert lib.rope3d_qkv_project(P(x), P(w), None, M, 200, c["N"], D, *map(P, outs),
                                  None) == rope3d.ROPE3D_EINVAL        # K % 64
    assert lib.rope3d_qkv_project(P(x) + 2, P(w), None, M, c["K"], c["N"], D, *map(P, outs),
                                  None) == rope3d.ROPE3D_EALIGN
    assert lib.rope3d_qkv_project(P(x), P(w), None, M, c["K"], c["N"], D, P(outs[0]),
                                  P(outs[0]), P(outs[2]), None) == rope3d.ROPE3D_EOVERLAP
    assert lib.rope3d_qkv_project(P(x), P(w), None, M, c["K"], c["N"], D, P(x), P(outs[1]),
                                  P(outs[2]), None) == rope3d.ROPE3D_EOVERLAP
    qo = torch.empty((c["B"], c["L"], c["N"], D), dtype=torch.bfloat16, device="cuda")
    ws = _workspace(c["B"], c["L"], c["N"])
    kc = torch.zeros((c["B"], c["C"], c["N"], D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    wq = torch.from_numpy(c["wq"]).cuda()

    def fused(opts=None, work=ws, nbytes=None):
        nbytes = work.numel() * work.element_size() if nbytes is None else nbytes
        return lib.rope3d_qkv_norm_rope_append(
            P(x), P(w), None, c["K"], c["B"], c["N"], D, 0, c["L"], c["s"], c["T"], c["H"],
            c["W"], P(wq), P(wq), 1e-6, P(qo), P(work), nbytes, P(kc), P(vc), c["C"],
            c["slot"], tables.handle, 0, opts, None)

    assert fused() == rope3d.ROPE3D_OK
    half = rope3d.rope3d_options(rope3d.ROPE3D_PAIRING_HALF, TOKEN)
    assert fused(ctypes.byref(half)) == rope3d.ROPE3D_EINVAL
    assert fused(work=kc) == rope3d.ROPE3D_EOVERLAP
    assert fused(nbytes=ws.numel() - 1) == rope3d.ROPE3D_EINVAL
    assert rope3d.rope3d_qkv_workspace_bytes(0, 10, 4) == 0
    torch.cuda.synchronize()


def test_projection_wait_timeout_reports_status(gemm_form):
    """A projection whose stages can never fill (the test hook makes every stage wait for
    16 bytes that no copy delivers) gives up after the wait limit: the tables' status word
    reports ROPE3D_ETIMEOUT, the kernel's copies and tensor-core work are drained and its
    tensor memory released, and the next call runs normally and correctly."""
    c = _fused_case(TOKEN)
    tables = rope3d.rope3d_tables_init(max_t=c["s"] + c["T"], max_h=c["H"], max_w=c["W"])
    rope3d.rope3d_testing_set_waits(20_000_000, 16)  # 20 ms
    try:
        _run_fused(c, tables, 0, c["L"])
        assert rope3d.rope3d_check_device_status(tables) == rope3d.ROPE3D_ETIMEOUT
    finally:
        rope3d.rope3d_testing_set_waits(0, 0)
    assert rope3d.rope3d_check_device_status(tables) == rope3d.ROPE3D_OK
    qo, _, kc, vc = _run_fused(c, tables, 0, c["L"])
    assert rope3d.rope3d_check_device_status(tables) == rope3d.ROPE3D_OK
    x64 = wl.bf16_bits_to_f64(c["x"])
    w64 = wl.bf16_bits_to_f64(c["w"])
    kr, vr = np.full(tuple(kc.shape), 2.0), np.full(tuple(vc.shape), -2.0)
    q_ref = oracle.default().qkv_norm_rope_append(
        x64, w64, c["b"], c["N"], 0, c["L"], c["s"], c["T"], c["H"], c["W"],
        c["wq"].astype(np.float64), c["wk"].astype(np.float64), 1e-6, kr, vr, c["slot"],
        round_bf16=False)
    assert_close(to_f64(qo), q_ref, "bf16", "q_out after a timed-out call")
    assert_close(to_f64(kc), kr, "bf16", "k_cache after a timed-out call")
