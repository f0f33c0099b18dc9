"""The all-to-all after attention (rope3d_sp_output_all_to_all) against the oracle.

"Accelerating Video Generation Inference with Sequential-Parallel 3D Positional Encoding
Using a Global Time Index", Algorithm 3, last step: o <- AllToAll(o, scatter_dim=1,
gather_dim=2).  Each rank holds every token for its own heads; afterwards each rank holds
its token slice with every head.  On one GPU the ranks are emulated as separate launches
over their own o into local destination buffers (the launches never wait on one another).
It is a bit copy, so every element must equal the oracle's exactly; rows of an output
that no rank writes do not exist (outputs are exactly the slices)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_support import to_bits, to_device, torch_dtype
from rotary_position_encoding_b200 import rope3d, workloads as wl

pytestmark = pytest.mark.gpu

D = wl.HEAD_DIM


def _run(dtype, B, L, N, P, cuts, seed):
    hl = N // P
    rng = np.random.default_rng(seed)
    raw = [wl.normal_tensor(rng, (B, L, hl, D), dtype) for _ in range(P)]
    o = [to_device(x, dtype) for x in raw]
    td = torch_dtype(dtype)
    out = [torch.full((B, cuts[r + 1] - cuts[r], N, D), 5.0, dtype=td, device="cuda")
           for r in range(P)]
    for r in range(P):  # rank r's launch: its heads of every token
        rope3d.rope3d_sp_output_all_to_all(o[r], out, r, cuts)
    torch.cuda.synchronize()
    ref = oracle.Oracle.sp_output_all_to_all(raw, cuts)  # float32 values or bf16 bits
    for r in range(P):
        want = np.ascontiguousarray(ref[r])
        if dtype == "f32":
            want = want.view(np.uint32)
        assert np.array_equal(to_bits(out[r]), want), f"rank {r}"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("P,cuts", [(1, [0, 23]), (2, [0, 9, 23]), (3, [0, 7, 16, 23]),
                                    (4, [0, 5, 5, 17, 23]), (8, [0, 1, 3, 6, 9, 12, 16, 20, 23])])
def test_small_every_element(dtype, P, cuts):
    _run(dtype, B=2, L=23, N=8 if P != 3 else 6, P=P, cuts=cuts, seed=800 + P)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_buffers_aligned_to_16_bytes_only(dtype):
    """o and every output start 16 bytes past a 32-byte boundary: the copy falls back from
    32-byte to 16-byte units, with the same result."""
    B, L, N, P = 2, 23, 8, 4
    cuts = [0, 5, 5, 17, 23]
    hl = N // P
    td = torch_dtype(dtype)
    pad = 16 // torch.empty((), dtype=td).element_size()
    rng = np.random.default_rng(840)
    raw = [wl.normal_tensor(rng, (B, L, hl, D), dtype) for _ in range(P)]

    def shifted(shape, fill):
        n = int(np.prod(shape))
        buf = torch.full((n + pad,), fill, dtype=td, device="cuda")
        t = buf[pad:].view(shape)
        assert n == 0 or t.data_ptr() % 32 == 16  # an empty slice has no address
        return t

    o = []
    for x in raw:
        t = shifted((B, L, hl, D), 0.0)
        t.copy_(to_device(x, dtype))
        o.append(t)
    out = [shifted((B, cuts[r + 1] - cuts[r], N, D), 5.0) for r in range(P)]
    for r in range(P):
        rope3d.rope3d_sp_output_all_to_all(o[r], out, r, cuts)
    torch.cuda.synchronize()
    ref = oracle.Oracle.sp_output_all_to_all(raw, cuts)
    for r in range(P):
        want = np.ascontiguousarray(ref[r])
        if dtype == "f32":
            want = want.view(np.uint32)
        assert np.array_equal(to_bits(out[r]), want), f"rank {r}"


def test_720p_eight_ranks_even_split():
    """The 720P chunk of a 40-head backbone over 8 ranks: 1350 tokens and 5 heads each."""
    _run("bf16", B=1, L=10800, N=40, P=8, cuts=[r * 1350 for r in range(9)], seed=808)


def test_round_trip_with_the_head_scatter():
    """The step with the head scatter on every rank's slice, then the output all-to-all
    of each owner's gathered q rows: every rank gets back exactly the plain step's q_out
    rows of its own slice, all heads."""
    w = wl.chunk_480p()
    P = 4
    n = w.tokens_per_chunk
    chunk = w.chunks[2]
    q, k, v = (to_device(x, w.dtype) for x in wl.chunk_inputs(w, 2))
    wq_np, wk_np = wl.norm_weights(w.seed, w.dim)
    wq, wk = torch.from_numpy(wq_np).cuda(), torch.from_numpy(wk_np).cuda()
    tables = rope3d.rope3d_tables_init(max_t=21, max_h=w.H, max_w=w.W)
    hl = w.N // P
    q_dst = [torch.empty((1, n, hl, D), dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    k_dst = [torch.zeros((1, w.cache_tokens, hl, D), dtype=torch.bfloat16, device="cuda")
             for _ in range(P)]
    v_dst = [torch.zeros_like(k_dst[0]) for _ in range(P)]
    cuts = [(r * n) // P for r in range(P + 1)]
    for a, e in zip(cuts[:-1], cuts[1:]):
        rope3d.rope3d_qk_norm_rope_append_sp(
            q[:, a:e].contiguous(), k[:, a:e].contiguous(), v[:, a:e].contiguous(), a, e,
            chunk.frame_offset, w.T, w.H, w.W, wq, wk, w.eps, q_dst, k_dst, v_dst, chunk.slot,
            tables)
    back = [torch.empty((1, cuts[r + 1] - cuts[r], w.N, D), dtype=torch.bfloat16,
                        device="cuda") for r in range(P)]
    for r in range(P):
        rope3d.rope3d_sp_output_all_to_all(q_dst[r], back, r)
    qo = torch.empty_like(q)
    kc = torch.zeros((1, w.cache_tokens, w.N, D), dtype=torch.bfloat16, device="cuda")
    rope3d.rope3d_qk_norm_rope_append(q, k, v, qo, 0, n, chunk.frame_offset, w.T, w.H, w.W,
                                      wq, wk, w.eps, kc, torch.zeros_like(kc), chunk.slot,
                                      tables)
    torch.cuda.synchronize()
    for r in range(P):
        assert torch.equal(back[r].view(torch.int16),
                           qo[:, cuts[r]:cuts[r + 1]].contiguous().view(torch.int16))
    tables.close()


def test_binding_checks_shapes():
    o = torch.zeros((1, 10, 2, D), dtype=torch.bfloat16, device="cuda")
    good = [torch.zeros((1, 5, 4, D), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    with pytest.raises(ValueError):
        rope3d.rope3d_sp_output_all_to_all(o, [good[0], good[1][:, :4].contiguous()], 0)
    with pytest.raises(TypeError):
        rope3d.rope3d_sp_output_all_to_all(o, [good[0], good[1].float()], 0)
    with pytest.raises(rope3d.Rope3dError) as e:
        rope3d.rope3d_sp_output_all_to_all(o, good, 2)
    assert e.value.status == rope3d.ROPE3D_EINVAL
