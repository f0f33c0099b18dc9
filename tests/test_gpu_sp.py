"""The sequence-parallel step with the all-to-all folded in (rope3d_qk_norm_rope_append_sp)
against the fp64 oracle and against the plain CUDA step.

"Accelerating Video Generation Inference with Sequential-Parallel 3D Positional Encoding
Using a Global Time Index", Algorithm 3 steps 3-5 and Section 3.4.1 item 1: every rank
normalises and rotates its own token slice, then an all-to-all gathers the sequence and
scatters the heads, and each rank appends its heads to its KV cache.  Here the all-to-all
is the kernel's own stores: each head goes straight to the rank that owns it.  On one GPU
the ranks are emulated as separate launches over their slices that share one destination
table of local buffers; the launches never wait on one another, so they need not run at
the same time.  Checks: every element of every destination against the oracle (bf16
tolerance, fp32 1e-5, V bit-exact), the destinations bit-identical to the plain step on
the whole sequence split by heads, untouched rows left alone, and argument errors."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gpu_support import assert_close, to_bits, to_device, to_f64, torch_dtype
from rotary_position_encoding_b200 import rope3d, workloads as wl

pytestmark = pytest.mark.gpu

D = wl.HEAD_DIM
TOKEN, HEAD = rope3d.ROPE3D_CACHE_TOKEN_MAJOR, rope3d.ROPE3D_CACHE_HEAD_MAJOR


class Setup:
    def __init__(self, dtype, B, N, T, H, W, s, C, slot, P, layout, seed, q_row0=0,
                 extra_rows=0, trig=rope3d.ROPE3D_TRIG_TABLE):
        self.dtype, self.B, self.N, self.T, self.H, self.W = dtype, B, N, T, H, W
        self.s, self.C, self.slot, self.P, self.layout, self.trig = s, C, slot, P, layout, trig
        self.L = T * H * W
        self.q_row0 = q_row0
        self.q_rows = self.L - q_row0 + extra_rows
        self.hl = N // P
        rng = np.random.default_rng(seed)
        self.raw = [wl.normal_tensor(rng, (B, self.L, N, D), dtype) for _ in range(3)]
        self.wq_np = rng.uniform(0.5, 1.5, N * D).astype(np.float32)
        self.wk_np = rng.uniform(0.5, 1.5, N * D).astype(np.float32)
        self.dev = [to_device(x, dtype) for x in self.raw]
        self.wq = torch.from_numpy(self.wq_np).cuda()
        self.wk = torch.from_numpy(self.wk_np).cuda()
        self.tables = rope3d.rope3d_tables_init(max_t=s + T, max_h=H, max_w=W)
        td = torch_dtype(dtype)
        self.cshape = (B, C, self.hl, D) if layout == TOKEN else (B, self.hl, C, D)
        self.q_dst = [torch.full((B, self.q_rows, self.hl, D), 3.0, dtype=td, device="cuda")
                      for _ in range(P)]
        self.k_dst = [torch.full(self.cshape, 2.0, dtype=td, device="cuda") for _ in range(P)]
        self.v_dst = [torch.full(self.cshape, -2.0, dtype=td, device="cuda") for _ in range(P)]

    def run_rank(self, a, e):
        q, k, v = (x[:, a:e].contiguous() for x in self.dev)
        rope3d.rope3d_qk_norm_rope_append_sp(
            q, k, v, a, e, self.s, self.T, self.H, self.W, self.wq, self.wk, 1e-6,
            self.q_dst, self.k_dst, self.v_dst, self.slot, self.tables, self.trig,
            self.layout, q_row0=self.q_row0)

    def oracle_dst(self, cuts):
        f64 = [wl.to_f64(x, self.dtype) for x in self.raw]
        q_dst = [np.full((self.B, self.q_rows, self.hl, D), 3.0) for _ in range(self.P)]
        k_dst = [np.full(self.cshape, 2.0) for _ in range(self.P)]
        v_dst = [np.full(self.cshape, -2.0) for _ in range(self.P)]
        orc = oracle.default()
        for a, e in zip(cuts[:-1], cuts[1:]):
            orc.qk_norm_rope_append_sp(*(x[:, a:e].copy() for x in f64), a, e, self.s, self.T,
                                       self.H, self.W, self.wq_np.astype(np.float64),
                                       self.wk_np.astype(np.float64), 1e-6, q_dst, k_dst,
                                       v_dst, self.slot, q_row0=self.q_row0,
                                       cache_layout=self.layout)
        return q_dst, k_dst, v_dst

    def plain_whole(self, a, e):
        """The plain CUDA step over [a, e) into full-width buffers."""
        q, k, v = (x[:, a:e].contiguous() for x in self.dev)
        shape = ((self.B, self.C, self.N, D) if self.layout == TOKEN
                 else (self.B, self.N, self.C, D))
        kc = torch.full(shape, 2.0, dtype=q.dtype, device="cuda")
        vc = torch.full(shape, -2.0, dtype=q.dtype, device="cuda")
        qo = torch.empty_like(q)
        rope3d.rope3d_qk_norm_rope_append_ex(q, k, v, qo, a, e, self.s, self.T, self.H, self.W,
                                             self.wq, self.wk, 1e-6, kc, vc, self.slot,
                                             self.tables, self.trig, cache_layout=self.layout)
        return qo, kc, vc

    def check_against_plain(self, a, e):
        qo, kc, vc = self.plain_whole(a, e)
        torch.cuda.synchronize()
        span = np.arange(a, e)
        rows = torch.from_numpy((self.slot + span) % self.C).cuda()
        for r in range(self.P):
            heads = slice(r * self.hl, (r + 1) * self.hl)
            assert torch.equal(self.q_dst[r][:, a - self.q_row0:e - self.q_row0],
                               qo[:, :, heads]), f"q of rank {r}"
            if self.layout == TOKEN:
                got_k, got_v = self.k_dst[r][:, rows], self.v_dst[r][:, rows]
                ref_k, ref_v = kc[:, rows][:, :, heads], vc[:, rows][:, :, heads]
            else:
                got_k, got_v = self.k_dst[r][:, :, rows], self.v_dst[r][:, :, rows]
                ref_k, ref_v = kc[:, heads][:, :, rows], vc[:, heads][:, :, rows]
            assert torch.equal(got_k, ref_k), f"K of rank {r}"
            assert torch.equal(got_v, ref_v), f"V of rank {r}"


def _cuts(L, P, uneven):
    if not uneven:
        n = L // P
        return [r * n for r in range(P)] + [L]
    raw = sorted(set(np.random.default_rng(L + P).integers(1, L, size=max(P - 1, 0)).tolist()))
    return [0] + raw + [L]


@pytest.mark.parametrize("dtype,N,P", [("f32", 2, 2), ("f32", 4, 4), ("bf16", 4, 2),
                                       ("bf16", 12, 3), ("bf16", 40, 8), ("bf16", 8, 8)])
@pytest.mark.parametrize("layout", [TOKEN, HEAD])
@pytest.mark.parametrize("uneven", [False, True])
def test_small_every_element(dtype, N, P, layout, uneven):
    st = Setup(dtype, B=2, N=N, T=2, H=3, W=5, s=4, C=64, slot=50, P=P, layout=layout,
               seed=500 + N + P, extra_rows=3)
    cuts = _cuts(st.L, P, uneven)
    for a, e in zip(cuts[:-1], cuts[1:]):
        st.run_rank(a, e)
    torch.cuda.synchronize()
    q_ref, k_ref, v_ref = st.oracle_dst(cuts)
    for r in range(P):
        assert_close(to_f64(st.q_dst[r]), q_ref[r], dtype, f"q of rank {r}")
        assert_close(to_f64(st.k_dst[r]), k_ref[r], dtype, f"K of rank {r}")
        assert np.array_equal(to_f64(st.v_dst[r]), v_ref[r]), f"V of rank {r}"
    st.check_against_plain(0, st.L)


@pytest.mark.parametrize("P", [2, 3, 4, 6])
@pytest.mark.parametrize("trig", [rope3d.ROPE3D_TRIG_TABLE, rope3d.ROPE3D_TRIG_ONTHEFLY])
def test_480p_chunk_matches_plain_step_and_oracle(P, trig):
    w = wl.chunk_480p()
    st = Setup("bf16", B=1, N=w.N, T=w.T, H=w.H, W=w.W, s=12, C=w.cache_tokens,
               slot=12 * 1560, P=P, layout=TOKEN, seed=600 + P, trig=trig)
    cuts = _cuts(st.L, P, uneven=False)  # the pages' even split L / P
    for a, e in zip(cuts[:-1], cuts[1:]):
        st.run_rank(a, e)
    torch.cuda.synchronize()
    st.check_against_plain(0, st.L)
    if P == 4:
        q_ref, k_ref, v_ref = st.oracle_dst(cuts)
        rows = (st.slot + np.arange(st.L)) % st.C
        for r in range(P):
            assert_close(to_f64(st.q_dst[r]), q_ref[r], "bf16", f"q of rank {r}")
            assert_close(to_f64(st.k_dst[r][:, rows]), k_ref[r][:, rows], "bf16", f"K {r}")
            assert np.array_equal(to_f64(st.v_dst[r][:, rows]), v_ref[r][:, rows])


@pytest.mark.slow
@pytest.mark.parametrize("layout", [TOKEN, HEAD])
def test_720p_chunk_eight_ranks(layout):
    """40 heads over 8 ranks (5 heads each), the pages' even split of 10800 tokens."""
    w = wl.chunk_720p()
    st = Setup("bf16", B=1, N=w.N, T=w.T, H=w.H, W=w.W, s=18, C=w.cache_tokens,
               slot=18 * 3600, P=8, layout=layout, seed=700)
    cuts = _cuts(st.L, 8, uneven=False)
    for a, e in zip(cuts[:-1], cuts[1:]):
        st.run_rank(a, e)
    torch.cuda.synchronize()
    st.check_against_plain(0, st.L)
    orc = oracle.default()
    sample = sorted(set(np.random.default_rng(8).integers(0, st.L, 24).tolist()) | {0, st.L - 1})
    for i in sample:
        q64, k64, v64 = (wl.to_f64(x[0, i], "bf16") for x in st.raw)
        eq, ek, ev, pos = orc.token(q64, k64, v64, i, st.s, st.T, st.H, st.W,
                                    st.wq_np.astype(np.float64), st.wk_np.astype(np.float64),
                                    1e-6, st.slot, st.C)
        row = int(pos[3])
        for r in range(8):
            heads = slice(r * 5, (r + 1) * 5)
            assert_close(to_f64(st.q_dst[r][0, i]), eq[heads], "bf16", f"q {i} rank {r}")
            kd = st.k_dst[r][0, row] if layout == TOKEN else st.k_dst[r][0, :, row]
            vd = st.v_dst[r][0, row] if layout == TOKEN else st.v_dst[r][0, :, row]
            assert_close(to_f64(kd), ek[heads], "bf16", f"K {i} rank {r}")
            assert np.array_equal(to_bits(vd), st.raw[2][0, i, heads])


def test_argument_errors():
    st = Setup("bf16", B=1, N=4, T=2, H=3, W=5, s=0, C=64, slot=0, P=2, layout=TOKEN, seed=9)
    q, k, v = st.dev
    L = st.L

    def call(q_dst=None, k_dst=None, v_dst=None, tb=0, te=None, q_row0=0, layout=TOKEN):
        te = L if te is None else te
        rope3d.rope3d_qk_norm_rope_append_sp(
            q[:, tb:te].contiguous(), k[:, tb:te].contiguous(), v[:, tb:te].contiguous(), tb, te,
            0, 2, 3, 5, st.wq, st.wk, 1e-6, q_dst or st.q_dst, k_dst or st.k_dst,
            v_dst or st.v_dst, 0, st.tables, cache_layout=layout, q_row0=q_row0)

    def status(**kw):
        with pytest.raises(rope3d.Rope3dError) as e:
            call(**kw)
        return e.value.status

    call()  # valid
    # the token range must lie inside the q buffers' rows
    assert status(tb=0, te=10, q_row0=5) == rope3d.ROPE3D_ERANGE
    # a destination that overlaps another one
    assert status(k_dst=[st.k_dst[0], st.k_dst[0]]) == rope3d.ROPE3D_EOVERLAP
    assert status(v_dst=[st.k_dst[0], st.v_dst[1]]) == rope3d.ROPE3D_EOVERLAP
    # misaligned destination (raw address 2 bytes into a buffer)
    addr = st.q_dst[1].data_ptr() + 2
    with pytest.raises(rope3d.Rope3dError) as e:
        rope3d.rope3d_qk_norm_rope_append_sp(q, k, v, 0, L, 0, 2, 3, 5, st.wq, st.wk, 1e-6,
                                             [st.q_dst[0], addr], st.k_dst, st.v_dst, 0,
                                             st.tables, q_rows=st.q_rows, cache_tokens=64)
    assert e.value.status == rope3d.ROPE3D_EALIGN
    # the C entry point directly: N not divisible by P, too many ranks, half pairing, FP8
    lib = rope3d.load_library()
    dest = rope3d.rope3d_sp_dest()
    dest.ranks, dest.q_rows, dest.q_row0 = 3, st.q_rows, 0
    for r in range(3):
        dest.q[r] = st.q_dst[r % 2].data_ptr()
        dest.k_cache[r] = st.k_dst[r % 2].data_ptr()
        dest.v_cache[r] = st.v_dst[r % 2].data_ptr()

    def c_call(d, opts=None):
        return lib.rope3d_qk_norm_rope_append_sp(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), 1, 4, D, rope3d.ROPE3D_BF16, 0, L, 0, 2, 3,
            5, st.wq.data_ptr(), st.wk.data_ptr(), 1e-6, ctypes.byref(d), 64, 0,
            st.tables.handle, rope3d.ROPE3D_TRIG_TABLE, opts, None)

    assert c_call(dest) == rope3d.ROPE3D_EINVAL  # 4 heads over 3 ranks
    dest.ranks = rope3d.ROPE3D_SP_MAX_RANKS + 1
    assert c_call(dest) == rope3d.ROPE3D_EINVAL
    dest.ranks = 2
    dest.reserved0 = 1
    assert c_call(dest) == rope3d.ROPE3D_EINVAL
    dest.reserved0 = 0
    assert c_call(dest) == rope3d.ROPE3D_OK
    half = rope3d.rope3d_options(rope3d.ROPE3D_PAIRING_HALF, TOKEN)
    assert c_call(dest, ctypes.byref(half)) == rope3d.ROPE3D_EINVAL
    scale = torch.zeros(64 * 4, device="cuda")
    fp8 = rope3d.rope3d_options(0, TOKEN, rope3d.ROPE3D_CACHE_FP8_E4M3, 0, scale.data_ptr(),
                                scale.data_ptr())
    assert c_call(dest, ctypes.byref(fp8)) == rope3d.ROPE3D_EINVAL
    torch.cuda.synchronize()


def test_symmetric_memory_wiring_one_rank():
    """The multi-GPU wiring (one symmetric-memory allocation per rank, the table of every
    rank's addresses, the step, the device barrier) on a one-rank NCCL group: the rank's
    own buffers hold the plain step's results bit for bit.  Runs with more ranks need
    more than one GPU."""
    import datetime
    import socket

    import torch.distributed as dist

    from rotary_position_encoding_b200 import sp
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        st = Setup("bf16", B=2, N=4, T=2, H=3, W=5, s=4, C=64, slot=50, P=1, layout=TOKEN,
                   seed=31)
        wiring = sp.SequenceParallelStep(dist.group.WORLD, 0, 1, B=2, N=4, q_rows=st.L,
                                         cache_tokens=64, dtype=torch.bfloat16, device="cuda")
        wiring.q.fill_(3.0)
        wiring.k_cache.fill_(2.0)
        wiring.v_cache.fill_(-2.0)
        q, k, v = st.dev
        wiring.step(q, k, v, 0, st.L, 4, 2, 3, 5, st.wq, st.wk, 1e-6, 50, st.tables)
        wiring.barrier()
        torch.cuda.synchronize()
        st.q_dst, st.k_dst, st.v_dst = [wiring.q], [wiring.k_cache], [wiring.v_cache]
        st.check_against_plain(0, st.L)
        # the exchange back after attention (identity on one rank): the gathered q rows
        # land in the output region as [B, L, N, 128]
        back = wiring.output_all_to_all(wiring.q)
        wiring.barrier()
        torch.cuda.synchronize()
        assert torch.equal(back.view(torch.int16), wiring.q.view(torch.int16))
        del wiring, st, back
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
