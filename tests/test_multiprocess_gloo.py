"""Multi-process host logic on CPU with the gloo backend, world size 2.

The step shards with no exchange: the paper's Causal-RoPE SP lets each rank compute its
own token slice [r L/P, (r+1) L/P) with the global index offset Delta = r L_local and no
communication ("Accelerating Video Generation Inference with Sequential-Parallel 3D
Positional Encoding Using a Global Time Index", Section 3.3.3; Algorithm 3 steps 2-3).
These tests run ranks as processes: (1) each rank computes its slice with the oracle
and rank 0 checks the gathered result against the whole sequence; (2) the oracle's
sequence-parallel step with the all-to-all folded in (each head stored at the rank that
owns it) equals the pages' separate FusedAllToAll -- an all-to-all that gathers the
sequence and scatters the heads (Algorithm 3 step 4), here torch's gloo all_to_all_single
-- applied to each rank's plain results; (3) the benchmark's timing reduction takes the
maximum over ranks and scales the token count by the ranks."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)


def _sp_rank(rank, world, port, q_path):
    _init(rank, world, port)
    import datetime

    import oracle
    from rotary_position_encoding_b200 import workloads as wl
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        w = wl.tiny()
        chunk = w.chunks[1]  # start frame 3, slot 72
        n = w.tokens_per_chunk
        q, k, v = (wl.to_f64(x, w.dtype) for x in wl.chunk_inputs(w, 1))
        wq, wk = (x.astype(np.float64) for x in wl.norm_weights(w.seed, w.dim))
        L_local = n // world
        delta = rank * L_local  # Algorithm 3 step 2
        a, e = delta, delta + L_local
        kc = np.zeros((w.B, w.cache_tokens, w.N, wl.HEAD_DIM))
        vc = np.zeros_like(kc)
        q_loc = oracle.default().qk_norm_rope_append(
            q[:, a:e].copy(), k[:, a:e].copy(), v[:, a:e].copy(), a, e, chunk.frame_offset,
            w.T, w.H, w.W, wq, wk, w.eps, kc, vc, chunk.slot)
        gathered = [torch.zeros(q_loc.shape, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, torch.from_numpy(q_loc))
        kc_t = torch.from_numpy(kc)
        dist.all_reduce(kc_t)  # each cache row is written by exactly one rank
        if rank == 0:
            q_sp = torch.cat(gathered, dim=1).numpy()
            kc0 = np.zeros_like(kc)
            vc0 = np.zeros_like(kc)
            q_whole = oracle.default().qk_norm_rope_append(
                q, k, v, 0, n, chunk.frame_offset, w.T, w.H, w.W, wq, wk, w.eps, kc0, vc0,
                chunk.slot)
            ok = np.array_equal(q_sp, q_whole) and np.array_equal(kc_t.numpy(), kc0)
            with open(q_path, "w") as f:
                f.write("ok" if ok else "mismatch")
    finally:
        dist.destroy_process_group()


def _a2a_rank(rank, world, port, out_path):
    _init(rank, world, port)
    import datetime

    import oracle
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        B, N, D, T, H, W, s, C, slot = 1, 4, 128, 3, 4, 6, 3, 96, 80
        L = T * H * W
        hl = N // world
        rng = np.random.default_rng(77)  # the same inputs on every rank
        q, k, v = (rng.standard_normal((B, L, N, D)).astype(np.float32).astype(np.float64)
                   for _ in range(3))
        wq, wk = (rng.uniform(0.5, 1.5, N * D).astype(np.float32).astype(np.float64)
                  for _ in range(2))
        n = L // world
        a, e = rank * n, (rank + 1) * n  # Algorithm 3 step 2: Delta = r L_local
        orc = oracle.default()
        # the pages' order: local step, then an all-to-all over (sequence, heads)
        kc = np.zeros((B, C, N, D))
        vc = np.zeros_like(kc)
        q_loc = orc.qk_norm_rope_append(q[:, a:e].copy(), k[:, a:e].copy(), v[:, a:e].copy(),
                                        a, e, s, T, H, W, wq, wk, 1e-6, kc, vc, slot)
        rows = (slot + np.arange(a, e)) % C

        def exchange(x):  # x: [B, n, N, D] -> this rank's heads of every rank's rows
            send = torch.from_numpy(np.ascontiguousarray(
                x.reshape(B, n, world, hl, D).transpose(2, 0, 1, 3, 4)))
            recv = torch.empty_like(send)
            dist.all_to_all_single(recv, send)
            return np.concatenate(list(recv.numpy()), axis=1)  # [B, L, hl, D]

        q_a2a = exchange(q_loc)
        k_a2a, v_a2a = exchange(kc[:, rows]), exchange(vc[:, rows])
        # the fused form: every rank writes each head straight to its owner's buffers
        q_dst = [np.zeros((B, L, hl, D)) for _ in range(world)]
        k_dst = [np.zeros((B, C, hl, D)) for _ in range(world)]
        v_dst = [np.zeros((B, C, hl, D)) for _ in range(world)]
        orc.qk_norm_rope_append_sp(q[:, a:e].copy(), k[:, a:e].copy(), v[:, a:e].copy(), a, e,
                                   s, T, H, W, wq, wk, 1e-6, q_dst, k_dst, v_dst, slot)
        mine = []
        for x in q_dst + k_dst + v_dst:  # land every rank's stores at the owner
            t = torch.from_numpy(x)
            dist.all_reduce(t)  # each element is written by exactly one rank
            mine.append(t.numpy())
        q_f, k_f, v_f = mine[rank], mine[world + rank], mine[2 * world + rank]
        all_rows = (slot + np.arange(L)) % C
        ok = (np.array_equal(q_f, q_a2a) and np.array_equal(k_f[:, all_rows], k_a2a) and
              np.array_equal(v_f[:, all_rows], v_a2a) and
              not np.delete(k_f, all_rows, axis=1).any())
        with open(f"{out_path}.{rank}", "w") as f:
            f.write("ok" if ok else "mismatch")
    finally:
        dist.destroy_process_group()


def _out_a2a_rank(rank, world, port, out_path):
    """Algorithm 3's last step on two gloo ranks: torch's all_to_all_single with the
    sequence scattered and the heads gathered (uneven token slices) against the oracle's
    definition."""
    _init(rank, world, port)
    import datetime

    import oracle
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        B, L, hl, D = 2, 13, 3, 128
        cuts = [0, 5, L]
        o_mine = np.random.default_rng(300 + rank).standard_normal((B, L, hl, D))
        # all_to_all_single splits dim 0: tokens first, then [B, hl, D]
        send = torch.from_numpy(np.ascontiguousarray(o_mine.transpose(1, 0, 2, 3)))
        mine = cuts[rank + 1] - cuts[rank]
        recv = torch.empty((world * mine, B, hl, D), dtype=torch.float64)
        dist.all_to_all_single(recv, send,
                               output_split_sizes=[mine] * world,
                               input_split_sizes=[cuts[j + 1] - cuts[j] for j in range(world)])
        got = np.concatenate([c.transpose(1, 0, 2, 3) for c in np.split(recv.numpy(), world)],
                             axis=2)  # source rank j's heads at [j hl, (j+1) hl)
        everyone = [None] * world
        dist.all_gather_object(everyone, o_mine)
        ref = oracle.Oracle.sp_output_all_to_all(everyone, cuts)[rank]
        with open(f"{out_path}.{rank}", "w") as f:
            f.write("ok" if got.shape == ref.shape and np.array_equal(got, ref) else "mismatch")
    finally:
        dist.destroy_process_group()


def _sp_table_rank(rank, world, port, out_path):
    """The multi-GPU wiring's address bookkeeping with a CPU stand-in for the symmetric
    allocation: every rank's destination table lists, in rank order, the regions that
    each rank exposes as its own q and cache tensors."""
    _init(rank, world, port)
    import datetime

    from rotary_position_encoding_b200 import rope3d, sp
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        def exchange(nbytes, device, group):
            buf = torch.zeros(nbytes, dtype=torch.uint8)
            bases = [None] * world
            dist.all_gather_object(bases, buf.data_ptr(), group=group)
            return buf, bases, lambda: dist.barrier(group=group)

        ok = True
        for layout in (rope3d.ROPE3D_CACHE_TOKEN_MAJOR, rope3d.ROPE3D_CACHE_HEAD_MAJOR):
            st = sp.SequenceParallelStep(dist.group.WORLD, rank, world, B=2, N=6, q_rows=77,
                                         cache_tokens=131, dtype=torch.bfloat16, device="cpu",
                                         cache_layout=layout, exchange=exchange)
            own = (st.q.data_ptr(), st.k_cache.data_ptr(), st.v_cache.data_ptr(),
                   st.out(st.layout.out_rows).data_ptr())
            everyone = [None] * world
            dist.all_gather_object(everyone, own)
            ok &= ([list(x) for x in zip(st.q_dst, st.k_dst, st.v_dst, st.out_dst)]
                   == [list(e) for e in everyone])
            cshape = (2, 131, 3, 128) if layout == rope3d.ROPE3D_CACHE_TOKEN_MAJOR else (2, 3, 131, 128)
            ok &= tuple(st.q.shape) == (2, 77, 3, 128) and tuple(st.k_cache.shape) == cshape
            lay = st.layout  # regions start on 256-byte boundaries of the allocation
            ok &= all(off % 256 == 0 for off in (lay.q_off, lay.k_off, lay.v_off, lay.out_off,
                                                 lay.nbytes))
            ends = sorted((t.data_ptr(), t.data_ptr() + t.numel() * 2)
                          for t in (st.q, st.k_cache, st.v_cache, st.out(st.layout.out_rows)))
            ok &= all(a[1] <= b[0] for a, b in zip(ends, ends[1:]))
            ok &= ends[-1][1] <= st.buffer.data_ptr() + st.buffer.numel()
            st.barrier()
        with open(f"{out_path}.{rank}", "w") as f:
            f.write("ok" if ok else "mismatch")
    finally:
        dist.destroy_process_group()


def _timing_rank(rank, world, port, out_path):
    _init(rank, world, port)
    import bench
    d = bench.Dist()
    d.init("gloo")
    try:
        worst = d.max(10.0 * (rank + 1), torch.device("cpu"))
        d.barrier()
        if rank == 0:
            tokens = 75600 * 3 * d.world  # every rank processed its own full job
            with open(out_path, "w") as f:
                f.write(f"{d.world} {worst} {tokens / (worst / 1e3)}")
    finally:
        d.close()


def test_sequence_parallel_slices_on_two_ranks(tmp_path):
    out = str(tmp_path / "sp.txt")
    mp.start_processes(_sp_rank, args=(2, _free_port(), out), nprocs=2, start_method="spawn",
                       join=True)
    assert open(out).read() == "ok"


def test_fused_head_scatter_equals_all_to_all_on_two_ranks(tmp_path):
    out = str(tmp_path / "a2a")
    mp.start_processes(_a2a_rank, args=(2, _free_port(), out), nprocs=2, start_method="spawn",
                       join=True)
    assert [open(f"{out}.{r}").read() for r in range(2)] == ["ok", "ok"]


def test_output_all_to_all_equals_torch_all_to_all_on_two_ranks(tmp_path):
    out = str(tmp_path / "oa2a")
    mp.start_processes(_out_a2a_rank, args=(2, _free_port(), out), nprocs=2,
                       start_method="spawn", join=True)
    assert open(out + ".0").read() == "ok" and open(out + ".1").read() == "ok"


def test_sp_destination_tables_on_two_ranks(tmp_path):
    out = str(tmp_path / "sptab")
    mp.start_processes(_sp_table_rank, args=(2, _free_port(), out), nprocs=2,
                       start_method="spawn", join=True)
    assert [open(f"{out}.{r}").read() for r in range(2)] == ["ok", "ok"]


def test_bench_timing_is_max_over_ranks(tmp_path):
    out = str(tmp_path / "timing.txt")
    mp.start_processes(_timing_rank, args=(2, _free_port(), out), nprocs=2,
                       start_method="spawn", join=True)
    world, worst, value = open(out).read().split()
    assert int(world) == 2
    assert float(worst) == 20.0
    assert float(value) == pytest.approx(75600 * 3 * 2 / 0.020)


def test_sp_plan_layout():
    """The per-rank allocation plan: regions 256-byte aligned, in order q, K, V, sized for
    the rank's heads; uneven head splits are refused."""
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    from rotary_position_encoding_b200 import rope3d, sp
    lay = sp.plan(B=2, N=40, P=8, q_rows=10800, cache_tokens=75600, dtype=torch.bfloat16)
    assert lay.q_shape == (2, 10800, 5, 128) and lay.cache_shape == (2, 75600, 5, 128)
    q_bytes = 2 * 10800 * 5 * 128 * 2
    c_bytes = 2 * 75600 * 5 * 128 * 2
    assert lay.q_off == 0 and lay.k_off >= q_bytes and lay.v_off >= lay.k_off + c_bytes
    o_bytes = 2 * 1350 * 40 * 128 * 2  # the largest of 8 even slices of 10800 tokens
    assert lay.out_rows == 1350 and lay.out_off >= lay.v_off + c_bytes
    assert lay.nbytes >= lay.out_off + o_bytes
    assert all(x % 256 == 0 for x in (lay.k_off, lay.v_off, lay.out_off, lay.nbytes))
    assert sp.even_cuts(10, 4) == [0, 2, 5, 7, 10]
    assert sp.plan(1, 12, 4, 10, 64, torch.bfloat16).out_rows == 3
    head = sp.plan(1, 12, 4, 100, 64, torch.bfloat16, rope3d.ROPE3D_CACHE_HEAD_MAJOR)
    assert head.cache_shape == (1, 3, 64, 128)
    with pytest.raises(ValueError):
        sp.plan(1, 12, 5, 100, 64, torch.bfloat16)
