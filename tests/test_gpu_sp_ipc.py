"""The sequence-parallel step with its destinations in another process's memory.

"Accelerating Video Generation Inference with Sequential-Parallel 3D Positional Encoding
Using a Global Time Index", Algorithm 3 step 4 and Section 3.4.1 item 1: after each rank
rotates its own token slice, a FusedAllToAll gathers the sequence and scatters the heads.
rope3d_qk_norm_rope_append_sp folds that exchange into its stores, so on a multi-GPU node
every rank writes the heads it does not own straight into the owners' buffers through
peer mappings.  Here two processes share one GPU: each allocates its own destination
buffers (q rows and K/V caches for its half of the heads), hands them to the other
process through CUDA IPC (torch.multiprocessing), and runs the step on its half of the
sequence with a destination table that mixes its own buffers and the other process's
mapped ones.  The kernels never wait on each other; the processes meet only on the host
(a barrier) after both have synchronised.  Then each process checks its own buffers
against the plain step on the whole sequence split by heads: bit-identical, so every
store through the mapped addresses landed where it belongs and nothing else moved.  Then
the output all-to-all (Algorithm 3, last step) runs the other way across the processes:
each sends its gathered q rows back as the other's token slice with every head, and each
checks that it got exactly the plain step's rows of its own slice."""
import os
import sys

import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# shape: 2 ranks, 8 heads (4 per rank), a 2 x 6 x 10 grid (120 tokens) at start frame 3,
# cache of 160 rows at slot 30 (so the rows wrap), bf16
P, N, T, H, W, S, C, SLOT = 2, 8, 2, 6, 10, 3, 160, 30


def _worker(rank, shared, barrier, results):
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import numpy as np
    import torch

    from rotary_position_encoding_b200 import rope3d, workloads as wl
    try:
        torch.cuda.set_device(0)
        D = wl.HEAD_DIM
        L = T * H * W
        hl = N // P
        rng = np.random.default_rng(77)  # both processes draw the same inputs
        raw = [wl.normal_tensor(rng, (1, L, N, D), "bf16") for _ in range(3)]
        wq_np = rng.uniform(0.5, 1.5, N * D).astype(np.float32)
        wk_np = rng.uniform(0.5, 1.5, N * D).astype(np.float32)

        def dev(x):
            return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
        q, k, v = (dev(x) for x in raw)
        wq, wk = torch.from_numpy(wq_np).cuda(), torch.from_numpy(wk_np).cuda()
        tables = rope3d.rope3d_tables_init(max_t=S + T, max_h=H, max_w=W)

        # this process's destination buffers, with sentinels
        mine = (torch.full((1, L, hl, D), 3.0, dtype=torch.bfloat16, device="cuda"),
                torch.full((1, C, hl, D), 2.0, dtype=torch.bfloat16, device="cuda"),
                torch.full((1, C, hl, D), -2.0, dtype=torch.bfloat16, device="cuda"))
        torch.cuda.synchronize()
        shared[rank].put(mine)              # exported through CUDA IPC
        theirs = shared[1 - rank].get(timeout=60)  # the other process's buffers, mapped here
        dst = [None, None]
        dst[rank], dst[1 - rank] = mine, theirs
        a, e = wl.slices(L, P)[rank]
        rope3d.rope3d_qk_norm_rope_append_sp(
            q[:, a:e].contiguous(), k[:, a:e].contiguous(), v[:, a:e].contiguous(), a, e, S,
            T, H, W, wq, wk, 1e-6, [d[0] for d in dst], [d[1] for d in dst],
            [d[2] for d in dst], SLOT, tables, q_row0=0)
        torch.cuda.synchronize()
        barrier.wait(timeout=60)            # both processes' stores are done

        # the plain step on the whole sequence, split by heads
        qo = torch.empty_like(q)
        kc = torch.full((1, C, N, D), 2.0, dtype=torch.bfloat16, device="cuda")
        vc = torch.full((1, C, N, D), -2.0, dtype=torch.bfloat16, device="cuda")
        rope3d.rope3d_qk_norm_rope_append(q, k, v, qo, 0, L, S, T, H, W, wq, wk, 1e-6, kc, vc,
                                          SLOT, tables)
        torch.cuda.synchronize()
        heads = slice(rank * hl, (rank + 1) * hl)
        ok = all(torch.equal(x.view(torch.int16), y.contiguous().view(torch.int16))
                 for x, y in ((mine[0], qo[:, :, heads]), (mine[1], kc[:, :, heads]),
                              (mine[2], vc[:, :, heads])))
        # Algorithm 3's last step across the processes: each one sends its gathered q rows
        # (every token, its heads) back as the other's token slice with all heads
        cuts = wl.slices(L, P)
        cuts = [c[0] for c in cuts] + [L]
        back = torch.full((1, cuts[rank + 1] - cuts[rank], N, D), 9.0, dtype=torch.bfloat16,
                          device="cuda")
        torch.cuda.synchronize()            # the fill lands before the other process writes
        shared[rank].put(back)
        their_back = shared[1 - rank].get(timeout=60)
        outs = [None, None]
        outs[rank], outs[1 - rank] = back, their_back
        barrier.wait(timeout=60)            # both outputs are mapped before either writes
        rope3d.rope3d_sp_output_all_to_all(mine[0], outs, rank, cuts)
        torch.cuda.synchronize()
        barrier.wait(timeout=60)            # both processes' stores are done
        ok2 = torch.equal(back.view(torch.int16),
                          qo[:, cuts[rank]:cuts[rank + 1]].contiguous().view(torch.int16))
        msg = ("" if ok and ok2 else
               "destination buffers differ from the plain step" if not ok else
               "the output all-to-all did not return this rank's slice")
        results.put((rank, ok and ok2, msg))
        del their_back, outs
        del theirs, dst
        torch.cuda.synchronize()
        barrier.wait(timeout=60)            # the mapping is released before either exits
        tables.close()
    except Exception as exc:  # report, then let the parent fail the test
        results.put((rank, False, repr(exc)))
        try:
            barrier.abort()
        except Exception:
            pass


def test_sp_step_stores_heads_into_another_process_buffers():
    ctx = mp.get_context("spawn")
    shared = [ctx.Queue(), ctx.Queue()]
    barrier = ctx.Barrier(P)
    results = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, shared, barrier, results)) for r in range(P)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(P):
            rank, ok, msg = results.get(timeout=240)
            got[rank] = (ok, msg)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert sorted(got) == [0, 1], got
    for rank, (ok, msg) in got.items():
        assert ok, f"rank {rank}: {msg}"
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
