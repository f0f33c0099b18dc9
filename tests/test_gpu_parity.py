"""The CUDA path against the fp64 oracle on the five seeded workloads, through the C ABI.

Small cases compare every element; the full-size workloads compare sampled rows (the
oracle computes them one token at a time) in the launch configuration the benchmark
times, plus properties that hold at any size (V bit copy, untouched cache rows,
bit-identical slices).  Paper: "Accelerating Video Generation Inference with
Sequential-Parallel 3D Positional Encoding Using a Global Time Index" (Yuan & Li)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_support import (PATHS, Case, assert_close, kernel_path, oracle_rows, to_bits, to_device,
                         to_f64)
from rotary_position_encoding_b200 import rope3d, workloads as wl

pytestmark = pytest.mark.gpu

TABLE, ONTHEFLY = rope3d.ROPE3D_TRIG_TABLE, rope3d.ROPE3D_TRIG_ONTHEFLY


@pytest.fixture(params=sorted(PATHS))
def path(request):
    """Both kernel paths of the fused step: the shared-memory bulk-copy ring and the
    register kernel."""
    with kernel_path(PATHS[request.param]):
        yield request.param


def _inputs(w, chunk_index, n_tok=None):
    """Device tensors and the host workload tensors (float32 or bf16 bits) of one call."""
    q, k, v = wl.chunk_inputs(w, chunk_index, n_tok)
    dev = [to_device(x, w.dtype) for x in (q, k, v)]
    return dev, (q, k, v)


def _f64(raw, w):
    return [wl.to_f64(x, w.dtype) for x in raw]


def _full_oracle(w, case, f64, chunk):
    orc = oracle.default()
    kc = np.zeros((w.B, w.cache_tokens, w.N, wl.HEAD_DIM))
    vc = np.zeros_like(kc)
    qo = orc.qk_norm_rope_append(f64[0], f64[1], f64[2], chunk.token_begin, chunk.token_end,
                                 chunk.frame_offset, w.T, w.H, w.W,
                                 case.wq_np.astype(np.float64), case.wk_np.astype(np.float64),
                                 w.eps, kc, vc, chunk.slot, schedule=case.schedule)
    return qo, kc, vc


def _cache_rows(chunk, w, token_begin, token_end):
    return np.array([(chunk.slot + i) % w.cache_tokens for i in range(token_begin, token_end)])


# ---------------------------------------------------------------- tiny, fp32, every element

@pytest.mark.parametrize("trig", [TABLE, ONTHEFLY])
@pytest.mark.parametrize("schedule", [0, 1])
def test_tiny_fp32_every_element(trig, schedule, path):
    w = wl.tiny()
    case = Case(w, schedule=schedule)
    expect_k = np.zeros((w.B, w.cache_tokens, w.N, wl.HEAD_DIM))
    expect_v = np.zeros_like(expect_k)
    for ci, chunk in enumerate(w.chunks):
        dev, raw = _inputs(w, ci)
        qo = case.run(*dev, chunk, trig=trig)
        torch.cuda.synchronize()
        ref_q, kc, vc = _full_oracle(w, case, _f64(raw, w), chunk)
        rows = _cache_rows(chunk, w, chunk.token_begin, chunk.token_end)
        expect_k[:, rows] = kc[:, rows]
        expect_v[:, rows] = vc[:, rows]
        assert_close(to_f64(qo), ref_q, "f32", f"q_out chunk {ci}")
    assert_close(to_f64(case.k_cache), expect_k, "f32", "k_cache")
    assert np.array_equal(to_f64(case.v_cache), expect_v), "v_cache is not a bit copy"


# ---------------------------------------------------------------- 480p chunk, every element

@pytest.mark.slow
def test_chunk_480p_every_element_all_offsets(path):
    w = wl.chunk_480p()
    case = Case(w)
    written = np.zeros(w.cache_tokens, dtype=bool)
    for ci, chunk in enumerate(w.chunks):
        dev, raw = _inputs(w, ci)
        qo = case.run(*dev, chunk)
        torch.cuda.synchronize()
        ref_q, kc, vc = _full_oracle(w, case, _f64(raw, w), chunk)
        rows = _cache_rows(chunk, w, chunk.token_begin, chunk.token_end)
        assert_close(to_f64(qo), ref_q, "bf16", f"q_out s={chunk.frame_offset}")
        assert_close(to_f64(case.k_cache[:, rows]), kc[:, rows], "bf16",
                     f"k_cache s={chunk.frame_offset}")
        assert np.array_equal(to_bits(case.v_cache[:, rows]), raw[2]), "v_cache bit copy"
        written[rows] = True
    assert written.all(), "the seven chunks must fill the 21-frame cache"


# ---------------------------------------------------------------- full 480p: slices vs whole

@pytest.mark.slow
def test_full_480p_slices_bit_identical_to_whole(path):
    w = wl.full_480p()
    n = w.tokens_per_chunk
    chunk = w.chunks[0]
    dev, raw = _inputs(w, 0)
    whole = Case(w)
    q_whole = whole.run(*dev, chunk)
    parts = Case(w)
    q_parts = torch.empty_like(q_whole)
    for (a, e) in wl.slices(n, 8):
        sub = [x[:, a:e].contiguous() for x in dev]
        out = parts.run(*sub, chunk, token_begin=a, token_end=e)
        q_parts[:, a:e] = out
    torch.cuda.synchronize()
    assert torch.equal(q_whole.view(torch.int16), q_parts.view(torch.int16))
    assert torch.equal(whole.k_cache.view(torch.int16), parts.k_cache.view(torch.int16))
    assert torch.equal(whole.v_cache.view(torch.int16), parts.v_cache.view(torch.int16))
    # and both match the oracle on sampled rows, including slice boundaries
    rng = np.random.default_rng(33)
    sample = sorted(set(rng.integers(0, n, 96).tolist()) |
                    {0, n - 1} | {a for a, _ in wl.slices(n, 8)} | {e - 1 for _, e in wl.slices(n, 8)})
    got_q = to_f64(q_whole)
    got_k = to_f64(whole.k_cache)
    for (b, r, qo, ko, vo, pos) in oracle_rows(w, whole, *raw, chunk, [(0, r) for r in sample], 0):
        assert_close(got_q[b, r], qo, "bf16", f"q_out row {r}")
        assert_close(got_k[b, pos[3]], ko, "bf16", f"k_cache row {pos[3]}")


# ---------------------------------------------------------------- 720p, sampled rows

@pytest.mark.slow
def test_chunk_720p_sampled_rows_all_chunks(path):
    w = wl.chunk_720p()
    case = Case(w)
    rng = np.random.default_rng(44)
    hw = w.H * w.W
    for ci, chunk in enumerate(w.chunks):
        dev, raw = _inputs(w, ci)
        qo = case.run(*dev, chunk)
        torch.cuda.synchronize()
        n = chunk.token_end - chunk.token_begin
        sample = sorted(set(rng.integers(0, n, 48).tolist()) |
                        {0, n - 1, hw - 1, hw, 2 * hw, w.W - 1, w.W})
        got_q = to_f64(qo[:, sample])
        rows = [(chunk.slot + r) % w.cache_tokens for r in sample]
        got_k = to_f64(case.k_cache[:, rows])
        got_v = to_bits(case.v_cache[:, rows])
        for si, (b, r, q_ref, k_ref, v_ref, pos) in enumerate(
                oracle_rows(w, case, *raw, chunk, [(0, r) for r in sample], 0)):
            assert pos[3] == rows[si]
            assert_close(got_q[b, si], q_ref, "bf16", f"720p chunk {ci} q row {r}")
            assert_close(got_k[b, si], k_ref, "bf16", f"720p chunk {ci} k row {r}")
            assert np.array_equal(got_v[b, si], raw[2][b, r])
    # after seven chunks every cache row has been written exactly by its own token
    assert bool((case.v_cache.view(torch.int16) != 0).any(dim=(0, 2, 3)).all())


# ---------------------------------------------------------------- long horizon, rolling window

@pytest.mark.slow
def test_long_horizon_rolling_window_table_and_onthefly(path):
    w = wl.long_horizon()
    tab = Case(w, max_t=240)
    fly = Case(w, max_t=240)
    rng = np.random.default_rng(55)
    hw = w.H * w.W
    max_diff = 0.0
    last_writer = {}
    for ci, chunk in enumerate(w.chunks):
        dev, raw = _inputs(w, ci)
        q_tab = tab.run(*dev, chunk, trig=TABLE)
        q_fly = fly.run(*dev, chunk, trig=ONTHEFLY)
        for r in range(0, chunk.token_end, hw):
            last_writer[(chunk.slot + r) % w.cache_tokens] = (ci, r)
        if ci % 8 == 0 or ci >= len(w.chunks) - 2:
            torch.cuda.synchronize()
            sample = sorted(set(rng.integers(0, chunk.token_end, 12).tolist()) | {0, 3 * hw - 1})
            rows = [(b, r) for b in range(w.B) for r in sample]
            gq_t, gq_f = to_f64(q_tab), to_f64(q_fly)
            for (b, r, q_ref, k_ref, v_ref, pos) in oracle_rows(w, tab, *raw, chunk, rows, 0):
                assert pos[0] == chunk.frame_offset + r // hw
                assert_close(gq_t[b, r], q_ref, "bf16", f"table chunk {ci} row {r}")
                assert_close(gq_f[b, r], q_ref, "bf16", f"on-the-fly chunk {ci} row {r}")
                max_diff = max(max_diff, float(np.abs(gq_t[b, r] - gq_f[b, r]).max()))
    torch.cuda.synchronize()
    # the two trig paths differ by at most one bf16 rounding step of the outputs
    assert max_diff <= 0.0625, max_diff
    # the final window holds frames 219..239: check one token per window frame
    assert sorted({ci for ci, _ in last_writer.values()}) == list(range(73, 80))
    regenerated = {}
    for row, (ci, r) in sorted(last_writer.items()):
        chunk = w.chunks[ci]
        if ci not in regenerated:
            regenerated[ci] = _inputs(w, ci, None)
        dev, raw = regenerated[ci]
        got = to_bits(tab.v_cache[:, row])
        assert np.array_equal(got, raw[2][:, r]), (row, ci, r)
        (b, rr, q_ref, k_ref, v_ref, pos) = oracle_rows(w, tab, *raw, chunk, [(1, r)], 0)[0]
        assert pos[3] == row
        assert_close(to_f64(tab.k_cache[1, row]), k_ref, "bf16", f"final window row {row}")


# ---------------------------------------------------------------- the two kernel paths agree

@pytest.mark.slow
@pytest.mark.parametrize("make", [wl.chunk_480p, wl.chunk_720p, wl.long_horizon, wl.tiny])
def test_kernel_paths_bit_identical(make):
    """The register kernel and the bulk-copy ring kernel run the same per-row arithmetic
    in the same order, so their outputs agree bit for bit."""
    w = make()
    chunk = w.chunks[1]
    dev, raw = _inputs(w, 1)
    outs = {}
    for name in sorted(PATHS):
        case = Case(w)
        with kernel_path(PATHS[name]):
            q = case.run(*dev, chunk)
        torch.cuda.synchronize()
        outs[name] = (q, case.k_cache, case.v_cache)
    for other in ("tma",):
        for a, b in zip(outs["registers"], outs[other]):
            assert torch.equal(
                a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32)), other
