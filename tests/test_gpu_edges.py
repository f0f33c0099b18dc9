"""Edge cases of the CUDA path against the fp64 oracle: ragged and single-token ranges,
in-place q_out, cache wrap inside a call, batch > 1, head counts from 1 to the maximum,
degenerate grids, zero rows, the rotation-only entry point, and argument errors (which
must return a status, launch nothing and leave every output untouched)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_support import PATHS, assert_close, kernel_path, to_bits, to_device, to_f64, torch_dtype
from rotary_position_encoding_b200 import rope3d, workloads as wl

pytestmark = pytest.mark.gpu

D = wl.HEAD_DIM
EPS = 1e-6


def _setup(B, n_tok, N, dtype, seed, C, max_t, H, W, schedule=0):
    rng = np.random.default_rng(seed)
    raw = [wl.normal_tensor(rng, (B, n_tok, N, D), dtype) for _ in range(3)]
    wq = rng.uniform(0.5, 1.5, N * D).astype(np.float32)
    wk = rng.uniform(0.5, 1.5, N * D).astype(np.float32)
    dev = [to_device(x, dtype) for x in raw]
    kc = torch.full((B, C, N, D), 3.0, dtype=torch_dtype(dtype), device="cuda")
    vc = torch.full((B, C, N, D), -3.0, dtype=torch_dtype(dtype), device="cuda")
    tables = rope3d.rope3d_tables_init(max_t=max_t, max_h=H, max_w=W, schedule=schedule)
    return raw, dev, wq, wk, kc, vc, tables


def _check_against_oracle(raw, dtype, wq, wk, qo, kc, vc, tb, te, s, T, H, W, C, slot,
                          schedule=0):
    B, n_tok, N, _ = raw[0].shape
    f64 = [wl.to_f64(x, dtype) for x in raw]
    kc_ref = np.full((B, C, N, D), 3.0)
    vc_ref = np.full((B, C, N, D), -3.0)
    ref_q = oracle.default().qk_norm_rope_append(
        f64[0], f64[1], f64[2], tb, te, s, T, H, W, wq.astype(np.float64),
        wk.astype(np.float64), EPS, kc_ref, vc_ref, slot, schedule=schedule)
    assert_close(to_f64(qo), ref_q, dtype, "q_out")
    assert_close(to_f64(kc), kc_ref, dtype, "k_cache (written and untouched rows)")
    assert np.array_equal(to_f64(vc), vc_ref), "v_cache"


@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("rng_", [(0, 1), (71, 72), (5, 42), (23, 25), (0, 72), (17, 71)])
def test_ragged_and_single_token_ranges(dtype, rng_, path):
    tb, te = rng_
    T, H, W, s, C, slot = 3, 4, 6, 6, 144, 100
    raw, dev, wq, wk, kc, vc, tables = _setup(2, te - tb, 2, dtype, 7, C, 9, H, W)
    qo = torch.empty_like(dev[0])
    with kernel_path(PATHS[path]):
        rope3d.rope3d_qk_norm_rope_append(dev[0], dev[1], dev[2], qo, tb, te, s, T, H, W,
                                          torch.from_numpy(wq).cuda(),
                                          torch.from_numpy(wk).cuda(), EPS, kc, vc, slot, tables)
    torch.cuda.synchronize()
    _check_against_oracle(raw, dtype, wq, wk, qo, kc, vc, tb, te, s, T, H, W, C, slot)


@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("trig", [rope3d.ROPE3D_TRIG_TABLE, rope3d.ROPE3D_TRIG_ONTHEFLY])
def test_in_place_q_and_cache_wrap(trig, path):
    T, H, W, s, C = 3, 30, 52, 12, 5000
    n = T * H * W
    slot = C - 777  # the range wraps around the end of the cache
    raw, dev, wq, wk, kc, vc, tables = _setup(1, n, 12, "bf16", 8, C, 15, H, W)
    q_inplace = dev[0].clone()
    with kernel_path(PATHS[path]):
        rope3d.rope3d_qk_norm_rope_append(q_inplace, dev[1], dev[2], q_inplace, 0, n, s, T, H,
                                          W, torch.from_numpy(wq).cuda(),
                                          torch.from_numpy(wk).cuda(), EPS, kc, vc, slot, tables,
                                          trig)
    torch.cuda.synchronize()
    _check_against_oracle(raw, "bf16", wq, wk, q_inplace, kc, vc, 0, n, s, T, H, W, C, slot)


@pytest.mark.parametrize("path", ["auto", "registers"])
@pytest.mark.parametrize("dtype,N", [("bf16", 1), ("bf16", 3), ("bf16", 5), ("bf16", 12),
                                     ("bf16", 40), ("bf16", 64), ("bf16", 128), ("f32", 1),
                                     ("f32", 3), ("f32", 12), ("f32", 64)])
def test_head_counts_up_to_maximum(dtype, N, path):
    T, H, W, s, C, slot = 2, 3, 5, 4, 64, 7
    n = T * H * W
    raw, dev, wq, wk, kc, vc, tables = _setup(2, n, N, dtype, 100 + N, C, 6, H, W)
    qo = torch.empty_like(dev[0])
    forced = rope3d.ROPE3D_PATH_AUTO if path == "auto" else rope3d.ROPE3D_PATH_REGISTERS
    with kernel_path(forced):
        rope3d.rope3d_qk_norm_rope_append(dev[0], dev[1], dev[2], qo, 0, n, s, T, H, W,
                                          torch.from_numpy(wq).cuda(),
                                          torch.from_numpy(wk).cuda(), EPS, kc, vc, slot, tables)
    torch.cuda.synchronize()
    _check_against_oracle(raw, dtype, wq, wk, qo, kc, vc, 0, n, s, T, H, W, C, slot)


def test_head_count_beyond_maximum_is_rejected():
    raw, dev, wq, wk, kc, vc, tables = _setup(1, 4, 256, "bf16", 1, 8, 2, 2, 2)
    qo = torch.zeros_like(dev[0])
    with pytest.raises(rope3d.Rope3dError) as e:
        rope3d.rope3d_qk_norm_rope_append(dev[0], dev[1], dev[2], qo, 0, 4, 0, 1, 2, 2,
                                          torch.from_numpy(wq).cuda(),
                                          torch.from_numpy(wk).cuda(), EPS, kc, vc, 0, tables)
    assert e.value.status == rope3d.ROPE3D_EINVAL
    assert bool((qo == 0).all())


@pytest.mark.parametrize("grid", [(1, 1, 1), (1, 1, 9), (4, 1, 1), (1, 7, 1), (2, 3, 1)])
@pytest.mark.parametrize("schedule", [0, 1])
def test_degenerate_grids(grid, schedule):
    T, H, W = grid
    n = T * H * W
    s, C, slot = 237, n, 0
    raw, dev, wq, wk, kc, vc, tables = _setup(1, n, 2, "f32", 9, C, s + T, H, W, schedule)
    qo = torch.empty_like(dev[0])
    rope3d.rope3d_qk_norm_rope_append(dev[0], dev[1], dev[2], qo, 0, n, s, T, H, W,
                                      torch.from_numpy(wq).cuda(), torch.from_numpy(wk).cuda(),
                                      EPS, kc, vc, slot, tables)
    torch.cuda.synchronize()
    # fp32 angles at frame 237+ carry ~1e-5 rad of table rounding; stay within 1e-5 abs
    # by comparing in the table path, which is built in fp64
    _check_against_oracle(raw, "f32", wq, wk, qo, kc, vc, 0, n, s, T, H, W, C, slot, schedule)


def test_zero_rows_give_zero_with_positive_eps():
    T, H, W = 1, 2, 2
    raw, dev, wq, wk, kc, vc, tables = _setup(1, 4, 2, "bf16", 10, 4, 1, H, W)
    zeros = torch.zeros_like(dev[0])
    qo = torch.empty_like(zeros)
    rope3d.rope3d_qk_norm_rope_append(zeros, zeros, zeros, qo, 0, 4, 0, T, H, W,
                                      torch.from_numpy(wq).cuda(), torch.from_numpy(wk).cuda(),
                                      EPS, kc, vc, 0, tables)
    torch.cuda.synchronize()
    assert bool((qo.float() == 0).all()) and bool((kc.float() == 0).all())


def test_position_zero_rotation_is_identity_after_norm():
    """At (t, h, w) = (0, 0, 0) the rotation is the identity, so q_out is RMSNorm(q)."""
    T, H, W = 1, 1, 1
    raw, dev, wq, wk, kc, vc, tables = _setup(1, 1, 4, "f32", 11, 1, 1, H, W)
    qo = torch.empty_like(dev[0])
    rope3d.rope3d_qk_norm_rope_append(dev[0], dev[1], dev[2], qo, 0, 1, 0, T, H, W,
                                      torch.from_numpy(wq).cuda(), torch.from_numpy(wk).cuda(),
                                      EPS, kc, vc, 0, tables)
    torch.cuda.synchronize()
    expect = oracle.default().rms_norm(raw[0].astype(np.float64), wq.astype(np.float64), EPS)
    assert_close(to_f64(qo).ravel(), expect, "f32", "identity at position 0")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("trig", [rope3d.ROPE3D_TRIG_TABLE, rope3d.ROPE3D_TRIG_ONTHEFLY])
@pytest.mark.parametrize("inplace", [False, True])
def test_apply_matches_oracle(dtype, trig, inplace):
    T, H, W, s = 3, 30, 52, 9
    n = T * H * W
    tb, te = 1000, 3333
    rng = np.random.default_rng(12)
    raw = wl.normal_tensor(rng, (2, te - tb, 3, D), dtype)
    x = to_device(raw, dtype)
    tables = rope3d.rope3d_tables_init(max_t=12, max_h=H, max_w=W)
    out = x if inplace else torch.empty_like(x)
    rope3d.rope3d_apply(x, out, tb, te, s, T, H, W, tables, trig)
    torch.cuda.synchronize()
    ref = oracle.default().apply(wl.to_f64(raw, dtype), tb, te, s, T, H, W)
    assert_close(to_f64(out), ref, dtype, "apply")
    assert n >= te


# ---------------------------------------------------------------- argument errors

def _err_case():
    T, H, W, C = 3, 4, 6, 144
    raw, dev, wq, wk, kc, vc, tables = _setup(1, 72, 2, "bf16", 13, C, 6, H, W)
    return dict(dev=dev, wq=torch.from_numpy(wq).cuda(), wk=torch.from_numpy(wk).cuda(),
                kc=kc, vc=vc, tables=tables)


def _call(c, q=None, k=None, v=None, qo=None, tb=0, te=72, s=0, T=3, H=4, W=6, kc=None,
          vc=None, slot=0, trig=rope3d.ROPE3D_TRIG_TABLE, eps=EPS, tables=None, N=2,
          dtype=rope3d.ROPE3D_BF16, Dh=128, C=144):
    lib = rope3d.load_library()
    q = c["dev"][0] if q is None else q
    k = c["dev"][1] if k is None else k
    v = c["dev"][2] if v is None else v
    qo = c["qo"] if qo is None else qo
    kc = c["kc"] if kc is None else kc
    vc = c["vc"] if vc is None else vc
    tables = c["tables"] if tables is None else tables
    return lib.rope3d_qk_norm_rope_append(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), qo.data_ptr(), 1, N, Dh, dtype, tb, te, s,
        T, H, W, c["wq"].data_ptr(), c["wk"].data_ptr(), eps, kc.data_ptr(), vc.data_ptr(), C,
        slot, tables.handle, trig, torch.cuda.current_stream().cuda_stream)


def test_errors_return_status_and_touch_nothing():
    c = _err_case()
    c["qo"] = torch.full_like(c["dev"][0], 5.0)
    kc0, vc0 = c["kc"].clone(), c["vc"].clone()
    big = torch.zeros(1, 72 * 2 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    misaligned = big.view(-1)[1:1 + 72 * 2 * 128]
    cases = {
        "empty range": (dict(tb=5, te=5), rope3d.ROPE3D_ERANGE),
        "past the grid": (dict(tb=0, te=73), rope3d.ROPE3D_ERANGE),
        "negative begin": (dict(tb=-1, te=71), rope3d.ROPE3D_ERANGE),
        "bad grid": (dict(T=0), rope3d.ROPE3D_EINVAL),
        "negative offset": (dict(s=-3), rope3d.ROPE3D_EINVAL),
        "frames past table": (dict(s=4), rope3d.ROPE3D_ERANGE),
        "H past table": (dict(H=5, te=72), rope3d.ROPE3D_ERANGE),
        "head size": (dict(Dh=64), rope3d.ROPE3D_EINVAL),
        "dtype": (dict(dtype=7), rope3d.ROPE3D_EINVAL),
        "trig": (dict(trig=9), rope3d.ROPE3D_EINVAL),
        "eps": (dict(eps=-1.0), rope3d.ROPE3D_EINVAL),
        "negative slot": (dict(slot=-1), rope3d.ROPE3D_EINVAL),
        "range longer than cache": (dict(C=71), rope3d.ROPE3D_ERANGE),
        "misaligned q": (dict(q=misaligned), rope3d.ROPE3D_EALIGN),
        "q_out is k": (dict(qo=c["dev"][1]), rope3d.ROPE3D_EOVERLAP),
        "k_cache is v_cache": (dict(kc=c["vc"]), rope3d.ROPE3D_EOVERLAP),
        "v_cache over q": (dict(vc=c["dev"][0]), rope3d.ROPE3D_EOVERLAP),
    }
    for name, (kw, status) in cases.items():
        rc = _call(c, **kw)
        assert rc == status, (name, rc, rope3d.rope3d_last_error())
        assert rope3d.rope3d_last_error(), name
    torch.cuda.synchronize()
    assert bool((c["qo"].float() == 5.0).all())
    assert torch.equal(c["kc"], kc0) and torch.equal(c["vc"], vc0)
    # and a valid call right after still works
    assert _call(c) == rope3d.ROPE3D_OK
    torch.cuda.synchronize()
    assert not bool((c["qo"].float() == 5.0).all())


def test_onthefly_only_tables_reject_table_path():
    c = _err_case()
    c["qo"] = torch.empty_like(c["dev"][0])
    bare = rope3d.rope3d_tables_init()  # no cos/sin rows
    assert _call(c, tables=bare) == rope3d.ROPE3D_ERANGE
    assert _call(c, tables=bare, trig=rope3d.ROPE3D_TRIG_ONTHEFLY) == rope3d.ROPE3D_OK
    torch.cuda.synchronize()
