"""Helpers shared by the gpu-marked tests: move seeded workload tensors to the device,
run the CUDA path through the C ABI binding, and compare with the fp64 oracle."""
from __future__ import annotations

import contextlib

import numpy as np
import torch

import oracle
from rotary_position_encoding_b200 import rope3d, workloads as wl

# Tolerances, elementwise |gpu - ref| <= ATOL + RTOL |ref| against the unrounded fp64
# oracle.  bf16: one rounding of a value up to ~8 is half an ulp of 0.031, which the
# absolute part alone does not cover, so the relative part carries it.  fp32: max-abs.
BF16_ATOL, BF16_RTOL = 1.6e-2, 8e-3
F32_MAX_ABS = 1e-5


def to_device(x: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)
    bits = np.ascontiguousarray(x, dtype=np.uint16).view(np.int16)
    return torch.from_numpy(bits).view(torch.bfloat16).to(device)


def to_f64(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.numpy().astype(np.float64)
    if t.dtype == torch.bfloat16:
        return wl.bf16_bits_to_f64(t.view(torch.int16).numpy().view(np.uint16))
    raise TypeError(t.dtype)


def to_bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy().view(np.uint32)


def torch_dtype(dtype: str):
    return torch.float32 if dtype == "f32" else torch.bfloat16


def assert_close(gpu: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    err = np.abs(gpu - ref)
    if dtype == "f32":
        worst = float(err.max()) if err.size else 0.0
        assert worst <= F32_MAX_ABS, f"{what}: max abs error {worst:.3g} > {F32_MAX_ABS}"
    else:
        bound = BF16_ATOL + BF16_RTOL * np.abs(ref)
        bad = err > bound
        if bad.any():
            idx = np.argwhere(bad)[0]
            raise AssertionError(
                f"{what}: {int(bad.sum())} of {err.size} elements out of tolerance; first at "
                f"{tuple(idx)}: gpu {gpu[tuple(idx)]!r} ref {ref[tuple(idx)]!r}; "
                f"max err {float(err.max()):.3g}")


class Case:
    """Device-side state of one workload: weights, caches and the tables."""

    def __init__(self, w: wl.Workload, max_t: int | None = None, schedule: int = 0):
        self.w = w
        wq, wk = wl.norm_weights(w.seed, w.dim)
        self.wq_np, self.wk_np = wq, wk
        self.wq = torch.from_numpy(wq).cuda()
        self.wk = torch.from_numpy(wk).cuda()
        shape = (w.B, w.cache_tokens, w.N, wl.HEAD_DIM)
        self.k_cache = torch.zeros(shape, dtype=torch_dtype(w.dtype), device="cuda")
        self.v_cache = torch.zeros(shape, dtype=torch_dtype(w.dtype), device="cuda")
        frames = max([c.frame_offset for c in w.chunks] + [0]) + w.T
        self.tables = rope3d.rope3d_tables_init(
            max_t=max_t or frames, max_h=w.H, max_w=w.W, schedule=schedule)
        self.schedule = schedule

    def run(self, q, k, v, chunk: wl.Chunk, trig=rope3d.ROPE3D_TRIG_TABLE, q_out=None,
            token_begin=None, token_end=None):
        tb = chunk.token_begin if token_begin is None else token_begin
        te = chunk.token_end if token_end is None else token_end
        if q_out is None:
            q_out = torch.empty_like(q)
        rope3d.rope3d_qk_norm_rope_append(
            q, k, v, q_out, tb, te, chunk.frame_offset, self.w.T, self.w.H, self.w.W,
            self.wq, self.wk, self.w.eps, self.k_cache, self.v_cache, chunk.slot, self.tables,
            trig)
        return q_out


def oracle_rows(w: wl.Workload, case: Case, q, k, v, chunk: wl.Chunk, rows,
                token_begin: int):
    """Oracle outputs for selected (b, r) rows of the workload tensors q, k, v (float32 or
    bf16 bits, widened exactly per row): q_out rows and the cache rows they map to."""
    orc = oracle.default()
    out = []
    for (b, r) in rows:
        i = token_begin + r
        q64, k64, v64 = (wl.to_f64(x[b, r], w.dtype) for x in (q, k, v))
        qo, ko, vo, pos = orc.token(q64, k64, v64, i, chunk.frame_offset,
                                    w.T, w.H, w.W, case.wq_np.astype(np.float64),
                                    case.wk_np.astype(np.float64), w.eps, chunk.slot,
                                    w.cache_tokens, schedule=case.schedule)
        out.append((b, r, qo, ko, vo, pos))
    return out


@contextlib.contextmanager
def kernel_path(path: int):
    """Run the block with the fused step forced onto one kernel path."""
    rope3d.rope3d_testing_force_path(path)
    try:
        yield
    finally:
        rope3d.rope3d_testing_force_path(rope3d.ROPE3D_PATH_AUTO)


PATHS = {"tma": rope3d.ROPE3D_PATH_TMA, "registers": rope3d.ROPE3D_PATH_REGISTERS}
