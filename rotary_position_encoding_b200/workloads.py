"""Seeded synthetic inputs and the workload shapes they come in.

This module holds random-number generation and bf16 bit handling only; none of the
method's arithmetic lives here, so the CUDA path and the fp64 CPU oracle can both take
their inputs from it.

Shapes follow the workloads of "Accelerating Video Generation Inference with
Sequential-Parallel 3D Positional Encoding Using a Global Time Index" (Yuan & Li):
Self-Forcing chunks of three latent frames (Section 3.3.2, item 1: start frames 0, 3,
6, ...), 480P generation (Section 4.1) on a Wan2.1-1.3B-shaped backbone (12 heads of
128) and a Wan2.1-14B-shaped 720P backbone (40 heads of 128).  The pages publish no
dataset for this step; every tensor is drawn here: q, k, v ~ N(0, 1) as float32,
rounded to bfloat16 with round-to-nearest-even for the bf16 workloads; RMSNorm weights
~ U(0.5, 1.5) float32.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

HEAD_DIM = 128


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bit patterns.
    Inputs are finite normals, so no NaN handling is needed."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float64."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32)


@dataclass
class Chunk:
    """One call of the step: token range [token_begin, token_end) of a chunk with grid
    (T, H, W), start frame ``frame_offset`` and cache slot ``slot``."""
    frame_offset: int
    slot: int
    token_begin: int
    token_end: int


@dataclass
class Workload:
    name: str
    B: int
    T: int
    H: int
    W: int
    N: int
    dtype: str            # "f32" or "bf16"
    cache_tokens: int
    seed: int
    chunks: list = field(default_factory=list)
    eps: float = 1e-6

    @property
    def dim(self) -> int:
        return self.N * HEAD_DIM

    @property
    def tokens_per_chunk(self) -> int:
        return self.T * self.H * self.W

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def algorithmic_bytes(self, n_tok: int) -> int:
        """Bytes one call must move: read q, k, v and write q_out, k_cache, v_cache."""
        return 6 * self.B * n_tok * self.dim * self.elem_bytes


def _three_frame_chunks(hw: int, frames: int, window_frames: int):
    out = []
    for s in range(0, frames, 3):
        out.append(Chunk(frame_offset=s, slot=(s % window_frames) * hw,
                         token_begin=0, token_end=3 * hw))
    return out


def tiny() -> Workload:
    """72-token grid (3x4x6), 2 heads, fp32; chunks at start frames 0 and 3 into a
    6-frame (144-token) cache."""
    return Workload("tiny_3x4x6_h2_f32", B=1, T=3, H=4, W=6, N=2, dtype="f32",
                    cache_tokens=144, seed=1,
                    chunks=[Chunk(0, 0, 0, 72), Chunk(3, 72, 0, 72)])


def chunk_480p() -> Workload:
    """Self-Forcing-1.3B-shaped 480P chunk: 3x30x52 = 4680 tokens, 12 heads, bf16,
    start frames 0, 3, ..., 18 appended into a 21-frame (32760-token) cache."""
    return Workload("chunk480p_3x30x52_h12_bf16", B=1, T=3, H=30, W=52, N=12, dtype="bf16",
                    cache_tokens=21 * 1560, seed=2,
                    chunks=_three_frame_chunks(1560, 21, 21))


def full_480p() -> Workload:
    """Whole 480P sequence: 21x30x52 = 32760 tokens, 12 heads, bf16, start frame 0, run
    once whole and once as 8 contiguous token-range slices."""
    n = 21 * 30 * 52
    return Workload("full480p_21x30x52_h12_bf16", B=1, T=21, H=30, W=52, N=12, dtype="bf16",
                    cache_tokens=n, seed=3, chunks=[Chunk(0, 0, 0, n)])


def slices(n_tokens: int, parts: int):
    """Contiguous [begin, end) ranges covering [0, n_tokens) in ``parts`` pieces."""
    bounds = [(p * n_tokens) // parts for p in range(parts + 1)]
    return [(bounds[p], bounds[p + 1]) for p in range(parts)]


def chunk_720p() -> Workload:
    """Wan-14B-shaped 720P: 21 latent frames of 45x80, 40 heads, bf16, in 3-frame chunks
    of 10800 tokens appended into a 75600-token cache (start frames 0..18)."""
    return Workload("chunk720p_3x45x80_h40_bf16", B=1, T=3, H=45, W=80, N=40, dtype="bf16",
                    cache_tokens=21 * 3600, seed=4,
                    chunks=_three_frame_chunks(3600, 21, 21))


def long_horizon() -> Workload:
    """Batch 2, 12 heads, 30x52 grid, 80 chunks of 3 frames (global frames up to 239)
    into a rolling 21-frame (32760-token) window with wrap-around slots."""
    return Workload("longhorizon_b2_3x30x52_h12_bf16", B=2, T=3, H=30, W=52, N=12,
                    dtype="bf16", cache_tokens=21 * 1560, seed=5,
                    chunks=_three_frame_chunks(1560, 240, 21))


ALL = {w.name: w for w in (tiny(), chunk_480p(), full_480p(), chunk_720p(), long_horizon())}


def rng_for(seed: int, *stream: int) -> np.random.Generator:
    return np.random.default_rng([seed, *stream])


def normal_tensor(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    """N(0,1) float32 draws; for bf16 returned as uint16 bit patterns (RNE-rounded)."""
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if dtype == "f32":
        return x
    return f32_to_bf16_bits(x)


def norm_weights(seed: int, dim: int):
    """RMSNorm weights for q and k, U(0.5, 1.5) float32."""
    rng = rng_for(seed, 1000)
    wq = rng.uniform(0.5, 1.5, size=dim).astype(np.float32)
    wk = rng.uniform(0.5, 1.5, size=dim).astype(np.float32)
    return wq, wk


def chunk_inputs(w: Workload, chunk_index: int, n_tok: int | None = None):
    """q, k, v of one call: [B, n_tok, N, 128] (float32, or bf16 bits as uint16)."""
    n = w.tokens_per_chunk if n_tok is None else n_tok
    rng = rng_for(w.seed, chunk_index)
    shape = (w.B, n, w.N, HEAD_DIM)
    return tuple(normal_tensor(rng, shape, w.dtype) for _ in range(3))


def hidden_states(w: Workload, chunk_index: int, K: int, n_tok: int | None = None):
    """Token rows x [B, n_tok, K] entering the QKV projection: N(0,1), bf16 bits."""
    n = w.tokens_per_chunk if n_tok is None else n_tok
    rng = rng_for(w.seed, 2000 + chunk_index)
    return f32_to_bf16_bits(rng.standard_normal(size=(w.B, n, K), dtype=np.float32))


def projection_weights(seed: int, dim: int, K: int):
    """A QKV projection: weight [3 dim, K] ~ N(0, 4/K) as bf16 bits (so that the projected
    values are about N(0, 4): the RMSNorm then halves them) and bias [3 dim] ~ N(0, 0.1^2)
    float32."""
    rng = rng_for(seed, 3000)
    w = rng.standard_normal(size=(3 * dim, K), dtype=np.float32) * np.float32(2.0 / np.sqrt(K))
    b = (rng.standard_normal(size=3 * dim, dtype=np.float32) * np.float32(0.1))
    return f32_to_bf16_bits(w), b


def to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 view of a workload tensor (float32 or bf16 bits)."""
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float64)
    return bf16_bits_to_f64(x)
