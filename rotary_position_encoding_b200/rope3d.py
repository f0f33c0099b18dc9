"""ctypes binding of librope3d.so (include/rope3d.h): argument marshalling only.

Every function here has the name of the C entry point it calls and does nothing but
turn torch tensors into device pointers and sizes, call the library on the current
CUDA stream, and turn a negative status into an exception.  All the work runs in the
library's CUDA kernels; there is no CPU path.  If the library has not been built,
the first call raises ``RuntimeError`` naming the build command.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(_PKG, "librope3d.so")

ROPE3D_OK = 0
ROPE3D_EINVAL = -1
ROPE3D_ERANGE = -2
ROPE3D_ECUDA = -3
ROPE3D_EDEVICE = -4
ROPE3D_EALIGN = -5
ROPE3D_EOVERLAP = -6
ROPE3D_ETIMEOUT = -7
ROPE3D_EINDEX = -8

ROPE3D_F32 = 0
ROPE3D_BF16 = 1

ROPE3D_SCHEDULE_PER_AXIS = 0
ROPE3D_SCHEDULE_HEAD_WIDE = 1

ROPE3D_TRIG_TABLE = 0
ROPE3D_TRIG_ONTHEFLY = 1

ROPE3D_PAIRING_ADJACENT = 0
ROPE3D_PAIRING_HALF = 1
ROPE3D_CACHE_TOKEN_MAJOR = 0
ROPE3D_CACHE_HEAD_MAJOR = 1
ROPE3D_CACHE_SAME = 0
ROPE3D_CACHE_FP8_E4M3 = 1
ROPE3D_CACHE_NVFP4 = 2


class rope3d_options(ctypes.Structure):
    """struct rope3d_options of include/rope3d.h."""
    _fields_ = [("pairing", ctypes.c_int), ("cache_layout", ctypes.c_int),
                ("cache_dtype", ctypes.c_int), ("reserved0", ctypes.c_int),
                ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
                ("nvfp4_k_global", ctypes.c_float), ("nvfp4_v_global", ctypes.c_float),
                ("reserved", ctypes.c_int * 2)]

ROPE3D_SP_MAX_RANKS = 8


class rope3d_sp_out_dest(ctypes.Structure):
    """struct rope3d_sp_out_dest of include/rope3d.h."""
    _fields_ = [("ranks", ctypes.c_int), ("rank", ctypes.c_int),
                ("cuts", ctypes.c_int64 * (ROPE3D_SP_MAX_RANKS + 1)),
                ("out", ctypes.c_void_p * ROPE3D_SP_MAX_RANKS)]


class rope3d_sp_dest(ctypes.Structure):
    """struct rope3d_sp_dest of include/rope3d.h."""
    _fields_ = [("ranks", ctypes.c_int), ("reserved0", ctypes.c_int),
                ("q_rows", ctypes.c_int64), ("q_row0", ctypes.c_int64),
                ("q", ctypes.c_void_p * ROPE3D_SP_MAX_RANKS),
                ("k_cache", ctypes.c_void_p * ROPE3D_SP_MAX_RANKS),
                ("v_cache", ctypes.c_void_p * ROPE3D_SP_MAX_RANKS)]

# include/rope3d_testing.h
ROPE3D_PATH_AUTO = 0
ROPE3D_PATH_REGISTERS = 1
ROPE3D_PATH_TMA = 2

_VP = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int

# name -> (argtypes, restype), in the order of include/rope3d.h and include/rope3d_testing.h
SIGNATURES = {
    "rope3d_tables_init": ([ctypes.POINTER(_VP), _INT, _INT, _INT, _INT, ctypes.c_double,
                            _INT, _INT, _INT, _INT, _VP], _INT),
    "rope3d_tables_destroy": ([_VP], None),
    "rope3d_qk_norm_rope_append": ([_VP, _VP, _VP, _VP, _I64, _I64, _INT, _INT, _I64, _I64, _I64,
                                    _INT, _INT, _INT, _VP, _VP, ctypes.c_float, _VP, _VP, _I64,
                                    _I64, _VP, _INT, _VP], _INT),
    "rope3d_qk_norm_rope_append_ex": ([_VP, _VP, _VP, _VP, _I64, _I64, _INT, _INT, _I64, _I64,
                                       _I64, _INT, _INT, _INT, _VP, _VP, ctypes.c_float, _VP,
                                       _VP, _I64, _I64, _VP, _INT,
                                       ctypes.POINTER(rope3d_options), _VP], _INT),
    "rope3d_qk_norm_rope_append_sp": ([_VP, _VP, _VP, _I64, _I64, _INT, _INT, _I64, _I64, _I64,
                                       _INT, _INT, _INT, _VP, _VP, ctypes.c_float,
                                       ctypes.POINTER(rope3d_sp_dest), _I64, _I64, _VP, _INT,
                                       ctypes.POINTER(rope3d_options), _VP], _INT),
    "rope3d_sp_output_all_to_all": ([_VP, _I64, _I64, _I64, _INT, _INT,
                                     ctypes.POINTER(rope3d_sp_out_dest), _VP], _INT),
    "rope3d_qkv_project": ([_VP, _VP, _VP, _I64, _I64, _I64, _INT, _VP, _VP, _VP, _VP], _INT),
    "rope3d_qkv_workspace_bytes": ([_I64, _I64, _I64, _INT], ctypes.c_size_t),
    "rope3d_qkv_norm_rope_append": ([_VP, _VP, _VP, _I64, _I64, _I64, _INT, _I64, _I64, _I64,
                                     _INT, _INT, _INT, _VP, _VP, ctypes.c_float, _VP, _VP,
                                     ctypes.c_size_t, _VP, _VP, _I64, _I64, _VP, _INT,
                                     ctypes.POINTER(rope3d_options), _VP], _INT),
    "rope3d_apply": ([_VP, _VP, _I64, _I64, _INT, _INT, _I64, _I64, _I64, _INT, _INT, _INT, _VP,
                      _INT, _VP], _INT),
    "rope3d_apply_ex": ([_VP, _VP, _I64, _I64, _INT, _INT, _I64, _I64, _I64, _INT, _INT, _INT,
                         _VP, _INT, ctypes.POINTER(rope3d_options), _VP], _INT),
    "rope3d_decode_positions": ([_I64, _I64, _I64, _INT, _INT, _INT, _I64, _I64, _VP, _VP], _INT),
    "rope3d_check_device_status": ([_VP, _VP], _INT),
    "rope3d_noalloc_check_status": ([_VP], _INT),
    "rope3d_qk_norm_rope_append_noalloc": ([_VP, _VP, _VP, _VP, _I64, _I64, _INT, _INT, _I64,
                                            _I64, _I64, _INT, _INT, _INT, _VP, _VP,
                                            ctypes.c_float, _VP, _VP, _I64, _I64, _INT, _INT,
                                            _INT, ctypes.c_double, _INT, _INT, _VP], _INT),
    "rope3d_strerror": ([_INT], ctypes.c_char_p),
    "rope3d_last_error": ([], ctypes.c_char_p),
    "rope3d_version": ([], _INT),
    "rope3d_testing_set_waits": ([ctypes.c_uint64, ctypes.c_uint32], None),
    "rope3d_testing_force_path": ([_INT], _INT),
    "rope3d_testing_gemm_cta_group": ([_INT], _INT),
    "rope3d_testing_last_path": ([], _INT),
    "rope3d_testing_shrink_checked_cache": ([_I64], _INT),
    "rope3d_testing_fast_divide": ([ctypes.c_uint32, ctypes.c_uint32], ctypes.c_uint32),
}

_lib = None


def load_library(path: str = LIBRARY) -> ctypes.CDLL:
    """Load librope3d.so and declare its entry points (no CUDA call is made)."""
    global _lib
    if _lib is not None and path == LIBRARY:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m rotary_position_encoding_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    for name, (args, res) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    if path == LIBRARY:
        _lib = lib
    return lib


class Rope3dError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(f"rope3d status {status}: {detail}")


def _check(status: int) -> None:
    if status != ROPE3D_OK:
        lib = load_library()
        msg = lib.rope3d_last_error().decode() or lib.rope3d_strerror(status).decode()
        raise Rope3dError(status, msg)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return ROPE3D_BF16
    if t.dtype == torch.float32:
        return ROPE3D_F32
    raise TypeError(f"unsupported dtype {t.dtype}; use torch.bfloat16 or torch.float32")


def _dev_ptr(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


class Tables:
    """Owns a ``rope3d_tables*``; frees it when garbage-collected or on ``close()``."""

    def __init__(self, handle: int, head_dim, n_t, n_h, n_w, theta, max_t, max_h, max_w,
                 schedule):
        self.handle = handle
        self.head_dim, self.n_t, self.n_h, self.n_w = head_dim, n_t, n_h, n_w
        self.theta, self.schedule = theta, schedule
        self.max_t, self.max_h, self.max_w = max_t, max_h, max_w

    def close(self) -> None:
        if self.handle:
            load_library().rope3d_tables_destroy(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def rope3d_tables_init(head_dim: int = 128, n_t: int = 22, n_h: int = 21, n_w: int = 21,
                       theta: float = 10000.0, max_t: int = 0, max_h: int = 0, max_w: int = 0,
                       schedule: int = ROPE3D_SCHEDULE_PER_AXIS, stream=None) -> Tables:
    lib = load_library()
    handle = _VP()
    _check(lib.rope3d_tables_init(ctypes.byref(handle), head_dim, n_t, n_h, n_w, theta, max_t,
                                  max_h, max_w, schedule, _stream(stream)))
    return Tables(handle.value, head_dim, n_t, n_h, n_w, theta, max_t, max_h, max_w, schedule)


def rope3d_tables_destroy(tables: Tables) -> None:
    tables.close()


def _check_step_tensors(q, k, v, q_out, token_begin: int, token_end: int, q_norm_w, k_norm_w,
                        k_cache, v_cache):
    """Shape and dtype checks of the fused step's tensors, shared by every wrapper that
    passes same-dtype caches: the C ABI sees only pointers and sizes, so a mismatch here
    would make the kernel read or write past the end of a tensor.  Returns (B, N, D)."""
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape or q_out.shape != q.shape:
        raise ValueError("q, k, v and q_out must all be [B, n_tok, N, D]")
    if k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache must both be [B, cache_tokens, N, D]")
    B, n_tok, N, D = q.shape
    if k_cache.shape[0] != B or k_cache.shape[2:] != q.shape[2:]:
        raise ValueError("cache shape does not match q")
    if n_tok != token_end - token_begin:
        raise ValueError("q has n_tok rows but the range holds token_end - token_begin")
    _dtype_code(q)
    for name, t in (("k", k), ("v", v), ("q_out", q_out), ("k_cache", k_cache),
                    ("v_cache", v_cache)):
        if t.dtype != q.dtype:
            raise TypeError(f"{name} must have q's dtype {q.dtype}")
    for name, t in (("q_norm_w", q_norm_w), ("k_norm_w", k_norm_w)):
        if t.dtype != torch.float32 or t.numel() != N * D:
            raise ValueError(f"{name} must be float32 with N*D elements")
    return B, N, D


def rope3d_qk_norm_rope_append(q, k, v, q_out, token_begin: int, token_end: int,
                               frame_offset: int, T: int, H: int, W: int, q_norm_w, k_norm_w,
                               eps: float, k_cache, v_cache, slot: int, tables: Tables,
                               trig: int = ROPE3D_TRIG_TABLE, stream=None) -> None:
    """q, k, v, q_out: [B, n_tok, N, 128]; k_cache, v_cache: [B, cache_tokens, N, 128];
    q_norm_w, k_norm_w: [N*128] float32.  Enqueued on ``stream`` (default: current)."""
    B, N, D = _check_step_tensors(q, k, v, q_out, token_begin, token_end, q_norm_w, k_norm_w,
                                  k_cache, v_cache)
    _check(load_library().rope3d_qk_norm_rope_append(
        _dev_ptr(q, "q"), _dev_ptr(k, "k"), _dev_ptr(v, "v"), _dev_ptr(q_out, "q_out"),
        B, N, D, _dtype_code(q), token_begin, token_end, frame_offset, T, H, W,
        _dev_ptr(q_norm_w, "q_norm_w"), _dev_ptr(k_norm_w, "k_norm_w"), eps,
        _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"), k_cache.shape[1], slot,
        tables.handle, trig, _stream(stream)))


def rope3d_qk_norm_rope_append_noalloc(q, k, v, q_out, token_begin: int, token_end: int,
                                       frame_offset: int, T: int, H: int, W: int, q_norm_w,
                                       k_norm_w, eps: float, k_cache, v_cache, slot: int,
                                       n_t: int = 22, n_h: int = 21, n_w: int = 21,
                                       theta: float = 10000.0,
                                       schedule: int = ROPE3D_SCHEDULE_PER_AXIS,
                                       trig: int = ROPE3D_TRIG_TABLE, stream=None) -> None:
    """The fused step with no device allocation (frequency configuration passed directly;
    its cos/sin rows and status word live in the library's fixed scratch array).  The
    tensors are checked as in rope3d_qk_norm_rope_append."""
    B, N, D = _check_step_tensors(q, k, v, q_out, token_begin, token_end, q_norm_w, k_norm_w,
                                  k_cache, v_cache)
    _check(load_library().rope3d_qk_norm_rope_append_noalloc(
        _dev_ptr(q, "q"), _dev_ptr(k, "k"), _dev_ptr(v, "v"), _dev_ptr(q_out, "q_out"),
        B, N, D, _dtype_code(q), token_begin, token_end, frame_offset, T, H, W,
        _dev_ptr(q_norm_w, "q_norm_w"), _dev_ptr(k_norm_w, "k_norm_w"), eps,
        _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"), k_cache.shape[1], slot,
        n_t, n_h, n_w, theta, schedule, trig, _stream(stream)))


def rope3d_qk_norm_rope_append_ex(q, k, v, q_out, token_begin: int, token_end: int,
                                  frame_offset: int, T: int, H: int, W: int, q_norm_w, k_norm_w,
                                  eps: float, k_cache, v_cache, slot: int, tables: Tables,
                                  trig: int = ROPE3D_TRIG_TABLE,
                                  pairing: int = ROPE3D_PAIRING_ADJACENT,
                                  cache_layout: int = ROPE3D_CACHE_TOKEN_MAJOR,
                                  k_scale=None, v_scale=None, k_global: float = 0.0,
                                  v_global: float = 0.0, stream=None) -> None:
    """rope3d_qk_norm_rope_append with options; head-major caches are [B, N, C, ...].
    Passing k_scale and v_scale selects a quantized cache (k_cache and v_cache are then
    uint8 code tensors): float32 scales [B, C, N] / [B, N, C] for FP8 E4M3 (caches
    [..., 128]); uint8 block scales [B, C, N, 8] / [B, N, C, 8] for NVFP4 (caches
    [..., 64]) with per-tensor scales k_global, v_global (0 = 1)."""
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape or q_out.shape != q.shape:
        raise ValueError("q, k, v and q_out must all be [B, n_tok, N, D]")
    B, n_tok, N, D = q.shape
    quant = k_scale is not None or v_scale is not None
    fp4 = quant and k_scale is not None and k_scale.dtype == torch.uint8
    row = D // 2 if fp4 else D
    if k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache must have one 4-d shape")
    if cache_layout == ROPE3D_CACHE_HEAD_MAJOR:
        C = k_cache.shape[2]
        ok = k_cache.shape[0] == B and k_cache.shape[1] == N and k_cache.shape[3] == row
    else:
        C = k_cache.shape[1]
        ok = k_cache.shape[0] == B and k_cache.shape[2] == N and k_cache.shape[3] == row
    if not ok:
        raise ValueError("cache shape does not match q and the cache layout")
    if n_tok != token_end - token_begin:
        raise ValueError("q has n_tok rows but the range holds token_end - token_begin")
    for name, t in (("k", k), ("v", v), ("q_out", q_out)) + (
            () if quant else (("k_cache", k_cache), ("v_cache", v_cache))):
        if t.dtype != q.dtype:
            raise TypeError(f"{name} must have q's dtype {q.dtype}")
    opts = rope3d_options(pairing, cache_layout)
    if quant:
        if k_cache.dtype != torch.uint8 or v_cache.dtype != torch.uint8:
            raise TypeError("a quantized cache is uint8 codes")
        sshape = (B, C, N) if cache_layout == ROPE3D_CACHE_TOKEN_MAJOR else (B, N, C)
        sdtype = torch.uint8 if fp4 else torch.float32
        if fp4:
            sshape = sshape + (D // 16,)
        for name, t in (("k_scale", k_scale), ("v_scale", v_scale)):
            if t is None or t.dtype != sdtype or tuple(t.shape) != sshape:
                raise ValueError(f"{name} must be {sdtype} of shape {sshape}")
        opts.cache_dtype = ROPE3D_CACHE_NVFP4 if fp4 else ROPE3D_CACHE_FP8_E4M3
        opts.k_scale = _dev_ptr(k_scale, "k_scale")
        opts.v_scale = _dev_ptr(v_scale, "v_scale")
        if fp4:
            opts.nvfp4_k_global = k_global
            opts.nvfp4_v_global = v_global
    _check(load_library().rope3d_qk_norm_rope_append_ex(
        _dev_ptr(q, "q"), _dev_ptr(k, "k"), _dev_ptr(v, "v"), _dev_ptr(q_out, "q_out"),
        B, N, D, _dtype_code(q), token_begin, token_end, frame_offset, T, H, W,
        _dev_ptr(q_norm_w, "q_norm_w"), _dev_ptr(k_norm_w, "k_norm_w"), eps,
        _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"), C, slot,
        tables.handle, trig, ctypes.byref(opts), _stream(stream)))


def rope3d_qk_norm_rope_append_sp(q, k, v, token_begin: int, token_end: int,
                                  frame_offset: int, T: int, H: int, W: int, q_norm_w, k_norm_w,
                                  eps: float, q_dst, k_cache_dst, v_cache_dst, slot: int,
                                  tables: Tables, trig: int = ROPE3D_TRIG_TABLE,
                                  cache_layout: int = ROPE3D_CACHE_TOKEN_MAJOR, q_row0: int = 0,
                                  q_rows: int | None = None, cache_tokens: int | None = None,
                                  stream=None) -> None:
    """The step with head-scatter stores: q, k, v are this rank's [B, n_tok, N, 128]; the
    three destination lists hold, in rank order, each rank's q buffer [B, q_rows, N/P, 128]
    and caches [B, C, N/P, 128] (head-major: [B, N/P, C, 128]) -- tensors on this device,
    or integer device addresses of peer mappings (then q_rows and cache_tokens are given)."""
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k and v must all be [B, n_tok, N, D]")
    B, n_tok, N, D = q.shape
    if n_tok != token_end - token_begin:
        raise ValueError("q has n_tok rows but the range holds token_end - token_begin")
    P = len(q_dst)
    if not 1 <= P <= ROPE3D_SP_MAX_RANKS or len(k_cache_dst) != P or len(v_cache_dst) != P:
        raise ValueError(f"one q, k and v destination per rank, 1 to {ROPE3D_SP_MAX_RANKS} ranks")
    for name, t in (("k", k), ("v", v)):
        if t.dtype != q.dtype:
            raise TypeError(f"{name} must have q's dtype {q.dtype}")
    if N % P:
        raise ValueError(f"N={N} heads do not split evenly over {P} ranks")
    hl = N // P
    dest = rope3d_sp_dest()
    dest.ranks = P
    dest.q_row0 = q_row0

    def addr(t, name, shape_ok):
        if isinstance(t, int):
            return t
        if t.dtype != q.dtype:
            raise TypeError(f"{name} must have q's dtype {q.dtype}")
        if not shape_ok(tuple(t.shape)):
            raise ValueError(f"{name} has shape {tuple(t.shape)}")
        return _dev_ptr(t, name)

    for r in range(P):
        if not isinstance(q_dst[r], int):
            q_rows = q_dst[r].shape[1] if q_rows is None else q_rows
        kc = k_cache_dst[r]
        if not isinstance(kc, int):
            c = kc.shape[2] if cache_layout == ROPE3D_CACHE_HEAD_MAJOR else kc.shape[1]
            cache_tokens = c if cache_tokens is None else cache_tokens
    if q_rows is None or cache_tokens is None:
        raise ValueError("q_rows and cache_tokens are needed when every destination is an address")
    cshape = ((B, hl, cache_tokens, D) if cache_layout == ROPE3D_CACHE_HEAD_MAJOR
              else (B, cache_tokens, hl, D))
    dest.q_rows = q_rows
    for r in range(P):
        dest.q[r] = addr(q_dst[r], f"q_dst[{r}]", lambda s: s == (B, q_rows, hl, D))
        dest.k_cache[r] = addr(k_cache_dst[r], f"k_cache_dst[{r}]", lambda s: s == cshape)
        dest.v_cache[r] = addr(v_cache_dst[r], f"v_cache_dst[{r}]", lambda s: s == cshape)
    opts = rope3d_options(ROPE3D_PAIRING_ADJACENT, cache_layout)
    _check(load_library().rope3d_qk_norm_rope_append_sp(
        _dev_ptr(q, "q"), _dev_ptr(k, "k"), _dev_ptr(v, "v"), B, N, D, _dtype_code(q),
        token_begin, token_end, frame_offset, T, H, W, _dev_ptr(q_norm_w, "q_norm_w"),
        _dev_ptr(k_norm_w, "k_norm_w"), eps, ctypes.byref(dest), cache_tokens, slot,
        tables.handle, trig, ctypes.byref(opts), _stream(stream)))


def rope3d_sp_output_all_to_all(o, out, rank: int, cuts=None, stream=None) -> None:
    """Algorithm 3's last step on this rank: o is [B, L, N/P, D] (every token, this rank's
    heads); out lists, in rank order, each rank's output [B, cuts[r'+1] - cuts[r'], N, D]
    -- tensors on this device, or integer device addresses of peer mappings.  cuts
    defaults to the even split r L // P."""
    if o.dim() != 4:
        raise ValueError("o must be [B, L, N/P, D]")
    B, L, hl, D = o.shape
    P = len(out)
    if not 1 <= P <= ROPE3D_SP_MAX_RANKS:
        raise ValueError(f"1 to {ROPE3D_SP_MAX_RANKS} ranks")
    if cuts is None:
        cuts = [(r * L) // P for r in range(P + 1)]
    if len(cuts) != P + 1:
        raise ValueError("one slice per rank: len(cuts) == P + 1")
    dest = rope3d_sp_out_dest()
    dest.ranks = P
    dest.rank = rank
    for r in range(P + 1):
        dest.cuts[r] = cuts[r]
    for r in range(P):
        t = out[r]
        if isinstance(t, int):
            dest.out[r] = t
            continue
        if t.dtype != o.dtype:
            raise TypeError(f"out[{r}] must have o's dtype {o.dtype}")
        if tuple(t.shape) != (B, cuts[r + 1] - cuts[r], P * hl, D):
            raise ValueError(f"out[{r}] has shape {tuple(t.shape)}")
        dest.out[r] = _dev_ptr(t, f"out[{r}]")
    _check(load_library().rope3d_sp_output_all_to_all(
        _dev_ptr(o, "o"), B, L, hl, D, _dtype_code(o), ctypes.byref(dest), _stream(stream)))


def rope3d_qkv_project(x, w_qkv, b_qkv, q_out, k_out, v_out, stream=None) -> None:
    """x [M, K] (or [..., K]) bf16, w_qkv [3 N 128, K] bf16, b_qkv [3 N 128] float32 or None;
    q_out, k_out, v_out [..., N, 128] bf16 with M rows."""
    K = x.shape[-1]
    M = x.numel() // K
    n_out = w_qkv.shape[0]
    if w_qkv.dim() != 2 or w_qkv.shape[1] != K or n_out % (3 * 128):
        raise ValueError("w_qkv must be [3 N 128, K]")
    N = n_out // 384
    for name, t in (("x", x), ("w_qkv", w_qkv), ("q_out", q_out), ("k_out", k_out),
                    ("v_out", v_out)):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16")
    for name, t in (("q_out", q_out), ("k_out", k_out), ("v_out", v_out)):
        if t.numel() != M * N * 128:
            raise ValueError(f"{name} must hold M x N x 128 elements")
    if b_qkv is not None and (b_qkv.dtype != torch.float32 or b_qkv.numel() != n_out):
        raise ValueError("b_qkv must be float32 with 3 N 128 elements")
    _check(load_library().rope3d_qkv_project(
        _dev_ptr(x, "x"), _dev_ptr(w_qkv, "w_qkv"),
        None if b_qkv is None else _dev_ptr(b_qkv, "b_qkv"), M, K, N, 128,
        _dev_ptr(q_out, "q_out"), _dev_ptr(k_out, "k_out"), _dev_ptr(v_out, "v_out"),
        _stream(stream)))


def rope3d_qkv_workspace_bytes(B: int, n_tok: int, N: int, D: int = 128) -> int:
    return int(load_library().rope3d_qkv_workspace_bytes(B, n_tok, N, D))


def rope3d_qkv_norm_rope_append(x, w_qkv, b_qkv, q_out, workspace, token_begin: int,
                                token_end: int, frame_offset: int, T: int, H: int, W: int,
                                q_norm_w, k_norm_w, eps: float, k_cache, v_cache, slot: int,
                                tables: Tables, trig: int = ROPE3D_TRIG_TABLE,
                                cache_layout: int = ROPE3D_CACHE_TOKEN_MAJOR,
                                stream=None) -> None:
    """x [B, n_tok, K] bf16 -> q_out [B, n_tok, N, 128] and the caches, through the QKV
    projection (w_qkv [3 N 128, K], b_qkv [3 N 128] float32 or None).  workspace: a uint8
    device tensor of at least rope3d_qkv_workspace_bytes(B, n_tok, N) bytes (scratch)."""
    if x.dim() != 3 or q_out.dim() != 4:
        raise ValueError("x must be [B, n_tok, K] and q_out [B, n_tok, N, D]")
    B, n_tok, K = x.shape
    N, D = q_out.shape[2], q_out.shape[3]
    if tuple(q_out.shape[:2]) != (B, n_tok):
        raise ValueError("q_out must be [B, n_tok, N, D]")
    if n_tok != token_end - token_begin:
        raise ValueError("x has n_tok rows but the range holds token_end - token_begin")
    if tuple(w_qkv.shape) != (3 * N * D, K):
        raise ValueError("w_qkv must be [3 N D, K]")
    C = k_cache.shape[2] if cache_layout == ROPE3D_CACHE_HEAD_MAJOR else k_cache.shape[1]
    for name, t in (("x", x), ("w_qkv", w_qkv), ("q_out", q_out), ("k_cache", k_cache),
                    ("v_cache", v_cache)):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16")
    nbytes = workspace.numel() * workspace.element_size()
    opts = rope3d_options(ROPE3D_PAIRING_ADJACENT, cache_layout)
    _check(load_library().rope3d_qkv_norm_rope_append(
        _dev_ptr(x, "x"), _dev_ptr(w_qkv, "w_qkv"),
        None if b_qkv is None else _dev_ptr(b_qkv, "b_qkv"), K, B, N, D, token_begin,
        token_end, frame_offset, T, H, W, _dev_ptr(q_norm_w, "q_norm_w"),
        _dev_ptr(k_norm_w, "k_norm_w"), eps, _dev_ptr(q_out, "q_out"),
        _dev_ptr(workspace, "workspace"), nbytes, _dev_ptr(k_cache, "k_cache"),
        _dev_ptr(v_cache, "v_cache"), C, slot, tables.handle, trig, ctypes.byref(opts),
        _stream(stream)))


def rope3d_apply_ex(x, out, token_begin: int, token_end: int, frame_offset: int, T: int, H: int,
                    W: int, tables: Tables, trig: int = ROPE3D_TRIG_TABLE,
                    pairing: int = ROPE3D_PAIRING_ADJACENT, stream=None) -> None:
    if x.dim() != 4 or out.shape != x.shape or out.dtype != x.dtype:
        raise ValueError("x and out must be [B, n_tok, N, D] of one dtype")
    B, n_tok, N, D = x.shape
    opts = rope3d_options(pairing, 0)
    _check(load_library().rope3d_apply_ex(
        _dev_ptr(x, "x"), _dev_ptr(out, "out"), B, N, D, _dtype_code(x), token_begin,
        token_end, frame_offset, T, H, W, tables.handle, trig, ctypes.byref(opts),
        _stream(stream)))


def rope3d_apply(x, out, token_begin: int, token_end: int, frame_offset: int, T: int, H: int,
                 W: int, tables: Tables, trig: int = ROPE3D_TRIG_TABLE, stream=None) -> None:
    """x, out: [B, n_tok, N, 128] (out may be x)."""
    if x.dim() != 4 or out.shape != x.shape or out.dtype != x.dtype:
        raise ValueError("x and out must be [B, n_tok, N, D] of one dtype")
    B, n_tok, N, D = x.shape
    if n_tok != token_end - token_begin:
        raise ValueError("x has n_tok rows but the range holds token_end - token_begin")
    _check(load_library().rope3d_apply(
        _dev_ptr(x, "x"), _dev_ptr(out, "out"), B, N, D, _dtype_code(x), token_begin,
        token_end, frame_offset, T, H, W, tables.handle, trig, _stream(stream)))


def rope3d_decode_positions(token_begin: int, token_end: int, frame_offset: int, T: int,
                            H: int, W: int, cache_tokens: int, slot: int, out,
                            stream=None) -> None:
    """out: int64 CUDA tensor [n_tok, 4] receiving (t_g, h, w, cache row)."""
    if out.dtype != torch.int64 or out.shape != (token_end - token_begin, 4):
        raise ValueError("out must be int64 [token_end - token_begin, 4]")
    _check(load_library().rope3d_decode_positions(
        token_begin, token_end, frame_offset, T, H, W, cache_tokens, slot,
        _dev_ptr(out, "out"), _stream(stream)))


def rope3d_check_device_status(tables: Tables, stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status of kernels launched
    with these tables: ROPE3D_OK, ROPE3D_ETIMEOUT, or (checked build) ROPE3D_EINDEX.
    Raises on a failure to read it."""
    status = load_library().rope3d_check_device_status(tables.handle, _stream(stream))
    if status not in (ROPE3D_OK, ROPE3D_ETIMEOUT, ROPE3D_EINDEX):
        _check(status)
    return status


def rope3d_noalloc_check_status(stream=None) -> int:
    """The same for the no-allocation entry point's status word on the current device."""
    status = load_library().rope3d_noalloc_check_status(_stream(stream))
    if status not in (ROPE3D_OK, ROPE3D_ETIMEOUT, ROPE3D_EINDEX):
        _check(status)
    return status


def rope3d_testing_set_waits(wait_limit_ns: int = 0, tx_extra_bytes: int = 0) -> None:
    load_library().rope3d_testing_set_waits(wait_limit_ns, tx_extra_bytes)


def rope3d_testing_force_path(path: int = ROPE3D_PATH_AUTO) -> None:
    _check(load_library().rope3d_testing_force_path(path))


def rope3d_testing_gemm_cta_group(group: int = 0) -> None:
    _check(load_library().rope3d_testing_gemm_cta_group(group))


def rope3d_testing_shrink_checked_cache(shrink_rows: int = 0) -> None:
    _check(load_library().rope3d_testing_shrink_checked_cache(shrink_rows))


def rope3d_testing_last_path() -> int:
    return load_library().rope3d_testing_last_path()


def rope3d_strerror(status: int) -> str:
    return load_library().rope3d_strerror(status).decode()


def rope3d_last_error() -> str:
    return load_library().rope3d_last_error().decode()


def rope3d_version() -> int:
    return load_library().rope3d_version()
