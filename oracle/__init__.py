"""fp64 CPU oracle of the Causal-RoPE SP Q/K preparation step -- TEST INFRASTRUCTURE.

Only the test suite, the smoke check (``__graft_entry__.smoke``) and the benchmark's
CPU-baseline and reference legs may import this package; the CUDA product path never
does.  The arithmetic lives in ``rope3d_oracle.c`` (plain C, double precision); this
module builds that file with gcc and exposes it through ctypes on numpy float64 arrays.
It shares no code with the CUDA library.

Paper: "Accelerating Video Generation Inference with Sequential-Parallel 3D
Positional Encoding Using a Global Time Index" (Yuan & Li) -- Section 3.3.1 (complex
rotation), Section 3.3.2 (global time index, localized formula), Algorithm 2 (per-axis
tables, adjacent-pair complex view, fp64), Section 3.3.3 (local-to-global index decode)
and Algorithms 1 and 3, step 5 (KV-cache update).  ``Oracle.qk_norm_rope_append_sp`` adds
the all-to-all of Algorithm 3 step 4 (Section 3.4.1 item 1: gather the sequence, scatter
the heads) as plain per-head stores on top of the C step.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "rope3d_oracle.c")
LIBRARY = os.path.join(_HERE, "librope3d_oracle.so")

# Default split of a 128-wide head: 22 t pairs, 21 h pairs, 21 w pairs; theta 10000.
N_T, N_H, N_W, THETA = 22, 21, 21, 10000.0

# Pairing of a head's elements and KV-cache layouts (the layout-variant functions).
PAIRING_ADJACENT, PAIRING_HALF = 0, 1
CACHE_TOKEN_MAJOR, CACHE_HEAD_MAJOR = 0, 1


def build(force: bool = False, source: str = SOURCE, library: str = LIBRARY) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction, OpenMP on)."""
    if (not force and os.path.exists(library)
            and os.path.getmtime(library) >= os.path.getmtime(source)):
        return library
    tmp = library + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-Wall", "-Wextra",
           source, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, library)
    return library


_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.c_int64
_INT = ctypes.c_int
_DBL = ctypes.c_double
_F = ctypes.POINTER(ctypes.c_float)
_U8 = ctypes.POINTER(ctypes.c_uint8)


def _declare(lib):
    sig = {
        "rope3d_oracle_inv_freq": ([_INT, _INT, _INT, _DBL, _INT, _D], _INT),
        "rope3d_oracle_decode": ([_I64, _I64, _I64, _I64, _I64, ctypes.POINTER(_I64),
                                  ctypes.POINTER(_I64), ctypes.POINTER(_I64)], None),
        "rope3d_oracle_cache_row": ([_I64, _I64, _I64], _I64),
        "rope3d_oracle_angles": ([_I64, _I64, _I64, _INT, _INT, _INT, _D, _D], None),
        "rope3d_oracle_rotate": ([_D, _I64, _I64, _D, _D], None),
        "rope3d_oracle_rms_norm": ([_D, _D, _I64, _DBL, _D], None),
        "rope3d_oracle_token": ([_D, _D, _D, _I64, _I64, _I64, _I64, _I64, _I64, _I64,
                                 _D, _D, _DBL, _I64, _I64, _INT, _INT, _INT, _D,
                                 _D, _D, _D, ctypes.POINTER(_I64)], _INT),
        "rope3d_oracle_qk_norm_rope_append": ([_D, _D, _D, _D, _I64, _I64, _I64, _I64, _I64,
                                               _I64, _I64, _I64, _I64, _D, _D, _DBL, _D, _D,
                                               _I64, _I64, _INT, _INT, _INT, _DBL, _INT,
                                               _INT], _INT),
        "rope3d_oracle_apply": ([_D, _D, _I64, _I64, _I64, _I64, _I64, _I64, _I64, _I64,
                                 _I64, _INT, _INT, _INT, _DBL, _INT], _INT),
        "rope3d_oracle_max_threads": ([], _INT),
        "rope3d_oracle_rotate_half": ([_D, _I64, _I64, _D, _D], None),
        "rope3d_oracle_rotate_pairing": ([_D, _I64, _I64, _D, _INT, _D], _INT),
        "rope3d_oracle_token_pairing": ([_D, _D, _D, _I64, _I64, _I64, _I64, _I64, _I64, _I64,
                                         _D, _D, _DBL, _I64, _I64, _INT, _INT, _INT, _D, _INT,
                                         _D, _D, _D, ctypes.POINTER(_I64)], _INT),
        "rope3d_oracle_qk_norm_rope_append_layout": ([_D, _D, _D, _D, _I64, _I64, _I64, _I64,
                                                      _I64, _I64, _I64, _I64, _I64, _D, _D,
                                                      _DBL, _D, _D, _I64, _I64, _INT, _INT,
                                                      _INT, _DBL, _INT, _INT, _INT, _INT], _INT),
        "rope3d_oracle_apply_pairing": ([_D, _D, _I64, _I64, _I64, _I64, _I64, _I64, _I64,
                                         _I64, _I64, _INT, _INT, _INT, _DBL, _INT, _INT], _INT),
        "rope3d_oracle_e4m3_value": ([_INT], _DBL),
        "rope3d_oracle_e4m3_encode": ([ctypes.c_float], _INT),
        "rope3d_oracle_e4m3_scale_exponent": ([ctypes.c_float], _INT),
        "rope3d_oracle_quantize_head_e4m3": ([_F, _I64, _U8, _F], None),
        "rope3d_oracle_qk_norm_rope_append_fp8": ([_D, _D, _D, _D, _I64, _I64, _I64, _I64, _I64,
                                                   _I64, _I64, _I64, _I64, _D, _D, _DBL, _U8,
                                                   _U8, _F, _F, _I64, _I64, _INT, _INT, _INT,
                                                   _DBL, _INT, _INT, _INT], _INT),
        "rope3d_oracle_e2m1_value": ([_INT], _DBL),
        "rope3d_oracle_e2m1_encode": ([ctypes.c_float], _INT),
        "rope3d_oracle_quantize_block_nvfp4": ([_F, _I64, ctypes.c_float, _U8, _U8], None),
        "rope3d_oracle_qk_norm_rope_append_nvfp4": ([_D, _D, _D, _D, _I64, _I64, _I64, _I64,
                                                     _I64, _I64, _I64, _I64, _I64, _D, _D, _DBL,
                                                     _U8, _U8, _U8, _U8, ctypes.c_float,
                                                     ctypes.c_float, _I64, _I64, _INT, _INT,
                                                     _INT, _DBL, _INT, _INT, _INT], _INT),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


class OracleError(ValueError):
    pass


def _f64(a, name):
    if not (isinstance(a, np.ndarray) and a.dtype == np.float64 and a.flags.c_contiguous):
        raise TypeError(f"{name} must be a C-contiguous float64 numpy array")
    return a.ctypes.data_as(_D)


def _f32(a, name):
    if not (isinstance(a, np.ndarray) and a.dtype == np.float32 and a.flags.c_contiguous):
        raise TypeError(f"{name} must be a C-contiguous float32 numpy array")
    return a.ctypes.data_as(_F)


def _u8(a, name):
    if not (isinstance(a, np.ndarray) and a.dtype == np.uint8 and a.flags.c_contiguous):
        raise TypeError(f"{name} must be a C-contiguous uint8 numpy array")
    return a.ctypes.data_as(_U8)


def _check(rc):
    if rc != 0:
        raise OracleError(f"oracle rejected the arguments (status {rc})")


class Oracle:
    """The compiled oracle library behind numpy-friendly methods."""

    def __init__(self, library: str | None = None):
        if library is None:
            library = build()
        self.path = library
        self.lib = _declare(ctypes.CDLL(library))

    def inv_freq(self, n_t=N_T, n_h=N_H, n_w=N_W, theta=THETA, schedule=0) -> np.ndarray:
        out = np.zeros(max(1, n_t + n_h + n_w), dtype=np.float64)
        _check(self.lib.rope3d_oracle_inv_freq(n_t, n_h, n_w, theta, schedule,
                                               _f64(out, "out")))
        return out[: n_t + n_h + n_w]

    def decode(self, i, frame_offset, T, H, W):
        t, h, w = _I64(), _I64(), _I64()
        self.lib.rope3d_oracle_decode(i, frame_offset, T, H, W, ctypes.byref(t),
                                      ctypes.byref(h), ctypes.byref(w))
        return t.value, h.value, w.value

    def cache_row(self, i, slot, cache_tokens):
        return self.lib.rope3d_oracle_cache_row(i, slot, cache_tokens)

    def angles(self, t_g, h, w, n_t=N_T, n_h=N_H, n_w=N_W, theta=THETA, schedule=0):
        inv = self.inv_freq(n_t, n_h, n_w, theta, schedule)
        phi = np.zeros(n_t + n_h + n_w, dtype=np.float64)
        self.lib.rope3d_oracle_angles(t_g, h, w, n_t, n_h, n_w, _f64(inv, "inv"),
                                      _f64(phi, "phi"))
        return phi

    def rotate(self, x, phi):
        """x: [n_heads, head_dim] float64 (one token row); phi: [head_dim/2]."""
        x = np.ascontiguousarray(x, dtype=np.float64)
        n_heads, head_dim = x.shape[-2], x.shape[-1]
        phi = np.ascontiguousarray(phi, dtype=np.float64)
        assert phi.shape == (head_dim // 2,)
        y = np.empty_like(x)
        self.lib.rope3d_oracle_rotate(_f64(x, "x"), n_heads, head_dim, _f64(phi, "phi"),
                                      _f64(y, "y"))
        return y

    def rms_norm(self, x, weight, eps):
        x = np.ascontiguousarray(x, dtype=np.float64).ravel()
        weight = np.ascontiguousarray(weight, dtype=np.float64).ravel()
        assert weight.shape == x.shape
        y = np.empty_like(x)
        self.lib.rope3d_oracle_rms_norm(_f64(x, "x"), _f64(weight, "weight"), x.size, eps,
                                        _f64(y, "y"))
        return y

    def token(self, q, k, v, i, frame_offset, T, H, W, q_norm_w, k_norm_w, eps, slot,
              cache_tokens, n_t=N_T, n_h=N_H, n_w=N_W, theta=THETA, schedule=0):
        """One token row ([N, D] each): returns (q_out, k_row, v_row, (t_g, h, w, row))."""
        q = np.ascontiguousarray(q, dtype=np.float64)
        k = np.ascontiguousarray(k, dtype=np.float64)
        v = np.ascontiguousarray(v, dtype=np.float64)
        N, D = q.shape[-2], q.shape[-1]
        inv = self.inv_freq(n_t, n_h, n_w, theta, schedule)
        qw = np.ascontiguousarray(q_norm_w, dtype=np.float64)
        kw = np.ascontiguousarray(k_norm_w, dtype=np.float64)
        qo, ko, vo = np.empty_like(q), np.empty_like(k), np.empty_like(v)
        pos = (_I64 * 4)()
        _check(self.lib.rope3d_oracle_token(
            _f64(q, "q"), _f64(k, "k"), _f64(v, "v"), N, D, i, frame_offset, T, H, W,
            _f64(qw, "q_norm_w"), _f64(kw, "k_norm_w"), eps, slot, cache_tokens,
            n_t, n_h, n_w, _f64(inv, "inv"), _f64(qo, "q_out"), _f64(ko, "k_row"),
            _f64(vo, "v_row"), pos))
        return qo, ko, vo, tuple(pos)

    def qk_norm_rope_append(self, q, k, v, token_begin, token_end, frame_offset, T, H, W,
                            q_norm_w, k_norm_w, eps, k_cache, v_cache, slot,
                            n_t=N_T, n_h=N_H, n_w=N_W, theta=THETA, schedule=0, nthreads=0):
        """Whole step.  q, k, v: [B, n_tok, N, D] float64; k_cache, v_cache:
        [B, cache_tokens, N, D] float64, updated in place.  Returns q_out."""
        B, n_tok, N, D = q.shape
        assert k.shape == q.shape and v.shape == q.shape
        assert k_cache.shape[0] == B and k_cache.shape[2:] == (N, D)
        assert v_cache.shape == k_cache.shape
        q_out = np.empty_like(q)
        _check(self.lib.rope3d_oracle_qk_norm_rope_append(
            _f64(q, "q"), _f64(k, "k"), _f64(v, "v"), _f64(q_out, "q_out"), B, N, D,
            token_begin, token_end, frame_offset, T, H, W,
            _f64(np.ascontiguousarray(q_norm_w, dtype=np.float64), "q_norm_w"),
            _f64(np.ascontiguousarray(k_norm_w, dtype=np.float64), "k_norm_w"), eps,
            _f64(k_cache, "k_cache"), _f64(v_cache, "v_cache"), k_cache.shape[1], slot,
            n_t, n_h, n_w, theta, schedule, nthreads))
        return q_out

    def apply(self, x, token_begin, token_end, frame_offset, T, H, W,
              n_t=N_T, n_h=N_H, n_w=N_W, theta=THETA, schedule=0):
        """Rotation alone over [B, n_tok, N, D] float64."""
        B, n_tok, N, D = x.shape
        out = np.empty_like(x)
        _check(self.lib.rope3d_oracle_apply(_f64(x, "x"), _f64(out, "out"), B, N, D,
                                            token_begin, token_end, frame_offset, T, H, W,
                                            n_t, n_h, n_w, theta, schedule))
        return out

    # ---- FP8 E4M3 KV cache

    def e4m3_value(self, code: int) -> float:
        return self.lib.rope3d_oracle_e4m3_value(code)

    def e4m3_encode(self, x: float) -> int:
        return self.lib.rope3d_oracle_e4m3_encode(x)

    def e4m3_scale_exponent(self, amax: float) -> int:
        return self.lib.rope3d_oracle_e4m3_scale_exponent(amax)

    def quantize_head_e4m3(self, x):
        x = np.ascontiguousarray(x, dtype=np.float32).ravel()
        codes = np.empty(x.size, dtype=np.uint8)
        scale = np.zeros(1, dtype=np.float32)
        self.lib.rope3d_oracle_quantize_head_e4m3(_f32(x, "x"), x.size, _u8(codes, "codes"),
                                                  _f32(scale, "scale"))
        return codes, float(scale[0])

    def qk_norm_rope_append_fp8(self, q, k, v, token_begin, token_end, frame_offset, T, H, W,
                                q_norm_w, k_norm_w, eps, k_codes, v_codes, k_scale, v_scale,
                                slot, pairing=PAIRING_ADJACENT, cache_layout=CACHE_TOKEN_MAJOR,
                                n_t=N_T, n_h=N_H, n_w=N_W, theta=THETA, schedule=0):
        """Whole step with an FP8 cache: codes uint8 [B,C,N,D] / [B,N,C,D], scales float32
        [B,C,N] / [B,N,C], updated in place.  Returns q_out (fp64)."""
        B, n_tok, N, D = q.shape
        C = k_codes.shape[1] if cache_layout == CACHE_TOKEN_MAJOR else k_codes.shape[2]
        q_out = np.empty_like(q)
        _check(self.lib.rope3d_oracle_qk_norm_rope_append_fp8(
            _f64(q, "q"), _f64(k, "k"), _f64(v, "v"), _f64(q_out, "q_out"), B, N, D,
            token_begin, token_end, frame_offset, T, H, W,
            _f64(np.ascontiguousarray(q_norm_w, dtype=np.float64), "q_norm_w"),
            _f64(np.ascontiguousarray(k_norm_w, dtype=np.float64), "k_norm_w"), eps,
            _u8(k_codes, "k_codes"), _u8(v_codes, "v_codes"), _f32(k_scale, "k_scale"),
            _f32(v_scale, "v_scale"), C, slot, n_t, n_h, n_w, theta, schedule, pairing,
            cache_layout))
        return q_out

    # ---- NVFP4 KV cache

    def e2m1_value(self, code: int) -> float:
        return self.lib.rope3d_oracle_e2m1_value(code)

    def e2m1_encode(self, x: float) -> int:
        return self.lib.rope3d_oracle_e2m1_encode(x)

    def quantize_block_nvfp4(self, x, g: float = 1.0):
        """n (even) values -> (n/2 code bytes, E4M3 scale byte)."""
        x = np.ascontiguousarray(x, dtype=np.float32).ravel()
        codes = np.zeros(x.size // 2, dtype=np.uint8)
        scale = np.zeros(1, dtype=np.uint8)
        self.lib.rope3d_oracle_quantize_block_nvfp4(_f32(x, "x"), x.size, g,
                                                    _u8(codes, "codes"), _u8(scale, "scale"))
        return codes, int(scale[0])

    def qk_norm_rope_append_nvfp4(self, q, k, v, token_begin, token_end, frame_offset, T, H,
                                  W, q_norm_w, k_norm_w, eps, k_codes, v_codes, k_scales,
                                  v_scales, slot, k_global=1.0, v_global=1.0,
                                  pairing=PAIRING_ADJACENT, cache_layout=CACHE_TOKEN_MAJOR,
                                  n_t=N_T, n_h=N_H, n_w=N_W, theta=THETA, schedule=0):
        """Whole step with an NVFP4 cache: codes uint8 [B,C,N,D/2] / [B,N,C,D/2], block
        scales uint8 [B,C,N,D/16] / [B,N,C,D/16], updated in place.  Returns q_out."""
        B, n_tok, N, D = q.shape
        C = k_codes.shape[1] if cache_layout == CACHE_TOKEN_MAJOR else k_codes.shape[2]
        q_out = np.empty_like(q)
        _check(self.lib.rope3d_oracle_qk_norm_rope_append_nvfp4(
            _f64(q, "q"), _f64(k, "k"), _f64(v, "v"), _f64(q_out, "q_out"), B, N, D,
            token_begin, token_end, frame_offset, T, H, W,
            _f64(np.ascontiguousarray(q_norm_w, dtype=np.float64), "q_norm_w"),
            _f64(np.ascontiguousarray(k_norm_w, dtype=np.float64), "k_norm_w"), eps,
            _u8(k_codes, "k_codes"), _u8(v_codes, "v_codes"), _u8(k_scales, "k_scales"),
            _u8(v_scales, "v_scales"), k_global, v_global, C, slot, n_t, n_h, n_w, theta,
            schedule, pairing, cache_layout))
        return q_out

    def max_threads(self) -> int:
        return self.lib.rope3d_oracle_max_threads()

    # ---- layout variants: rotate_half pairing, head-major cache

    def rotate_pairing(self, x, phi, pairing):
        """x: [n_heads, head_dim] float64 (one token row); phi: [head_dim/2]."""
        x = np.ascontiguousarray(x, dtype=np.float64)
        n_heads, head_dim = x.shape[-2], x.shape[-1]
        phi = np.ascontiguousarray(phi, dtype=np.float64)
        y = np.empty_like(x)
        _check(self.lib.rope3d_oracle_rotate_pairing(_f64(x, "x"), n_heads, head_dim,
                                                     _f64(phi, "phi"), pairing, _f64(y, "y")))
        return y

    def token_pairing(self, q, k, v, i, frame_offset, T, H, W, q_norm_w, k_norm_w, eps, slot,
                      cache_tokens, pairing, n_t=N_T, n_h=N_H, n_w=N_W, theta=THETA,
                      schedule=0):
        q = np.ascontiguousarray(q, dtype=np.float64)
        k = np.ascontiguousarray(k, dtype=np.float64)
        v = np.ascontiguousarray(v, dtype=np.float64)
        N, D = q.shape[-2], q.shape[-1]
        inv = self.inv_freq(n_t, n_h, n_w, theta, schedule)
        qw = np.ascontiguousarray(q_norm_w, dtype=np.float64)
        kw = np.ascontiguousarray(k_norm_w, dtype=np.float64)
        qo, ko, vo = np.empty_like(q), np.empty_like(k), np.empty_like(v)
        pos = (_I64 * 4)()
        _check(self.lib.rope3d_oracle_token_pairing(
            _f64(q, "q"), _f64(k, "k"), _f64(v, "v"), N, D, i, frame_offset, T, H, W,
            _f64(qw, "q_norm_w"), _f64(kw, "k_norm_w"), eps, slot, cache_tokens,
            n_t, n_h, n_w, _f64(inv, "inv"), pairing, _f64(qo, "q_out"), _f64(ko, "k_row"),
            _f64(vo, "v_row"), pos))
        return qo, ko, vo, tuple(pos)

    def qk_norm_rope_append_layout(self, q, k, v, token_begin, token_end, frame_offset, T,
                                   H, W, q_norm_w, k_norm_w, eps, k_cache, v_cache, slot,
                                   pairing=PAIRING_ADJACENT, cache_layout=CACHE_TOKEN_MAJOR,
                                   n_t=N_T, n_h=N_H, n_w=N_W, theta=THETA, schedule=0,
                                   nthreads=0):
        """Whole step; caches are [B, C, N, D] (token-major) or [B, N, C, D] (head-major)."""
        B, n_tok, N, D = q.shape
        C = k_cache.shape[1] if cache_layout == CACHE_TOKEN_MAJOR else k_cache.shape[2]
        q_out = np.empty_like(q)
        _check(self.lib.rope3d_oracle_qk_norm_rope_append_layout(
            _f64(q, "q"), _f64(k, "k"), _f64(v, "v"), _f64(q_out, "q_out"), B, N, D,
            token_begin, token_end, frame_offset, T, H, W,
            _f64(np.ascontiguousarray(q_norm_w, dtype=np.float64), "q_norm_w"),
            _f64(np.ascontiguousarray(k_norm_w, dtype=np.float64), "k_norm_w"), eps,
            _f64(k_cache, "k_cache"), _f64(v_cache, "v_cache"), C, slot,
            n_t, n_h, n_w, theta, schedule, pairing, cache_layout, nthreads))
        return q_out

    def qk_norm_rope_append_sp(self, q, k, v, token_begin, token_end, frame_offset, T, H, W,
                               q_norm_w, k_norm_w, eps, q_dst, k_dst, v_dst, slot,
                               q_row0=0, cache_layout=CACHE_TOKEN_MAJOR, n_t=N_T, n_h=N_H,
                               n_w=N_W, theta=THETA, schedule=0):
        """One rank's sequence-parallel step with the all-to-all (Algorithm 3, steps 3-5;
        the FusedAllToAll of Section 3.4.1 item 1: gather over the sequence, scatter over
        heads).  q, k, v: this rank's rows [B, n, N, D] for tokens [token_begin,
        token_end), all heads.  The step is computed as usual; then every head n goes to
        its owner rank r = n // (N/P) as local head n - r N/P: q to q_dst[r][b, i - q_row0],
        K and V to k_dst[r], v_dst[r] at cache row (slot + i) mod C
        ([B, C, N/P, D], or [B, N/P, C, D] head-major).  P = len(q_dst); the destination
        arrays (float64) are written in place."""
        B, n, N, D = q.shape
        P = len(q_dst)
        if N % P:
            raise ValueError("heads do not split evenly over the ranks")
        hl = N // P
        if token_begin < q_row0 or token_end - q_row0 > q_dst[0].shape[1]:
            raise ValueError("the token range is not inside the q buffers' rows")
        C = k_dst[0].shape[1] if cache_layout == CACHE_TOKEN_MAJOR else k_dst[0].shape[2]
        kc = np.zeros((B, C, N, D))
        vc = np.zeros((B, C, N, D))
        q_out = self.qk_norm_rope_append_layout(
            q, k, v, token_begin, token_end, frame_offset, T, H, W, q_norm_w, k_norm_w, eps,
            kc, vc, slot, PAIRING_ADJACENT, CACHE_TOKEN_MAJOR, n_t, n_h, n_w, theta, schedule)
        i = np.arange(token_begin, token_end)
        rows = (slot + i) % C
        for head in range(N):
            r, local = divmod(head, hl)
            q_dst[r][:, i - q_row0, local] = q_out[:, :, head]
            if cache_layout == CACHE_TOKEN_MAJOR:
                k_dst[r][:, rows, local] = kc[:, rows, head]
                v_dst[r][:, rows, local] = vc[:, rows, head]
            else:
                k_dst[r][:, local, rows] = kc[:, rows, head]
                v_dst[r][:, local, rows] = vc[:, rows, head]

    @staticmethod
    def sp_output_all_to_all(o_ranks, cuts):
        """The all-to-all after attention (Algorithm 3, last step: o <- AllToAll(o,
        scatter_dim=1, gather_dim=2)).  Rank r holds o_ranks[r] = [B, L, N/P, D]: the whole
        sequence for its own heads [r N/P, (r+1) N/P).  Afterwards rank r' holds its token
        slice [cuts[r'], cuts[r'+1]) with every head: out[r'][b, i - cuts[r'], r N/P + h]
        = o_ranks[r][b, i, h].  Returns the P outputs [B, cuts[r'+1] - cuts[r'], N, D]."""
        P = len(o_ranks)
        B, L, hl, D = o_ranks[0].shape
        if len(cuts) != P + 1 or cuts[0] != 0 or cuts[-1] != L or any(
                cuts[j] > cuts[j + 1] for j in range(P)):
            raise ValueError("cuts must rise from 0 to L with one slice per rank")
        outs = [np.zeros((B, cuts[r + 1] - cuts[r], P * hl, D), dtype=o_ranks[0].dtype)
                for r in range(P)]
        for r in range(P):              # source rank: its heads
            for dst in range(P):        # destination rank: its tokens
                a, e = cuts[dst], cuts[dst + 1]
                outs[dst][:, :, r * hl:(r + 1) * hl] = o_ranks[r][:, a:e]
        return outs

    # ---- QKV projection feeding the step (Algorithm 1/3 step 1, Section 3.4.1 item 3)

    @staticmethod
    def bf16_round(a):
        return bf16_round(a)

    @staticmethod
    def qkv_project(x, w_qkv, b_qkv=None):
        """q, k, v = QKV(x): x [B, n, dim_in] @ w_qkv.T + b_qkv, in fp64, with w_qkv
        [3 dim, dim_in] holding the q rows, then the k rows, then the v rows (an
        nn.Linear weight); each result is returned as [B, n, dim]."""
        x = np.asarray(x, dtype=np.float64)
        w = np.asarray(w_qkv, dtype=np.float64)
        y = x @ w.T
        if b_qkv is not None:
            y = y + np.asarray(b_qkv, dtype=np.float64)
        dim = w.shape[0] // 3
        return y[..., :dim], y[..., dim:2 * dim], y[..., 2 * dim:]

    def qkv_norm_rope_append(self, x, w_qkv, b_qkv, N, token_begin, token_end, frame_offset,
                             T, H, W, q_norm_w, k_norm_w, eps, k_cache, v_cache, slot,
                             round_bf16=True, **freq):
        """Step 1 (the projection) then the step.  With round_bf16 the projected q, k, v
        are rounded to bf16 first (round to nearest even), as a projection that stores
        bf16 activations hands them on; the step then runs on those values."""
        q, k, v = self.qkv_project(x, w_qkv, b_qkv)
        if round_bf16:
            q, k, v = (self.bf16_round(a) for a in (q, k, v))
        B, n = q.shape[:2]
        shape = (B, n, N, q.shape[-1] // N)
        return self.qk_norm_rope_append_layout(
            q.reshape(shape).copy(), k.reshape(shape).copy(), v.reshape(shape).copy(),
            token_begin, token_end, frame_offset, T, H, W, q_norm_w, k_norm_w, eps, k_cache,
            v_cache, slot, **freq)

    def apply_pairing(self, x, token_begin, token_end, frame_offset, T, H, W, pairing,
                      n_t=N_T, n_h=N_H, n_w=N_W, theta=THETA, schedule=0):
        B, n_tok, N, D = x.shape
        out = np.empty_like(x)
        _check(self.lib.rope3d_oracle_apply_pairing(
            _f64(x, "x"), _f64(out, "out"), B, N, D, token_begin, token_end, frame_offset,
            T, H, W, n_t, n_h, n_w, theta, schedule, pairing))
        return out


def bf16_round(a):
    """fp64 values rounded to the nearest bfloat16 (8 significant bits, ties to even,
    the fp32 exponent range with its subnormal spacing 2^-133), returned as fp64."""
    a = np.asarray(a, dtype=np.float64)
    _, e = np.frexp(a)               # a = m 2^e with 0.5 <= |m| < 1
    e = np.maximum(e, -125)          # below 2^-126 the spacing stays 2^-133
    return np.ldexp(np.rint(np.ldexp(a, 8 - e)), e - 8)


_default = None


def default() -> Oracle:
    """The oracle built from ``rope3d_oracle.c`` beside this file (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
