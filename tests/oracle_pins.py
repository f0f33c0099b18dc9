"""Checks that tie the fp64 oracle to what the paper and the mathematics fix.

Every check takes an ``oracle.Oracle`` and raises AssertionError on a mismatch.  The
same checks run against the real oracle (tests/test_oracle_pins.py) and against copies
of its source with a planted mistake (tests/test_oracle_mutants.py), which must each fail
at least one of them.

Paper: "Accelerating Video Generation Inference with Sequential-Parallel 3D Positional
Encoding Using a Global Time Index" (Yuan & Li).
"""
from __future__ import annotations

import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
D = 128
P = 64
NT, NH, NW = 22, 21, 21
CACHE_TOKEN_MAJOR, CACHE_HEAD_MAJOR = 0, 1  # the oracle's cache layouts


def _f32(x):
    """float64 values that are exactly float32 (as the workloads' inputs are)."""
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def _rows(name):
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                out.append(line)
    return out


def _rng(seed):
    return np.random.default_rng(seed)


# ---------------------------------------------------------------- frequency schedule

def check_inv_freq_special_values(orc):
    """Per-axis schedule: pair j of an axis with n_a pairs turns at theta^(-j/n_a).
    Closed forms: the first pair of each axis is 1; t pair 11 is 10000^(-1/2) = 0.01;
    h pair 7 is 10000^(-1/3); w pair 14 is 10000^(-2/3)."""
    inv = orc.inv_freq(NT, NH, NW, 10000.0, 0)
    assert inv.shape == (P,)
    for first in (0, NT, NT + NH):
        assert inv[first] == 1.0
    assert abs(inv[11] - 0.01) < 1e-17
    assert abs(inv[NT + 7] - 0.046415888336127795) < 1e-16
    assert abs(inv[NT + NH + 14] - 0.0021544346900318843) < 1e-17
    # strictly decreasing within each axis, equal ratios between neighbours
    for lo, n in ((0, NT), (NT, NH), (NT + NH, NW)):
        seg = inv[lo:lo + n]
        assert np.all(np.diff(seg) < 0)
        ratios = seg[1:] / seg[:-1]
        assert np.allclose(ratios, ratios[0], rtol=1e-13, atol=0)


def check_inv_freq_single_schedule(orc):
    """Alternative reading: one head-wide schedule theta^(-2j/128) split 22/21/21.
    Pair 32 is 10000^(-1/2) = 0.01, pair 22 is 10^(-11/8), pair 0 is 1."""
    inv = orc.inv_freq(NT, NH, NW, 10000.0, 1)
    assert inv[0] == 1.0
    assert abs(inv[32] - 0.01) < 1e-17
    assert abs(inv[22] - 0.042169650342858224) < 1e-16
    assert np.all(np.diff(inv) < 0)


# ---------------------------------------------------------------- position decode

def check_decode_golden(orc):
    """Hand-derived decode of a (2, 2, 3) grid at s = 3 split over 4 ranks."""
    L_local = 3
    for line in _rows("decode_F2_H2_W3_s3_P4.txt"):
        r, i_local, i_global, t_g, h, w = map(int, line.split())
        assert r * L_local + i_local == i_global
        assert orc.decode(i_global, 3, 2, 2, 3) == (t_g, h, w)


def check_decode_brute_force(orc):
    """Row-major enumeration (t outermost, w innermost) of several grids and offsets."""
    for (T, H, W) in ((3, 4, 6), (1, 1, 1), (2, 5, 1), (4, 1, 7), (3, 30, 52)):
        for s in (0, 3, 6, 237):
            i = 0
            for t in range(T):
                for h in range(H):
                    for w in range(W):
                        if (T, H, W) != (3, 30, 52) or i % 97 == 0:
                            assert orc.decode(i, s, T, H, W) == (s + t, h, w), (T, H, W, s, i)
                        i += 1


def check_start_frames_golden(orc):
    """tau = 3: block k starts at frame 3k, so local frame t of block k is global 3k + t."""
    H, W = 4, 6
    for line in _rows("start_frames_tau3.txt"):
        k, s = map(int, line.split())
        assert s == 3 * k
        for t in range(3):
            assert orc.decode(t * H * W, s, 3, H, W)[0] == s + t
            assert orc.decode(t * H * W + H * W - 1, s, 3, H, W)[0] == s + t


def check_cache_rows_rolling_window(orc):
    """Frame-level simulation of a rolling window of `window` frames: the tokens of global
    frame f sit in window frame f mod window, spatial order kept.  The oracle places token
    i of the chunk starting at frame s, with slot = (s mod window) * HW, at
    (slot + i) mod cache_tokens; both must agree, wrap-around included."""
    H, W, window = 2, 3, 5
    hw = H * W
    cache_tokens = window * hw
    for s in range(0, 40, 3):
        slot = (s % window) * hw
        for i in range(3 * hw):
            f = s + i // hw
            expect = (f % window) * hw + i % hw
            assert orc.cache_row(i, slot, cache_tokens) == expect, (s, i)
    # a slot that is not frame aligned still places the range contiguously modulo the cache
    rows = [orc.cache_row(i, 7, 20) for i in range(20)]
    assert sorted(rows) == list(range(20))
    assert rows[0] == 7 and rows[12] == 19 and rows[13] == 0


# ---------------------------------------------------------------- rotation

def _one_token_rotate(orc, x, t_g, h, w, schedule=0):
    phi = orc.angles(t_g, h, w, NT, NH, NW, 10000.0, schedule)
    return orc.rotate(x, phi)


def check_rotation_golden(orc):
    """Closed-form rotations at whole-radian angles (golden file)."""
    for line in _rows("rotation_unit_angles.txt"):
        t_g, h, w, j, re_in, im_in, re_out, im_out = line.split()
        x = np.zeros((1, D))
        x[0, 2 * int(j)] = float(re_in)
        x[0, 2 * int(j) + 1] = float(im_in)
        y = _one_token_rotate(orc, x, int(t_g), int(h), int(w))
        assert abs(y[0, 2 * int(j)] - float(re_out)) < 1e-14, line
        assert abs(y[0, 2 * int(j) + 1] - float(im_out)) < 1e-14, line
        others = np.delete(y[0], [2 * int(j), 2 * int(j) + 1])
        assert np.all(others == 0.0)


def check_position_zero_identity(orc):
    x = _rng(1).standard_normal((3, D))
    y = _one_token_rotate(orc, x, 0, 0, 0)
    assert np.array_equal(x, y)


def check_one_hot_axis_ownership(orc):
    """e_{2j} rotates to (cos phi_j, sin phi_j); each pair moves only with its own axis."""
    inv = orc.inv_freq()
    for (t_g, h, w) in ((5, 0, 0), (0, 4, 0), (0, 0, 6), (9, 2, 11)):
        for j in range(P):
            x = np.zeros((1, D))
            x[0, 2 * j] = 1.0
            y = _one_token_rotate(orc, x, t_g, h, w)
            pos = t_g if j < NT else (h if j < NT + NH else w)
            phi = pos * inv[j]
            assert abs(y[0, 2 * j] - math.cos(phi)) < 1e-14
            assert abs(y[0, 2 * j + 1] - math.sin(phi)) < 1e-14


def check_rotation_matches_complex_exp(orc):
    """The rotation equals numpy's complex multiply by exp(i phi) on adjacent pairs."""
    rng = _rng(2)
    inv = orc.inv_freq()
    for _ in range(10):
        t_g, h, w = (int(v) for v in rng.integers(0, 240, size=3))
        x = rng.standard_normal((4, D))
        pos = np.array([t_g] * NT + [h] * NH + [w] * NW, dtype=np.float64)
        z = x.reshape(4, P, 2)
        zc = (z[..., 0] + 1j * z[..., 1]) * np.exp(1j * pos * inv)
        expect = np.stack([zc.real, zc.imag], axis=-1).reshape(4, D)
        y = _one_token_rotate(orc, x, t_g, h, w)
        assert np.allclose(y, expect, rtol=0, atol=1e-13)


def check_pair_norms_preserved(orc):
    rng = _rng(3)
    x = rng.standard_normal((5, D))
    y = _one_token_rotate(orc, x, 17, 29, 51)
    nx = np.hypot(x[:, 0::2], x[:, 1::2])
    ny = np.hypot(y[:, 0::2], y[:, 1::2])
    assert np.allclose(nx, ny, rtol=0, atol=1e-12)


def check_relative_offset_brute_force(orc):
    """<R(p_m) q, R(p_n) k> = <q, R(p_n - p_m) k> for every pair of tokens of the 3x4x6
    grid at start frame 3 (all 72 x 72 pairs); so the score depends only on the 3D offset."""
    rng = _rng(4)
    T, H, W, s = 3, 4, 6, 3
    n = T * H * W
    q = rng.standard_normal((n, 2, D))
    k = rng.standard_normal((n, 2, D))
    pos = [orc.decode(i, s, T, H, W) for i in range(n)]
    rq = [_one_token_rotate(orc, q[m], *pos[m]) for m in range(n)]
    rk = [_one_token_rotate(orc, k[m], *pos[m]) for m in range(n)]
    for m in range(n):
        for nn in range(n):
            lhs = float(np.sum(rq[m] * rk[nn]))
            d = tuple(pos[nn][a] - pos[m][a] for a in range(3))
            rhs = float(np.sum(q[m] * _one_token_rotate(orc, k[nn], *d)))
            assert abs(lhs - rhs) < 1e-10, (m, nn)


def check_rotation_group_property(orc):
    """R(a) R(b) = R(a + b) and R(a) R(-a) = identity."""
    rng = _rng(5)
    x = rng.standard_normal((2, D))
    a, b = (3, 7, 11), (40, -2, 5)
    ab = tuple(a[i] + b[i] for i in range(3))
    y1 = _one_token_rotate(orc, _one_token_rotate(orc, x, *a), *b)
    y2 = _one_token_rotate(orc, x, *ab)
    assert np.allclose(y1, y2, rtol=0, atol=1e-12)
    y3 = _one_token_rotate(orc, _one_token_rotate(orc, x, *a), *(-v for v in a))
    assert np.allclose(y3, x, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- RMSNorm

def check_rms_norm_golden(orc):
    for line in _rows("rmsnorm_examples.txt"):
        eps, xs, ws, ys = (part.split() for part in line.split("|"))
        y = orc.rms_norm(np.array(xs, float), np.array(ws, float), float(eps[0]))
        assert np.allclose(y, np.array(ys, float), rtol=0, atol=1e-14), line


def check_rms_norm_closed_forms(orc):
    rng = _rng(6)
    dim = 256
    w = rng.uniform(0.5, 1.5, dim)
    for c, eps in ((2.0, 1e-6), (0.1, 1e-2), (-3.0, 0.5)):
        y = orc.rms_norm(np.full(dim, c), w, eps)
        assert np.allclose(y, c / math.sqrt(c * c + eps) * w, rtol=1e-14, atol=0)
    x = rng.standard_normal(dim)
    ones = np.ones(dim)
    y = orc.rms_norm(x, ones, 0.0)
    assert abs(float(np.sum(y * y)) - dim) < 1e-10
    for alpha in (1e-3, 7.0, 1e4):
        assert np.allclose(orc.rms_norm(alpha * x, w, 0.0), orc.rms_norm(x, w, 0.0),
                           rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- fused token and step

def check_token_norms_and_weights(orc):
    """With eps = 0 and constant weights c_q, c_k: |q_out|^2 = c_q^2 dim and
    |k_row|^2 = c_k^2 dim (RMSNorm fixes the mean square, rotation keeps it); v is copied
    bit for bit; the returned position and cache row are the decode and the rolling row."""
    rng = _rng(7)
    N = 3
    dim = N * D
    q, k, v = (rng.standard_normal((N, D)) for _ in range(3))
    qo, ko, vo, pos = orc.token(q, k, v, 29, 6, 3, 4, 6, np.full(dim, 1.0), np.full(dim, 2.0),
                                0.0, 100, 144)
    assert abs(float(np.sum(qo * qo)) - dim) < 1e-9
    assert abs(float(np.sum(ko * ko)) - 4.0 * dim) < 1e-9
    assert np.array_equal(vo, v)
    assert pos == (6 + 1, (29 // 6) % 4, 29 % 6, (100 + 29) % 144)


def check_token_is_norm_then_rotate(orc):
    """q_out = RoPE(RMSNorm(q)) -- the norm of one row is taken before rotating, with the
    q weights for q and the k weights for k.  Weights differ per element, so swapping the
    order or the weights changes the result."""
    rng = _rng(8)
    N = 2
    dim = N * D
    q, k, v = (rng.standard_normal((N, D)) for _ in range(3))
    wq, wk = rng.uniform(0.5, 1.5, dim), rng.uniform(0.5, 1.5, dim)
    qo, ko, _, (t_g, h, w, _) = orc.token(q, k, v, 50, 3, 3, 4, 6, wq, wk, 1e-6, 0, 144)
    phi = orc.angles(t_g, h, w)
    expect_q = orc.rotate(orc.rms_norm(q, wq, 1e-6).reshape(N, D), phi)
    expect_k = orc.rotate(orc.rms_norm(k, wk, 1e-6).reshape(N, D), phi)
    assert np.allclose(qo, expect_q, rtol=0, atol=1e-13)
    assert np.allclose(ko, expect_k, rtol=0, atol=1e-13)
    # independent recomputation of the mean square for one element
    rs = 1.0 / math.sqrt(np.mean(q.ravel() ** 2) + 1e-6)
    a, b = q[1, 2 * 30] * rs * wq[D + 60], q[1, 2 * 30 + 1] * rs * wq[D + 61]
    c, s = math.cos(phi[30]), math.sin(phi[30])
    assert abs(qo[1, 60] - (a * c - b * s)) < 1e-13
    assert abs(qo[1, 61] - (a * s + b * c)) < 1e-13


def _step_inputs(seed, B, n_tok, N):
    rng = _rng(seed)
    q, k, v = (rng.standard_normal((B, n_tok, N, D)) for _ in range(3))
    wq, wk = rng.uniform(0.5, 1.5, N * D), rng.uniform(0.5, 1.5, N * D)
    return q, k, v, wq, wk


def check_step_matches_tokens(orc):
    """The whole step writes, for each (b, r), the token function's rows: q_out at row r,
    K and V at (slot + i) mod cache_tokens of sample b; other cache rows stay untouched."""
    B, N, T, H, W = 2, 2, 3, 4, 6
    tb, te, s, slot, C = 10, 50, 3, 130, 144
    q, k, v, wq, wk = _step_inputs(9, B, te - tb, N)
    kc = np.full((B, C, N, D), 7.0)
    vc = np.full((B, C, N, D), -7.0)
    qo = orc.qk_norm_rope_append(q, k, v, tb, te, s, T, H, W, wq, wk, 1e-6, kc, vc, slot)
    touched = set()
    for b in range(B):
        for r in range(te - tb):
            i = tb + r
            eq, ek, ev, pos = orc.token(q[b, r], k[b, r], v[b, r], i, s, T, H, W, wq, wk, 1e-6,
                                        slot, C)
            row = pos[3]
            assert row == (slot + i) % C
            assert np.array_equal(qo[b, r], eq)
            assert np.array_equal(kc[b, row], ek)
            assert np.array_equal(vc[b, row], ev)
            touched.add((b, row))
    for b in range(B):
        for row in range(C):
            if (b, row) not in touched:
                assert np.all(kc[b, row] == 7.0) and np.all(vc[b, row] == -7.0)


def check_slices_equal_whole(orc):
    """Section 3.3.3: processing [r L/P, (r+1) L/P) on each of P ranks gives the whole-
    sequence result.  Uneven slices cut through rows and frames."""
    B, N, T, H, W, s, C = 1, 2, 3, 4, 6, 6, 144
    n = T * H * W
    q, k, v, wq, wk = _step_inputs(10, B, n, N)
    kc0, vc0 = np.zeros((B, C, N, D)), np.zeros((B, C, N, D))
    q0 = orc.qk_norm_rope_append(q, k, v, 0, n, s, T, H, W, wq, wk, 1e-6, kc0, vc0, 72)
    kc1, vc1 = np.zeros((B, C, N, D)), np.zeros((B, C, N, D))
    q1 = np.empty_like(q0)
    for (a, e) in ((0, 5), (5, 29), (29, 30), (30, 72)):
        q1[:, a:e] = orc.qk_norm_rope_append(q[:, a:e].copy(), k[:, a:e].copy(),
                                             v[:, a:e].copy(), a, e, s, T, H, W, wq, wk,
                                             1e-6, kc1, vc1, 72)
    assert np.array_equal(q0, q1)
    assert np.array_equal(kc0, kc1)
    assert np.array_equal(vc0, vc1)


def check_frame_shift_invariant(orc):
    """Causal-RoPE SP on a chunk starting at frame s equals full-sequence RoPE on the
    longer video: out(i, s) on grid (T, H, W) == out(i + s H W, 0) on grid (T + s, H, W)."""
    B, N, T, H, W, s = 1, 2, 3, 4, 6, 6
    hw = H * W
    n = T * hw
    q, k, v, wq, wk = _step_inputs(11, B, n, N)
    C = (T + s) * hw
    kc_a, vc_a = np.zeros((B, C, N, D)), np.zeros((B, C, N, D))
    qa = orc.qk_norm_rope_append(q, k, v, 0, n, s, T, H, W, wq, wk, 1e-6, kc_a, vc_a, s * hw)
    kc_b, vc_b = np.zeros((B, C, N, D)), np.zeros((B, C, N, D))
    qb = orc.qk_norm_rope_append(q, k, v, s * hw, s * hw + n, 0, T + s, H, W, wq, wk, 1e-6,
                                 kc_b, vc_b, 0)
    assert np.array_equal(qa, qb)
    assert np.array_equal(kc_a, kc_b)
    assert np.array_equal(vc_a, vc_b)


def check_apply_matches_rotation(orc):
    """The rotation-only entry point rotates row r by the angles of index begin + r."""
    B, N, T, H, W, s = 2, 2, 3, 4, 6, 9
    rng = _rng(12)
    x = rng.standard_normal((B, 40, N, D))
    y = orc.apply(x, 20, 60, s, T, H, W)
    for b in range(B):
        for r in range(40):
            t_g, h, w = orc.decode(20 + r, s, T, H, W)
            assert (t_g, h, w) == (s + (20 + r) // 24, ((20 + r) // 6) % 4, (20 + r) % 6)
            assert np.array_equal(y[b, r], _one_token_rotate(orc, x[b, r], t_g, h, w))


# ---------------------------------------------------------------- layout variants

def _half_to_adjacent_perm(D=128):
    """Index map: element j (j < D/2) -> 2j and element D/2 + j -> 2j + 1."""
    perm = np.empty(D, dtype=np.int64)
    half = D // 2
    for j in range(half):
        perm[2 * j] = j
        perm[2 * j + 1] = half + j
    return perm


def check_half_pairing_golden(orc):
    """Closed-form rotate_half rotations at whole-radian angles (golden file), on the
    16/24/24 head-wide split of M-RoPE."""
    for line in _rows("rotation_half_unit_angles.txt"):
        t_g, h, w, j, re_in, im_in, re_out, im_out = line.split()
        j = int(j)
        x = np.zeros((1, D))
        x[0, j] = float(re_in)
        x[0, 64 + j] = float(im_in)
        phi = orc.angles(int(t_g), int(h), int(w), 16, 24, 24, 10000.0, 1)
        y = orc.rotate_pairing(x, phi, 1)
        assert abs(y[0, j] - float(re_out)) < 1e-14, line
        assert abs(y[0, 64 + j] - float(im_out)) < 1e-14, line
        others = np.delete(y[0], [j, 64 + j])
        assert np.all(others == 0.0)


def check_half_pairing_is_permuted_adjacent(orc):
    """rotate_half on x equals the adjacent-pair rotation on x with each pair's two
    elements brought next to each other, mapped back."""
    rng = _rng(20)
    perm = _half_to_adjacent_perm()
    for (t_g, h, w) in ((0, 0, 0), (3, 7, 11), (239, 44, 79)):
        x = rng.standard_normal((3, D))
        phi = orc.angles(t_g, h, w)
        y_half = orc.rotate_pairing(x, phi, 1)
        y_adj = orc.rotate(x[:, perm], phi)
        back = np.empty_like(y_adj)
        back[:, perm] = y_adj
        assert np.array_equal(y_half, back)


def check_half_pairing_matches_complex_exp(orc):
    rng = _rng(21)
    inv = orc.inv_freq(16, 24, 24, 10000.0, 1)
    for _ in range(5):
        t_g, h, w = (int(v) for v in rng.integers(0, 100, size=3))
        x = rng.standard_normal((2, D))
        pos = np.array([t_g] * 16 + [h] * 24 + [w] * 24, dtype=np.float64)
        z = (x[:, :64] + 1j * x[:, 64:]) * np.exp(1j * pos * inv)
        expect = np.concatenate([z.real, z.imag], axis=1)
        phi = orc.angles(t_g, h, w, 16, 24, 24, 10000.0, 1)
        assert np.allclose(orc.rotate_pairing(x, phi, 1), expect, rtol=0, atol=1e-13)


def check_half_pairing_relative_offset(orc):
    """<R(p_m) q, R(p_n) k> = <q, R(p_n - p_m) k> with the rotate_half pairing, all pairs
    of 24 tokens of a 2x3x4 grid."""
    rng = _rng(22)
    T, H, W, s = 2, 3, 4, 5
    n = T * H * W
    q = rng.standard_normal((n, 2, D))
    k = rng.standard_normal((n, 2, D))
    pos = [orc.decode(i, s, T, H, W) for i in range(n)]

    def rot(x, p):
        return orc.rotate_pairing(x, orc.angles(*p), 1)
    rq = [rot(q[m], pos[m]) for m in range(n)]
    rk = [rot(k[m], pos[m]) for m in range(n)]
    for m in range(n):
        for nn in range(n):
            d = tuple(pos[nn][a] - pos[m][a] for a in range(3))
            assert abs(float(np.sum(rq[m] * rk[nn])) - float(np.sum(q[m] * rot(k[nn], d)))) < 1e-10


def check_layout_step_default_equals_base_step(orc):
    """Adjacent pairing with a token-major cache is the base step, bit for bit."""
    B, N, T, H, W, s, slot, C = 2, 2, 3, 4, 6, 3, 50, 144
    q, k, v, wq, wk = _step_inputs(23, B, 72, N)
    kc0, vc0 = np.zeros((B, C, N, D)), np.zeros((B, C, N, D))
    q0 = orc.qk_norm_rope_append(q, k, v, 0, 72, s, T, H, W, wq, wk, 1e-6, kc0, vc0, slot)
    kc1, vc1 = np.zeros((B, C, N, D)), np.zeros((B, C, N, D))
    q1 = orc.qk_norm_rope_append_layout(q, k, v, 0, 72, s, T, H, W, wq, wk, 1e-6, kc1, vc1, slot,
                                        0, 0)
    assert np.array_equal(q0, q1) and np.array_equal(kc0, kc1) and np.array_equal(vc0, vc1)


def check_head_major_cache_is_transpose(orc):
    """A head-major cache holds exactly the token-major cache with heads moved forward."""
    B, N, T, H, W, s, slot, C = 2, 3, 3, 4, 6, 6, 100, 144
    q, k, v, wq, wk = _step_inputs(24, B, 72, N)
    for pairing in (0, 1):
        kt, vt = np.zeros((B, C, N, D)), np.zeros((B, C, N, D))
        qt = orc.qk_norm_rope_append_layout(q, k, v, 0, 72, s, T, H, W, wq, wk, 1e-6, kt, vt,
                                            slot, pairing, 0)
        kh, vh = np.zeros((B, N, C, D)), np.zeros((B, N, C, D))
        qh = orc.qk_norm_rope_append_layout(q, k, v, 0, 72, s, T, H, W, wq, wk, 1e-6, kh, vh,
                                            slot, pairing, 1)
        assert np.array_equal(qt, qh)
        assert np.array_equal(kh, kt.transpose(0, 2, 1, 3))
        assert np.array_equal(vh, vt.transpose(0, 2, 1, 3))


def check_layout_step_slices_and_rows(orc):
    """A token range that starts mid-chunk, in either pairing and layout, writes row r of
    q_out from global index begin + r and cache row (slot + begin + r) mod C, exactly as
    the per-token function computes them."""
    B, N, T, H, W, s, slot, C = 1, 2, 3, 4, 6, 3, 130, 144
    tb, te = 13, 60
    q, k, v, wq, wk = _step_inputs(27, B, te - tb, N)
    for pairing in (0, 1):
        for layout in (0, 1):
            shape = (B, C, N, D) if layout == 0 else (B, N, C, D)
            kc, vc = np.zeros(shape), np.zeros(shape)
            qo = orc.qk_norm_rope_append_layout(q, k, v, tb, te, s, T, H, W, wq, wk, 1e-6, kc,
                                                vc, slot, pairing, layout)
            for r in (0, 11, te - tb - 1):
                eq, ek, ev, pos = orc.token_pairing(q[0, r], k[0, r], v[0, r], tb + r, s, T, H,
                                                    W, wq, wk, 1e-6, slot, C, pairing)
                assert pos[3] == (slot + tb + r) % C
                assert np.array_equal(qo[0, r], eq)
                got_k = kc[0, pos[3]] if layout == 0 else kc[0, :, pos[3]]
                got_v = vc[0, pos[3]] if layout == 0 else vc[0, :, pos[3]]
                assert np.array_equal(got_k, ek) and np.array_equal(got_v, ev)


def check_half_step_is_norm_then_rotate_half(orc):
    """With the rotate_half pairing the step's q and K rows are rotate_half(RMSNorm(x))
    built from the separately pinned pieces; V is copied."""
    B, N, T, H, W, s, slot, C = 1, 2, 3, 4, 6, 3, 0, 72
    q, k, v, wq, wk = _step_inputs(25, B, 72, N)
    kc, vc = np.zeros((B, C, N, D)), np.zeros((B, C, N, D))
    qo = orc.qk_norm_rope_append_layout(q, k, v, 0, 72, s, T, H, W, wq, wk, 1e-6, kc, vc, slot,
                                        1, 0)
    for r in (0, 17, 71):
        phi = orc.angles(*orc.decode(r, s, T, H, W))
        eq = orc.rotate_pairing(orc.rms_norm(q[0, r], wq, 1e-6).reshape(N, D), phi, 1)
        ek = orc.rotate_pairing(orc.rms_norm(k[0, r], wk, 1e-6).reshape(N, D), phi, 1)
        assert np.allclose(qo[0, r], eq, rtol=0, atol=1e-13)
        assert np.allclose(kc[0, r], ek, rtol=0, atol=1e-13)
        assert np.array_equal(vc[0, r], v[0, r])


def check_apply_half_matches_rotation(orc):
    B, N, T, H, W, s = 1, 2, 3, 4, 6, 9
    rng = _rng(26)
    x = rng.standard_normal((B, 30, N, D))
    y = orc.apply_pairing(x, 10, 40, s, T, H, W, 1)
    for r in range(30):
        phi = orc.angles(*orc.decode(10 + r, s, T, H, W))
        assert np.array_equal(y[0, r], orc.rotate_pairing(x[0, r], phi, 1))


# ---------------------------------------------------------------- FP8 E4M3 KV cache

def check_e4m3_closed_form_values(orc):
    """E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits, subnormals, max 448, NaN at
    the all-ones code."""
    expect = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0,
              0x39: 1.125, 0x3C: 1.5, 0x40: 2.0, 0x77: 240.0, 0x7E: 448.0, 0xB8: -1.0,
              0xFE: -448.0}
    for code, value in expect.items():
        assert orc.e4m3_value(code) == value, hex(code)
    assert math.isnan(orc.e4m3_value(0x7F)) and math.isnan(orc.e4m3_value(0xFF))
    assert math.copysign(1.0, orc.e4m3_value(0x80)) == -1.0


def check_e4m3_encode_round_trip_ties_saturation(orc):
    vals = [orc.e4m3_value(c) for c in range(0x7F)]
    assert all(b > a for a, b in zip(vals, vals[1:]))        # strictly increasing
    for c in range(0x7F):
        assert orc.e4m3_encode(vals[c]) == c
        assert orc.e4m3_encode(-vals[c]) == 0x80 | c
    for c in range(0x7E):                                     # midpoints go to the even code
        mid = (vals[c] + vals[c + 1]) / 2
        if np.float32(mid) == mid:
            assert orc.e4m3_encode(mid) == (c if c % 2 == 0 else c + 1), hex(c)
    assert orc.e4m3_encode(1000.0) == 0x7E and orc.e4m3_encode(-1e9) == 0xFE
    assert orc.e4m3_encode(448.0) == 0x7E and orc.e4m3_encode(463.99) == 0x7E


def check_e4m3_encode_matches_torch(orc):
    """In range, the encoder equals torch's float32 -> float8_e4m3fn conversion."""
    import torch
    rng = _rng(30)
    xs = np.concatenate([rng.uniform(-447, 447, 300), rng.standard_normal(300),
                         rng.standard_normal(200) * 1e-3,
                         np.array([orc.e4m3_value(c) for c in range(0x7E)]) * 1.0625])
    xs = xs.astype(np.float32)
    got = np.array([orc.e4m3_encode(float(x)) for x in xs], dtype=np.uint8)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def check_e4m3_scale_exponent_closed_forms(orc):
    """The power-of-two scale: smallest 2^e with amax / 2^e <= 448."""
    cases = {448.0: 0, 449.0: 1, 1.0: -8, 3.5: -7, 3.5000002: -6, 224.0: -1, 224.00002: 0,
             896.0: 1, 1e-3: -18, 3.0e38: 120}
    for amax, e in cases.items():
        assert orc.e4m3_scale_exponent(amax) == e, amax
    assert orc.e4m3_scale_exponent(1e-40) == -126      # clamped at the smallest normal 2^e
    assert orc.e4m3_scale_exponent(0.0) == -126        # the same rule for an all-zero head
    assert orc.e4m3_scale_exponent(448.0 * 2.0 ** -126) == -126
    assert orc.e4m3_scale_exponent(float(np.nextafter(np.float32(448.0 * 2.0 ** -126),
                                                      np.float32(1)))) == -125


def check_e4m3_head_quantizer(orc):
    """scale = 2^e with the head's largest magnitude in (224, 448] after scaling; codes are
    E4M3(x / scale) of the exactly scaled values; every value is recovered within half an
    E4M3 step; an all-zero head has scale 2^-126 (the rule's smallest) and zero codes."""
    rng = _rng(31)
    for _ in range(5):
        x = (rng.standard_normal(128) * rng.uniform(0.1, 5)).astype(np.float32)
        codes, scale = orc.quantize_head_e4m3(x)
        amax = float(np.max(np.abs(x)))
        m, ex = math.frexp(scale)
        assert m == 0.5 and 224.0 < amax / scale <= 448.0
        assert np.array_equal(codes, [orc.e4m3_encode(float(np.float32(v) / np.float32(scale)))
                                      for v in x])
        deq = np.array([orc.e4m3_value(int(c)) for c in codes]) * scale
        y = np.abs(x.astype(np.float64) / scale)
        step = np.where(y >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(y, 2.0 ** -6))) - 3),
                        2.0 ** -9)
        assert np.all(np.abs(deq - x) <= 0.5 * step * scale * (1 + 1e-12))
    codes, scale = orc.quantize_head_e4m3(np.zeros(128, dtype=np.float32))
    assert scale == 2.0 ** -126 and np.all((codes & 0x7F) == 0)


def check_fp8_step_matches_layout_step(orc):
    """The FP8-cache step leaves q_out as the plain step does and stores, per (token,
    head), the quantization of the plain step's K and V rows (rounded to fp32)."""
    B, N, T, H, W, s, slot, C = 1, 2, 3, 4, 6, 3, 100, 144
    tb, te = 5, 60
    q, k, v, wq, wk = _step_inputs(32, B, te - tb, N)
    for pairing in (0, 1):
        for layout in (0, 1):
            shape = (B, C, N, D) if layout == 0 else (B, N, C, D)
            kf, vf = np.zeros(shape), np.zeros(shape)
            q0 = orc.qk_norm_rope_append_layout(q, k, v, tb, te, s, T, H, W, wq, wk, 1e-6, kf, vf,
                                                slot, pairing, layout)
            kc = np.zeros(shape, dtype=np.uint8)
            vc = np.zeros(shape, dtype=np.uint8)
            ks = np.zeros(shape[:3], dtype=np.float32)
            vs = np.zeros(shape[:3], dtype=np.float32)
            q1 = orc.qk_norm_rope_append_fp8(q, k, v, tb, te, s, T, H, W, wq, wk, 1e-6, kc, vc,
                                             ks, vs, slot, pairing, layout)
            assert np.array_equal(q0, q1)
            for r in (0, 20, te - tb - 1):
                row = (slot + tb + r) % C
                for n in range(N):
                    idx = (0, row, n) if layout == 0 else (0, n, row)
                    ek, esk = orc.quantize_head_e4m3(kf[idx])
                    ev, esv = orc.quantize_head_e4m3(vf[idx])
                    assert np.array_equal(kc[idx], ek) and ks[idx] == esk
                    assert np.array_equal(vc[idx], ev) and vs[idx] == esv


# ---------------------------------------------------------------- NVFP4 cache

E2M1_MAGNITUDES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]  # the format's 8 magnitudes


def check_e2m1_closed_forms(orc):
    """E2M1 (sign, 2 exponent bits with bias 1, 1 mantissa bit): codes 0..7 are the
    magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 and codes 8..15 their negatives; every value
    encodes to itself; midpoints go to the even code; magnitudes from 6 up saturate to
    code 7; just off a midpoint goes to the nearer value; -0 keeps its sign."""
    for c in range(16):
        mag = E2M1_MAGNITUDES[c & 7]
        assert orc.e2m1_value(c) == (-mag if c & 8 else mag), c
        assert orc.e2m1_encode(float(orc.e2m1_value(c))) == (c if c != 8 else 8)
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for x, c in ties.items():
        assert orc.e2m1_encode(x) == c, x
        assert orc.e2m1_encode(-x) == c | 8, -x
        lo, hi = np.nextafter(np.float32(x), np.float32(0)), np.nextafter(np.float32(x), np.float32(9))
        assert orc.e2m1_encode(float(lo)) == E2M1_MAGNITUDES.index(max(m for m in E2M1_MAGNITUDES if m < x))
        assert orc.e2m1_encode(float(hi)) == E2M1_MAGNITUDES.index(min(m for m in E2M1_MAGNITUDES if m > x))
    for x in (6.0, 6.5, 7.0, 1e30):
        assert orc.e2m1_encode(x) == 7 and orc.e2m1_encode(-x) == 15
    assert orc.e2m1_encode(-0.0) == 8 and orc.e2m1_encode(0.0) == 0
    assert orc.e2m1_encode(-0.2) == 8  # rounds to a negative zero


def check_nvfp4_block_worked_example(orc):
    """The block 0, 1, ..., 15 worked by hand: amax 15, 15 fp32(1/6) rounds to 2.5 in
    fp32, S = E4M3(2.5) = 0x42 (1.25 * 2^1, exact), r = fp32(1 / 2.5), and
    x r = 0, 0.4, ..., 6.0 rounds to
    0, 0.5, 1, 1, 1.5, 2, 2, 3, 3, 4, 4, 4, 4, 6, 6, 6, packed low nibble first."""
    codes, scale = orc.quantize_block_nvfp4(np.arange(16, dtype=np.float32))
    assert scale == 0x42
    want = [0, 1, 2, 2, 3, 4, 4, 5, 5, 6, 6, 6, 6, 7, 7, 7]
    assert list(codes) == [want[2 * j] | (want[2 * j + 1] << 4) for j in range(8)]


def check_nvfp4_block_quantizer(orc):
    """Block scale and codes follow the recipe (S = E4M3(amax fp32(1 / (6 g))), codes =
    E2M1(x / (value(S) g)) through an fp32 reciprocal); every value is recovered within
    half an E2M1 step of value(S) g, except where amax / (value(S) g) exceeds 6 and the
    largest values saturate; a zero block has scale 0 and zero codes; a power-of-two
    global scale g = 2^k gives the same codes and scale for x 2^k."""
    rng = _rng(43)
    for g in (1.0, 0.25, 3.0):
        for _ in range(6):
            x = (rng.standard_normal(16) * rng.uniform(0.05, 20)).astype(np.float32)
            codes, S = orc.quantize_block_nvfp4(x, g)
            amax = np.float32(np.max(np.abs(x)))
            k = np.float32(1.0) / np.float32(6.0 * g)
            assert S == orc.e4m3_encode(float(amax * k))
            sv = np.float32(orc.e4m3_value(S))
            r = np.float32(1.0) / np.float32(sv * np.float32(g))
            got = [(c >> 4 * (e & 1)) & 15 for e, c in enumerate(np.repeat(codes, 2))]
            assert got == [orc.e2m1_encode(float(np.float32(xe) * r)) for xe in x]
            deq = np.array([orc.e2m1_value(c) for c in got]) * float(sv) * g
            y = np.abs(x.astype(np.float64)) / (float(sv) * g)
            step = np.where(y < 2, 0.5, np.where(y < 4, 1.0, 2.0))
            bound = np.where(y <= 6, 0.5 * step, y - 6) * float(sv) * g
            assert np.all(np.abs(deq - x) <= bound * (1 + 1e-6) + 1e-30)
    codes, S = orc.quantize_block_nvfp4(np.zeros(16, dtype=np.float32))
    assert S == 0 and not codes.any()
    x = (rng.standard_normal(16) * 3).astype(np.float32)
    c1, s1 = orc.quantize_block_nvfp4(x, 1.0)
    c2, s2 = orc.quantize_block_nvfp4(x * np.float32(8.0), 8.0)
    assert np.array_equal(c1, c2) and s1 == s2


def check_nvfp4_step_matches_layout_step(orc):
    """The NVFP4-cache step leaves q_out as the plain step does and stores, per block of
    16 elements of each (token, head), the block quantization of the plain step's K and V
    values (rounded to fp32) with the K and V global scales."""
    B, N, T, H, W, s, slot, C = 1, 2, 3, 4, 6, 3, 100, 144
    tb, te = 5, 60
    kg, vg = 0.75, 2.0
    q, k, v, wq, wk = _step_inputs(33, B, te - tb, N)
    for pairing in (0, 1):
        for layout in (0, 1):
            shape = (B, C, N, D) if layout == 0 else (B, N, C, D)
            kf, vf = np.zeros(shape), np.zeros(shape)
            q0 = orc.qk_norm_rope_append_layout(q, k, v, tb, te, s, T, H, W, wq, wk, 1e-6, kf, vf,
                                                slot, pairing, layout)
            kc = np.zeros(shape[:3] + (D // 2,), dtype=np.uint8)
            vc = np.zeros_like(kc)
            ks = np.zeros(shape[:3] + (D // 16,), dtype=np.uint8)
            vs = np.zeros_like(ks)
            q1 = orc.qk_norm_rope_append_nvfp4(q, k, v, tb, te, s, T, H, W, wq, wk, 1e-6, kc, vc,
                                               ks, vs, slot, kg, vg, pairing, layout)
            assert np.array_equal(q0, q1)
            for r in (0, 20, te - tb - 1):
                row = (slot + tb + r) % C
                for n in range(N):
                    idx = (0, row, n) if layout == 0 else (0, n, row)
                    for blk in range(D // 16):
                        sl = slice(16 * blk, 16 * blk + 16)
                        ek, esk = orc.quantize_block_nvfp4(kf[idx][sl], kg)
                        ev, esv = orc.quantize_block_nvfp4(vf[idx][sl], vg)
                        assert np.array_equal(kc[idx][8 * blk:8 * blk + 8], ek)
                        assert np.array_equal(vc[idx][8 * blk:8 * blk + 8], ev)
                        assert ks[idx][blk] == esk and vs[idx][blk] == esv


# ---------------------------------------------------------------- QKV projection

def check_qkv_project_brute_force(orc):
    """q, k, v = QKV(x) (Algorithm 1/3 step 1) as an nn.Linear: out[t][o] = sum_i x[t][i]
    w[o][i] + b[o], with output rows [0, dim) -> q, [dim, 2 dim) -> k, [2 dim, 3 dim) -> v;
    checked by explicit loops on a tiny case, with and without bias."""
    rng = _rng(51)
    B, n, din, dim = 2, 3, 5, 4
    x = rng.standard_normal((B, n, din))
    w = rng.standard_normal((3 * dim, din))
    b = rng.standard_normal(3 * dim)
    for bias in (b, None):
        q, k, v = orc.qkv_project(x, w, bias)
        for bb in range(B):
            for t in range(n):
                for o in range(3 * dim):
                    acc = 0.0
                    for i in range(din):
                        acc += x[bb, t, i] * w[o, i]
                    if bias is not None:
                        acc += bias[o]
                    got = (q, k, v)[o // dim][bb, t, o % dim]
                    assert abs(got - acc) <= 1e-12 * (1 + abs(acc))


def check_qkv_project_closed_forms(orc):
    """A one-hot token e_j picks column j of each projection plus its bias; a zero token
    gives the bias alone."""
    rng = _rng(52)
    din, dim = 6, 4
    w = rng.standard_normal((3 * dim, din))
    b = rng.standard_normal(3 * dim)
    x = np.zeros((1, din + 1, din))
    for j in range(din):
        x[0, j, j] = 1.0
    q, k, v = orc.qkv_project(x, w, b)
    for j in range(din):
        assert np.allclose(q[0, j], w[:dim, j] + b[:dim], rtol=0, atol=1e-15)
        assert np.allclose(k[0, j], w[dim:2 * dim, j] + b[dim:2 * dim], rtol=0, atol=1e-15)
        assert np.allclose(v[0, j], w[2 * dim:, j] + b[2 * dim:], rtol=0, atol=1e-15)
    assert np.array_equal(np.concatenate([q[0, din], k[0, din], v[0, din]]), b)


def check_bf16_round(orc):
    """Rounding to bfloat16: equal to torch's float32 -> bfloat16 conversion (a library
    routine) on float32 values across the exponent range; exact midpoints go to the even
    significand; below 2^-126 the spacing is 2^-133."""
    import torch
    rng = _rng(53)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-80, 80, 20000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(orc.bf16_round(x.astype(np.float64)), ref)
    ulp = 2.0 ** -7
    mids = np.array([1 + ulp / 2, 1 + 3 * ulp / 2, -(1 + ulp / 2), 3 + ulp, 3 + 3 * ulp])
    assert list(orc.bf16_round(mids)) == [1.0, 1 + 2 * ulp, -1.0, 3.0, 3 + 4 * ulp]
    tiny = np.array([2.0 ** -133 * 2.5, 2.0 ** -133 * 3.5, 2.0 ** -126 * (1 + 2 ** -9)])
    assert list(orc.bf16_round(tiny)) == [2.0 ** -132, 2.0 ** -131, 2.0 ** -126]


def check_sp_head_scatter_is_whole_step_split_by_heads(orc):
    """Algorithm 3 steps 3-5 with the all-to-all folded in: ranks with uneven token
    ranges, each storing every head at its owner, together leave in owner r exactly the
    whole-sequence step's heads [r N/P, (r+1) N/P) -- q at rows i - q_row0 of its buffer,
    K/V at the rolling cache rows -- and nothing else (sentinels elsewhere stay).  Both
    cache layouts; P = 1, 2, 4; q buffers longer than the range, and buffers that start
    mid-chunk (q_row0 > 0)."""
    rng = _rng(41)
    B, N, T, H, W, s, C, slot = 2, 4, 3, 4, 6, 6, 100, 90
    L = T * H * W
    q, k, v = (_f32(rng.standard_normal((B, L, N, D))) for _ in range(3))
    wq, wk = (_f32(rng.uniform(0.5, 1.5, N * D)) for _ in range(2))
    kw, vw = np.zeros((B, C, N, D)), np.zeros((B, C, N, D))
    whole = orc.qk_norm_rope_append_layout(q, k, v, 0, L, s, T, H, W, wq, wk, 1e-6, kw, vw,
                                           slot)
    for P, cuts, q_row0, q_rows in ((1, [0, L], 0, L), (2, [0, 17, 40, L], 0, L + 9),
                                    (4, [0, 17, 40, L], 0, L), (2, [24, 50, L], 24, L - 24 + 3)):
        hl = N // P
        span = np.arange(cuts[0], cuts[-1])
        rows = (slot + span) % C
        for layout in (CACHE_TOKEN_MAJOR, CACHE_HEAD_MAJOR):
            cshape = (B, C, hl, D) if layout == CACHE_TOKEN_MAJOR else (B, hl, C, D)
            q_dst = [np.full((B, q_rows, hl, D), 7.0) for _ in range(P)]
            k_dst = [np.full(cshape, 7.0) for _ in range(P)]
            v_dst = [np.full(cshape, 7.0) for _ in range(P)]
            for a, e in zip(cuts[:-1], cuts[1:]):
                orc.qk_norm_rope_append_sp(q[:, a:e].copy(), k[:, a:e].copy(),
                                           v[:, a:e].copy(), a, e, s, T, H, W, wq, wk, 1e-6,
                                           q_dst, k_dst, v_dst, slot, q_row0=q_row0,
                                           cache_layout=layout)
            for r in range(P):
                heads = slice(r * hl, (r + 1) * hl)
                got = q_dst[r][:, span - q_row0]
                assert np.array_equal(got, whole[:, span][:, :, heads])
                assert np.all(np.delete(q_dst[r], span - q_row0, axis=1) == 7.0)
                kt, vt = k_dst[r], v_dst[r]
                if layout == CACHE_HEAD_MAJOR:
                    kt, vt = kt.transpose(0, 2, 1, 3), vt.transpose(0, 2, 1, 3)
                assert np.array_equal(kt[:, rows], kw[:, rows][:, :, heads])
                assert np.array_equal(vt[:, rows], v[:, span][:, :, heads])
                assert np.all(np.delete(kt, rows, axis=1) == 7.0)


def check_sp_output_all_to_all_inverts_the_head_split(orc):
    """Algorithm 3's last step, o <- AllToAll(o, scatter_dim=1, gather_dim=2): if every
    rank holds the whole sequence for its own heads -- a tensor X split by heads -- then
    afterwards rank r holds its token slice of X with every head, i.e. X split by tokens
    (numpy.split on the other axis).  P = 1, 2, 4, uneven slices and an empty one."""
    rng = _rng(43)
    B, L, N = 2, 23, 8
    X = rng.standard_normal((B, L, N, D))
    for P, cuts in ((1, [0, L]), (2, [0, 9, L]), (4, [0, 5, 5, 17, L]), (4, [0, 6, 12, 18, L])):
        hl = N // P
        o_ranks = np.split(X, P, axis=2)  # rank r: heads [r hl, (r+1) hl), all tokens
        outs = orc.sp_output_all_to_all([x.copy() for x in o_ranks], cuts)
        want = np.split(X, cuts[1:-1], axis=1)  # rank r: tokens [cuts[r], cuts[r+1])
        assert len(outs) == P
        for got, ref in zip(outs, want):
            assert got.shape == ref.shape and np.array_equal(got, ref)


def check_sp_round_trip_returns_each_slice_with_every_head(orc):
    """The two exchanges of Algorithm 3 compose: rank slices through the step with the
    head scatter (step 4 folded into the stores) give each owner the whole sequence for
    its heads; the output all-to-all then gives each rank back its own token slice with
    every head, equal to the whole-sequence step's rows of that slice."""
    rng = _rng(44)
    B, N, T, H, W, s, C, slot = 1, 4, 2, 3, 5, 3, 40, 7
    L = T * H * W
    q, k, v = (_f32(rng.standard_normal((B, L, N, D))) for _ in range(3))
    wq, wk = (_f32(rng.uniform(0.5, 1.5, N * D)) for _ in range(2))
    kw, vw = np.zeros((B, C, N, D)), np.zeros((B, C, N, D))
    whole = orc.qk_norm_rope_append_layout(q, k, v, 0, L, s, T, H, W, wq, wk, 1e-6, kw, vw,
                                           slot)
    P, cuts = 2, [0, 11, L]
    hl = N // P
    q_dst = [np.zeros((B, L, hl, D)) for _ in range(P)]
    k_dst = [np.zeros((B, C, hl, D)) for _ in range(P)]
    v_dst = [np.zeros((B, C, hl, D)) for _ in range(P)]
    for a, e in zip(cuts[:-1], cuts[1:]):
        orc.qk_norm_rope_append_sp(q[:, a:e].copy(), k[:, a:e].copy(), v[:, a:e].copy(), a, e,
                                   s, T, H, W, wq, wk, 1e-6, q_dst, k_dst, v_dst, slot)
    back = orc.sp_output_all_to_all(q_dst, cuts)
    for r in range(P):
        assert np.array_equal(back[r], whole[:, cuts[r]:cuts[r + 1]])


ALL_CHECKS = [v for k, v in sorted(globals().items()) if k.startswith("check_")]
