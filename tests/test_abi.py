"""The C ABI library without a GPU: it loads, exports every entry point that
include/rope3d.h declares, and rejects bad arguments with a status (never a crash).
Compute calls need a GPU and live in the gpu-marked tests."""
import ctypes
import os
import re

import pytest
import torch

from rotary_position_encoding_b200 import build as native_build
from rotary_position_encoding_b200 import rope3d

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("rope3d.h", "rope3d_testing.h")]


@pytest.fixture(scope="module")
def lib():
    native_build.build()
    return rope3d.load_library()


def _header_text():
    return "\n".join(open(h).read() for h in HEADERS)


def header_functions():
    return re.findall(r"ROPE3D_API\s+[\w\s\*]+?\b(rope3d_\w+)\s*\(", _header_text())


def header_constants():
    text = _header_text()
    return {m[0]: int(m[1]) for m in re.findall(r"#define\s+(ROPE3D_[A-Z0-9_]+)\s+\(?(-?\d+)\)?",
                                                  text)}


def test_header_declares_the_boundary():
    names = header_functions()
    for required in ("rope3d_tables_init", "rope3d_tables_destroy",
                     "rope3d_qk_norm_rope_append", "rope3d_apply", "rope3d_decode_positions",
                     "rope3d_strerror"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    names = header_functions()
    assert names
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(rope3d.SIGNATURES), "binding and header disagree"


def test_binding_constants_match_header():
    for name, value in header_constants().items():
        if hasattr(rope3d, name):
            assert getattr(rope3d, name) == value, name


def test_strerror_and_version(lib):
    for status in (0, -1, -2, -3, -4, -5, -6, -7, -99):
        assert lib.rope3d_strerror(status)
    assert rope3d.rope3d_version() >= 10000


def test_null_and_bad_arguments_rejected_without_device(lib):
    handle = ctypes.c_void_p(12345)
    # head_dim must equal 2 (n_t + n_h + n_w): rejected before any CUDA call
    assert lib.rope3d_tables_init(ctypes.byref(handle), 128, 22, 21, 20, 1e4, 0, 0, 0, 0,
                                  None) == rope3d.ROPE3D_EINVAL
    assert handle.value is None
    assert lib.rope3d_tables_init(None, 128, 22, 21, 21, 1e4, 0, 0, 0, 0, None) == rope3d.ROPE3D_EINVAL
    assert lib.rope3d_tables_init(ctypes.byref(handle), 128, 22, 21, 21, 0.5, 0, 0, 0, 0,
                                  None) == rope3d.ROPE3D_EINVAL
    assert lib.rope3d_tables_init(ctypes.byref(handle), 128, 22, 21, 21, 1e4, 0, 0, 0, 7,
                                  None) == rope3d.ROPE3D_EINVAL
    assert lib.rope3d_tables_init(ctypes.byref(handle), 128, 22, 21, 21, 1e4, 10, 0, 5, 0,
                                  None) == rope3d.ROPE3D_EINVAL
    assert "head_dim" in rope3d.rope3d_last_error() or rope3d.rope3d_last_error()
    # the fused step and the rotation with NULL tables
    p = ctypes.c_void_p(0x10000)
    assert lib.rope3d_qk_norm_rope_append(p, p, p, p, 1, 2, 128, 1, 0, 72, 0, 3, 4, 6, p, p,
                                          1e-6, p, p, 144, 0, None, 0, None) == rope3d.ROPE3D_EINVAL
    assert lib.rope3d_apply(p, p, 1, 2, 128, 1, 0, 72, 0, 3, 4, 6, None, 0, None) == rope3d.ROPE3D_EINVAL
    # decode: empty range, range past the grid, bad grid, misaligned output
    assert lib.rope3d_decode_positions(5, 5, 0, 3, 4, 6, 144, 0, p, None) == rope3d.ROPE3D_ERANGE
    assert lib.rope3d_decode_positions(0, 73, 0, 3, 4, 6, 144, 0, p, None) == rope3d.ROPE3D_ERANGE
    assert lib.rope3d_decode_positions(0, 10, 0, 0, 4, 6, 144, 0, p, None) == rope3d.ROPE3D_EINVAL
    assert lib.rope3d_decode_positions(0, 10, 0, 3, 4, 6, 0, 0, p, None) == rope3d.ROPE3D_EINVAL
    assert lib.rope3d_decode_positions(0, 10, 0, 3, 4, 6, 144, 0, ctypes.c_void_p(0x10004),
                                       None) == rope3d.ROPE3D_EALIGN
    assert lib.rope3d_decode_positions(0, 10, -1, 3, 4, 6, 144, 0, p, None) == rope3d.ROPE3D_EINVAL


def test_testing_hooks_validate_without_device(lib):
    assert lib.rope3d_testing_force_path(7) == rope3d.ROPE3D_EINVAL
    assert lib.rope3d_testing_force_path(rope3d.ROPE3D_PATH_AUTO) == rope3d.ROPE3D_OK
    lib.rope3d_testing_set_waits(0, 0)
    assert lib.rope3d_check_device_status(None, None) == rope3d.ROPE3D_EINVAL
    assert lib.rope3d_testing_shrink_checked_cache(-1) == rope3d.ROPE3D_EINVAL
    assert lib.rope3d_testing_shrink_checked_cache(0) == rope3d.ROPE3D_OK


def test_checked_build_compiles_and_exports_every_declared_symbol():
    """librope3d_checked.so is the same source built with -DROPE3D_DEVICE_CHECKS."""
    native_build.build_all()
    checked = rope3d.load_library(native_build.CHECKED_LIBRARY)
    assert checked is not rope3d.load_library()
    for name in header_functions():
        assert hasattr(checked, name), name
    assert checked.rope3d_strerror(rope3d.ROPE3D_EINDEX).decode().startswith("a device-side")
    assert checked.rope3d_version() == rope3d.load_library().rope3d_version()


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        rope3d.load_library(str(tmp_path / "librope3d.so"))


def test_options_struct_layout_matches_header(tmp_path):
    """The ctypes mirror of rope3d_options has the C struct's size and field offsets."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("needs gcc")
    src = tmp_path / "layout.c"
    src.write_text('#include <stddef.h>\n#include <stdio.h>\n#include "rope3d.h"\n'
                   'int main(void){printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu",'
                   ' sizeof(rope3d_options),'
                   ' offsetof(rope3d_options, pairing), offsetof(rope3d_options, cache_layout),'
                   ' offsetof(rope3d_options, cache_dtype), offsetof(rope3d_options, k_scale),'
                   ' offsetof(rope3d_options, v_scale), offsetof(rope3d_options, nvfp4_k_global),'
                   ' offsetof(rope3d_options, nvfp4_v_global), offsetof(rope3d_options, reserved));'
                   ' return 0;}\n')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    got = list(map(int, subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()))
    S = rope3d.rope3d_options
    assert got == [ctypes.sizeof(S), S.pairing.offset, S.cache_layout.offset,
                   S.cache_dtype.offset, S.k_scale.offset, S.v_scale.offset,
                   S.nvfp4_k_global.offset, S.nvfp4_v_global.offset, S.reserved.offset]


def test_sp_dest_struct_layout_matches_header(tmp_path):
    """The ctypes mirror of rope3d_sp_dest has the C struct's size and field offsets."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("needs gcc")
    fields = ("ranks", "reserved0", "q_rows", "q_row0", "q", "k_cache", "v_cache")
    src = tmp_path / "layout_sp.c"
    src.write_text('#include <stddef.h>\n#include <stdio.h>\n#include "rope3d.h"\n'
                   'int main(void){printf("%zu", sizeof(rope3d_sp_dest));'
                   + "".join(f'printf(" %zu", offsetof(rope3d_sp_dest, {f}));' for f in fields)
                   + ' return 0;}\n')
    exe = tmp_path / "layout_sp"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    got = list(map(int, subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()))
    S = rope3d.rope3d_sp_dest
    assert got == [ctypes.sizeof(S)] + [getattr(S, f).offset for f in fields]


def test_sp_out_dest_struct_layout_matches_header(tmp_path):
    """The ctypes mirror of rope3d_sp_out_dest has the C struct's size and field offsets."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("needs gcc")
    fields = ("ranks", "rank", "cuts", "out")
    src = tmp_path / "layout_spo.c"
    src.write_text('#include <stddef.h>\n#include <stdio.h>\n#include "rope3d.h"\n'
                   'int main(void){printf("%zu", sizeof(rope3d_sp_out_dest));'
                   + "".join(f'printf(" %zu", offsetof(rope3d_sp_out_dest, {f}));'
                             for f in fields)
                   + ' return 0;}\n')
    exe = tmp_path / "layout_spo"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True)
    got = list(map(int, subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()))
    S = rope3d.rope3d_sp_out_dest
    assert got == [ctypes.sizeof(S)] + [getattr(S, f).offset for f in fields]


def test_sp_output_all_to_all_rejects_bad_arguments_without_device(lib):
    """Every host-side check of the output all-to-all fails before any CUDA call."""
    o = 0x100000
    dest = rope3d.rope3d_sp_out_dest()
    dest.ranks, dest.rank = 2, 0
    dest.cuts[0], dest.cuts[1], dest.cuts[2] = 0, 5, 10
    dest.out[0], dest.out[1] = 0x200000, 0x300000

    def call(o=o, B=1, L=10, hl=2, D=128, dtype=rope3d.ROPE3D_BF16, d=dest):
        return lib.rope3d_sp_output_all_to_all(o, B, L, hl, D, dtype,
                                               None if d is None else ctypes.byref(d), None)
    assert call(o=0) == rope3d.ROPE3D_EINVAL
    assert call(d=None) == rope3d.ROPE3D_EINVAL
    assert call(D=64) == rope3d.ROPE3D_EINVAL
    assert call(dtype=7) == rope3d.ROPE3D_EINVAL
    assert call(L=11) == rope3d.ROPE3D_ERANGE  # cuts end at 10
    assert call(o=o + 8) == rope3d.ROPE3D_EALIGN
    bad = rope3d.rope3d_sp_out_dest.from_buffer_copy(dest)
    bad.rank = 2
    assert call(d=bad) == rope3d.ROPE3D_EINVAL
    bad = rope3d.rope3d_sp_out_dest.from_buffer_copy(dest)
    bad.ranks = 9
    assert call(d=bad) == rope3d.ROPE3D_EINVAL
    bad = rope3d.rope3d_sp_out_dest.from_buffer_copy(dest)
    bad.cuts[1] = 11
    assert call(d=bad) == rope3d.ROPE3D_ERANGE  # cuts fall
    bad = rope3d.rope3d_sp_out_dest.from_buffer_copy(dest)
    bad.out[1] = 0
    assert call(d=bad) == rope3d.ROPE3D_EINVAL
    bad = rope3d.rope3d_sp_out_dest.from_buffer_copy(dest)
    bad.out[1] = 0x200000 + 16
    assert call(d=bad) == rope3d.ROPE3D_EOVERLAP  # outputs overlap each other
    bad = rope3d.rope3d_sp_out_dest.from_buffer_copy(dest)
    bad.out[0] = o + 16
    assert call(d=bad) == rope3d.ROPE3D_EOVERLAP  # an output overlaps o


def test_sp_step_rejects_null_arguments_without_device(lib):
    """NULL tables or a NULL destination table fail on the host (the destination checks that
    need real tables run in the gpu-marked tests)."""
    p = ctypes.c_void_p(0x10000)
    dest = rope3d.rope3d_sp_dest()
    dest.ranks, dest.q_rows, dest.q_row0 = 2, 72, 0
    for r in range(2):
        dest.q[r] = dest.k_cache[r] = dest.v_cache[r] = 0x100000 * (r + 1)
    for d in (ctypes.byref(dest), None):
        assert lib.rope3d_qk_norm_rope_append_sp(p, p, p, 1, 2, 128, 1, 0, 72, 0, 3, 4, 6, p, p,
                                                 1e-6, d, 144, 0, None, 0, None,
                                                 None) == rope3d.ROPE3D_EINVAL


@pytest.mark.parametrize("entry", ["rope3d_qk_norm_rope_append",
                                   "rope3d_qk_norm_rope_append_noalloc"])
def test_step_wrappers_check_tensors_before_any_call(entry):
    """Both step wrappers check shapes and dtypes before the C call (host logic only: the
    tensors here never reach the library)."""
    fn = getattr(rope3d, entry)
    extra = {"tables": None} if entry == "rope3d_qk_norm_rope_append" else {}
    q = torch.zeros((1, 4, 2, 128), dtype=torch.bfloat16)
    kc = torch.zeros((1, 8, 2, 128), dtype=torch.bfloat16)
    wq = torch.ones(256)
    args = dict(frame_offset=0, T=1, H=2, W=4, q_norm_w=wq, k_norm_w=wq, eps=1e-6, slot=0,
                **extra)
    with pytest.raises(ValueError, match="n_tok"):
        fn(q, q, q, q.clone(), token_begin=0, token_end=5, k_cache=kc, v_cache=kc.clone(), **args)
    with pytest.raises(TypeError, match="k_cache"):
        fn(q, q, q, q.clone(), token_begin=0, token_end=4, k_cache=kc.float(),
           v_cache=kc.float(), **args)
    with pytest.raises(ValueError, match="cache shape"):
        fn(q, q, q, q.clone(), token_begin=0, token_end=4, k_cache=kc[:, :, :1].contiguous(),
           v_cache=kc[:, :, :1].contiguous(), **args)
    with pytest.raises(ValueError, match="float32"):
        fn(q, q, q, q.clone(), token_begin=0, token_end=4, k_cache=kc, v_cache=kc.clone(),
           **dict(args, q_norm_w=wq[:8]))
    with pytest.raises(ValueError, match="all be"):
        fn(q, q[:, :3], q, q.clone(), token_begin=0, token_end=4, k_cache=kc, v_cache=kc.clone(),
           **args)


def test_fast_divide_matches_integer_division(lib):
    """The multiply-and-shift division the kernels' 32-bit decode uses, on the host: exact
    floor(n / d) for every dividend below 2^31, at random and at the edges (powers of two
    and their neighbours, the grid sizes of the workloads, n = q d - 1, q d, q d + 1)."""
    import numpy as np
    rng = np.random.default_rng(11)
    top = (1 << 31) - 1
    divisors = {1, 2, 3, 5, 7, 52, 80, 1560, 3600, 4680, 10800, 32760, 75600, top, top - 1}
    divisors |= {(1 << k) + e for k in range(1, 31) for e in (-1, 0, 1)}
    divisors |= set(int(x) for x in rng.integers(1, top, 300))
    for d in sorted(x for x in divisors if 1 <= x <= top):
        ns = {0, 1, d - 1, d, d + 1, top, top - 1, top - d}
        for q in (1, 2, 3, top // d, top // d - 1):
            ns |= {q * d - 1, q * d, q * d + 1}
        ns |= set(int(x) for x in rng.integers(0, top + 1, 40))
        for n in ns:
            if 0 <= n <= top:
                assert lib.rope3d_testing_fast_divide(n, d) == n // d, (n, d)
    assert lib.rope3d_testing_fast_divide(5, 0) == 0xFFFFFFFF
    assert lib.rope3d_testing_fast_divide(1 << 31, 3) == 0xFFFFFFFF


def test_projection_rejects_a_tile_count_over_int_range(lib):
    """M = 2^30 token rows against 3 N D = 3 * 43690 * 128 output columns passes the per-size
    limits but is 2^23 x 65535 output tiles: ERANGE before any device work."""
    p = 0x100000
    rc = lib.rope3d_qkv_project(p, p, None, 1 << 30, 64, 43690, 128, p, p, p, None)
    assert rc == rope3d.ROPE3D_ERANGE
    assert "tiles" in lib.rope3d_last_error().decode()
