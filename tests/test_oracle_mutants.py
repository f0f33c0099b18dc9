"""Plant plausible mistakes in a copy of the oracle's C source and require that the pins
catch every one: a dropped term, a wrong sign, a swapped or transposed operand, an
off-by-one.  The mistakes are planted on the CPU only, in a temporary build."""
import os
import shutil

import pytest

import oracle
from oracle_pins import ALL_CHECKS

MUTANTS = {
    "e2m1_ties_to_odd": ("            else best = (c % 2 == 0) ? c : c + 1;  /* tie: even mantissa */\n"
                         "            break;\n        }\n    }\n    return sign | best;\n}\n\n/* One block",
                         "            else best = (c % 2 == 0) ? c + 1 : c;\n"
                         "            break;\n        }\n    }\n    return sign | best;\n}\n\n/* One block"),
    "e2m1_no_saturation": ("if (a >= 6.0) return sign | 0x7;", "if (a >= 8.0) return sign | 0x7;"),
    "nvfp4_scale_over_4": ("float k = 1.0f / (6.0f * g);", "float k = 1.0f / (4.0f * g);"),
    "nvfp4_nibbles_swapped": ("codes[e / 2] = (unsigned char)(rope3d_oracle_e2m1_encode(lo) |\n"
                              "                                       (rope3d_oracle_e2m1_encode(hi) << 4));",
                              "codes[e / 2] = (unsigned char)(rope3d_oracle_e2m1_encode(hi) |\n"
                              "                                       (rope3d_oracle_e2m1_encode(lo) << 4));"),
    "nvfp4_one_scale_per_head": ("int64_t scale_off = head_off * (D / 16) + blk;",
                                 "int64_t scale_off = head_off * (D / 16);"),
    "nvfp4_v_uses_k_global": ("rope3d_oracle_quantize_block_nvfp4(head, 16, v_global, v_codes + code_off,",
                              "rope3d_oracle_quantize_block_nvfp4(head, 16, k_global, v_codes + code_off,"),
    "nvfp4_reciprocal_ignores_global": ("float r = sv > 0.0f ? 1.0f / (sv * g) : 0.0f;",
                                        "float r = sv > 0.0f ? 1.0f / sv : 0.0f;"),
    "rotate_real_sign": ("y[n * head_dim + 2 * j] = a * c - b * s;",
                         "y[n * head_dim + 2 * j] = a * c + b * s;"),
    "rotate_imag_transposed": ("y[n * head_dim + 2 * j + 1] = a * s + b * c;",
                               "y[n * head_dim + 2 * j + 1] = b * s + a * c;"),
    "pair_layout_rotate_half": ("double a = x[n * head_dim + 2 * j];     /* real part */",
                                "double a = x[n * head_dim + j];"),
    "axis_subdim_off_by_one": ("double d_a = 2.0 * n_axis[a];",
                               "double d_a = 2.0 * n_axis[a] + 2.0;"),
    "single_schedule_wrong_offset": ("exponent = (2.0 * (first + j)) / d;",
                                     "exponent = (2.0 * j) / d;"),
    "decode_drops_start_frame": ("*t_g = s + i / hw;", "*t_g = i / hw;"),
    "decode_h_w_swapped": ("*h = (i / W) % H;", "*h = (i / H) % W;"),
    "angle_h_uses_w": ("phi[n_t + j] = (double)h * inv[n_t + j];",
                       "phi[n_t + j] = (double)w * inv[n_t + j];"),
    "rms_mean_wrong_count": ("double mean_sq = sum_sq / (double)dim;",
                             "double mean_sq = sum_sq / (double)(dim - 1);"),
    "rms_drops_eps": ("double inv_rms = 1.0 / sqrt(mean_sq + eps);",
                      "double inv_rms = 1.0 / sqrt(mean_sq);"),
    "rms_drops_weight": ("y[e] = x[e] * inv_rms * weight[e];", "y[e] = x[e] * inv_rms;"),
    "k_uses_q_weights": ("rope3d_oracle_rms_norm(k, k_norm_w, dim, eps, k_row);",
                         "rope3d_oracle_rms_norm(k, q_norm_w, dim, eps, k_row);"),
    "rotate_before_norm": (
        "    rope3d_oracle_rms_norm(q, q_norm_w, dim, eps, q_out);\n"
        "    rope3d_oracle_rotate(q_out, N, D, phi, q_out);",
        "    rope3d_oracle_rotate(q, N, D, phi, q_out);\n"
        "    rope3d_oracle_rms_norm(q_out, q_norm_w, dim, eps, q_out);"),
    "v_copies_k": ("memcpy(v_row, v, (size_t)dim * sizeof(double));",
                   "memcpy(v_row, k, (size_t)dim * sizeof(double));"),
    "cache_row_ignores_slot": ("return (slot + i) % cache_tokens;", "return i % cache_tokens;"),
    "cache_offset_wrong_stride": ("int64_t cache_off = (b * cache_tokens + row) * dim;",
                                  "int64_t cache_off = (b * n_tok + row) * dim;"),
    "step_index_ignores_begin": ("int64_t i = token_begin + r;", "int64_t i = r;"),
    "half_pairs_reversed": ("double b = x[n * head_dim + pairs + j];  /* imaginary part: second half */",
                            "double b = x[n * head_dim + 2 * pairs - 1 - j];"),
    "half_real_sign": ("y[n * head_dim + j] = a * c - b * s;",
                       "y[n * head_dim + j] = a * c + b * s;"),
    "half_k_not_rotated_half": ("rope3d_oracle_rotate_pairing(k_row, N, D, phi, pairing, k_row);",
                                "rope3d_oracle_rotate(k_row, N, D, phi, k_row);"),
    "head_major_offset_is_token_major": (": ((b * N + n) * cache_tokens + row) * D;",
                                         ": ((b * cache_tokens + row) * N + n) * D;"),
    # the same mistakes made only in the layout-variant functions (second occurrence)
    "k_uses_q_weights_in_pairing_token": ("rope3d_oracle_rms_norm(k, k_norm_w, dim, eps, k_row);",
                                          "rope3d_oracle_rms_norm(k, q_norm_w, dim, eps, k_row);",
                                          1),
    "v_copies_k_in_pairing_token": ("memcpy(v_row, v, (size_t)dim * sizeof(double));",
                                    "memcpy(v_row, k, (size_t)dim * sizeof(double));", 1),
    "layout_step_ignores_begin": ("int64_t i = token_begin + r;", "int64_t i = r;", 1),
    "layout_step_row_ignores_slot": ("int64_t row = rope3d_oracle_cache_row(i, slot, cache_tokens);",
                                     "int64_t row = rope3d_oracle_cache_row(i, 0, cache_tokens);",
                                     1),
    # FP8 E4M3 quantizer
    "e4m3_ties_to_odd": ("else best = (c % 2 == 0) ? c : c + 1;  /* tie: even mantissa */",
                         "else best = (c % 2 == 0) ? c + 1 : c;"),
    "e4m3_bias_8": ("else v = ldexp(1.0 + (double)m / 8.0, e - 7);",
                    "else v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "e4m3_no_saturation": ("if (a >= 448.0) return sign | 0x7E;", "if (a >= 464.0) return sign | 0x7F;"),
    "fp8_scale_exponent_240": ("while ((double)amax > ldexp(448.0, e)) ++e;",
                               "while ((double)amax > ldexp(240.0, e)) ++e;"),
    "fp8_scale_exponent_strict": ("while ((double)amax > ldexp(448.0, e)) ++e;",
                                  "while ((double)amax >= ldexp(448.0, e)) ++e;"),
    "fp8_codes_unscaled_by_half": ("codes[e] = (unsigned char)rope3d_oracle_e4m3_encode(ldexpf(x[e], -ex));  /* exact */",
                                   "codes[e] = (unsigned char)rope3d_oracle_e4m3_encode(ldexpf(x[e], -ex - 1));"),
    "fp8_v_scale_from_k": ("rope3d_oracle_quantize_head_e4m3(head, D, v_codes + code_off, v_scale + scale_off);",
                           "rope3d_oracle_quantize_head_e4m3(head, D, v_codes + code_off, k_scale + scale_off);"),
}


def _build_mutant(tmp_path, name, old, new, occurrence=None):
    """Plant the mistake at every occurrence of `old`, or only at the given one (0-based)."""
    src = open(oracle.SOURCE).read()
    count = src.count(old)
    assert count >= 1, f"mutation site for {name} not found"
    if occurrence is None:
        mutated = src.replace(old, new)
    else:
        assert occurrence < count, f"{name}: only {count} occurrences"
        at = -1
        for _ in range(occurrence + 1):
            at = src.index(old, at + 1)
        mutated = src[:at] + new + src[at + len(old):]
    path = os.path.join(tmp_path, f"{name}.c")
    with open(path, "w") as f:
        f.write(mutated)
    return oracle.build(force=True, source=path, library=os.path.join(tmp_path, f"{name}.so"))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(tmp_path, name):
    old, new, *occurrence = MUTANTS[name]
    orc = oracle.Oracle(_build_mutant(str(tmp_path), name, old, new,
                                      occurrence[0] if occurrence else None))
    caught = []
    for check in ALL_CHECKS:
        try:
            check(orc)
        except AssertionError:
            caught.append(check.__name__)
        except Exception as e:  # a crash also counts as caught, but say which
            caught.append(f"{check.__name__} ({type(e).__name__})")
    assert caught, f"no pin catches the planted mistake {name}"


# Planted mistakes in the oracle's Python-level head scatter (the sequence-parallel step's
# all-to-all folded into stores): a copy of oracle/__init__.py with one line changed.
PY_MUTANTS = {
    "qkv_weight_not_transposed": ("y = x @ w.T", "y = x @ w.reshape(w.shape[::-1])"),
    "qkv_q_and_k_swapped": ("return y[..., :dim], y[..., dim:2 * dim], y[..., 2 * dim:]",
                            "return y[..., dim:2 * dim], y[..., :dim], y[..., 2 * dim:]"),
    "qkv_bias_dropped": ("            y = y + np.asarray(b_qkv, dtype=np.float64)",
                         "            y = y + 0.0"),
    "bf16_round_half_up": ("return np.ldexp(np.rint(np.ldexp(a, 8 - e)), e - 8)",
                           "return np.ldexp(np.floor(np.ldexp(a, 8 - e) + 0.5), e - 8)"),
    "sp_round_robin_owner": ("r, local = divmod(head, hl)", "r, local = head % P, head // P"),
    "sp_q_row_ignores_row0": ("q_dst[r][:, i - q_row0, local]", "q_dst[r][:, i, local]"),
    "sp_cache_rows_drop_slot": ("rows = (slot + i) % C", "rows = i % C"),
    "sp_out_heads_at_destination_offset": (
        "outs[dst][:, :, r * hl:(r + 1) * hl] = o_ranks[r][:, a:e]",
        "outs[dst][:, :, dst * hl:(dst + 1) * hl] = o_ranks[r][:, a:e]"),
    "sp_out_tokens_of_source_slice": ("a, e = cuts[dst], cuts[dst + 1]",
                                      "a, e = cuts[r], cuts[r + 1]"),
    "sp_head_major_as_token_major": (
        "                k_dst[r][:, local, rows] = kc[:, rows, head]",
        "                k_dst[r][:, rows, local] = kc[:, rows, head]"),
}


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_pins_catch_python_mutant(name):
    import types
    old, new = PY_MUTANTS[name]
    src = open(oracle.__file__).read()
    assert src.count(old) == 1, f"mutant site of {name} not found exactly once"
    mod = types.ModuleType(f"oracle_{name}")
    mod.__file__ = oracle.__file__
    exec(compile(src.replace(old, new), oracle.__file__, "exec"), mod.__dict__)
    orc = mod.Oracle()
    caught = []
    for check in ALL_CHECKS:
        try:
            check(orc)
        except AssertionError:
            caught.append(check.__name__)
        except Exception as e:
            caught.append(f"{check.__name__} ({type(e).__name__})")
    assert caught, f"no pin catches the planted mistake {name}"
