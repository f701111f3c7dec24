"""Mutation check of the oracle's pins (CPU only).

The oracle is trusted because ``tests/test_oracle_*.py`` pin it to things
other than itself.  This file checks that those pins have teeth: each case
below plants one plausible mistake (a dropped term, a wrong sign, bias or
index, a swapped operand, a changed tie or comparison rule) in a temporary
copy of ``oracle/`` and runs the pin files against that copy in a child
process.  Every mutant must make at least one pin fail; the unmodified copy
must pass.  The real ``oracle/`` is never modified.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_FILES = ["test_oracle_formats.py", "test_oracle_quant.py",
             "test_oracle_route_gemm.py", "test_oracle_tdc_decomp.py"]

Q = "qlinear_oracle.py"
T = "tdc_oracle.py"

# (name, file, exact text in the oracle, replacement).  Each text must occur
# exactly once, so a mutant can never silently stop applying.
MUTANTS = [
    # number formats
    ("e2m1_subnormal_value", Q, "vals.append(m * 0.5)", "vals.append(m * 0.25)"),
    ("e2m1_exponent_bias", Q, "vals.append((1.0 + m / 2.0) * 2.0 ** (e - 1))",
     "vals.append((1.0 + m / 2.0) * 2.0 ** e)"),
    ("e4m3_exponent_bias", Q, "vals.append((1.0 + m / 8.0) * 2.0 ** (e - 7))",
     "vals.append((1.0 + m / 8.0) * 2.0 ** (e - 8))"),
    ("e4m3_subnormal_scale", Q, "vals.append(m / 8.0 * 2.0 ** -6)", "vals.append(m / 8.0 * 2.0 ** -7)"),
    ("ties_to_odd", Q, "((d_hi == d_lo) & (hi % 2 == 0))", "((d_hi == d_lo) & (hi % 2 == 1))"),
    ("ties_upward", Q, "pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))",
     "pick_hi = d_hi <= d_lo"),
    ("e2m1_sign_bit", Q, "(mag_code | (sign << 3))", "(mag_code | (sign << 2))"),
    ("e2m1_decode_sign_ignored", Q, "return np.where(code & 8, -mag, mag)", "return mag"),
    ("nibble_order", Q, "(codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)",
     "(codes[:, 1::2] & 0xF) | ((codes[:, 0::2] & 0xF) << 4)"),
    # Hadamard
    ("hadamard_negated", Q, "np.where(pop % 2 == 0, 1, -1)", "np.where(pop % 2 == 1, 1, -1)"),
    ("butterfly_sign", Q, "v[:, :, :, 1, :] = a - b", "v[:, :, :, 1, :] = b - a"),
    ("butterfly_last_stage_dropped", Q, "while s < HADAMARD_N:", "while s < HADAMARD_N // 2:"),
    # NVFP4
    ("tensor_scale_drops_e2m1_max", Q, "np.float32(a_t / np.float32(E2M1_MAX * E4M3_MAX))",
     "np.float32(a_t / np.float32(E4M3_MAX))"),
    ("tensor_amax_signed", Q, "a_t = np.float32(np.max(np.abs(h)))", "a_t = np.float32(np.max(h))"),
    ("block_amax_signed", Q, "a_b = np.max(np.abs(blocks), axis=2)", "a_b = np.max(blocks, axis=2)"),
    ("block_scale_drops_six", Q, "d = np.float32(np.float32(E2M1_MAX) * g)", "d = np.float32(g)"),
    ("codes_use_unrounded_scale", Q, "denom = (e4m3_decode(sb) * g).astype(np.float32)",
     "denom = (sf * g).astype(np.float32)"),
    ("zero_block_keeps_sign", Q, "    q[~nz] = 0 ", "    pass "),
    ("dequant_drops_block_scale", Q, "return (vals * scales[:, :, None]).reshape(rows, k)",
     "return vals.reshape(rows, k)"),
    # activation decomposition
    ("residual_sign", Q, "r = (h - nvfp4_values(p1, s1, g)).astype(np.float32)",
     "r = (nvfp4_values(p1, s1, g) - h).astype(np.float32)"),
    ("residual_own_tensor_scale", Q, "p2, s2, _ = nvfp4_quantize(r, g)", "p2, s2, _ = nvfp4_quantize(r)"),
    ("values_drop_tensor_scale", Q, "s = (e4m3_decode(sb) * np.float32(g)).astype(np.float32)",
     "s = e4m3_decode(sb).astype(np.float32)"),
    # integer activations
    ("int_scale_off_by_one", Q, "(amax / np.float32(qmax)).astype(np.float32), np.float32(0))",
     "(amax / np.float32(qmax + 1)).astype(np.float32), np.float32(0))"),
    ("int_round_floor", Q, "q = np.clip(np.rint(y), -qmax, qmax)", "q = np.clip(np.floor(y), -qmax, qmax)"),
    ("int_round_half_away", Q, "q = np.clip(np.rint(y), -qmax, qmax)",
     "q = np.clip(np.trunc(y + np.copysign(np.float32(0.5), y)), -qmax, qmax)"),
    ("int_clamp_narrow", Q, "q = np.clip(np.rint(y), -qmax, qmax)", "q = np.clip(np.rint(y), -qmax + 1, qmax - 1)"),
    ("token_amax_signed", Q, "amax = np.max(np.abs(h), axis=1) if h.shape[1]",
     "amax = np.max(h, axis=1) if h.shape[1]"),
    ("int6_range", Q, "INT6_QMAX = 31", "INT6_QMAX = 32"),
    # router
    ("gamma_normalised_by_output", Q, "s0 = float(np.sum(np.abs(x).astype(np.float64)))",
     "s0 = float(np.sum(np.abs(y).astype(np.float64)))"),
    ("gamma_signed_sum", Q, "s1 = float(np.sum(np.abs(d).astype(np.float64)))",
     "s1 = abs(float(np.sum(d.astype(np.float64))))"),
    ("route_not_strict", Q, "return ROUTE_INT8 if gamma > threshold else ROUTE_NVFP4",
     "return ROUTE_INT8 if gamma >= threshold else ROUTE_NVFP4"),
    # Q-ARVD
    ("median_even_upper", Q, "return float((s[n // 2 - 1] + s[n // 2]) / 2.0)", "return float(s[n // 2])"),
    ("mad_signed", Q, "mad = median_sorted(np.abs(v - med))", "mad = median_sorted(v - med)"),
    ("zscore_sign", Q, "m = (v - med) / mad", "m = (med - v) / mad"),
    ("alpha_condition_dropped", Q, "mask = (m > tau) & (v > alpha * med)", "mask = m > tau"),
    ("norms_l1", Q, "return np.sqrt(np.sum(w * w, axis=0))", "return np.sum(np.abs(w), axis=0)"),
    ("norms_over_output_channels", Q, "return np.sqrt(np.sum(w * w, axis=0))", "return np.sqrt(np.sum(w * w, axis=1))"),
    ("outliers_first", Q, "perm = np.concatenate([normal, outl])", "perm = np.concatenate([outl, normal])"),
    ("class_padding_16", Q, "QARVD_K_ALIGN = 32 ", "QARVD_K_ALIGN = 16 "),
    ("int4_range", Q, "INT4_QMAX = 7", "INT4_QMAX = 8"),
    # GEMMs
    ("w4a4_rotation_scale_dropped", Q, "np.float64(g_x) * np.float64(g_w) / HADAMARD_N)",
     "np.float64(g_x) * np.float64(g_w))"),
    ("w4a4_weight_scale_dropped", Q, "np.float64(g_x) * np.float64(g_w) / HADAMARD_N)",
     "np.float64(g_x) / HADAMARD_N)"),
    ("w4a8_weight_scale_dropped", Q, "(s[:, None] * np.float64(g_w) / c)", "(s[:, None] / c)"),
    ("w4a8_rotation_always", Q, "c = HADAMARD_N if hadamard else 1", "c = HADAMARD_N"),
    ("qarvd_class_scales_swapped", Q, "acc_n.astype(np.float64) * np.asarray(s_norm, np.float64)",
     "acc_n.astype(np.float64) * np.asarray(s_out, np.float64)"),
    ("bf16_product_transposed_weight", Q, "return x @ bf16_bits_to_f32(w_bits).astype(np.float64).T",
     "return x @ bf16_bits_to_f32(w_bits).astype(np.float64).T[::-1]"),
    # temporal delta cache and PDR
    ("bf16_round_half_up", T, "rounded = (b + 0x7FFF + ((b >> 16) & 1)) >> 16", "rounded = (b + 0x8000) >> 16"),
    ("delta_reversed", T, "d = (bf16_bits_to_f32(out_bits) - bf16_bits_to_f32(inp_bits))",
     "d = (bf16_bits_to_f32(inp_bits) - bf16_bits_to_f32(out_bits))"),
    ("skip_output_subtracts", T, "y = (bf16_bits_to_f32(inp_bits) + bf16_bits_to_f32(delta_bits))",
     "y = (bf16_bits_to_f32(inp_bits) - bf16_bits_to_f32(delta_bits))"),
    ("delta_error_normalised_by_new", T, "return dmpq_gamma(old_bits, new_bits)", "return dmpq_gamma(new_bits, old_bits)"),
    ("skip_ignores_accumulated_error", T, "st.acc + st.eps <= prm.acc_max", "st.acc <= prm.acc_max"),
    ("skip_count_off_by_one", T, "and st.skips < prm.max_skips)", "and st.skips <= prm.max_skips)"),
    ("skip_no_error_threshold", T, "st.eps < prm.eps_threshold and", "True and"),
    ("skip_error_threshold_not_strict", T, "st.eps < prm.eps_threshold and", "st.eps <= prm.eps_threshold and"),
    ("no_forced_int8_after_skip", T, "    if st.last_skipped:\n        return ROUTE_INT8",
     "    if st.last_skipped:\n        return ROUTE_NVFP4"),
    ("forced_int8_before_bf16", T,
     "    if st.rho > prm.rho_max:\n        return ROUTE_BF16\n    if st.last_skipped:\n        return ROUTE_INT8",
     "    if st.last_skipped:\n        return ROUTE_INT8\n    if st.rho > prm.rho_max:\n        return ROUTE_BF16"),
    ("compute_keeps_skip_error", T, "    st.acc = 0.0\n    st.skips = 0", "    st.skips = 0"),
    ("skip_error_not_accumulated", T, "    st.acc += st.eps\n", ""),
    ("delta_error_against_oldest", T, "tdc_delta_error(d, st.deltas[-1])", "tdc_delta_error(d, st.deltas[0])"),
    ("outlier_count_sixteen", T, "flagged = (a * np.float32(15))", "flagged = (a * np.float32(16))"),
    ("outlier_rest_includes_max", T, "others = (s - a).astype(np.float32)", "others = s"),
    ("outlier_ratio_not_strict", T, "(a * np.float32(15)).astype(np.float32) > (", "(a * np.float32(15)).astype(np.float32) >= ("),
]

_CHILD = r"""
import os, sys
root, copy, needle, fname = sys.argv[1], sys.argv[2], sys.argv[3], sys.argv[4]
sys.path.insert(0, copy)
import oracle, oracle.qlinear_oracle, oracle.tdc_oracle
assert os.path.dirname(oracle.__file__) == os.path.join(copy, "oracle"), oracle.__file__
if needle:
    with open(os.path.join(copy, "oracle", fname)) as f:
        assert needle in f.read()
import pytest
files = [os.path.join(root, "tests", n) for n in %r]
sys.exit(pytest.main(["-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu", *files]))
""" % (PIN_FILES,)


def _mutate(dst, fname, old, new):
    path = os.path.join(dst, "oracle", fname)
    with open(path) as f:
        src = f.read()
    assert src.count(old) == 1, f"{fname}: mutation site found {src.count(old)} times: {old!r}"
    with open(path, "w") as f:
        f.write(src.replace(old, new))


def _run(copy, needle="", fname=""):
    env = dict(os.environ, PYTHONDONTWRITEBYTECODE="1", OMP_NUM_THREADS="1", MKL_NUM_THREADS="1",
               OPENBLAS_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-c", _CHILD, ROOT, copy, needle, fname],
                       cwd=copy, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-2000:] + r.stderr[-2000:]


def _copy_oracle(base, name):
    dst = os.path.join(base, name)
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(dst, "oracle"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    return dst


def test_unmodified_copy_passes(tmp_path):
    rc, out = _run(_copy_oracle(str(tmp_path), "control"))
    assert rc == 0, out


def test_every_mutant_fails_a_pin(tmp_path):
    names = [m[0] for m in MUTANTS]
    assert len(set(names)) == len(names)
    jobs = []
    for name, fname, old, new in MUTANTS:
        dst = _copy_oracle(str(tmp_path), name)
        _mutate(dst, fname, old, new)
        jobs.append((name, dst, new, fname))
    workers = max(1, min(8, (os.cpu_count() or 2) - 1))
    with ThreadPoolExecutor(workers) as ex:
        results = list(ex.map(lambda j: (j[0], *_run(j[1], j[2], j[3])), jobs))
    survived = [(n, out) for n, rc, out in results if rc == 0]
    broken = [(n, rc, out) for n, rc, out in results if rc not in (0, 1)]
    assert not broken, "child runs that neither passed nor failed a test:\n" + \
        "\n".join(f"{n}: rc={rc}\n{out}" for n, rc, out in broken)
    assert not survived, "mutants no pin caught: " + ", ".join(n for n, _ in survived)
