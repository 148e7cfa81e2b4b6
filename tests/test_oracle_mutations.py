"""The pins must catch plausible mistakes planted in the oracle (CPU only).

Each mutant is a copy of oracle/lk_oracle.py with one textual change (a
reciprocal instead of a true division, ties away from zero, a transposed
factor, a dropped scale or residual, swapped nibbles, a wrong int4 divisor
or group index, a reversed scale vector, ...).  The copy, the pin tests and
their golden files are written to a temporary directory; the pins run
against the copy in a subprocess and must fail.  The unchanged copy must
pass.  Nothing here touches the real oracle file.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
 "recip_mul": ("ratio = _fl32_div(v, safe[..., None])\n    codes = np.clip(np.rint(ratio), -127, 127)",
               "ratio = (v * (np.float32(1.0) / safe[..., None])).astype(np.float32)\n    codes = np.clip(np.rint(ratio), -127, 127)"),
 "ties_away": ("codes = np.clip(np.rint(ratio), -127, 127)", "codes = np.clip(np.sign(ratio)*np.floor(np.abs(ratio)+0.5), -127, 127)"),
 "bk_transpose": ("K = np.asarray(Ck_hat, np.float64) @ np.asarray(B_K, np.float64)   # [T, H]",
                  "K = np.asarray(Ck_hat, np.float64) @ np.asarray(B_K, np.float64).T   # [T, H]"),
 "no_scale": ("s = (K @ np.asarray(q, np.float64)) * float(softmax_scale)", "s = (K @ np.asarray(q, np.float64))"),
 "scale_swap": ("* np.asarray(s_D, np.float16).astype(np.float64)[None, :])", "* np.asarray(s_V if s_V is not None else s_D, np.float16).astype(np.float64)[None, :])"),
 "nibble_swap": ("return (lo | (hi << 4)).astype(np.uint8)", "return (hi | (lo << 4)).astype(np.uint8)"),
 "i4_div8": ("s32 = _fl32_div(absmax, np.float32(7.0))", "s32 = _fl32_div(absmax, np.float32(8.0))"),
 "no_requant_sU": ("* np.asarray(s_U, np.float16).astype(np.float32)[None, :]).astype(np.float32)\n    return quantize_rows_i8(t)",
                   "* 1.0).astype(np.float32)\n    return quantize_rows_i8(t)"),
 "rms_eps_out": ("np.mean(x * x, axis=-1, keepdims=True) + eps)", "np.mean(x * x, axis=-1, keepdims=True)) + eps"),
 "drop_residual": ("    if residual is not None:\n        y += np.asarray(residual, np.float64)", "    pass"),
 "v_not_BV": ("V = np.asarray(Cv_hat, np.float64) @ np.asarray(B_V, np.float64)   # [T, H]", "V = np.asarray(Cv_hat, np.float64) @ np.asarray(B_K, np.float64)   # [T, H]"),
 "svd_no_sigma": ("return U[:, :r] * sig[None, :r], Vt[:r, :]", "return U[:, :r], Vt[:r, :]"),
 "w8a8_sa_order": ("* np.asarray(a_scale, np.float16).astype(np.float32)[None, :]).astype(np.float32)\n    return v", "* np.asarray(a_scale, np.float16).astype(np.float32)[::-1][None, :]).astype(np.float32)\n    return v"),
 "i4_group_index": ("idx = np.arange(r) // group", "idx = np.arange(r) % (-(-r // group))"),
 "layer_swiglu_swap": ("act = swiglu(gate, upv).astype(np.float32)", "act = swiglu(upv, gate).astype(np.float32)"),
 "layer_ffn_fed_h1": ("h2 = rmsnorm(x2, eps).astype(np.float32)", "h2 = h1"),
 "layer_attn_quant_before_store": (
     "attn = round_bf16(attn.reshape(Bsz, n_h * H))\n    aq, sa = quantize_rows_i8(attn.astype(np.float32))",
     "aq, sa = quantize_rows_i8(attn.reshape(Bsz, n_h * H).astype(np.float32))\n"
     "    attn = round_bf16(attn.reshape(Bsz, n_h * H))"),
 "layer_no_attn_residual": ("layer[\"s_O\"], residual=x))", "layer[\"s_O\"], residual=None))"),
 "layer_ffn_residual_x": ("d[\"s_V\"], residual=x2)", "d[\"s_V\"], residual=x)"),
 "hadamard_unnormalised": ("    return h / math.sqrt(n)", "    return h"),
 "rotation_block_cap_32": ("    while r % (2 * n) == 0 and 2 * n <= 64:", "    while r % (2 * n) == 0 and 2 * n <= 32:"),
 "rotate_latents_skips_head": ("        out[..., off:off + r] = v[..., off:off + r] @ latent_rotation(r)",
                               "        out[..., off:off + r] = v[..., off:off + r] @ latent_rotation(r) if off else v[..., :r]"),
 "rope_interleaved_pairs": ("    x1, x2 = x[:, :h], x[:, h:]\n    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=1)",
                            "    x1, x2 = x[:, 0::2], x[:, 1::2]\n    return np.stack([x1 * c - x2 * s, x2 * c + x1 * s], axis=2).reshape(x.shape)"),
 "rope_sign": ("x2 * c + x1 * s], axis=1)", "x2 * c - x1 * s], axis=1)"),
 "rope_freq_exponent": ("theta = float(base) ** (-2.0 * i / H)", "theta = float(base) ** (-1.0 * i / H)"),
 "rope_query_unrotated": ("    q_rot = rope(np.asarray(q, np.float64)[None, :], [q_pos], base)[0]",
                          "    q_rot = np.asarray(q, np.float64)"),
 "rope_query_at_len": ("softmax_scale, T - 1, base)", "softmax_scale, T, base)"),
 "outsplit_lr_scaled_by_sx": ("        y[:, np.asarray(lr_out)] = (acc_V.astype(np.float64) * s_t.astype(np.float64)[:, None]",
                              "        y[:, np.asarray(lr_out)] = (acc_V.astype(np.float64) * sx.astype(np.float64)[:, None]"),
 "outsplit_dense_inputs_reversed": ("        acc_D = x @ np.asarray(W_D, np.int64)", "        acc_D = x[:, ::-1] @ np.asarray(W_D, np.int64)"),
 "ffn_gate_up_swapped": ("    return swiglu(g, u)", "    return swiglu(u, g)"),
 "layer_q_from_x": ("q = round_bf16(_linear_dense_w8a8(xq, sx, layer[\"W_Q\"], layer[\"s_Q\"]))",
                    "q = round_bf16(_linear_dense_w8a8(*quantize_rows_i8(x.astype(np.float32)), layer[\"W_Q\"], layer[\"s_Q\"]))"),
}


def _run_pins(tmp_root, name, change):
    d = os.path.join(tmp_root, name)
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(d, "oracle"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    os.makedirs(os.path.join(d, "tests"))
    shutil.copy(os.path.join(ROOT, "tests", "test_oracle_pins.py"), os.path.join(d, "tests"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(d, "tests", "golden"))
    if change is not None:
        path = os.path.join(d, "oracle", "lk_oracle.py")
        with open(path) as f:
            text = f.read()
        old, new = change
        assert text.count(old) == 1, f"mutant {name}: anchor not found once"
        with open(path, "w") as f:
            f.write(text.replace(old, new))
    env = dict(os.environ, PYTHONPATH=d, PYTHONDONTWRITEBYTECODE="1")
    p = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(d, "tests", "test_oracle_pins.py")],
                       cwd=d, env=env, capture_output=True, text=True, timeout=600)
    return p.returncode


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    tmp_root = str(tmp_path_factory.mktemp("oracle_mutants"))
    jobs = [("unchanged", None)] + sorted(MUTANTS.items())
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        codes = list(ex.map(lambda job: _run_pins(tmp_root, *job), jobs))
    return dict(zip([j[0] for j in jobs], codes))


def test_unchanged_copy_passes(outcomes):
    assert outcomes["unchanged"] == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(outcomes, name):
    assert outcomes[name] != 0, f"no pin fails when the oracle has the mistake '{name}'"
