"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a private copy of oracle/oracle.c (a dropped
term, a wrong sign or index, a transposed operand), builds it on the CPU, and
runs the pin tests against it: every mutant must make at least one pin fail.
"""
import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")
PINS = ["tests/test_oracle_bf16.py", "tests/test_oracle_qk.py", "tests/test_oracle_adaln.py",
        "tests/test_oracle_residual_swiglu.py", "tests/test_oracle_packing.py", "tests/test_oracle_fused.py",
        "tests/test_oracle_frames.py", "tests/test_oracle_rope_modes.py",
        "tests/test_oracle_modulation_f32.py", "tests/test_oracle_av_modulation.py",
        "tests/test_oracle_shard.py"]

# (name, original text, planted mistake)
MUTANTS = [
    ("rope_sign", "y0 * c - y1 * s", "y0 * c + y1 * s"),
    ("rope_interleaved_read_as_half_split",
     "int i0 = rope_mode == ORACLE_ROPE_HALF ? j : 2 * j;\n        int i1 = rope_mode == ORACLE_ROPE_HALF ? j + D / 2 : 2 * j + 1;",
     "int i0 = j;\n        int i1 = j + D / 2;"),
    ("rope_half_wrong_partner", "int i1 = rope_mode == ORACLE_ROPE_HALF ? j + D / 2 : 2 * j + 1;",
     "int i1 = rope_mode == ORACLE_ROPE_HALF ? D - 1 - j : 2 * j + 1;"),
    ("rope_none_drops_weight", "put(out_bits, out_f64, i, y[i]);", "put(out_bits, out_f64, i, ld(&x[i]) * inv_rms);"),
    ("rms_eps_dropped", "sqrt(ms + eps)", "sqrt(ms)"),
    ("rms_mean_not_divided", "ms /= (double)D;", ""),
    ("rms_weight_dropped", "y[i] = ld(&x[i]) * inv_rms * ld(&w[i]);", "y[i] = ld(&x[i]) * inv_rms;"),
    ("rope_3d_freq_whole_head", "(double)jl / (double)sec[s]", "(double)jl / (double)head_dim"),
    ("rope_3d_h_index", "pos3[1] = (g / W) % H;", "pos3[1] = (g / H) % W;"),
    ("rope_tail_position", "pos1 = g - thw;", "pos1 = g;"),
    ("rope_k_uses_q_weight", "rmsnorm_rope_head(k + off, k_weight,", "rmsnorm_rope_head(k + off, q_weight,"),
    ("adaln_scale_without_one", "xhat * (1.0 + ldm(scale, mb + c, mod_f32))", "xhat * ldm(scale, mb + c, mod_f32)"),
    ("adaln_unbiased_variance", "var /= (double)hidden;", "var /= (double)(hidden - 1);"),
    ("adaln_shift_scale_swapped", "xhat * (1.0 + ldm(scale, mb + c, mod_f32)) + ldm(shift, mb + c, mod_f32)",
     "xhat * (1.0 + ldm(shift, mb + c, mod_f32)) + ldm(scale, mb + c, mod_f32)"),
    ("gate_dropped", "ldm(gate, gb + c, gate_f32) * ld(&y[row * y_row_stride + c])",
     "ld(&y[row * y_row_stride + c])"),
    ("fused_gate_dropped", "ldm(gate, gb + c, mod_f32) * ld(&y[row * y_row_stride + c])",
     "ld(&y[row * y_row_stride + c])"),
    ("vectors_not_per_sequence", "int64_t off = (int64_t)b * seq_stride;", "int64_t off = 0;"),
    ("audio_split_off_by_one", "if (g >= thw)\n            off += audio_offset;", "if (g > thw)\n            off += audio_offset;"),
    ("audio_vectors_ignored", "off += audio_offset;", "off += 0;"),
    ("rope_position_offset_ignored", "const int64_t g = r + (pos_offset ? pos_offset[b] : 0);",
     "const int64_t g = r;"),
    ("stream_split_offset_ignored", "int64_t g = r + (pos_offset ? pos_offset[b] : 0); /* index in the whole sequence */",
     "int64_t g = r;"),
    ("silu_sign", "exp(-av)", "exp(av)"),
    ("swiglu_operands_transposed", "double silu = av / (1.0 + exp(-av));\n            put(out, out_f64, row * out_row_stride + c, silu * bv);",
     "double silu = bv / (1.0 + exp(-bv));\n            put(out, out_f64, row * out_row_stride + c, silu * av);"),
    ("bf16_truncates", "nearbyint(ax / spacing)", "floor(ax / spacing)"),
    ("padding_row_read", "if (r < len) {", "if (r <= len) {"),
    ("fused_mean_over_x_not_residual", "mean += ld(&rr[c]);", "mean += ld(&x[row * x_row_stride + c]);"),
    ("fused_residual_not_rounded_before_norm",
     "double xhat = (ld(&rr[c]) - mean) * inv_std;",
     "double xhat = (ld(&x[row * x_row_stride + c]) + ldm(gate, gb + c, mod_f32) * ld(&y[row * y_row_stride + c]) - mean) * inv_std;"),
    ("fp32_modulation_read_as_bf16", "return (double)((const float*)base)[idx];",
     "return oracle_bf16_to_f64(((const uint16_t*)base)[idx]);"),
    ("frames_truncates", "return (uint8_t)nearbyintf(u);", "return (uint8_t)u;"),
    ("frames_no_clamp_top", "if (u >= 255.0f)\n        return 255;", ""),
    ("frames_wrong_layout", "? (((b * frames + t) * height + h) * width + w) * channels + c",
     "? (((b * frames + t) * width + w) * height + h) * channels + c"),
    ("rows_located_by_valid_offsets", "if (row >= cu_seqlens_padded[b] && row < cu_seqlens_padded[b + 1]) {",
     "if (row >= cu_seqlens[b] && row < cu_seqlens[b + 1]) {"),
]


def _run_mutant(name, old, new, workdir):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"{name}: pattern not found in oracle.c"
    d = os.path.join(workdir, name)
    os.makedirs(d)
    shutil.copy(os.path.join(ROOT, "oracle", "oracle.h"), d)
    with open(os.path.join(d, "oracle.c"), "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(d, "liboracle.so")
    subprocess.check_call(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
                           "-o", lib, os.path.join(d, "oracle.c"), "-lm"])
    env = dict(os.environ, DIT_ORACLE_LIB=lib, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PINS],
                       cwd=ROOT, env=env, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True,
                       timeout=600)
    return name, r.returncode, r.stdout[-400:]


def test_every_planted_mistake_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(max(1, min(8, os.cpu_count() or 1))) as ex:
            results = list(ex.map(lambda m: _run_mutant(*m, tmp), MUTANTS))
    survivors = [(n, out) for n, rc, out in results if rc == 0]
    assert not survivors, f"mutants not caught by any pin: {survivors}"
    # a clean copy must pass (the harness itself is sound)
    with tempfile.TemporaryDirectory() as tmp:
        name, rc, out = _run_mutant("clean", "int oracle_num_threads(void)", "int oracle_num_threads(void)", tmp)
    assert rc == 0, out
