"""Plant plausible mistakes in copies of the oracle and check that the pins
catch every one of them (no GPU).

Each mutant replaces one exact snippet of oracle/attention_ref.c, is compiled
to a temporary shared library and is run against every pin in a child
process (so a copy that crashes also counts as caught).  A mutant that passes
every pin would mean the pins cannot tell that mistake from the oracle.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "attention_ref.c")
RUNNER = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_mutant_runner.py")

MUTANTS = {
    "causal_off_by_one": ("(!J->causal || j <= i + off)", "(!J->causal || j < i + off)"),
    "bottom_right_offset_off_by_one": ("(int64_t)len - J->Nq : 0", "(int64_t)len - J->Nq + 1 : 0"),
    "bottom_right_ignores_length": ("(int64_t)len - J->Nq : 0", "(int64_t)J->N - J->Nq : 0"),
    "padding_off_by_one": ("(j < len) &&", "(j <= len) &&"),
    "scale_dropped": ("Srow[j] = J->scale * acc;", "Srow[j] = acc;"),
    "gqa_interleaved": ("const int g = h / (J->Hq / J->Hkv);", "const int g = h % J->Hkv;"),
    "q_row_transposed": ("qbase + i * d + c", "qbase + (int64_t)c * N + i"),
    "v_operand_from_k": ("orow[c] += p * in_at(J->v,", "orow[c] += p * in_at(J->k,"),
    "max_not_subtracted_in_sum": ("denom += exp(Srow[j] - m);", "denom += exp(Srow[j]);"),
    "softmax_sign_flipped": ("Srow[j] = exp(Srow[j] - m) / denom;",
                             "Srow[j] = exp(m - Srow[j]) / denom;"),
    "lse_drops_max": ("= m + log(denom);", "= log(denom);"),
    "lse_log2": ("= m + log(denom);", "= m + log2(denom);"),
    "o_overwritten_not_accumulated": ("orow[c] += p *", "orow[c] = p *"),
    "head_batch_swapped": ("((int64_t)b * J->Hq + h) * J->Nq * d",
                           "((int64_t)h * J->B + b) * J->Nq * d"),
    "kv_head_dropped": ("((int64_t)b * J->Hkv + g) * N * d", "((int64_t)b * J->Hkv) * N * d"),
    "seqlen_of_batch_0": ("J->seqlens ? J->seqlens[b] : N", "J->seqlens ? J->seqlens[0] : N"),
    "bwd_missing_row_term": ("const double ds = p * (dP[j] - D);", "const double ds = p * dP[j];"),
    "bwd_dk_without_scale": ("dkg[(int64_t)j * d + c] += J->scale * ds * qrow[c];",
                             "dkg[(int64_t)j * d + c] += ds * qrow[c];"),
    "bwd_dv_from_ds": ("dvg[(int64_t)j * d + c] += p * dorow[c];",
                       "dvg[(int64_t)j * d + c] += ds * dorow[c];"),
    "bwd_dq_from_v": ("dqrow[c] += J->scale * ds * in_at(J->k,", "dqrow[c] += J->scale * ds * in_at(J->v,"),
    "bwd_causal_off_by_one": ("(j < len) && (!J->causal || j <= i);",
                              "(j < len) && (!J->causal || j < i);"),
    "e4m3_bias_off_by_one": ("ldexp(1.0 + m / 8.0, e - 7)", "ldexp(1.0 + m / 8.0, e - 8)"),
    "e4m3_subnormal_scale": ("ldexp((double)m, -9)", "ldexp((double)m, -10)"),
    "masked_row_not_zeroed": ("for (int j = 0; j < N; ++j) Srow[j] = 0.0;",
                              "for (int j = 0; j < N; ++j) Srow[j] = 1.0 / N;"),
}


def _compile(src_text, out):
    path_c = out + ".c"
    with open(path_c, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O1", "-fPIC", "-shared", "-std=c11", "-pthread", "-ffp-contract=off",
                    "-o", out, path_c, "-lm"], check=True)


def test_unmutated_copy_passes(tmp_path):
    with open(SRC) as f:
        text = f.read()
    lib = str(tmp_path / "clean.so")
    _compile(text, lib)
    r = subprocess.run([sys.executable, RUNNER, lib, "--all"], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    with open(SRC) as f:
        text = f.read()
    assert text.count(old) >= 1, f"snippet for {name} not found in the oracle"
    lib = str(tmp_path / f"{name}.so")
    _compile(text.replace(old, new), lib)
    r = subprocess.run([sys.executable, RUNNER, lib], capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} passed every pin: {r.stdout}"
