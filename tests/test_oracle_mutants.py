"""The oracle's pins must reject plausible mistakes.

Each case below plants one mistake in a private copy of oracle/kda_oracle.c
(on the CPU, in a temporary directory), builds it, and runs the pin suite
against that copy (forward and gradient pins); the suite has to fail.  The shipped oracle is untouched.
"""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(ROOT, "oracle", "kda_oracle.c")

DECAY = ("for (int c = 0; c < dk; ++c)\n"
         "                    for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= alpha[c];\n")
READ_MARK = "                /* read the updated state: o_t = S^T q_t */\n"
R_MARK = "                /* then remember: write only the error, scaled by beta_t */\n"
WRITE_BLOCK = ("                for (int c = 0; c < dk; ++c) {\n"
               "                    const double kc = k[tk + c];\n"
               "                    for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] += kc * r[j];\n"
               "                }\n")
READ_BLOCK = ("                for (int j = 0; j < dv; ++j) {\n"
              "                    double acc = 0.0;\n"
              "                    for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * q[tk + c];\n"
              "                    o[tv + j] = acc;\n"
              "                }\n")


def _move(src, block, before):
    """Cut `block` out of the source and paste it in front of `before`."""
    assert block in src and before in src
    src = src.replace(block, "", 1)
    return src.replace(before, block + before, 1)


MUTANTS = {
    "gate_on_value_axis": lambda s: s.replace("*= alpha[c];", "*= alpha[j % dk];", 1),
    "beta_dropped": lambda s: s.replace("r[j] = b * (v[tv + j] - r[j]);", "r[j] = (v[tv + j] - r[j]);", 1),
    "write_sign_flipped": lambda s: s.replace("S[(size_t)c * dv + j] += kc * r[j];",
                                              "S[(size_t)c * dv + j] -= kc * r[j];", 1),
    "read_with_key": lambda s: s.replace("acc += S[(size_t)c * dv + j] * q[tk + c];",
                                         "acc += S[(size_t)c * dv + j] * k[tk + c];", 1),
    "decay_after_write": lambda s: _move(s, "                " + DECAY, READ_MARK),
    "prediction_before_decay": lambda s: _move(s, "                " + DECAY, R_MARK),
    "read_before_write": lambda s: _move(s, READ_BLOCK, R_MARK),
    "alpha_not_exponentiated": lambda s: s.replace("alpha[c] = exp(log_alpha[tk + c]);",
                                                   "alpha[c] = 1.0 + log_alpha[tk + c];", 1),
    # reverse sweep (oracle.backward)
    "bwd_prediction_adjoint_dropped": lambda s: s.replace(
        "dS[(size_t)c * dv + j] += kt[c] * du[j];", "(void)0;", 1),
    "bwd_key_term_of_prediction_dropped": lambda s: s.replace(
        "dk_out[tk + c] += acc;", "dk_out[tk + c] += 0.0 * acc;", 1),
    "bwd_adjoint_not_decayed": lambda s: s.replace(
        "for (int j = 0; j < dv; ++j) dS[(size_t)c * dv + j] *= alpha[c];", "", 1),
    "bwd_value_grad_without_beta": lambda s: s.replace(
        "dv_out[tv + j] = bt * du[j];", "dv_out[tv + j] = du[j];", 1),
    "bwd_beta_grad_sign": lambda s: s.replace(
        "db += du[j] * (vt[j] - r[j]);", "db += du[j] * (vt[j] + r[j]);", 1),
    "bwd_query_grad_from_decayed_state": lambda s: s.replace(
        "acc += S[(size_t)c * dv + j] * dot[j];", "acc += Sp[(size_t)c * dv + j] * dot[j];", 1),
    "bwd_gate_grad_from_new_state": lambda s: s.replace(
        "acc += dS[(size_t)c * dv + j] * Sp[(size_t)c * dv + j];",
        "acc += dS[(size_t)c * dv + j] * S[(size_t)c * dv + j];", 1),
    "bwd_segment_restarts_from_first_checkpoint": lambda s: s.replace(
        "memcpy(S, ckpt + (size_t)sgi * kv, sizeof(double) * kv);",
        "memcpy(S, ckpt, sizeof(double) * kv);", 1),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, tmp_path):
    src = open(SRC).read()
    bad = MUTANTS[name](src)
    assert bad != src, f"mutation {name} did not apply"
    c = tmp_path / "kda_oracle_mutant.c"
    c.write_text(bad)
    so = tmp_path / "libkda_oracle_mutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o", str(so), str(c), "-lm"],
                   check=True)
    env = dict(os.environ, KDA_ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_oracle_pins.py"),
                        os.path.join(HERE, "test_oracle_backward_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"pins accepted mutant {name}:\n{r.stdout[-2000:]}"
