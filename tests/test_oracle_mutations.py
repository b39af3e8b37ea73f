"""Plant plausible mistakes in a copy of the oracle (CPU only) and check that
the pins of test_oracle_pins.py catch every one of them."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ckda_oracle.c")

MUTATIONS = {
    "delta_sign": ("S[i * dv + j] += beta * k[i] * (v[j] - kx[j]);",
                   "S[i * dv + j] += beta * k[i] * (v[j] + kx[j]);"),
    "gate_sign_dropped": ("double a = (double)sg[i] * exp(g[i]);\n        for (int j = 0; j < dv; ++j) S[i * dv + j] *= a;",
                          "double a = exp(g[i]);\n        for (int j = 0; j < dv; ++j) S[i * dv + j] *= a;"),
    "output_before_update": ("for (int j = 0; j < dv; ++j) o[j] += S[i * dv + j] * q[i];",
                             "for (int j = 0; j < dv; ++j) o[j] += (S[i * dv + j] - beta * k[i] * (v[j] - kx[j])) * q[i];"),
    "beta_on_value_only": ("S[i * dv + j] += beta * k[i] * (v[j] - kx[j]);",
                           "S[i * dv + j] += k[i] * (beta * v[j] - kx[j]);"),
    "transposed_key_read": ("for (int j = 0; j < dv; ++j) kx[j] += k[i] * S[i * dv + j];",
                            "for (int j = 0; j < dv; ++j) kx[j] += k[j % dk] * S[i * dv + j];"),
    "bwd_dg_sign": ("dg[i] = s;", "dg[i] = -s;"),
    "bwd_dv_beta": ("dv_[j] = beta * Gk[j];", "dv_[j] = Gk[j];"),
    "bwd_dk_term": ("dk_[i] = beta * (gr - xg);", "dk_[i] = beta * (gr + xg);"),
    "bwd_state_gate": ("G[i * dv + j] = a * dx;", "G[i * dv + j] = dx;"),
    "bwd_dbeta_residual": ("db += Gk[j] * r[j];", "db += Gk[j] * v[j];"),
    "bwd_output_term": ("G[i * dv + j] += q[i] * dO[j];", "G[i * dv + j] += q[i] * dO[j] * 0.5;"),
    "bwd_dq_prev_state": ("s += Snew[i * dv + j] * dO[j];", "s += Sprev[i * dv + j] * dO[j];"),
    "chunk_state_late_snapshot": ("if (p->chunk_states && (t - t0) % p->chunk == 0) {\n"
                                  "            int64_t c = p->chunk_off[n] + (t - t0) / p->chunk;",
                                  "if (p->chunk_states && (t - t0 + 1) % p->chunk == 0) {\n"
                                  "            int64_t c = p->chunk_off[n] + (t - t0 + 1) / p->chunk - 1;"),
    "chunk_state_sequence_offset": ("int64_t c = p->chunk_off[n] + (t - t0) / p->chunk;",
                                    "int64_t c = p->chunk_off[n > 0 ? n - 1 : 0] + (t - t0) / p->chunk;"),
    "bwd_checkpoint_off_by_one": ("memcpy(seg, ckpt + s * sz, sizeof(double) * sz);",
                                  "memcpy(seg, ckpt + (s > 0 ? s - 1 : 0) * sz, sizeof(double) * sz);"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor not found once: " + name
    mutated = tmp_path / "mut.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", str(lib),
                           str(mutated), "-lm", "-lpthread"])
    env = dict(os.environ, CKDA_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, "planted mistake %s passed every pin" % name
