"""The oracle's pins must catch plausible mistakes.

Each case copies the oracle to a temporary directory, plants one mistake in its
C source (CPU only), and runs the pin suite against the copy in a subprocess:
the suite has to fail.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    "decay_misplaced": ("row[j] = a * (row[j] - b * ki * y[j]) + b * ki * v[j];",
                        "row[j] = a * row[j] - b * ki * y[j] + b * ki * v[j];"),
    "write_strength_dropped": ("+ b * ki * v[j];", "+ ki * v[j];"),
    "erase_sign_flipped": ("(row[j] - b * ki * y[j])", "(row[j] + b * ki * y[j])"),
    "readout_before_update": ("    /* Sigma_t = a (Sigma - b k y) + b k v^T */",
                              "    if (o) { for (int j = 0; j < dv; ++j) { o[j] = 0.0;"
                              " for (int i = 0; i < dk; ++i) o[j] += q[i] * sig[(size_t)i * dv + j];"
                              " o[j] *= scale; } o = 0; }\n"
                              "    /* Sigma_t = a (Sigma - b k y) + b k v^T */"),
    "key_transposed_with_query": ("const double ki = k[i];\n        double *row",
                                  "const double ki = q[i];\n        double *row"),
}

# mistakes in the reverse mode, caught by its own pins
BWD_MUTATIONS = {
    "bwd_key_cross_term_dropped": ("dk_out[th * dk + r] = -at * bt * (gx + sy) + bt * gv;",
                                   "dk_out[th * dk + r] = -at * bt * gx + bt * gv;"),
    "bwd_adjoint_decay_dropped": ("G[(size_t)r * dv + j] = at * (G[(size_t)r * dv + j] - bt * kt[r] * y[j]);",
                                  "G[(size_t)r * dv + j] = (G[(size_t)r * dv + j] - bt * kt[r] * y[j]);"),
    "bwd_query_grad_uses_previous_state": ("acc += Sig[(size_t)r * dv + j] * dOt[j];",
                                           "acc += Sp[(size_t)r * dv + j] * dOt[j];"),
    "bwd_write_strength_sign": ("db[th] = yv - at * yx;", "db[th] = yv + at * yx;"),
}


# mistakes in the per-channel gate variant, caught by its own pins; a list of
# (anchor, replacement) pairs is applied in order
KDA_MUTATIONS = {
    "kda_decay_dropped": ("row[j] *= a[i];", "row[j] *= 1.0;"),
    "kda_decay_channel_reversed": ("row[j] *= a[i];", "row[j] *= a[dk - 1 - i];"),
    "kda_decay_after_delta": [("row[j] *= a[i];", "row[j] *= 1.0;"),
                              ("row[j] = row[j] - b * kc * y[j] + b * kc * v[j];",
                               "row[j] = a[i] * (row[j] - b * kc * y[j]) + b * kc * v[j];")],
    "kda_gate_of_first_channel": ("row[j] *= a[i];", "row[j] *= a[0];"),
}


# mistakes in the sliding-window attention, caught by its own pins
SWA_MUTATIONS = {
    "swa_window_one_wider": ("(t - window + 1 > cu_seqlens[s]) ? t - window + 1",
                             "(t - window > cu_seqlens[s]) ? t - window"),
    "swa_scale_dropped": ("sc[j - lo] = scale * acc;", "sc[j - lo] = acc;"),
    "swa_not_normalised": ("for (int c = 0; c < dv; ++c) ot[c] /= l;", "(void)l;"),
}


def _pairs(name):
    for table in (MUTATIONS, BWD_MUTATIONS, KDA_MUTATIONS, SWA_MUTATIONS):
        if name in table:
            m = table[name]
            return m if isinstance(m, list) else [m]
    raise KeyError(name)


@pytest.mark.parametrize("name", sorted(MUTATIONS) + sorted(BWD_MUTATIONS) + sorted(KDA_MUTATIONS)
                         + sorted(SWA_MUTATIONS))
def test_pins_catch_planted_mistake(tmp_path, name):
    pins = ("test_oracle_pins.py" if name in MUTATIONS else
            "test_oracle_bwd_pins.py" if name in BWD_MUTATIONS else
            "test_oracle_kda_pins.py" if name in KDA_MUTATIONS else "test_oracle_swa_pins.py")
    shutil.copytree(os.path.join(ROOT, "oracle"), tmp_path / "oracle",
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    shutil.copytree(os.path.join(ROOT, "tests"), tmp_path / "tests",
                    ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutations.py"))
    cfile = tmp_path / "oracle" / "gdn_oracle.c"
    text = cfile.read_text()
    for src, dst in _pairs(name):
        assert text.count(src) == 1, f"mutation anchor not found once: {src!r}"
        text = text.replace(src, dst)
    cfile.write_text(text)
    env = dict(os.environ, PYTHONPATH=str(tmp_path))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        str(tmp_path / "tests" / pins)],
                       cwd=tmp_path, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch mutation {name}:\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout
