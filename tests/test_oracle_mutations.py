"""Mutation check of the oracle's pins (CPU only).

Each case plants one plausible mistake in a copy of oracle/mmoe_oracle.c,
builds the copy with the oracle's own flags and runs tests/test_oracle.py
against that build (MMOE_ORACLE_SO); at least one pin must fail.  An
unmutated copy, built and run the same way, must pass, so a failure is the
planted mistake's and not the harness's.  The oracle source itself is never
modified.
"""
import os
import subprocess
import sys

import pytest

import oracle
from tests.conftest import ROOT

SRC_PATH = os.path.join(ROOT, "oracle", "mmoe_oracle.c")

# name: (text in the oracle, planted replacement)
MUTATIONS = {
    # Eq. (*) layer structure
    "shared_expert_dropped": ("for (int64_t m = 0; m < d; ++m) yrow[m] = o[m];",
                              "for (int64_t m = 0; m < d; ++m) yrow[m] = 0.0f;"),
    "shared_expert_gated": ("for (int64_t m = 0; m < d; ++m) yrow[m] = o[m];",
                            "for (int64_t m = 0; m < d; ++m) yrow[m] = 0.5f * o[m];"),
    "gates_reversed": ("float prod = gate[s] * o[m];", "float prod = gate[k - 1 - s] * o[m];"),
    # router (section on the FP32 router; softmax without renormalisation)
    "router_bias_missing": ("if (L->router_bias && L->gating != 2) l = l + L->router_bias[e];", ""),
    "tie_goes_to_high_index": ("if (best < 0 || key[e] > key[best]) best = e;",
                               "if (best < 0 || key[e] >= key[best]) best = e;"),
    # selection-only bias (gating 2, auxiliary-loss-free balancing)
    "sel_bias_enters_logit": ("if (L->router_bias && L->gating != 2) l = l + L->router_bias[e];",
                              "if (L->router_bias) l = l + L->router_bias[e];"),
    "sel_bias_ignored": ("key[e] = L->gating == 2 ? (L->router_bias ? probs[e] + L->router_bias[e] : probs[e])",
                         "key[e] = L->gating == 2 ? (L->router_bias ? probs[e] : probs[e])"),
    "sel_bias_on_logit": ("key[e] = L->gating == 2 ? (L->router_bias ? probs[e] + L->router_bias[e] : probs[e])",
                          "key[e] = L->gating == 2 ? (L->router_bias ? logits[e] + L->router_bias[e] : probs[e])"),
    "softmax_renormalised": ("for (int64_t j = 0; j < k; ++j) gate[j] = probs[idx[j]];",
                             "double ss = 0; for (int64_t j = 0; j < k; ++j) ss += probs[idx[j]]; "
                             "for (int64_t j = 0; j < k; ++j) gate[j] = (float)(probs[idx[j]] / ss);"),
    # SwiGLU
    "activation_scale_dropped": ("float gv = ga * sx;", "float gv = ga;"),
    "gate_and_up_swapped": ("float silu = gv / (1.0f + expf(-gv));\n        a[n] = silu * uv;",
                            "float silu = uv / (1.0f + expf(-uv));\n        a[n] = silu * gv;"),
    "silu_sign": ("expf(-gv)", "expf(gv)"),
    "up_uses_gate_scales": ("ua = fmaf((float)p_u, S[(hid + n) * ng + j], ua);",
                            "ua = fmaf((float)p_u, S[n * ng + j], ua);"),
    # down projection
    "down_weights_transposed": ("const uint8_t* wr = W + m * (hid / 2);",
                                "const uint8_t* wr = W + (m % hid) * (hid / 2);"),
    "down_group_scale_index": ("acc = fmaf((float)p, S[m * ng + j], acc);",
                               "acc = fmaf((float)p, S[m * ng], acc);"),
    "down_row_scale_dropped": ("o[m] = acc * sh;", "o[m] = acc;"),
    # Eq. (6) weights and INT4 packing
    "eq6_scale_max_over_7": ("float s = (2.0f * m) / 15.0f;", "float s = m / 7.0f;"),
    "eq6_truncates": ("float v = rintf(w[kk] / s);", "float v = truncf(w[kk] / s);"),
    "int4_high_nibble_first": ("int v = (row[k >> 1] >> ((k & 1) * 4)) & 15;",
                               "int v = (row[k >> 1] >> ((~k & 1) * 4)) & 15;"),
    "int4_unsigned": ("return v >= 8 ? v - 16 : v;", "return v;"),
    # dynamic INT8 activations
    "act_scale_over_128": ("float s = m / 127.0f;", "float s = m / 128.0f;"),
    "act_truncates": ("float v = rintf(a[i] / s);", "float v = truncf(a[i] / s);"),
    # (no mutation of the activation clamp: with s = absmax / 127 every quotient already lies
    # within [-127, 127], so a wrong clamp bound changes nothing observable)
}


def _run_pins(tmp_path, text):
    src = tmp_path / "mmoe_oracle.c"
    src.write_text(text)
    so = tmp_path / "liboracle.so"
    oracle.compile_oracle(str(src), str(so))
    env = dict(os.environ, MMOE_ORACLE_SO=str(so))
    return subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle.py"), "-x", "-q",
                           "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)


def test_unmutated_copy_passes_the_pins(tmp_path):
    r = _run_pins(tmp_path, open(SRC_PATH).read())
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(tmp_path, name):
    src = open(SRC_PATH).read()
    before, after = MUTATIONS[name]
    assert src.count(before) == 1, f"{name}: the text to mutate must occur exactly once"
    r = _run_pins(tmp_path, src.replace(before, after))
    # exit status 1: tests ran and at least one failed (not a collection or usage error)
    assert r.returncode == 1 and " failed" in r.stdout, (name, r.returncode, r.stdout[-2000:])
