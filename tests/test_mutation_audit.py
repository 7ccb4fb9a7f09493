"""Mutation audit of the oracle's pins (test infrastructure; collected, and skipped unless
SKV_MUTATION_AUDIT=1 is set, because it rebuilds and re-tests the oracle once per mutation, which
takes a few minutes).

Each entry plants one plausible mistake -- a dropped term, a wrong index, order or operand, a wrong
rounding, normaliser or comparison -- in a temporary copy of the oracle, rebuilds that copy and runs
the oracle's CPU pins (tests/test_oracle_*.py) against it. A mistake that no pin catches fails its
test case. The repository's own files are never modified.

    SKV_MUTATION_AUDIT=1 python -m pytest tests/test_mutation_audit.py -q       # every mutation
    SKV_MUTATION_AUDIT=1 python -m pytest tests/test_mutation_audit.py -k seg_gt

Conventions of the oracle's own readings that the pages do not fix are listed in CONVENTIONS:
there a planted change alters only which (equally valid) convention is followed, so surviving it
is expected (and asserted).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C = "oracle/skv_oracle.c"
STREAM = "oracle/stream.py"
INIT = "oracle/__init__.py"

MUTATIONS = [
    # projection (reading R2) and the fixed fp32 variation recipe
    ("proj_sqrt_r", C, "const double inv_sqrt_r = 1.0 / sqrt((double)r);",
     "const double inv_sqrt_r = 1.0 / (double)r;"),
    ("proj_sin", C, "cos(two_pi * u2)", "sin(two_pi * u2)"),
    ("feat_desc", C, "for (int j = 0; j < d; ++j) acc = fmaf(P[i * cols + j], k[j], acc);",
     "for (int j = d - 1; j >= 0; --j) acc = fmaf(P[i * cols + j], k[j], acc);"),
    ("feat_transpose", C, "acc = fmaf(P[i * cols + j], k[j], acc);\n        for (int j = 0; j < d; ++j) "
     "acc = fmaf(P[i * cols + d + j], v[j], acc);\n        z[i] = acc;",
     "acc = fmaf(P[j * ORC_PROJ_DIM + i], k[j], acc);\n        for (int j = 0; j < d; ++j) "
     "acc = fmaf(P[(d + j) * ORC_PROJ_DIM + i], v[j], acc);\n        z[i] = acc;"),
    ("feat_v_half", C, "for (int j = 0; j < d; ++j) acc = fmaf(P[i * cols + d + j], v[j], acc);\n        z[i] = acc;",
     "for (int j = 0; j < d; ++j) acc = fmaf(P[i * cols + j], v[j], acc);\n        z[i] = acc;"),
    ("feat_no_v", C, "for (int j = 0; j < d; ++j) acc = fmaf(P[i * cols + d + j], v[j], acc);\n        z[i] = acc;",
     "z[i] = acc;"),
    ("qstep_floor", C, "*D = (int64_t)llrintf(scaled);", "*D = (int64_t)floorf(scaled);"),
    ("qstep_nosqrt", C, "float dd = sqrtf(s);", "float dd = s;"),
    ("qstep_15", C, "    for (int i = 0; i < ORC_PROJ_DIM; ++i) {\n        float di = zc[i] - zp[i];",
     "    for (int i = 0; i < ORC_PROJ_DIM - 1; ++i) {\n        float di = zc[i] - zp[i];"),
    # boundaries and the sink / middle / recent split
    ("seg_gt", C, "while (j <= N - 1 && lhs >= (__int128)j * cT) {", "while (j <= N - 1 && lhs > (__int128)j * cT) {"),
    ("seg_next", C, "            b[j] = t;\n            ++j;", "            b[j] = t + 1;\n            ++j;"),
    ("split_noclamp", C, "int w = W < T - s ? W : T - s;", "int w = W < T ? W : T;"),
    # node statistics and the representative
    ("stats_sample", C, "        var_sum += acc / m;\n        if (var_vec) var_vec[i] = acc / m;",
     "        var_sum += m > 1 ? acc / (m - 1) : 0.0;\n        if (var_vec) var_vec[i] = m > 1 ? acc / (m - 1) : 0.0;"),
    ("stats_sig2_sum", C, "*sig2 = var_sum / d;", "*sig2 = var_sum;"),
    ("stats_beta_d", C, "*beta = *sig2 / (2.0 * d);", "*beta = *sig2 / d;"),
    ("stats_alpha", C, "*alpha = log((double)m);", "*alpha = log((double)m + 1.0);"),
    ("stats_vmean_k", C, "vt[i] = sv / m;\n    }", "vt[i] = sk / m;\n    }"),
    ("rep_shift", C, "? D + mid : NULL;", "? D + mid + 1 : NULL;"),
    ("stats_var_scale", C, "        var_sum += acc / m;", "        var_sum += acc / m * 1.0000001;"),
    # decode
    ("dec_sqrt", C, "s[j] = dot * inv_sqrt_d + alpha[j] + closure;", "s[j] = dot + alpha[j] + closure;"),
    ("dec_noalpha", C, "s[j] = dot * inv_sqrt_d + alpha[j] + closure;", "s[j] = dot * inv_sqrt_d + closure;"),
    ("dec_closure_sign", C, "s[j] = dot * inv_sqrt_d + alpha[j] + closure;",
     "s[j] = dot * inv_sqrt_d + alpha[j] - closure;"),
    ("dec_qnorm", C, "double closure = qn2 * beta[j];", "double closure = sqrt(qn2) * beta[j];"),
    ("dec_diag_noq2", C, "c += qr[i] * qr[i] * var[(long)j * d + i];", "c += qr[i] * var[(long)j * d + i];"),
    ("dec_diag_d", C, "closure = c / (2.0 * d);", "closure = c / d;"),
    ("dec_lse_log2", C, "const double l = mx + log(Z);", "const double l = mx + log2(Z);"),
    ("dec_out_unnorm", C, "const double p = exp(s[j] - l);", "const double p = exp(s[j] - mx);"),
    # the Python layer: GQA head mapping and option marshalling
    ("gqa_interleaved", INIT, "        rows = q[b, :, h * G:(h + 1) * G, :].reshape(R * G, d)",
     "        rows = q[b, :, h::Hkv, :].reshape(R * G, d)"),
    ("rows_order", INIT, "        rows = q[b, :, h * G:(h + 1) * G, :].reshape(R * G, d)",
     "        rows = q[b, :, h * G:(h + 1) * G, :].transpose(1, 0, 2).reshape(R * G, d)"),
    ("rep_codes_swapped", INIT, 'REPRESENTATIVES = {"mean": 0, "variation": 1}',
     'REPRESENTATIVES = {"mean": 1, "variation": 0}'),
    # streaming (readings S3-S5)
    ("stream_gt_for_ge", STREAM, "if self.N * (last.V + D) >= self.cT:", "if self.N * (last.V + D) > self.cT:"),
    ("stream_no_step_in_open", STREAM, "if self.N * (last.V + D) >= self.cT:", "if self.N * last.V >= self.cT:"),
    ("stream_cT_after_split", STREAM, "        self.cT += D\n        last = self.nodes[-1]\n",
     "        last = self.nodes[-1]\n        self.cT += 0\n"),
    ("stream_rightmost_tie", STREAM, "j = int(np.argmin(sums))", "j = len(sums) - 1 - int(np.argmin(sums[::-1]))"),
    ("stream_single_V", STREAM, "sums = [self.nodes[j].V + self.nodes[j + 1].V for j in range(len(self.nodes) - 1)]",
     "sums = [self.nodes[j].V for j in range(len(self.nodes) - 1)]"),
    ("stream_merge_M2", STREAM, "M2 = a.M2 + b.M2 + float(dk @ dk) * a.m * b.m / m",
     "M2 = a.M2 + b.M2"),
    # the centring option's fixed-order mean (reading R8)
    ("mean_one_block", C, "const int b1 = b0 + ORC_MEAN_BLOCK < T ? b0 + ORC_MEAN_BLOCK : T;",
     "const int b1 = T;"),
    ("mean_div_tminus1", C, "mu[i] = T > 0 ? total / (float)T : 0.0f;",
     "mu[i] = T > 1 ? total / (float)(T - 1) : 0.0f;"),
    ("center_keys_noop", INIT, "    return (k - key_mean_f32(k)[None, :]).astype(np.float32)",
     "    return k.astype(np.float32)"),
    # the given-steps path and the tensor projection's checks
    ("steps_prefix_exclusive", C, "            if (C) C[t] = run;\n            if (d64) d64[t] = 0.0;",
     "            if (C) C[t] = run - D_in[t];\n            if (d64) d64[t] = 0.0;"),
    ("steps_ignored", C, "            run += D_in[t];", "            run += 100;"),
    ("bf16_truncate", INIT, "    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16", "    r = (u >> 16) << 16"),
    ("tensor_ref_no_v", INIT, "    x = np.concatenate([k, v], axis=1)[s_eff:s_eff + M]",
     "    x = np.concatenate([k, 0 * v], axis=1)[s_eff:s_eff + M]"),

]

# the Box-Muller branch is part of reading R2's generator definition, which the pages leave open
CONVENTIONS = {"proj_sin"}

# applied after the main replacement (the c_T update moves to after the split decision; the
# interleaved GQA mapping also writes its outputs back interleaved)
EXTRA = {"stream_cT_after_split": ("        while len(self.nodes) > self.N:",
                                   "        self.cT += D\n        while len(self.nodes) > self.N:"),
         "gqa_interleaved": ("        out[b, :, h * G:(h + 1) * G, :] = o.reshape(R, G, d)\n"
                             "        lse[b, :, h * G:(h + 1) * G] = l.reshape(R, G)",
                             "        out[b, :, h::Hkv, :] = o.reshape(R, G, d)\n"
                             "        lse[b, :, h::Hkv] = l.reshape(R, G)")}


def _copy_tree(dst):
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(dst, "oracle"),
                    ignore=shutil.ignore_patterns("_build", "__pycache__"))
    shutil.copytree(os.path.join(ROOT, "workloads"), os.path.join(dst, "workloads"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    os.makedirs(os.path.join(dst, "tests"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dst, "tests", "golden"))
    for f in os.listdir(os.path.join(ROOT, "tests")):
        if f.startswith("test_oracle_") or f in ("conftest.py", "exact_f32.py"):
            shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(dst, "tests", f))




def _run_mutation(name, rel, old, new):
    """True if the pins catch the planted mistake (the pin suite fails on the mutated copy)."""
    with tempfile.TemporaryDirectory(prefix="oracle_mut_") as tmp:
        _copy_tree(tmp)
        path = os.path.join(tmp, rel)
        src = open(path).read()
        assert src.count(old) == 1, f"{name}: anchor found {src.count(old)} times"
        src = src.replace(old, new)
        if name in EXTRA:
            a, b = EXTRA[name]
            src = src.replace(a, b, 1)
        open(path, "w").write(src)
        env = dict(os.environ, PYTHONDONTWRITEBYTECODE="1")
        env.pop("SKV_MUTATION_AUDIT", None)
        subprocess.run([sys.executable, "-c", "import oracle; oracle.build(force=True)"], cwd=tmp, env=env,
                       check=True, capture_output=True)
        tests = sorted(os.path.join("tests", f) for f in os.listdir(os.path.join(tmp, "tests"))
                       if f.startswith("test_oracle_"))
        r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "not gpu", "-p", "no:cacheprovider",
                            *tests], cwd=tmp, env=env, capture_output=True, text=True)
        return r.returncode != 0


@pytest.mark.skipif(not os.environ.get("SKV_MUTATION_AUDIT"),
                    reason="rebuilds and re-tests the oracle per mutation (minutes): set SKV_MUTATION_AUDIT=1")
@pytest.mark.parametrize("name,rel,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught_by_a_pin(name, rel, old, new):
    caught = _run_mutation(name, rel, old, new)
    if name in CONVENTIONS:
        assert not caught, f"{name}: a convention change should leave every pin green"
    else:
        assert caught, f"{name}: no oracle pin catches this planted mistake"


def test_every_anchor_is_present_once():
    """Each mutation's anchor text occurs exactly once in the current oracle sources (so the audit
    keeps testing what it claims when the oracle is edited)."""
    for name, rel, old, _ in MUTATIONS:
        assert open(os.path.join(ROOT, rel)).read().count(old) == 1, name
