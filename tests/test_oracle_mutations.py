"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of oracle/ep_oracle.c (a dropped or
reordered term, a wrong index, a transposed operand, the wrong rounding
rule), builds it, and runs the CPU pin tests against it with EP_ORACLE_LIB
pointing at the mutant: they must fail.  The unmodified copy must pass."""

import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ep_oracle.c")

# (name, text in ep_oracle.c, replacement, pin test file expected to fail)
MUTATIONS = [
    ("e4m3 ties away from zero", "double r = rint(a / q) * q; /* a / q is exact; rint rounds half to even */",
     "double r = round(a / q) * q;", "test_oracle_formats.py"),
    # the encoder saturates twice (before and after rounding): remove both
    ("e4m3 no saturation", ("if (a > 448.0) return (uint8_t)(s | 0x7E);", "if (r > 448.0) r = 448.0;"),
     ("if (a > 1e30) return (uint8_t)(s | 0x7E);", ""), "test_oracle_formats.py"),
    ("e4m3 subnormal spacing", "double q = (a < ldexp(1.0, -6)) ? ldexp(1.0, -9)",
     "double q = (a < ldexp(1.0, -6)) ? ldexp(1.0, -10)", "test_oracle_formats.py"),
    ("bf16 ties away from zero", "double r = rint(a / q) * q;\n  if (r >= ldexp(1.0, 128))",
     "double r = round(a / q) * q;\n  if (r >= ldexp(1.0, 128))", "test_oracle_formats.py"),
    ("scale uses 447", "float scale = amax / 448.0f;", "float scale = amax / 447.0f;", "test_oracle_ops.py"),
    ("quantise multiplies by the scale", "q[g * 128 + c] = epo_e4m3_encode(v / scale);",
     "q[g * 128 + c] = epo_e4m3_encode(v * scale);", "test_oracle_ops.py"),
    ("amax ignores the sign", "float a = fabsf(epo_f32_from_bf16(x[t * H + g * 128 + c]));",
     "float a = epo_f32_from_bf16(x[t * H + g * 128 + c]);", "test_oracle_ops.py"),
    ("combine rounds the product first",
     "acc = fmaf(topk_weights[t * k + j], epo_f32_from_bf16(y[(int64_t)s * H + h]), acc);",
     "acc = acc + topk_weights[t * k + j] * epo_f32_from_bf16(y[(int64_t)s * H + h]);", "test_oracle_ops.py"),
    ("combine in reverse top-k order",
     "      for (int64_t j = 0; j < k; ++j) {\n        int32_t s = slot_of_pair[t * k + j];\n        if (s < 0) continue;\n        acc = fmaf(",
     "      for (int64_t j = k - 1; j >= 0; --j) {\n        int32_t s = slot_of_pair[t * k + j];\n        if (s < 0) continue;\n        acc = fmaf(",
     "test_oracle_ops.py"),
    ("combine drops the last pair",
     "      for (int64_t j = 0; j < k; ++j) {\n        int32_t s = slot_of_pair[t * k + j];\n        if (s < 0) continue;\n        acc = fmaf(",
     "      for (int64_t j = 0; j < k - 1; ++j) {\n        int32_t s = slot_of_pair[t * k + j];\n        if (s < 0) continue;\n        acc = fmaf(",
     "test_oracle_ops.py"),
    ("weight grad with a transposed operand",
     "dot += (double)g * (double)epo_f32_from_bf16(y[(int64_t)s * H + h]);",
     "dot += (double)g * (double)epo_f32_from_bf16(y[t * H + h]);", "test_oracle_ops.py"),
    ("grad_y without the weight", "float prod = w * g;", "float prod = g;", "test_oracle_ops.py"),
    ("dispatch backward skips the first pair",
     "        if (s < 0) continue;\n        acc = acc + epo_f32_from_bf16(grad_recv",
     "        if (s < 0 || j == 0) continue;\n        acc = acc + epo_f32_from_bf16(grad_recv", "test_oracle_ops.py"),
    ("slots in (j, t) order",
     "  for (int64_t t = 0; t < T; ++t) {\n    for (int64_t j = 0; j < k; ++j) {\n      int64_t e = topk_idx[t * k + j];\n      if (e < 0 || e >= E) { slot_of_pair",
     "  for (int64_t j = 0; j < k; ++j) {\n    for (int64_t t = 0; t < T; ++t) {\n      int64_t e = topk_idx[t * k + j];\n      if (e < 0 || e >= E) { slot_of_pair",
     "test_oracle_layout.py"),
    ("rank of an expert by modulo",
     "is_token_in_rank[t * R + e / Er] = 1;\n      count_src_rank_expert[(t / Tr) * E + e] += 1;",
     "is_token_in_rank[t * R + e % R] = 1;\n      count_src_rank_expert[(t / Tr) * E + e] += 1;",
     "test_oracle_layout.py"),
    ("source-rank offsets one rank late", "      src_rank_expert_offset[r * E + e] = run;\n      run += count_src_rank_expert[r * E + e];",
     "      run += count_src_rank_expert[r * E + e];\n      src_rank_expert_offset[r * E + e] = run;", "test_oracle_layout.py"),
    ("bad ids not flagged", "if (e < -1 || e >= E) { status = EPO_BAD_INDEX; continue; }",
     "if (e < -1 || e >= E) { continue; }", "test_oracle_layout.py"),
    ("padded blocks rank-major", "int64_t row = (e * R + r) * M + i;", "int64_t row = (r * E + e) * M + i;",
     "test_oracle_layout.py"),
    ("padded overflow not flagged", "if (i >= M) { status |= EPO_CAPACITY; continue; }",
     "if (i >= M) { continue; }", "test_oracle_layout.py"),
    ("router group ties to the higher index", "if (!gsel[g] && (best < 0 || gscore[g] > gscore[best])) best = g;",
     "if (!gsel[g] && (best < 0 || gscore[g] >= gscore[best])) best = g;", "test_oracle_router.py"),
    ("router ignores the group limit", "if (gsel[e / per] && !taken[e] && (best < 0 || s[e] > s[best])) best = e;",
     "if (!taken[e] && (best < 0 || s[e] > s[best])) best = e;", "test_oracle_router.py"),
    ("router group score is the first expert", "if (s[g * per + i] > m) m = s[g * per + i];",
     "if (0) m = s[g * per + i];", "test_oracle_router.py"),
]


def build_variant(tmp_path, name, old=None, new=None):
    src = open(SRC).read()
    if old is not None:
        olds, news = (old, new) if isinstance(old, tuple) else ((old,), (new,))
        for o, n in zip(olds, news):
            assert src.count(o) == 1, f"mutation site not unique or missing: {name}"
            src = src.replace(o, n)
    d = tmp_path / "src"
    d.mkdir(exist_ok=True)
    (d / "ep_oracle.c").write_text(src)
    (d / "ep_oracle.h").write_text(open(os.path.join(ROOT, "oracle", "ep_oracle.h")).read())
    lib = tmp_path / f"lib_{abs(hash(name))}.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
                    "-fno-builtin-fmaf", "-o", str(lib), str(d / "ep_oracle.c"), "-lm"], check=True)
    return lib


def run_pins(lib, test_file):
    env = dict(os.environ, EP_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", test_file)], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-2000:]


def test_unmodified_copy_passes(tmp_path):
    lib = build_variant(tmp_path, "unmodified")
    for f in ("test_oracle_formats.py", "test_oracle_ops.py", "test_oracle_layout.py", "test_oracle_router.py"):
        rc, out = run_pins(lib, f)
        assert rc == 0, out


def test_pins_reject_every_mutant(tmp_path):
    """All mutants, checked concurrently (each in its own pytest process)."""
    from concurrent.futures import ThreadPoolExecutor

    def check(i):
        name, old, new, test_file = MUTATIONS[i]
        sub = tmp_path / f"m{i}"
        sub.mkdir()
        rc, out = run_pins(build_variant(sub, name, old, new), test_file)
        return name, rc, out

    with ThreadPoolExecutor(min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(check, range(len(MUTATIONS))))
    survived = [(name, out) for name, rc, out in results if rc == 0]
    assert not survived, "the pins accepted: " + "; ".join(n for n, _ in survived)
    assert len(results) == len(MUTATIONS) >= 19
