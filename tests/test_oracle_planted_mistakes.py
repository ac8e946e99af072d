"""Planted mistakes: the oracle's pins must catch each plausible slip.

Each case edits one line of oracle/spec_verify_oracle.c, compiles the edited
copy with the oracle's own flags into a temporary library, and runs a chosen
subset of the CPU pins against it (the oracle loader takes the library from
SV_ORACLE_LIB).  The pins must FAIL on every mutant, and a control build of
the unedited source must pass the same pins.  Mistakes are planted in the
oracle only, on the CPU; nothing here touches the GPU library.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "spec_verify_oracle.c")
REPORT = "tests/test_oracle_report.py"
PINS = "tests/test_oracle_pins.py"

# (name, line as written, planted mistake, pins that must catch it)
MUTANTS = [
    ("near-tie gap: second best dropped when a new best arrives",
     "if (s->arg >= 0) s->second = s->best;", ";", [REPORT]),
    ("near-tie gap: second best updated only past the best",
     "} else if (score > s->second) {", "} else if (score > s->best) {", [REPORT]),
    ("near-tie gap: sign flipped",
     "return s->best - s->second;", "return s->second - s->best;", [REPORT]),
    ("acceptance margin: ratio inverted",
     "fabs(u - p / q)", "fabs(u - q / p)", [REPORT]),
    ("acceptance margin: the next position's draw",
     "fabs(u - p / q)",
     "fabs(accept_uniform(draw_word(seed, 0u, (uint32_t)i + 1u, seq, TAG_ACCEPT, 0)) - p / q)",
     [REPORT]),
    ("tree margin: residual mass ignored",
     "fabs(uj - p / R)", "fabs(uj - p)", [REPORT, "-k", "tree"]),
    ("acceptance: p and q swapped",
     "(u * q < p)", "(u * p < q)", [PINS, "-k", "closed_form or first_committed"]),
    ("correction: residual sign flipped",
     "double r = softmax_prob(rt, x, T, mt, st) - softmax_prob(rd, x, T, md, sd);",
     "double r = softmax_prob(rd, x, T, md, sd) - softmax_prob(rt, x, T, mt, st);",
     [PINS, "-k", "correction_follows_residual"]),
    ("bonus: drawn from row k - 1",
     "(int64_t)b * t_sb + (int64_t)k * t_sp};", "(int64_t)b * t_sb + (int64_t)(k - 1) * t_sp};",
     [PINS, "-k", "bonus_follows_last_target_row"]),
    ("softmax: temperature multiplied",
     "return exp(row_at(r, x) / T - m) / s;", "return exp(row_at(r, x) * T - m) / s;",
     [PINS, "-k", "probs_match_library_softmax"]),
    ("Gumbel noise: sign flipped",
     "return -log(-log(u));", "return log(-log(u));", [REPORT, "-k", "recomputed and not tree"]),
    ("greedy: last maximum instead of the first",
     "if (v > best) {", "if (v >= best) {", [PINS, "-k", "greedy_equals_argmax_decoding"]),
    ("Philox: Weyl constant off by two",
     "k[0] += 0x9E3779B9u;", "k[0] += 0x9E3779BBu;", [PINS, "-k", "philox_known_answers"]),
    ("multi-candidate: ties go to the last branch",
     "if (n > best_n) {", "if (n >= best_n) {", [PINS, "-k", "multi_bruteforce"]),
    ("tree: residual mass not reduced after a rejection",
     "R -= p;", ";", [REPORT, "-k", "tree"]),
    ("tree: rejected siblings not excluded from the final draw",
     "if (in_e) continue;", ";", [PINS, "-k", "final_draw_skips_rejected_siblings"]),
    ("tree: bonus tag at inner nodes",
     "has_child ? TAG_CORRECTION : TAG_BONUS", "TAG_BONUS",
     [PINS, "-k", "chain_is_stochastic_verify"]),
]


def build_variant(tmp_path, old=None, new=None):
    with open(SRC) as f:
        src = f.read()
    if old is not None:
        assert src.count(old) == 1, f"mutation site not unique: {old!r}"
        src = src.replace(old, new)
    c = tmp_path / "variant.c"
    c.write_text(src)
    lib = tmp_path / "libvariant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                    "-fno-fast-math", "-o", str(lib), str(c), "-lm"], check=True)
    return str(lib)


def run_pins(lib, args):
    env = dict(os.environ, SV_ORACLE_LIB=lib)
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
           "-m", "not gpu", *args]
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_control_build_passes(tmp_path):
    lib = build_variant(tmp_path)
    r = run_pins(lib, [REPORT])
    assert r.returncode == 0, r.stdout[-2000:]
    r = run_pins(lib, [PINS, "-k", "philox_known_answers or greedy_equals or multi_bruteforce"])
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("name,old,new,args", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, old, new, args):
    lib = build_variant(tmp_path, old, new)
    r = run_pins(lib, args)
    # 1 = tests ran and failed (not a crash, a collection error or no tests)
    assert r.returncode == 1, f"{name}: pins returned {r.returncode}\n{r.stdout[-2000:]}"
