"""Mutation check of the oracle's pins (test infrastructure).

Each entry below plants one plausible mistake in a temporary copy of
zero_oracle.c: a dropped term, a wrong coefficient, a moved epsilon, an
off-by-one in a rule. The script builds each copy and runs the oracle's pin
tests (tests/test_oracle_*.py: pages, closed forms, library routines, brute
force) against it through ZERO_ORACLE_LIB. A mutant that the pins do not
reject means a pin is missing, and the script exits non-zero.

    python oracle/mutation_check.py            # every mutant
    python oracle/mutation_check.py -k clip    # mutants whose name contains "clip"
"""
import argparse
import os
import subprocess
import sys
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "zero_oracle.c")

# (name, exact text in zero_oracle.c, replacement)
MUTANTS = [
    ("clip_without_min", "coef = (float)(cd < 1.0 ? cd : 1.0);", "coef = (float)cd;"),
    ("clip_without_eps", "sqrt(nrm) + 1e-6", "sqrt(nrm)"),
    ("accumulation_dropped", "acc[e] = acc[e] + part[e];", "acc[e] = part[e];"),
    ("divisor_missing",
     "c.inv = (float)(1.0 / (((double)R * opts->grad_divisor) * (double)scale));",
     "c.inv = (float)(1.0 / ((double)R * (double)scale));"),
    ("weight_decay_dropped", "float pp = master[e] * c.dec;", "float pp = master[e];"),
    ("beta2_coefficient", "c.omb2 = (float)(1.0 - hp->beta2);", "c.omb2 = (float)(1.0 - hp->beta1);"),
    ("bias_correction_no_sqrt", "c.bc2s = (float)sqrt(1.0 - pow(hp->beta2, (double)t));",
     "c.bc2s = (float)(1.0 - pow(hp->beta2, (double)t));"),
    ("eps_inside_sqrt", "float den = sqrtf(vv) / c->bc2s + c->epsf;",
     "float den = sqrtf(vv + c->epsf) / c->bc2s;"),
    ("fsm_growth_factor", "st->scale = st->scale * st->growth_factor;", "st->scale = st->scale * 4.0f;"),
    ("fsm_t_on_skip", "st->last_skipped = skip;", "st->last_skipped = skip; if (skip) st->t += 1;"),
    ("reduction_order", "s = s + oracle_half_to_float(grads[(int64_t)r * P + e], dtype);",
     "s = oracle_half_to_float(grads[(int64_t)r * P + e], dtype) + s * 1.0000001f;"),
    ("bucket_rule_strict", "total + numels[lo_k - 1] <= bucket_elems",
     "total + numels[lo_k - 1] < bucket_elems"),
    ("shard_rounding", "int64_t S = round_up((L + R - 1) / R, 8);", "int64_t S = round_up(L / R, 8);"),
    ("fp16_round_half_up", "double n = nearbyint(a / q);", "double n = floor(a / q + 0.5);"),
    ("memory_stage2", "case 2: return param_b * psi + (grad_b + optim_b) * psi / N;",
     "case 2: return (param_b + grad_b) * psi + optim_b * psi / N;"),
    ("memory_stage3_unsharded_params", "case 3: return (param_b + grad_b + optim_b) * psi / N;",
     "case 3: return param_b * psi + (grad_b + optim_b) * psi / N;"),
    ("momentum_gradient_term", "float mm = c->b1f * *m + c->omb1 * g;", "float mm = c->b1f * *m + g;"),
    ("update_sign", "    pp = pp - c->ss * (mm / den);\n    *p = pp;", "    pp = pp + c->ss * (mm / den);\n    *p = pp;"),
    ("bias_correction1_dropped", "c.ss = (float)(hp->lr / (1.0 - pow(hp->beta1, (double)t)));",
     "c.ss = (float)hp->lr;"),
    ("bias_correction_step_offset", "c.bc2s = (float)sqrt(1.0 - pow(hp->beta2, (double)t));",
     "c.bc2s = (float)sqrt(1.0 - pow(hp->beta2, (double)t + 1.0));"),
    ("unscale_without_R", "c.inv = (float)(1.0 / ((double)R * (double)scale));",
     "c.inv = (float)(1.0 / (double)scale);"),
    ("overflow_misses_inf", "if (!isfinite(s)) overflow = 1;", "if (isnan(s)) overflow = 1;"),
    ("backoff_without_floor", "st->scale = (s < st->min_scale) ? st->min_scale : s;", "st->scale = s;"),
    ("good_not_reset_on_overflow", "st->good = 0;\n            skip = 1;", "skip = 1;"),
    ("growth_interval_off_by_one", "if (st->good >= st->growth_interval)", "if (st->good > st->growth_interval)"),
    ("subnormal_quantum", "if (E < f->emin) E = f->emin;", "if (E < f->emin) return sign;"),
    ("nan_encoded_as_inf", "return (uint16_t)(sign | exp_all | (1u << (f->mant_bits - 1)));",
     "return (uint16_t)(sign | exp_all);"),
    ("fp16_overflow_threshold", "FMT_FP16 = {10, 5, 15, -14, 15}", "FMT_FP16 = {10, 5, 15, -14, 16}"),
    ("subnormal_decode_scale", "val = ldexp((double)frac, f->emin - f->mant_bits);",
     "val = ldexp((double)frac, f->emin - f->mant_bits - 1);"),
    ("tensor_alignment_ignored", "offsets[k] = round_up(cursor, align);", "offsets[k] = cursor;"),
    ("last_bucket_without_padding", "bucket_hi[nb] = (hi_k == n - 1) ? T : offsets[hi_k + 1];",
     "bucket_hi[nb] = (hi_k == n - 1) ? L : offsets[hi_k + 1];"),
    ("layer_end_includes_padding", "layer_hi[j] = (j + 1 < n) ? offsets[j + 1] : L;",
     "layer_hi[j] = (j + 1 < n) ? offsets[j + 1] : T;"),
    ("clip_not_applied", "float g = (acc[e] * c.inv) * coef;", "float g = acc[e] * c.inv;"),
    ("sharded_flag_one_owner", "overflow |= flag_o;", "overflow = flag_o;"),
    ("sharded_rank_stride", "s = s + oracle_half_to_float(grads[(int64_t)r * T + i], dtype);",
     "s = s + oracle_half_to_float(grads[(int64_t)r * S + i], dtype);"),
    ("sample_norm_ignored", "if (norm_sq_all) nrm = *norm_sq_all;", "(void)norm_sq_all;"),
]


def run_one(name, old, new, tmp):
    src = open(SRC).read()
    if src.count(old) != 1:
        return "stale", f"the text to mutate occurs {src.count(old)} times"
    c = os.path.join(tmp, name + ".c")
    so = os.path.join(tmp, name + ".so")
    with open(c, "w") as f:
        f.write(src.replace(old, new, 1))
    cc = subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-I", HERE,
                         c, "-o", so, "-lm"], capture_output=True, text=True)
    if cc.returncode != 0:
        return "stale", cc.stderr.strip().splitlines()[-1] if cc.stderr else "compile failed"
    env = dict(os.environ, ZERO_ORACLE_LIB=so)
    pins = sorted(os.path.join("tests", f) for f in os.listdir(os.path.join(ROOT, "tests"))
                  if f.startswith("test_oracle_") and f.endswith(".py"))
    r = subprocess.run([sys.executable, "-m", "pytest", *pins, "-q", "-x", "-m", "not gpu",
                        "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    last = r.stdout.strip().splitlines()[-1] if r.stdout.strip() else ""
    return ("caught" if r.returncode != 0 else "SURVIVED"), last


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("-k", default="", help="only mutants whose name contains this")
    args = ap.parse_args()
    bad = 0
    with tempfile.TemporaryDirectory() as tmp:
        for name, old, new in MUTANTS:
            if args.k not in name:
                continue
            verdict, detail = run_one(name, old, new, tmp)
            print(f"{name:28s} {verdict:9s} {detail}", flush=True)
            bad += verdict != "caught"
    sys.exit(1 if bad else 0)


if __name__ == "__main__":
    main()
