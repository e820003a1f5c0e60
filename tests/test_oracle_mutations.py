"""The oracle's pins bite: copies of the oracle with one planted, plausible
mistake each must fail the pin suite.  CPU only; mutants are built from a
temporary copy of the C source and never touch the real oracle."""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "zero_oracle.c")

# (name, exact text in the oracle source, replacement)
MUTANTS = [
    ("no bias correction of m", "double mhat = *m / (1.0 - pow(h->beta1, (double)t));",
     "double mhat = *m;"),
    ("no bias correction of v", "double vhat = *v / (1.0 - pow(h->beta2, (double)t));",
     "double vhat = *v;"),
    ("bias correction one step late", "pow(h->beta1, (double)t)", "pow(h->beta1, (double)(t + 1))"),
    ("eps inside the square root", "(sqrt(vhat) + h->eps)", "sqrt(vhat + h->eps)"),
    ("betas swapped in m", "*m = h->beta1 * *m + (1.0 - h->beta1) * g;",
     "*m = (1.0 - h->beta1) * *m + h->beta1 * g;"),
    ("v from |g| not g^2", "*v = h->beta2 * *v + (1.0 - h->beta2) * g * g;",
     "*v = h->beta2 * *v + (1.0 - h->beta2) * fabs(g);"),
    ("decay not scaled by w", "h->weight_decay * *w)", "h->weight_decay)"),
    ("sum instead of mean", "return s / (wsum * S);", "return s / S;"),
    ("loss scale not undone", "return s / (wsum * S);", "return s / wsum;"),
    ("equal weights ignore token counts", "s += (weights ? weights[r] : 1.0) *", "s += 1.0 *"),
    ("ceil ownership", "lo[r] = (uint64_t)(((unsigned __int128)P * r) / R);",
     "lo[r] = (uint64_t)(((unsigned __int128)P * r + R - 1) / R);"),
    ("64-bit overflow in ownership", "lo[r] = (uint64_t)(((unsigned __int128)P * r) / R);",
     "lo[r] = (uint64_t)(((uint64_t)P * r) / R);"),
    ("ties away from zero", "n = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0; /* tie: even */",
     "n = fl + 1.0;"),
    ("skip keeps the scale", "c->loss_scale *= 0.5;", "c->loss_scale *= 1.0;"),
    ("skip still counts a step", "c->skipped += 1;", "c->skipped += 1; c->t += 1;"),
    ("f16 subnormal off by one", "mag = ldexp((double)f, -24);", "mag = ldexp((double)f, -25);"),
    ("accumulation ignores first", "double prev = first ? 0.0 : (double)acc[k];", "double prev = (double)acc[k];"),
    ("accumulation drops the scale", "acc[k] = (float)(prev + scale * g);", "acc[k] = (float)(prev + g);"),
    ("growth one step early", "c->growth_tracker == c->growth_interval)",
     "c->growth_tracker + 1 == c->growth_interval)"),
    ("growth count kept across a skip", "    c->loss_scale *= 0.5;\n    c->growth_tracker = 0;",
     "    c->loss_scale *= 0.5;"),
    ("growth with the check off", "    if (check) {\n        c->growth_tracker += 1;",
     "    if (1) {\n        c->growth_tracker += 1;"),
    ("growth count not restarted after growth", "c->loss_scale *= 2.0;\n            c->growth_tracker = 0;",
     "c->loss_scale *= 2.0;"),
    ("growth triples the scale", "c->loss_scale *= 2.0;", "c->loss_scale *= 3.0;"),
    ("overflow check misses NaN", "if (!isfinite(zo_load(gdtype, grads[r], k))) found |= 1;",
     "if (isinf(zo_load(gdtype, grads[r], k))) found |= 1;"),
]


def _build_mutant(tmp, i, old, new):
    with open(SRC) as f:
        src = f.read()
    assert src.count(old) >= 1, old
    c = os.path.join(tmp, f"m{i}.c")
    with open(c, "w") as f:
        f.write(src.replace(old, new))
    so = os.path.join(tmp, f"m{i}.so")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                           "-ffp-contract=off", "-o", so, c, "-lm"])
    return so


def test_every_planted_mistake_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        procs = []
        for i, (name, old, new) in enumerate(MUTANTS):
            so = _build_mutant(tmp, i, old, new)
            env = dict(os.environ, ORACLE_LIB_OVERRIDE=so, OMP_NUM_THREADS="1")
            p = subprocess.Popen([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                                  os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                                 cwd=ROOT, env=env, stdout=subprocess.PIPE, stderr=subprocess.STDOUT)
            procs.append((name, p))
        survivors = []
        for name, p in procs:
            out, _ = p.communicate(timeout=900)
            if p.returncode == 0:
                survivors.append(name)
        assert not survivors, f"planted mistakes not caught by any pin: {survivors}"
