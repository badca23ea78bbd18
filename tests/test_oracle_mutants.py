"""The oracle pins have teeth: each plausible slip, planted in a copy of the
oracle's C source and built on the CPU, makes at least one pin in
tests/test_oracle_pins.py fail.  The mutations are applied at every place the
step computes the operation (decode and prefill alike), so that the two modes
stay consistent with each other and only the pins can catch the slip."""
import os
import re
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ODIR = os.path.join(ROOT, "oracle")

# (name, regex, replacement[, "c" for the wrapper file]): each must match at
# least once
MUTANTS = [
    ("gqa_interleaved", r"int gh = h / grp;", "int gh = h % nkv;"),
    ("swiglu_swapped", r"g\[i\] = F\(orc_silu\)\(g\[i\]\) \* u\[i\];", "g[i] = F(orc_silu)(u[i]) * g[i];"),
    ("rope_adjacent_pairs",
     r"R u = v\[i\], w = v\[i \+ h\];\s*v\[i\] = u \* c - w \* s;\s*v\[i \+ h\] = u \* s \+ w \* c;",
     "R u = v[2 * i], w = v[2 * i + 1];\n    v[2 * i] = u * c - w * s;\n    v[2 * i + 1] = u * s + w * c;"),
    ("rope_sign", r"v\[i\] = u \* c - w \* s;\s*v\[i \+ h\] = u \* s \+ w \* c;",
     "v[i] = u * c + w * s;\n    v[i + h] = -u * s + w * c;"),
    ("rope_frequency", r"pow\(theta, -2\.0 \* \(double\)i / \(double\)d\)", "pow(theta, -1.0 * (double)i / (double)d)"),
    ("rope_on_v_too", r"for \(int h = 0; h < nkv; \+\+h\) F\(orc_rope\)\(k \+ h \* d, d, (pos|p), sh->rope_theta\);",
     r"for (int h = 0; h < nkv; ++h) { F(orc_rope)(k + h * d, d, \1, sh->rope_theta); "
     r"F(orc_rope)(v + h * d, d, \1, sh->rope_theta); }"),
    ("rope_position_off_by_one", r"F\(orc_rope\)\(([qk]) \+ h \* d, d, (pos|p), sh->rope_theta\)",
     r"F(orc_rope)(\1 + h * d, d, \2 + 1, sh->rope_theta)"),
    ("rmsnorm_no_eps", r"\(double\)\(ss / \(R\)n \+ \(R\)eps\)", "(double)(ss / (R)n)"),
    ("rmsnorm_no_gamma", r"y\[i\] = x\[i\] \* inv \* F\(orc_bf16_to_real\)\(gamma\[i\]\);", "y[i] = x[i] * inv;"),
    ("norm_weights_swapped", r"L->(attn|ffn)_norm", lambda m: "L->" + ("ffn" if m.group(1) == "attn" else "attn") + "_norm"),
    ("attention_no_scale", r"R scale = \(R\)1 / \(R\)sqrt\(\(double\)d\);", "R scale = (R)1;"),
    ("attention_no_max_shift", r"s\[j\] = \(R\)exp\(\(double\)\(s\[j\] - mx\)\);", "s[j] = (R)exp((double)(s[j]));"),
    ("attention_one_short", r"\b(pos|p) \+ 1, d, o \+ h \* d\);", r"\1, d, o + h * d);"),
    ("v_read_from_k", r"F\(kv_row\)\(kv, 1, l, gh, 0, d\)", "F(kv_row)(kv, 0, l, gh, 0, d)"),
    ("no_attention_residual", r"(F\(orc_matvec\)\(L->wo, o, H, qd, t\);\s*for \(int i = 0; i < H; \+\+i\) x\[i\]) \+= t\[i\];",
     r"\1 = t[i];"),
    ("bf16_truncates", r"nearbyint\(ldexp\(m, 8\)\)", "trunc(ldexp(m, 8))"),
    ("rmsnorm_sum_not_mean", r"\(double\)\(ss / \(R\)n \+ \(R\)eps\)", "(double)(ss + (R)eps)"),
    ("silu_sign", r"\(R\)exp\(-\(double\)z\)", "(R)exp((double)z)"),
    ("final_norm_skipped", r"F\(orc_rmsnorm\)\((x|X \+ \(int64_t\)p \* H), m->final_norm, H, sh->rms_eps, a\);",
     r"for (int i_ = 0; i_ < H; ++i_) a[i_] = (\1)[i_];"),
    ("no_ffn_residual", r"(F\(orc_matvec\)\(L->w_down, g, H, Fd, t\);\s*for \(int i = 0; i < H; \+\+i\) x\[i\]) \+= t\[i\];",
     r"\1 = t[i];"),
    ("embedding_row_shifted", r"m->embed\[\(int64_t\)(token|tokens\[p\]) \* H \+ i\]",
     r"m->embed[(int64_t)((\1 + 1) % sh->vocab) * H + i]"),
    ("lm_head_reads_embedding", r"F\(orc_matvec\)\(m->lm_head,", "F(orc_matvec)(m->embed,"),
    ("argmax_last_maximum", r"if \(x\[i\] > x\[best\]\) best = i;", "if (x[i] >= x[best]) best = i;", "c"),
]


def _build_mutant(tmp, name, pat, rep, where="body"):
    """Copy the oracle source, apply one mutation to the body (or to the
    wrapper, where = "c") and build it with the oracle's own flags."""
    d = os.path.join(tmp, name)
    os.makedirs(d)
    files = {"body": "llama_oracle_body.h", "c": "llama_oracle.c"}
    for f in ("llama_oracle.c", "llama_oracle.h", "llama_oracle_body.h"):
        shutil.copy(os.path.join(ODIR, f), d)
    target = os.path.join(d, files[where])
    new, n = re.subn(pat, rep, open(target).read())
    assert n >= 1, f"mutation {name} does not apply"
    with open(target, "w") as fh:
        fh.write(new)
    so = os.path.join(d, "liboracle.so")
    subprocess.check_call(["gcc", *oracle.CFLAGS, "-o", so, os.path.join(d, "llama_oracle.c"), "-lm"])
    return so


def _pins_fail(so):
    env = dict(os.environ, MK_ORACLE_LIB=so, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(ROOT, "tests", "test_oracle_pins.py"), "-x", "-q",
                        "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-2000:]


def test_unmutated_copy_passes(tmp_path):
    """Control: the same build recipe on the unmodified source passes every pin."""
    so = _build_mutant(str(tmp_path), "control", r"\A", "")
    rc, out = _pins_fail(so)
    assert rc == 0, out


def test_every_planted_mistake_fails_a_pin(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    libs = [(m[0], _build_mutant(str(tmp_path), *m)) for m in MUTANTS]
    with ThreadPoolExecutor(max_workers=4) as ex:
        results = list(ex.map(lambda nl: (nl[0],) + _pins_fail(nl[1]), libs))
    survivors = [name for name, rc, _ in results if rc != 1]
    assert not survivors, {name: out for name, rc, out in results if name in survivors}
