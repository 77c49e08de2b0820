"""Each plausible slip in the oracle must fail at least one pin.

A mutant is the oracle's C source with one textual change (a dropped term, a wrong sign,
index, divisor or operand), compiled to a temporary library; the pins run against it in a
child process, which must fail. The unchanged source, compiled the same way, must pass.
CPU only; the mutants are planted in copies of the oracle, never in the CUDA path.
"""
import os
import subprocess
import sys

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

# (name, [(text, replacement, count)]) -- count 0 replaces every occurrence
MUTANTS = [
    ("means divide by rows not tokens",
     [("xm[((int64_t)b * R + r) * C + c] = sum / rs;", "xm[((int64_t)b * R + r) * C + c] = sum / hr;", 1)]),
    ("means number regions column-major",
     [("const int r = ry * n_win + rx;", "const int r = rx * n_win + ry;", 1)]),
    ("means drop the last token of a region",
     [("for (int xx = 0; xx < wr; ++xx)\n                            sum +=",
       "for (int xx = 0; xx < wr - (yy == hr - 1); ++xx)\n                            sum +=", 1)]),
    ("affinity scaled by R instead of C",
     [("const double scale = 1.0 / sqrt((double)C);", "const double scale = 1.0 / sqrt((double)R);", 1)]),
    ("affinity with a transposed operand",
     [("* km[((int64_t)b * R + s) * C + c];", "* km[((int64_t)b * R + r) * C + c];", 1)]),
    ("top-k ascending",
     [("if (a->value > b->value) return -1;", "if (a->value > b->value) return 1;", 1),
      ("if (a->value < b->value) return 1;", "if (a->value < b->value) return -1;", 1)]),
    ("ties to the higher region",
     [("return (a->region < b->region) ? -1 : (a->region > b->region ? 1 : 0);",
       "return (a->region > b->region) ? -1 : (a->region < b->region ? 1 : 0);", 1)]),
    ("NaN ranked first",
     [("if (a_nan != b_nan) return a_nan ? 1 : -1;", "if (a_nan != b_nan) return a_nan ? -1 : 1;", 1)]),
    ("attention scaled by C instead of head_dim",
     [("const double scale = 1.0 / sqrt((double)hd);", "const double scale = 1.0 / sqrt((double)C);", 1)]),
    ("attention without the scale",
     [("logits[n] = scale * dot;", "logits[n] = dot;", 1)]),
    ("values taken from k",
     [("const double *vt = v + token_offset", "const double *vt = k + token_offset", 1)]),
    ("every head uses head 0's query",
     [("dot += qt[c0 + c] * kt[c0 + c];", "dot += qt[c] * kt[c0 + c];", 1)]),
    ("keys from the query's own region",
     [("const int sy = routed[j] / n_win, sx = routed[j] % n_win;",
       "const int sy = r / n_win, sx = r % n_win;", 0)]),
    ("query region transposed",
     [("const int r = (y / hr) * n_win + (x / wr);", "const int r = (x / wr) * n_win + (y / hr);", 1)]),
    ("softmax denominator drops the first key",
     [("for (int i = 0; i < n; ++i) {\n            logits[i] = exp(logits[i] - max_logit);\n            denom += logits[i];",
       "for (int i = 0; i < n; ++i) {\n            logits[i] = exp(logits[i] - max_logit);\n            if (i) denom += logits[i];", 1)]),
    ("softmax without the exponential",
     [("logits[i] = exp(logits[i] - max_logit);", "logits[i] = logits[i] - max_logit + 1.0;", 1)]),
    ("last routed region ignored",
     [("for (int j = 0; j < topk; ++j) {\n            const int sy = routed[j] / n_win, sx = routed[j] % n_win;\n            for (int yy = 0; yy < hr; ++yy)\n                for (int xx = 0; xx < wr; ++xx) {\n                    const double *vt",
       "for (int j = 0; j < topk - (topk > 1); ++j) {\n            const int sy = routed[j] / n_win, sx = routed[j] % n_win;\n            for (int yy = 0; yy < hr; ++yy)\n                for (int xx = 0; xx < wr; ++xx) {\n                    const double *vt", 1)]),
    # per-head routing and attention
    ("per-head affinity scaled by C",
     [("const double head_scale = 1.0 / sqrt((double)hd);", "const double head_scale = 1.0 / sqrt((double)C);", 1)]),
    ("per-head routing without the topk clamp",
     [("const int k_eff = topk < R ? topk : R;", "const int k_eff = topk;", 1)]),
    ("per-head keys from head 0",
     [("km[((int64_t)b * R + s2) * C + h * hd + d];", "km[((int64_t)b * R + s2) * C + d];", 1)]),
    ("every head attends with head 0's index rows",
     [("(idx_heads > 1 ? h : 0)", "0", 1)]),
    # LePE
    ("LePE without the residual",
     [("y[token_offset(b, i, j, H, W, C) + c] = x[token_offset(b, i, j, H, W, C) + c] + conv;",
       "y[token_offset(b, i, j, H, W, C) + c] = conv;", 1)]),
    ("LePE without the bias", [("double conv = bias[c];", "double conv = 0.0;", 1)]),
    ("LePE with a flipped filter (convolution, not correlation)",
     [("w[(int64_t)c * 25 + di * 5 + dj]", "w[(int64_t)c * 25 + (4 - di) * 5 + (4 - dj)]", 1)]),
    ("LePE with padding 1",
     [("const int ii = i + di - 2, jj = j + dj - 2;", "const int ii = i + di - 1, jj = j + dj - 1;", 1)]),
    # backward
    ("backward without the softmax centring term",
     [("const double ds = p[i] * (dp[i] - pdp);", "const double ds = p[i] * dp[i];", 1)]),
    ("backward dk without the scale",
     [("dk[key[i] + c0 + c] += inv_sqrt_hd * ds", "dk[key[i] + c0 + c] += ds", 1)]),
    ("backward dq from the values",
     [("dq[qo + c0 + c] += inv_sqrt_hd * ds * k[key[i] + c0 + c];",
       "dq[qo + c0 + c] += inv_sqrt_hd * ds * v[key[i] + c0 + c];", 1)]),
    ("backward dv from the unnormalised weights",
     [("p[i] /= denom;", "p[i] /= 1.0;", 1)]),
    # auto_pad
    ("auto_pad pads at the top and left",
     [("xp[token_offset(b, i, j, Hp, Wp, C) + c] = x[token_offset(b, i, j, H, W, C) + c];",
       "xp[token_offset(b, i + Hp - H, j + Wp - W, Hp, Wp, C) + c] = x[token_offset(b, i, j, H, W, C) + c];", 1)]),
    ("auto_pad crops the bottom right",
     [("out[token_offset(b, i, j, H, W, C) + c] = op[token_offset(b, i, j, Hp, Wp, C) + c];",
       "out[token_offset(b, i, j, H, W, C) + c] = op[token_offset(b, i + Hp - H, j + Wp - W, Hp, Wp, C) + c];", 1)]),
    ("auto_pad rounds down", [("return (n + n_win - 1) / n_win * n_win;", "return n / n_win * n_win;", 1)]),
]


def _build(tmp_path, name, edits):
    with open(oracle.SOURCE) as f:
        src = f.read()
    for text, repl, count in edits:
        n = src.count(text)
        assert n >= 1 and (count == 0 or n == count), f"mutation text for {name!r} found {n} times"
        src = src.replace(text, repl)
    path = tmp_path / "mutant.c"
    path.write_text(src)
    return oracle.compile_oracle(str(path), str(tmp_path / "libmutant.so"))


def _pins_pass(lib):
    env = dict(os.environ, OMP_NUM_THREADS="2", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, os.path.join(HERE, "oracle_pins.py"), lib], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=300)
    return r.returncode == 0, (r.stdout + r.stderr)[-400:]


def test_unmutated_copy_passes(tmp_path):
    ok, log = _pins_pass(_build(tmp_path, "control", []))
    assert ok, log


@pytest.mark.parametrize("name,edits", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, edits):
    ok, _ = _pins_pass(_build(tmp_path, name, edits))
    assert not ok, f"no pin catches the mutant: {name}"
