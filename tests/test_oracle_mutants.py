"""Pins are strong enough: each plausible mistake, planted in a temporary copy
of the CPU oracle, is caught by at least one pin (no GPU).

Every mutant is a one-line textual change of ``oracle/binattn_oracle.c``
compiled into a temporary directory. The committed oracle is never modified.
"""
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

MUTANTS = [
    ("sign(0) = -1",
     "return x >= 0.0 ? 1.0 : -1.0;", "return x > 0.0 ? 1.0 : -1.0;"),
    ("signed mean instead of mean |x|",
     "sum_abs += fabs(v);", "sum_abs += v;"),
    ("alpha divided by the padded width",
     "alpha[t] = sum_abs / (double)d;", "alpha[t] = sum_abs / (double)(((d + 31) / 32) * 32);"),
    ("bit order MSB first",
     "|= (uint32_t)1u << (c % 32);", "|= (uint32_t)1u << (31 - c % 32);"),
    ("score sign flipped",
     "s += p->sq[qtok * p->d + c] * p->sk[ktok * p->d + c];",
     "s -= p->sq[qtok * p->d + c] * p->sk[ktok * p->d + c];"),
    ("first channel dropped from the score",
     "for (long c = 0; c < p->d; c++)", "for (long c = 1; c < p->d; c++)"),
    ("scores always against head 0",
     "double s = score_pm1(&p, qtok, bh * (size_t)N + (size_t)j);",
     "double s = score_pm1(&p, qtok, (size_t)j);"),
    ("alpha_k dropped",
     "double logit = softmax_scale * aq * p->ak[ktok] * s;",
     "double logit = softmax_scale * aq * s;"),
    ("alpha_q dropped",
     "double logit = softmax_scale * aq * p->ak[ktok] * s;",
     "double logit = softmax_scale * p->ak[ktok] * s;"),
    ("bias scaled by softmax_scale",
     "logit += load_elem(bias, ORACLE_BF16, ((size_t)h * N + i) * N + j);",
     "logit += softmax_scale * load_elem(bias, ORACLE_BF16, ((size_t)h * N + i) * N + j);"),
    ("bias transposed",
     "((size_t)h * N + i) * N + j", "((size_t)h * N + j) * N + i"),
    ("bias head index ignored",
     "long h = (long)(bh % (size_t)H);", "long h = 0;"),
    ("keys of the wrong head in the softmax",
     "size_t ktok = bh * (size_t)N + (size_t)j;", "size_t ktok = (size_t)j;"),
    ("exp of the negated logit",
     "P[j] = exp(P[j] - m);", "P[j] = exp(m - P[j]);"),
    ("softmax not normalised",
     "P[j] /= z;", "P[j] /= 1.0;"),
    ("V indexed by the query row",
     "o += P[j] * load_elem(v, ORACLE_BF16, (bh * (size_t)N + (size_t)j) * d + c);",
     "o += P[j] * load_elem(v, ORACLE_BF16, qtok * d + c);"),
    ("last key dropped from P.V",
     "for (long j = 0; j < N; j++)\n                o +=", "for (long j = 0; j < N - 1; j++)\n                o +="),
    ("spread without the absolute value",
     "e += P[j] * fabs(load_elem(", "e += P[j] * (load_elem("),
    ("spread not weighted by P",
     "e += P[j] * fabs(", "e += fabs("),
    ("8-bit P on 256 levels",
     "U[j] = nearbyint(255.0 * U[j]);", "U[j] = nearbyint(256.0 * U[j]);"),
    ("8-bit P truncated",
     "U[j] = nearbyint(255.0 * U[j]);", "U[j] = floor(255.0 * U[j]);"),
    ("V code scale over 128",
     "const float sc = mx / 127.0f;", "const float sc = mx / 128.0f;"),
    ("V code truncated",
     "q = nearbyintf((float)load_elem(v, ORACLE_BF16, idx) / sc);",
     "q = truncf((float)load_elem(v, ORACLE_BF16, idx) / sc);"),
    ("8-bit row sum dropped",
     "O_rows[(size_t)r * d + c] = (double)s[bh * (size_t)d + c] * acc / usum;",
     "O_rows[(size_t)r * d + c] = (double)s[bh * (size_t)d + c] * acc / 255.0;"),
    ("relative position with the key and query swapped",
     "const long dy = pi / gw - pj / gw, dx = pi % gw - pj % gw;",
     "const long dy = pj / gw - pi / gw, dx = pj % gw - pi % gw;"),
    ("relative position rows of width gw instead of 2 gw - 1",
     "idx = (dy + gh - 1) * (2 * gw - 1) + (dx + gw - 1);", "idx = (dy + gh - 1) * gw + (dx + gw - 1);"),
    ("class entries swapped",
     "idx = R0;\n", "idx = R0 + 1;\n"),
    ("backward without the softmax's D_i term",
     "dL[(size_t)i * N + j] = P[(size_t)i * N + j] * (dL[(size_t)i * N + j] - Di);",
     "dL[(size_t)i * N + j] = P[(size_t)i * N + j] * dL[(size_t)i * N + j];"),
    ("dV from the transposed probabilities",
     "acc += P[(size_t)i * N + j] * load_elem(dO,", "acc += P[(size_t)j * N + i] * load_elem(dO,"),
    ("ds without softmax_scale",
     "ds[(tok0 + i) * d + c] = softmax_scale * acc;", "ds[(tok0 + i) * d + c] = acc;"),
    ("ds against the query's own signs",
     "acc += dL[(size_t)i * N + j] * p.ak[tok0 + j] * p.sk[(tok0 + j) * d + c];",
     "acc += dL[(size_t)i * N + j] * p.ak[tok0 + j] * p.sq[(tok0 + i) * d + c];"),
    ("dt from the rows of dlogit",
     "acc += dL[(size_t)i * N + j] * p.aq[tok0 + i] * p.sq[(tok0 + i) * d + c];",
     "acc += dL[(size_t)j * N + i] * p.aq[tok0 + i] * p.sq[(tok0 + i) * d + c];"),
    ("dbias of the last batch entry only",
     "dbias[(size_t)h * N * N + e] += dL[e];", "dbias[(size_t)h * N * N + e] = dL[e];"),
    ("dbias transposed",
     "dbias[(size_t)h * N * N + e] += dL[e];",
     "dbias[(size_t)h * N * N + (e % N) * N + e / N] += dL[e];"),
]


@pytest.mark.parametrize("name,find,repl", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, find, repl):
    src = open(oracle.SOURCE).read()
    assert src.count(find) == 1, f"mutation site not unique: {find!r}"
    mut_src = tmp_path / "mutant.c"
    mut_src.write_text(src.replace(find, repl))
    lib = oracle.build(str(mut_src), str(tmp_path / "libmutant.so"))
    orc = oracle.Oracle(lib)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
            break
    assert caught, f"no pin catches the mutant '{name}'"
