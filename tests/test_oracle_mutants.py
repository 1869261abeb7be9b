"""Plant one mistake at a time in a copy of the oracle and check the pins catch it.

Each mutant is a plausible slip (a dropped term, a wrong sign or index, a
swapped bound). A pin suite that let any of them through would not be pinning
the oracle to the pages.
"""
import os

import pytest

import oracle as O
import oracle_pins as P

MUTANTS = {
    "eviction candidates ignore the alive set":
        ("cand[j] = (uint8_t)(j < N && ps[j] && al[j]);", "cand[j] = (uint8_t)(j < N && ps[j]);"),
    "ties go to the higher index":
        ("return (x->idx < y->idx) ? -1 : (x->idx > y->idx);\n}\n\n/*\n * Top-m",
         "return (x->idx > y->idx) ? -1 : (x->idx < y->idx);\n}\n\n/*\n * Top-m"),
    "block pooling sums instead of max":
        ("if (u > out[j]) out[j] = u;", "out[j] = (out[j] == -INFINITY) ? u : out[j] + u;"),
    "attention drops the scale":
        ("z[nt] = c->scale * dot;", "z[nt] = dot;"),
    "query-aware set may repeat Gamma_e":
        ("cand[j] = (uint8_t)(j < N && !ge[j]);", "cand[j] = (uint8_t)(j < N);"),
    "attention reads one token past the end":
        ("tau < (j + 1) * c->bs && tau < L;", "tau < (j + 1) * c->bs && tau <= L;"),
    "sub-block mean divides by the full size":
        ("out[x] /= (double)(t1 - t0);", "out[x] /= (double)c->s;"),
    "victims are the most recently used":
        ("if (x->lu != y->lu) return (x->lu < y->lu) ? -1 : 1;", "if (x->lu != y->lu) return (x->lu > y->lu) ? -1 : 1;"),
    "eviction never removes a block":
        ("al[j] = 0; /* dropped", "al[j] = 1; /* dropped"),
    "score averages over a fixed 4 rows":
        ("u /= (double)R;", "u /= 4.0;"),
    "tail block not fetched":
        ("need[tail] = 1;", "need[tail] = 0;"),
    "free slots ignored":
        ("if (own[z] < 0) zl[nz++] = z;", "if (own[z] < -1) zl[nz++] = z;"),
    "window pools one sub-block":
        ("if (win && i + 1 < M) n1 =", "if (0 && win && i + 1 < M) n1 ="),
    "window weights its sub-blocks equally":
        ("kb[x] = (n0 * k0[x] + n1 * k1[x]) / (double)(n0 + n1);", "kb[x] = 0.5 * (k0[x] + k1[x]);"),
    "early stop compares the gain with the mass before the block":
        ("const double ratio = dl / l;", "const double ratio = dl / (l - dl + 1e-300);"),
    "early stop visits the blocks in index order":
        ("qsort(it, n, sizeof(orc_item), item_cmp);\n    double* acc", "(void)item_cmp;\n    double* acc"),
    "early stop keeps going past the threshold":
        ("if (ratio < tau_stop) break;", "if (ratio < 0.5 * tau_stop) break;"),
    "bf16 means truncated instead of rounded":
        ("u += 0x7FFFu + ((u >> 16) & 1u);", "u += 0u;"),
    "softmax without its normalizer":
        ("u += exp(z[(size_t)r * M + i] - mx[r]) / den[r];", "u += exp(z[(size_t)r * M + i] - mx[r]);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(O._SRC).read()
    assert src.count(old) == 1, f"mutation site not unique for {name!r}"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    so = O.compile_oracle(str(path), str(tmp_path / f"libm_{abs(hash(name))}.so"))
    with pytest.raises((AssertionError, RuntimeError, ValueError)):
        P.run_all(so)
