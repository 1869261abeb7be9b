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
    "query heads mapped to groups interleaved":
        ("const int h = g * G + r;\n      const int L = st->len[gi];\n      const uint16_t* qh",
         "const int h = r * c->Hkv + g;\n      const int L = st->len[gi];\n      const uint16_t* qh"),
    "attention output not normalised":
        ("o[x] = (nt > 0) ? o[x] / den : 0.0;", "o[x] = (nt > 0) ? o[x] : 0.0;"),
    "top-m takes the lowest keys":
        ("  if (x->key > y->key) return -1;\n  if (x->key < y->key) return 1;",
         "  if (x->key < y->key) return -1;\n  if (x->key > y->key) return 1;"),
    "query-aware set of fixed size k_q":
        ("const int mq = (k - ne < N - ne) ? k - ne : N - ne;", "const int mq = (c->k_q < N - ne) ? c->k_q : N - ne;"),
    "S(t) records only Gamma_q":
        ("ps[j] = (uint8_t)(ge[j] || gq[j]);", "ps[j] = (uint8_t)(gq[j]);"),
    "eviction candidates ignore S(t-1)":
        ("cand[j] = (uint8_t)(j < N && ps[j] && al[j]);", "cand[j] = (uint8_t)(j < N && al[j]);"),
    "last_used never refreshed":
        ("if (need[j]) lu[j] = L;", "if (need[j]) lu[j] = lu[j];"),
    "victims paired in least-recently-used order":
        ("for (int j = 0; j < nb; ++j)\n          if (isv[j]) vict[w++] = j;", "for (int r = 0; r < nv; ++r) vict[w++] = vc[r].idx;"),
    "free slots taken from the top":
        ("for (int z = 0; z < c->slots && nz < nm; ++z)\n      if (own[z] < 0) zl[nz++] = z;",
         "for (int z = c->slots - 1; z >= 0 && nz < nm; --z)\n      if (own[z] < 0) zl[nz++] = z;"),
    "tail block always counted a miss":
        ("if (need[j] && bsl[j] < 0) misses[nm++] = j;", "if (need[j] && (bsl[j] < 0 || j == tail)) misses[nm++] = j;"),
    "append refreshes the previous sub-block":
        ("const int i = pos / c->s;\n    sub_mean", "const int i = (pos > 0 ? pos - 1 : 0) / c->s;\n    sub_mean"),
    "sub-block assigned to the next block":
        ("const int j = i / spb;\n      if (u > out[j])", "const int j = (i + 1) / spb;\n      if (j < nb && u > out[j])"),
    "softmax exponent without the row max":
        ("for (int i = 0; i < M; ++i) den[r] += exp(zr[i] - mx[r]);", "for (int i = 0; i < M; ++i) den[r] += exp(zr[i]);"),
    "early stop without rescaling the accumulator":
        ("for (int x = 0; x < d; ++x) acc[x] *= rescale;", "for (int x = 0; x < d; ++x) acc[x] *= 1.0;"),
    "early stop normalises without the stopping block's mass":
        ("if (ratio < tau_stop) break;", "if (ratio < tau_stop) { l -= dl; break; }"),
    "window counts the next sub-block in full":
        ("if (win && i + 1 < M) n1 = (L - (i + 1) * c->s < c->s) ? L - (i + 1) * c->s : c->s;",
         "if (win && i + 1 < M) n1 = c->s;"),
    "eviction set ranked by block scores":
        ("ekey[j] = (double)evict[(size_t)gi * nb + j];", "ekey[j] = scores[(size_t)gi * nb + j];"),
    "scale applied twice in scores":
        ("z[(size_t)r * M + i] = c->scale * dot;", "z[(size_t)r * M + i] = c->scale * c->scale * dot;"),
    "append writes K and V one row late":
        ("memcpy(st->K + tok_off(c, gi, pos), k_new + (size_t)gi * c->d, sizeof(uint16_t) * c->d);\n"
         "    memcpy(st->V + tok_off(c, gi, pos), v_new",
         "memcpy(st->K + tok_off(c, gi, pos + 1 < c->max_blocks * c->bs ? pos + 1 : pos), k_new + (size_t)gi * c->d, sizeof(uint16_t) * c->d);\n"
         "    memcpy(st->V + tok_off(c, gi, pos + 1 < c->max_blocks * c->bs ? pos + 1 : pos), v_new"),
    "append copies V from k_new":
        ("memcpy(st->V + tok_off(c, gi, pos), v_new + (size_t)gi * c->d",
         "memcpy(st->V + tok_off(c, gi, pos), k_new + (size_t)gi * c->d"),
    "last prefill block starts outside S(-1)":
        ("st->prev_sel[(size_t)gi * nb + j] = (uint8_t)(j < n0);", "st->prev_sel[(size_t)gi * nb + j] = (uint8_t)(j < n0 - 1);"),
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


# Slips in the oracle's Python driver (the SparDA lookahead order of run_case). Each runs the
# lookahead pins in a child process on a copy of the oracle package with one change.
PY_MUTANTS = {
    "lookahead appends before selecting":
        [("        if not lookahead:\n            orc.append(inp.k_new[t], inp.v_new[t])",
          "        if True:\n            orc.append(inp.k_new[t], inp.v_new[t])"),
         ("        if lookahead:\n            orc.append(inp.k_new[t], inp.v_new[t])",
          "        if False:\n            orc.append(inp.k_new[t], inp.v_new[t])")],
    "lookahead plans residency after the append":
        [("        miss = orc.residency(sel)\n        if lookahead:\n            orc.append(inp.k_new[t], inp.v_new[t])",
          "        if lookahead:\n            orc.append(inp.k_new[t], inp.v_new[t])\n        miss = orc.residency(sel)")],
    "lookahead attends before the append":
        [("        if lookahead:\n            orc.append(inp.k_new[t], inp.v_new[t])\n        used = None",
          "        used = None"),
         ("            out = orc.attend(q16, sel)\n",
          "            out = orc.attend(q16, sel)\n            if lookahead:\n                orc.append(inp.k_new[t], inp.v_new[t])\n")],
}

_PY_DRIVER = """
import sys
sys.path.insert(0, {pkg!r})
sys.path.insert(1, {root!r})
sys.path.insert(2, {tests!r})
import oracle as O
assert O.__file__.startswith({pkg!r}), O.__file__
import nosa_synth as syn
import oracle_pins as P
P.check_lookahead_dense_sdpa()
cs = syn.configs()
for name in ("lookahead_tiny", "lookahead_ragged", "lookahead_small"):
    case = P.check_attention_subset(cs[name], lookahead=True)
    P.check_selection_trace(case, lookahead=True)
    if case.cfg.offload:
        P.check_residency_trace(case, lookahead=True)
print("LOOKAHEAD PINS PASS")
"""


def _run_py_mutant(tmp_path, edits):
    import shutil
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = tmp_path / "pkg"
    dst = pkg / "oracle"
    dst.mkdir(parents=True)
    src_dir = os.path.join(root, "oracle")
    for f in ("__init__.py", "nosa_oracle.c"):
        shutil.copy(os.path.join(src_dir, f), dst / f)
    shutil.copy(O.build(), dst / "libnosa_oracle.so")
    text = (dst / "__init__.py").read_text()
    for old, new in edits:
        assert text.count(old) == 1, f"mutation site not unique: {old[:60]!r}"
        text = text.replace(old, new)
    (dst / "__init__.py").write_text(text)
    drv = tmp_path / "drive.py"
    drv.write_text(_PY_DRIVER.format(pkg=str(pkg), root=root, tests=os.path.join(root, "tests")))
    return subprocess.run([sys.executable, str(drv)], capture_output=True, text=True, timeout=900)


def test_lookahead_pins_pass_on_the_unchanged_driver(tmp_path):
    r = _run_py_mutant(tmp_path, [])
    assert r.returncode == 0 and "LOOKAHEAD PINS PASS" in r.stdout, r.stderr[-3000:]


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_lookahead_pins_catch_driver_mutant(name, tmp_path):
    r = _run_py_mutant(tmp_path, PY_MUTANTS[name])
    assert r.returncode != 0 and "LOOKAHEAD PINS PASS" not in r.stdout, r.stdout[-2000:]
    assert "AssertionError" in r.stderr or "ValueError" in r.stderr, r.stderr[-3000:]
