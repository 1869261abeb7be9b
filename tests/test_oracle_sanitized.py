"""The oracle and the input generators under AddressSanitizer and UndefinedBehaviorSanitizer.

Both C libraries are rebuilt with -fsanitize=address,undefined and the pin suite plus a set of
edge-case workloads (empty prefill, k_q = 0, host pools, early stop, variants, bf16 means,
lookahead) runs on them in a child process with the sanitizer runtimes preloaded: an
out-of-bounds access, a use after free or undefined behaviour in either library fails the
test. CPU only.
"""
import os
import subprocess
import sys
import textwrap

import pytest

import oracle as O
import nosa_synth as syn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FLAGS = ["-O1", "-g", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fsanitize=address,undefined",
         "-fno-omit-frame-pointer"]

DRIVER = textwrap.dedent("""
    import sys
    sys.path.insert(0, {root!r})
    sys.path.insert(0, {tests!r})
    import nosa_synth as syn
    syn._lib = None
    syn._SO = {synth!r}
    syn.build = lambda force=False: syn._SO
    import oracle_pins as P
    lib = {oracle!r}
    P.run_all(lib)
    cs = syn.configs()
    for name in ("tiny", "empty", "short_kq0", "short_kq0_offload", "offload_small", "g8",
                 "bs128_d64", "tiny_stop", "ragged_window_softmax", "ragged_kc16"):
        c = cs[name]
        case = P.check_attention_subset(c, lib) if c.stop_tau == 0 else P.check_early_stop(c, lib)
        P.check_selection_trace(case)
        if c.offload:
            P.check_residency_trace(case)
    for name in ("lookahead_tiny", "lookahead_ragged"):
        case = P.check_attention_subset(cs[name], lib, lookahead=True)
        P.check_selection_trace(case, lookahead=True)
    print("SANITIZED RUN OK")
""")


def _runtime(name):
    p = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True, text=True).stdout.strip()
    return p if os.path.isabs(p) and os.path.exists(p) else None


def test_oracle_and_generators_are_clean_under_sanitizers(tmp_path):
    asan, ubsan = _runtime("libasan.so"), _runtime("libubsan.so")
    if not (asan and ubsan):
        pytest.skip("gcc has no sanitizer runtimes here")
    orc = str(tmp_path / "liboracle_san.so")
    syn_so = str(tmp_path / "libsynth_san.so")
    subprocess.check_call(["gcc", *FLAGS, "-o", orc, O._SRC, "-lm"])
    subprocess.check_call(["gcc", *FLAGS, "-o", syn_so, syn._SRC, "-lm"])
    drv = tmp_path / "drive.py"
    drv.write_text(DRIVER.format(root=ROOT, tests=os.path.join(ROOT, "tests"), synth=syn_so, oracle=orc))
    env = dict(os.environ, LD_PRELOAD=f"{asan}:{ubsan}",
               ASAN_OPTIONS="detect_leaks=0:halt_on_error=1",
               UBSAN_OPTIONS="print_stacktrace=1:halt_on_error=1")
    r = subprocess.run([sys.executable, str(drv)], env=env, capture_output=True, text=True, timeout=1200)
    log = r.stdout + r.stderr
    assert r.returncode == 0 and "SANITIZED RUN OK" in r.stdout, log[-4000:]
    assert "runtime error" not in log and "AddressSanitizer" not in log, log[-4000:]
