"""The oracle's C code under AddressSanitizer and UndefinedBehaviorSanitizer, no GPU.

The oracle is built a second time with -fsanitize=address,undefined and every
pin file runs against that build in a fresh interpreter (the sanitizer runtimes
preloaded), so an out-of-bounds index, a use after free or an undefined shift
in any oracle function fails here even where the numbers happen to come out
right.
"""
import os
import subprocess
import sys
import textwrap

import pytest

from oracle import build as obuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_FILES = ["test_oracle.py", "test_oracle_relpos.py", "test_oracle_bwd.py",
             "test_oracle_indexer.py", "test_oracle_paged.py", "test_oracle_splitkv.py",
             "test_oracle_properties.py"]

# -s: the inner pytest leaves stderr alone, so a sanitizer report reaches the caller
RUNNER = textwrap.dedent("""
    import sys
    sys.path.insert(0, {root!r})
    import oracle
    from oracle import build
    lib = oracle.load({lib!r})
    oracle._lib, oracle._lib_path = lib, build.LIB
    import pytest
    sys.exit(pytest.main(["-x", "-q", "-s", "-p", "no:cacheprovider"] + {tests!r}))
""")


def runtime(name):
    path = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True,
                          text=True).stdout.strip()
    return path if os.path.isabs(path) and os.path.exists(path) else None


def test_pins_pass_under_sanitizers(tmp_path):
    asan, ubsan = runtime("libasan.so"), runtime("libubsan.so")
    if not (asan and ubsan):
        pytest.skip("gcc sanitizer runtimes not installed")
    lib = obuild.build(out=str(tmp_path / "liboracle_san.so"),
                       extra=["-g", "-O1", "-fno-omit-frame-pointer",
                              "-fsanitize=address,undefined", "-fno-sanitize-recover=undefined"])
    tests = [os.path.join(ROOT, "tests", f) for f in PIN_FILES]
    env = dict(os.environ, LD_PRELOAD=f"{asan} {ubsan}", OMP_NUM_THREADS="2",
               ASAN_OPTIONS="detect_leaks=0", UBSAN_OPTIONS="print_stacktrace=1")
    res = subprocess.run([sys.executable, "-c", RUNNER.format(root=ROOT, lib=lib, tests=tests)],
                         capture_output=True, text=True, cwd=str(tmp_path), env=env, timeout=900)
    assert res.returncode == 0 and "runtime error" not in res.stderr, (
        res.stderr[:3000] + res.stdout[-2000:])
