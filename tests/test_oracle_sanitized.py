"""The fp64 oracle under AddressSanitizer and UndefinedBehaviorSanitizer: the
C source is built with -fsanitize=address,undefined into a temporary library
and every oracle pin test runs against it in a child process (the sanitizer
runtimes preloaded); an out-of-bounds access, a use after free or an
undefined operation aborts the child."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = ["test_oracle_pins.py", "test_oracle_producer_pins.py", "test_oracle_kl_pins.py",
        "test_oracle_mha_pins.py", "test_oracle_fp8_latent_pins.py"]

CHILD = """
import sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import oracle
oracle._LIB = {lib!r}
oracle.build = lambda force=False: oracle._LIB
import pytest
sys.exit(pytest.main(['-q', '-x', '-p', 'no:cacheprovider'] + {pins!r}))
"""


def _runtime(name):
    out = subprocess.run(["gcc", "-print-file-name=" + name], capture_output=True, text=True).stdout.strip()
    return out if os.path.isabs(out) and os.path.exists(out) else None


def test_oracle_pins_pass_under_asan_and_ubsan(tmp_path):
    asan, ubsan = _runtime("libasan.so"), _runtime("libubsan.so")
    if not asan or not ubsan:
        pytest.skip("gcc has no sanitizer runtimes here")
    lib = str(tmp_path / "dsa_oracle_sanitized.so")
    subprocess.run(["gcc", "-std=c11", "-O1", "-g", "-fsanitize=address,undefined", "-fno-omit-frame-pointer",
                    "-fno-sanitize-recover=undefined", "-fopenmp", "-fPIC", "-shared",
                    os.path.join(ROOT, "oracle", "dsa_oracle.c"), "-o", lib, "-lm"], check=True)
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"), lib=lib,
                        pins=[os.path.join(ROOT, "tests", p) for p in PINS])
    env = dict(os.environ, LD_PRELOAD=asan + " " + ubsan, ASAN_OPTIONS="detect_leaks=0:halt_on_error=1",
               UBSAN_OPTIONS="halt_on_error=1:print_stacktrace=1")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-3000:])
