"""Host-side sanitizers (compute-sanitizer is closed on this machine, so device
code is checked by the bounds of the GPU parity tests; host code here).

* The fp64 oracle built with AddressSanitizer and UndefinedBehaviorSanitizer
  (-fno-sanitize-recover) runs every pin in a child process.
* The tile rules of csrc/tiles.h, which the host API and the kernels share,
  run under both sanitizers in a C++ harness that checks them against a
  brute-force mask.
Any sanitizer report fails the test.
"""
import os
import subprocess
import sys

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "exact_blockwise_head_b200", "csrc")
SAN = ["-fsanitize=address,undefined", "-fno-sanitize-recover=all", "-fno-omit-frame-pointer",
       "-g", "-O1"]


def _runtime(name):
    p = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True, text=True)
    return p.stdout.strip()


def _run_pins_sanitized(tmp_path, source_text):
    src = tmp_path / "attn_oracle.c"
    src.write_text(source_text)
    hdr = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.h")
    (tmp_path / "attn_oracle.h").write_text(open(hdr).read())
    lib = tmp_path / "oracle_san.so"
    subprocess.run(["gcc", "-std=c11", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
                    *SAN, "-o", str(lib), str(src), "-lm"], check=True)
    script = (
        "import sys; sys.path.insert(0, %r)\n"
        "import oracle\n"
        "from tests import _pins\n"
        "orc = oracle.load_variant(%r)\n"
        "for pin in _pins.ALL_PINS:\n"
        "    pin(orc)\n"
        "print('pins ok')\n" % (ROOT, str(lib)))
    env = dict(os.environ)
    env["LD_PRELOAD"] = _runtime("libasan.so")
    env["ASAN_OPTIONS"] = "detect_leaks=0:abort_on_error=1"
    env["UBSAN_OPTIONS"] = "print_stacktrace=1:halt_on_error=1"
    p = subprocess.run([sys.executable, "-c", script], capture_output=True, text=True, env=env,
                       cwd=ROOT, timeout=900)
    return p.returncode, p.stdout, p.stdout + p.stderr


ORACLE_SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")


def test_oracle_pins_under_asan_and_ubsan(tmp_path):
    rc, out, report = _run_pins_sanitized(tmp_path, open(ORACLE_SRC).read())
    assert rc == 0 and "pins ok" in out, report[-3000:]
    assert "AddressSanitizer" not in report and "runtime error" not in report, report[-3000:]


def test_the_sanitizers_are_live(tmp_path):
    """Negative control: a copy of the oracle that reads one key row past the
    end of K must be stopped by AddressSanitizer."""
    src = open(ORACLE_SRC).read()
    planted = src.replace("  for (int64_t j = 0; j < L; ++j) {\n    if (!allowed(i, j, mask_kind, window)) continue;\n    const float* kj = kh + j * d;",
                          "  for (int64_t j = 0; j <= L; ++j) {\n    if (j < L && !allowed(i, j, mask_kind, window)) continue;\n    const float* kj = kh + j * d;", 1)
    assert planted != src
    rc, out, report = _run_pins_sanitized(tmp_path, planted)
    assert rc != 0 and "AddressSanitizer" in report, report[-2000:]


def test_tile_rules_under_asan_and_ubsan(tmp_path):
    exe = tmp_path / "tiles_check"
    subprocess.run(["g++", "-std=c++17", *SAN, "-I", CSRC, "-o", str(exe),
                    os.path.join(HERE, "sanitize", "tiles_check.cpp")], check=True)
    p = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, ASAN_OPTIONS="abort_on_error=1"))
    report = p.stdout + p.stderr
    assert p.returncode == 0 and "0 mismatches" in p.stdout, report[-3000:]
    assert "runtime error" not in report, report[-3000:]
