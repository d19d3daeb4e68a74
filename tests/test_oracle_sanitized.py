"""Every pin of ``test_oracle_pins.py`` against copies of the oracle built with the compiler's
undefined-behaviour and address sanitizers, entirely on the CPU: an out-of-bounds index, an
overflowing integer or float-to-int conversion, or a read past an array in the oracle would
stop the pin with a sanitizer report, even where the pinned value happens to come out right.
The undefined-behaviour copy runs in this process (recovery off, so the first report aborts);
the address-sanitizer copy runs in a child process that preloads the sanitizer runtime."""

import os
import subprocess
import sys

import pytest

import oracle
from tests import test_oracle_pins as pins

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(os.path.dirname(oracle.__file__), "bq_oracle.c")
BASE = ["gcc", "-std=c11", "-O1", "-g", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared", "-Wall",
        "-I", os.path.dirname(SRC)]


def _runtime(name):
    """Path of a sanitizer runtime library, or None when the compiler has none."""
    p = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True, text=True).stdout.strip()
    return p if os.path.isabs(p) and os.path.exists(p) else None


def test_pins_under_undefined_behaviour_sanitizer(tmp_path):
    if _runtime("libubsan.so") is None:
        pytest.skip("no undefined-behaviour sanitizer runtime")
    lib = str(tmp_path / "liboracle_ubsan.so")
    subprocess.run(BASE + ["-fsanitize=undefined,float-cast-overflow", "-fno-sanitize-recover=all", "-o", lib,
                           SRC, "-lm"], check=True)
    o = oracle.Oracle(lib)
    for pin in pins.PINS:
        pin(o)


def test_pins_under_address_sanitizer(tmp_path):
    asan = _runtime("libasan.so")
    if asan is None:
        pytest.skip("no address sanitizer runtime")
    lib = str(tmp_path / "liboracle_asan.so")
    subprocess.run(BASE + ["-fsanitize=address", "-fno-omit-frame-pointer", "-o", lib, SRC, "-lm"], check=True)
    code = ("import sys; sys.path.insert(0, %r)\n"
            "import oracle\n"
            "from tests import test_oracle_pins as pins\n"
            "o = oracle.Oracle(%r)\n"
            "for pin in pins.PINS:\n"
            "    pin(o)\n"
            "print('pins ok', len(pins.PINS))\n") % (ROOT, lib)
    env = dict(os.environ, LD_PRELOAD=asan, ASAN_OPTIONS="detect_leaks=0:abort_on_error=0")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "pins ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
    assert "AddressSanitizer" not in r.stderr, r.stderr[-4000:]
