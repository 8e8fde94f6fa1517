"""The oracle's C source is ISO C11 that compiles without a single warning.

The oracle library is built with every warning an error, so a compiler
release that turns a warning into an error (an implicit declaration, for
one) cannot silently change what every parity test runs against.
"""
import os
import subprocess
import tempfile

import oracle

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "fp8_oracle.c")


def _compile(path):
    return subprocess.run(["gcc", "-fsyntax-only", "-fopenmp"] + oracle.WARN_FLAGS + [path],
                          capture_output=True, text=True)


def test_oracle_compiles_without_warnings():
    r = _compile(SRC)
    assert r.returncode == 0 and r.stderr == "", r.stderr


def test_the_flags_reject_an_implicit_declaration():
    # the same flags on the oracle source with one call moved ahead of its
    # declaration: the build must fail
    src = open(SRC).read()
    planted = "static void planted_early_call(void) { orc_quant_rows(0, 0, 0, 0, 0, 0, 0); }\n"
    anchor = "/* ---------------------------------------------------------------- formats */"
    assert anchor in src
    with tempfile.TemporaryDirectory() as tmp:
        p = os.path.join(tmp, "o.c")
        open(p, "w").write(src.replace(anchor, planted + anchor, 1))
        r = _compile(p)
    assert r.returncode != 0 and "implicit" in r.stderr
