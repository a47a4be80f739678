"""The C boundary from plain C (CPU): tests/c_consumer.c includes
include/libmoe.h as C99 with warnings as errors, links lib/libmoe.so and
runs the calls that need no GPU."""
import os
import subprocess

import pytest

from mixture_experts_routing_top_b200 import build as B
from oracle import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def consumer():
    so = B.build()
    out = os.path.join(B.BUILD, "c_consumer")
    src = os.path.join(ROOT, "tests", "c_consumer.c")
    lib_dir = os.path.dirname(so)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    src, "-o", out, "-L", lib_dir, "-l:libmoe.so", "-Wl,-rpath," + lib_dir], check=True,
                   capture_output=True, text=True)
    return out


def test_c_program_uses_the_boundary(consumer):
    r = subprocess.run([consumer], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    got = dict(line.split(" ", 1) for line in r.stdout.strip().splitlines())
    assert got["abi"] == "1"
    assert got["status"] == "unsupported shape or alignment"
    assert int(got["capacity"]) == O.capacity(1.25, 8192, 2, 8) == 2560
    assert got["max_rows"].split() == [str(min(8192 * 2, 8 * 2560)), str(4096 * 8)]
    assert got["ws"] == "1"
    assert got["k>E"] == "1"            # MOE_ERR_ARG
    assert got["T=0"] == "0"            # MOE_OK, nothing launched
