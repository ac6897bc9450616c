"""ep.h is a C header: a C99 program (and the same source as C++) that
includes it compiles with every warning an error, links libep.so, and its
host-only calls behave as the header states.  No call reaches a GPU."""
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_consumer.c")
INCLUDE = os.path.join(ROOT, "include")


@pytest.fixture(scope="module")
def libdir():
    from combine_ep_layout_08_b200 import _build

    return os.path.dirname(_build.build())


def _compile(compiler, std_flags, libdir, out):
    cmd = [compiler, *std_flags, "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", INCLUDE,
           SRC, "-L", libdir, "-lep", "-Wl,-rpath," + libdir, "-o", out]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, " ".join(cmd) + "\n" + r.stderr


@pytest.mark.parametrize("compiler,std", [("gcc", ["-std=c99"]),
                                          ("g++", ["-x", "c++", "-std=c++11"])])
def test_header_compiles_links_and_runs(libdir, tmp_path, oracle, compiler, std):
    if shutil.which(compiler) is None:
        pytest.skip(compiler + " not installed")
    exe = str(tmp_path / "c_consumer")
    _compile(compiler, std, libdir, exe)
    rng = np.random.default_rng(11)
    sizes = [(0, 8, 256), (1, 1, 8), (8192, 8, 256), (128, 8, 256)]
    sizes += [(int(rng.integers(0, 20000)), int(rng.integers(1, 9)),
               int(rng.choice([8, 64, 256]))) for _ in range(20)]
    args = [str(v) for s in sizes for v in s]
    r = subprocess.run([exe, *args], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    got = [int(v) for v in r.stdout.split()]
    assert got == [oracle.recv_rows_bound(T, k, E, 128) for T, k, E in sizes]
