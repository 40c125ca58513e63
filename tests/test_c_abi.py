"""The boundary is a C ABI: a plain C11 program including only include/*.h
compiles with gcc, links libzero.so and gets the pages' ledger figures for
the running example (no GPU: host-only calls)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "zero_partitioned_mixed_02_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_caller(tmp_path):
    lib = os.path.join(PKG, "libzero.so")
    if not os.path.isfile(lib):
        pytest.skip("libzero.so not built")
    exe = str(tmp_path / "ledger")
    cmd = ["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi_ledger.c"), lib, "-Wl,-rpath," + PKG, "-o", exe]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    f = [float(x) for x in out[0].split()[1:]]
    # [P1] stage table for 7.5B, Nd = 64: 120 / 31.4 / 16.6 / 1.88 GB
    assert f == [120e9, 31.40625e9, 16.640625e9, 1.875e9]
    assert out[1] == "partition 117187500"
    host, dev = (int(x) for x in out[2].split()[1:])
    assert host == 12 * 117187500 and dev == 2 * 7500000000 + 2 * 117187500
    assert out[3] == "bad -1"
    assert out[4] == "peer 104 -1"
