"""CPU test of the file-backed store's reader pool (csrc/readpool.h): a read
that outlasts the caller's limit is abandoned with its thread still writing
its buffer; the pool must refuse new batches until that read ends, drop its
late result, and then work normally with a larger job table.  pread is
replaced by a stub (a blocking descriptor stands in for a slow device); the
program is built with the address and undefined-behaviour sanitizers, so an
out-of-bounds write by the late read fails the test."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "expert_streaming_decode_b200", "csrc")


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_read_pool_straggler_and_failures(tmp_path):
    exe = str(tmp_path / "readpool_test")
    cmd = ["g++", "-std=c++17", "-O1", "-g", "-pthread", "-fsanitize=address,undefined", "-fno-sanitize-recover=all",
           "-I", CSRC, os.path.join(HERE, "cpp", "readpool_test.cpp"), "-o", exe]
    subprocess.run(cmd, check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "readpool ok" in r.stdout, r.stdout + r.stderr
