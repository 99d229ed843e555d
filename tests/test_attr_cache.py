"""The decode kernel's shared-memory attribute is set per (kernel instance, device): the cache
behind it (csrc/rtp_attr_cache.h, host-only C++) compiled with g++ and driven by a fake setter."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_attr_cache_is_per_device(tmp_path):
    exe = tmp_path / "attr_cache_check"
    subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", "-o", str(exe),
                    os.path.join(HERE, "attr_cache_check.cpp")], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "attr cache: ok" in r.stdout
