"""Both decode arithmetic paths (CUDA cores and tensor cores) and both split-KV
modes (one CTA per partition with a fused merge; one warp per partition with a
second-pass merge kernel) against the oracle for every supported group size,
head_dim and storage type, 16-bit and 8-bit caches, with NaN patterns planted
in the unused slots of every partly filled block."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("split", ["cta", "warp"])
@pytest.mark.parametrize("path", ["cuda_cores", "tensor"])
def test_decode_path_parity(path, split):
    env = dict(os.environ, PA_DECODE_PATH=path, PA_DECODE_SPLIT=split)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "path_check.py")], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "ok" in r.stdout
