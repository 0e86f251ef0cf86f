"""Host check of the persistent batch-1 decode kernel's geometry (work split,
shared-memory layout and bulk-copy lists), compiled from the kernel's own
source with g++: for every CTA, copies are 16-byte aligned and in bounds,
copies in flight together do not overlap, and every row and scale row the
kernel reads holds the source bytes it wants."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    if shutil.which("g++") is None or not os.path.isdir("/usr/local/cuda/include"):
        pytest.skip("g++ or the CUDA headers are missing")
    exe = str(tmp_path_factory.mktemp("dlc") / "decode_layout_check")
    subprocess.run(["g++", "-O1", "-std=c++17", "-I", "/usr/local/cuda/include", "-o", exe,
                    os.path.join(HERE, "decode_layout_check.cpp")], check=True)
    return exe


@pytest.mark.parametrize("dims", [
    (2816, 704, 2112, 128, 8, 148),     # the 30-layer decode workload on 148 SMs
    (2816, 704, 2112, 128, 8, 160),
    (256, 128, 192, 16, 4, 148),        # the tiny test configuration
    (192, 128, 192, 16, 4, 148),        # an odd number of 64-groups along H
    (512, 192, 320, 32, 8, 100),
    (2048, 512, 1024, 64, 6, 148),
])
def test_layout(checker, dims):
    r = subprocess.run([checker, *map(str, dims)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.startswith("ok"), r.stdout


def test_too_small_grid_is_refused(checker):
    r = subprocess.run([checker, "2816", "704", "2112", "128", "8", "100"], capture_output=True, text=True)
    assert r.returncode == 3 and "does not fit" in r.stdout
