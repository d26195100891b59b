"""The SIMT forward (with per-chunk states), backward and decode-step kernels,
compiled for the host by tests/host_emu and run one std::thread per CUDA thread
under AddressSanitizer, against the FP64 oracle (gate variants included).  No GPU: this checks the kernels'
index arithmetic, their block-level synchronisation and the gradient they
compute before any device run; the GPU tests remain the parity tests proper."""
import os
import shutil
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "host_emu"))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_simt_kernels_under_host_emulation():
    import emu_build  # noqa: E402  (tests/host_emu on sys.path)
    emu_build.build()
    env = dict(os.environ, LD_PRELOAD=emu_build.asan_runtime(), ASAN_OPTIONS="detect_leaks=0")
    r = subprocess.run([sys.executable, os.path.join(HERE, "host_emu", "run_parity.py")], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-4000:]
    assert "MISMATCH" not in r.stdout and r.stdout.count(" ok ") == 16, r.stdout
