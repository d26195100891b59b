"""The library's kernels (SIMT chunk forward with per-chunk states, backward,
decode step, segment combine, layer prologue and epilogue, and the tcgen05
chunk kernel over a host model of its instructions), compiled for the host by
tests/host_emu and run one std::thread per CUDA thread
under AddressSanitizer against the FP64 oracle (gate variants included), and
under ThreadSanitizer for data races; two planted probes (CPU only) show that
the harness reports a shared-memory overrun and a missing barrier.  No GPU: this checks the kernels'
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
    assert "MISMATCH" not in r.stdout and r.stdout.count(" ok ") == 36, r.stdout


_PROBE = r"""
namespace kda { namespace {
__global__ void oob_kernel(float *out, int shift) {
    extern __shared__ float smem[];
    smem[threadIdx.x] = 1.f;
    __syncthreads();
    out[threadIdx.x] = smem[threadIdx.x + shift];
}
__global__ void race_kernel(float *out, int sync) {
    extern __shared__ float smem[];
    smem[threadIdx.x] = (float)threadIdx.x;
    if (sync) __syncthreads();
    out[threadIdx.x] = smem[(threadIdx.x + 1) % blockDim.x];
}
} }
"""
_PROBE_RUN = r"""
extern "C" int probe_oob(float *out, int shift) {
    kda::emu_poison(64 * sizeof(float));   // the launch asks for 64 floats of shared memory
    emu_launch(dim3(1), dim3(64), [&] { kda::oob_kernel(out, shift); });
    return 0;
}
extern "C" int probe_race(float *out, int sync) {
    emu_launch(dim3(1), dim3(64), [&] { kda::race_kernel(out, sync); });
    return 0;
}
"""


def _probe(tmp_path, sanitizer, call):
    import emu_build  # noqa: E402  (tests/host_emu on sys.path)
    text = emu_build.unit_from_text(_PROBE, _PROBE_RUN, poison=(sanitizer == "address"))
    if sanitizer != "address":
        text = text.replace("kda::emu_poison(64 * sizeof(float));", "")
    lib = emu_build.compile_units({"probe.cpp": text}, str(tmp_path / ("probe_%s.so" % sanitizer)), sanitizer)
    code = ("import ctypes, numpy as np\n"
            "lib = ctypes.CDLL(%r)\n"
            "out = np.zeros(64, np.float32)\n"
            "lib.%s\n") % (lib, call)
    env = dict(os.environ, LD_PRELOAD=emu_build.sanitizer_runtime(sanitizer), ASAN_OPTIONS="detect_leaks=0",
               TSAN_OPTIONS="halt_on_error=0", OMP_NUM_THREADS="1")
    return subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_harness_reports_a_shared_memory_overrun(tmp_path):
    """A kernel planted (on the CPU only) with a read past its launch's shared
    memory stops with an AddressSanitizer report; in bounds it runs clean."""
    ok = _probe(tmp_path, "address", "probe_oob(out.ctypes.data_as(ctypes.c_void_p), 0)")
    assert ok.returncode == 0, ok.stderr[-2000:]
    bad = _probe(tmp_path, "address", "probe_oob(out.ctypes.data_as(ctypes.c_void_p), 1)")
    assert bad.returncode != 0 and "AddressSanitizer" in bad.stderr


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_harness_reports_a_missing_barrier(tmp_path):
    """Without the __syncthreads between a shared write and another thread's
    read, ThreadSanitizer reports a data race; with it, none."""
    bad = _probe(tmp_path, "thread", "probe_race(out.ctypes.data_as(ctypes.c_void_p), 0)")
    assert "data race" in bad.stderr and bad.returncode != 0
    ok = _probe(tmp_path, "thread", "probe_race(out.ctypes.data_as(ctypes.c_void_p), 1)")
    assert "data race" not in ok.stderr and ok.returncode == 0, ok.stderr[-2000:]


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_simt_kernels_have_no_data_race():
    """The CUDA-core kernels under ThreadSanitizer."""
    import emu_build  # noqa: E402
    lib = emu_build.build(sanitizer="thread")
    env = dict(os.environ, LD_PRELOAD=emu_build.sanitizer_runtime("thread"), TSAN_OPTIONS="halt_on_error=0",
               OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, os.path.join(HERE, "host_emu", "run_parity.py"), "--races", lib],
                       env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and "data race" not in r.stderr, r.stderr[-4000:]
    assert "race run done" in r.stdout


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_autograd_binding_over_the_emulated_kernels():
    """torch.autograd through kda_chunk, with the library calls served by the
    host-emulated kernels: gradients of every input equal the oracle's."""
    import emu_build  # noqa: E402
    emu_build.build()
    env = dict(os.environ, LD_PRELOAD=emu_build.asan_runtime(), ASAN_OPTIONS="detect_leaks=0")
    r = subprocess.run([sys.executable, os.path.join(HERE, "host_emu", "run_autograd.py")], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert r.stdout.count(" ok ") == 2, r.stdout
