"""The bounds-checked build of the kernels (libqvae_debug.so, -DQVAE_DEBUG_CHECKS):
every TMA load's and store's coordinates and shared-memory range, every
direct store's index and every MMA's accumulator columns are checked before
the access, and a failed check is recorded (qvae_get_error() then returns
QVAE_ERR_BOUNDS).  This runs a cross-section of the parity tests -- CTA pairs
and single CTAs, one to four sub-tiles, one- and three-tap weight stages,
ring depths down to one, the sub-tile hand-off, ragged edges, few CTAs
walking many tiles, every k-step count, streamed chunks, row bands, the
fused and native-precision convolutions and the layer chain -- against the
debug library in a child process; each of those tests asserts
qvae_get_error() == 0 after its calls, so any recorded bounds failure fails
it."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

SELECT = [
    "tests/test_gpu_parity.py::test_conv_tilings_exact",
    "tests/test_gpu_parity.py::test_conv_few_ctas_many_tiles_exact",
    "tests/test_gpu_parity.py::test_conv_one_pair_every_kstep_count_exact",
    "tests/test_gpu_parity.py::test_conv_subtile_handoff_exact",
    "tests/test_gpu_parity.py::test_conv_tiny_and_odd",
    "tests/test_gpu_stream.py",
    "tests/test_gpu_bands.py",
    "tests/test_gpu_fused.py::test_fused_shapes_exact",
    "tests/test_gpu_native.py",
    "tests/test_gpu_graph.py",
]


@pytest.mark.gpu
def test_parity_cross_section_passes_on_the_bounds_checked_build():
    from video_vae_decode_b200 import build as cuda_build

    lib = cuda_build.build(debug=True)
    env = dict(os.environ, QVAE_LIBRARY=lib)
    # the child processes load the bounds-checked build
    probe = subprocess.run([sys.executable, "-c", "from video_vae_decode_b200 import qvae; "
                            "print(qvae.lib().qvae_build_flags(), qvae.LIB_PATH)"],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert probe.returncode == 0, probe.stderr[-2000:]
    flags, path = probe.stdout.split()
    assert flags == "1" and os.path.basename(path) == "libqvae_debug.so", probe.stdout
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                          *SELECT], cwd=ROOT, env=env, capture_output=True, text=True, timeout=3000)
    tail = res.stdout[-3000:] + res.stderr[-2000:]
    assert res.returncode == 0, tail
    assert " passed" in res.stdout and "failed" not in res.stdout, tail
