"""The package's helper submodules import without loading the CUDA library.

`build` must work in a checkout where the library has not been compiled yet,
and the oracle's timing leg of the benchmark uses `synth` without mapping
the library; both go through the package's lazy attribute hook.
"""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_submodules_do_not_load_the_binding():
    code = ("import sys\n"
            "from paged_kv_cache_402_b200 import build, synth, trace\n"
            "import paged_kv_cache_402_b200.synth\n"
            "assert 'paged_kv_cache_402_b200.binding' not in sys.modules, 'binding loaded'\n"
            "maps = open('/proc/self/maps').read()\n"
            "assert 'libpagedattn' not in maps, 'library mapped'\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr


def test_binding_names_still_resolve():
    import paged_kv_cache_402_b200 as pa
    assert callable(pa.pa_decode) and pa.PA_PARTITION_TOKENS == 512


def test_reference_arm_maps_only_the_oracle():
    """`bench.py --impl reference` times the oracle alone: the CUDA library is
    never mapped into that process."""
    code = ("import runpy, sys\n"
            "sys.argv = ['bench.py', '--impl', 'reference', '--steps', '1', '--warmup', '3']\n"
            "runpy.run_path('bench.py', run_name='__main__')\n"
            "maps = open('/proc/self/maps').read()\n"
            "assert 'libpagedattn' not in maps, 'library mapped'\n"
            "assert 'liboracle' in maps, 'oracle not mapped'\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    assert '"impl": "reference"' in r.stdout
