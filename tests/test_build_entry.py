"""build() must work in a tree that has no built library yet: it loads the build
scripts by file path, so nothing imports the package (which loads libvscan.so)
before the library exists."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_build_scripts_load_without_importing_the_package():
    code = (
        "import sys, __graft_entry__ as g\n"
        "m = g._load_build_script('vision_selective_state_b200/build.py', '_b')\n"
        "o = g._load_build_script('oracle/build.py', '_o')\n"
        "assert callable(m.build) and callable(o.build)\n"
        "assert m.LIB.endswith('libvscan.so')\n"
        "assert 'vision_selective_state_b200' not in sys.modules\n"
        "assert 'oracle' not in sys.modules\n"
    )
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
