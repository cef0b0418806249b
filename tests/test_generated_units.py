"""The instantiation units under csrc/ are exactly what gen_instances.py
writes: the generator, run on its own in a scratch directory, produces the
same set of files with the same bytes, so no table can fall out of step with
the dispatch code that indexes it."""
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_recurrent_state_decode_b200", "csrc")


def test_generated_units_are_current(tmp_path):
    shutil.copy(os.path.join(CSRC, "gen_instances.py"), tmp_path)
    subprocess.run([sys.executable, str(tmp_path / "gen_instances.py")], check=True,
                   capture_output=True, text=True)
    made = sorted(f for f in os.listdir(tmp_path) if f.startswith("qstate_inst_"))
    have = sorted(f for f in os.listdir(CSRC) if f.startswith("qstate_inst_"))
    assert made == have
    for f in made:
        with open(tmp_path / f, "rb") as a, open(os.path.join(CSRC, f), "rb") as b:
            assert a.read() == b.read(), f
