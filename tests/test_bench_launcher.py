"""bench.py --gpus N starts N ranks (CPU, gloo, a stand-in worker).

bench._relaunch is what `python bench.py --gpus N` calls when no launcher set
WORLD_SIZE: it runs the script as N ranks under torch.distributed.run.  Here
the script is tests/launcher_stub.py, which forms a gloo group and has rank
0 print a JSON line; the test checks that two ranks formed, that the max over
ranks saw both, and that the arguments reached the ranks.  Also: a WORLD_SIZE
that disagrees with --gpus is refused before any work.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
STUB = os.path.join(ROOT, "tests", "launcher_stub.py")


def test_gpus_flag_starts_that_many_ranks():
    code = ("import sys; sys.path.insert(0, %r); import bench; "
            "sys.exit(bench._relaunch(2, ['--gpus', '2', '--steps', '5'], script=%r))" % (ROOT, STUB))
    env = dict(os.environ, MASTER_ADDR="127.0.0.1")
    env.pop("WORLD_SIZE", None)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=240, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    out = json.loads(lines[0])
    assert out["n_gpus"] == 2 and out["ranks_formed"] == 2
    assert out["max_over_ranks"] == 2.0
    assert out["argv"] == ["--gpus", "2", "--steps", "5"]


def test_world_size_must_match_gpus():
    env = dict(os.environ, WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "4"], capture_output=True,
                       text=True, timeout=240, env=env)
    assert r.returncode != 0
    assert "WORLD_SIZE=2" in r.stderr
