"""bench.py --impl reference launched as two ranks (CPU only, as torchrun sets
RANK / WORLD_SIZE): rank 0 alone runs the oracle and prints one JSON line; the
other rank exits 0 at once, with no collective step that could time out while
rank 0 works."""
import json
import os
import subprocess
import sys
from pathlib import Path

ROOT = Path(__file__).resolve().parent.parent


def test_reference_arm_under_two_ranks():
    from paged_kv_cache_331_b200 import build as B
    B.build()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
                   MASTER_PORT="29511")
        procs.append(subprocess.Popen([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "2",
                                       "--warmup", "3", "--reference-seconds", "2"], cwd=ROOT, env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=600) for p in procs]
    assert [p.returncode for p in procs] == [0, 0], [o[1][-2000:] for o in outs]
    assert outs[1][0].strip() == ""
    lines = [ln for ln in outs[0][0].splitlines() if ln.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["value"] > 0 and rec["e2e"]["h2d_bytes_per_step"] == 0
