"""Host logic of the multi-GPU benchmark on CPU ranks (gloo, world size 2):
the decode has no exchange step, so the only cross-rank work is the barrier
and the max-over-ranks timing, and the reference arm runs on rank 0 alone."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import os, sys, json
sys.path.insert(0, os.environ["ROOT"])
import torch.distributed as dist
dist.init_process_group("gloo")
import bench
r = dist.get_rank()
vals = bench.max_over_ranks([10.0 + r, 5.0 - r, 3.0 * (r + 1)])
dist.barrier()
with open(os.path.join(os.environ["OUT_DIR"], f"rank{r}.json"), "w") as f:
    json.dump({"rank": r, "vals": vals}, f)
dist.destroy_process_group()
"""


def _torchrun(script, nproc=2, extra_env=None):
    env = dict(os.environ, ROOT=ROOT, **(extra_env or {}))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={nproc}",
           "--master-addr=127.0.0.1", "--master-port=29531", *script]
    return subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=240)


def test_max_over_ranks_gloo(tmp_path):
    f = tmp_path / "w.py"
    f.write_text(WORKER)
    p = _torchrun([str(f)], extra_env={"OUT_DIR": str(tmp_path)})
    assert p.returncode == 0, p.stderr[-2000:]
    import json
    lines = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    for ln in lines:
        assert ln["vals"] == [11.0, 5.0, 6.0]


def test_reference_arm_runs_on_rank0_only():
    p = _torchrun([os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1",
                   "--warmup", "3", "--workload", "single_1k", "--ref-sample", "65536"])
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    import json
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle"
