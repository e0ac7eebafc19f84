"""Data-parallel layer sharding and gradient averaging on the GPU, with the one
GPU a test box has: one-rank NCCL communicators drive the sharded copy path
(slice copy, in-place all-gather on the copy stream, ready event) and the
per-layer gradient all-reduce (reduction stream, the optimiser waiting for it),
and each step must equal the plain one bit for bit.  Several ranks whose all-gathers wait on one another
are never run on one GPU; the slice plan for G ranks is checked with gloo ranks
on the CPU (test_dist_gloo.py).  Runs in a fresh process, bounded by a timeout,
so that NCCL's set-up stays out of the rest of the suite."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def test_sharded_stack_step_equals_unsharded():
    env = dict(os.environ)
    env.setdefault("NCCL_SOCKET_IFNAME", "lo")     # one rank: its bootstrap stays on loopback
    r = subprocess.run([sys.executable, os.path.join(HERE, "shard_child.py")], env=env,
                       cwd=os.path.dirname(HERE), capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "shard ok" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]
