"""Multi-process host logic of the benchmark's replica mode, on CPU with the gloo backend: two
ranks rendezvous over 127.0.0.1, meet at the barrier, and every rank sees the max over ranks of
its timing, which is what the whole-job throughput is divided by."""
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RANK_CODE = r"""
import os, sys
sys.path.insert(0, {root!r})
import bench
d = bench.Dist()
d.init("gloo")
assert d.world == 2 and d.rank == int(os.environ["RANK"])
ms = 10.0 + 5.0 * d.rank          # rank 1 is the slower one
d.barrier()
print("MAX", d.max(ms))
d.barrier()
d.close()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_agree_on_the_max_time():
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", RANK_CODE.format(root=ROOT)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err[-2000:]
        outs.append(out)
    for out in outs:
        assert "MAX 15.0" in out, out


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    env_backup = {k: os.environ.pop(k) for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK") if k in os.environ}
    try:
        d = bench.Dist()
        d.init("gloo")
        assert d.world == 1 and not d.pg
        assert d.max(3.25) == 3.25
        d.barrier()
        d.close()
    finally:
        os.environ.update(env_backup)
