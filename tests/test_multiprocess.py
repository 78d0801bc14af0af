"""The N > 1 bench path on CPU: two gloo ranks rendezvous on 127.0.0.1, take
the max of per-rank times and pass barriers; non-zero ranks skip the oracle
arm. (Replicas only: the hot path has no data-path collective.)"""
import json
import os
import socket
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_max_and_barrier():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, os.path.join(HERE, "mp_worker.py")], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    try:
        for p in procs:
            o, e = p.communicate(timeout=120)
            assert p.returncode == 0, e[-2000:]
            outs.append(json.loads(o.strip().splitlines()[-1]))
    finally:
        for p in procs:
            if p.poll() is None:
                p.kill()
    outs.sort(key=lambda d: d["rank"])
    assert [d["rank"] for d in outs] == [0, 1]
    assert all(d["world"] == 2 and d["backend"] == "gloo" for d in outs)
    assert all(d["max"] == 2.5 for d in outs)
    assert outs[1]["reference_rc"] == 0
