"""The multi-process side of bench.py on CPU: two `gloo` ranks, each with its
own batch (weak scaling, no data-path collective), must agree on the max of
their times and on the summed token count, and the barrier must pair up."""
import os
import socket
import subprocess
import sys
import textwrap

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_two_gloo_ranks_reduce_like_the_bench():
    script = textwrap.dedent(f"""
        import os, sys
        sys.path.insert(0, {ROOT!r})
        import torch
        import bench
        class A: pass
        ws, rank = bench.dist_init(A())
        assert ws == 2
        bench.barrier(ws)
        t = bench.max_over_ranks(10.0 + rank, ws)          # rank 1 is the slower one
        n = bench.sum_over_ranks(1024.0 * (rank + 1), ws)  # per-rank tokens
        print(f"RESULT {{rank}} {{t}} {{n}}", flush=True)
        import torch.distributed as dist
        dist.destroy_process_group()
    """)
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", script], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=120)
        assert p.returncode == 0, err
        outs.append(out)
    for r, out in enumerate(outs):
        line = [l for l in out.splitlines() if l.startswith("RESULT")][0].split()
        assert int(line[1]) == r
        assert float(line[2]) == 11.0
        assert float(line[3]) == 3072.0
