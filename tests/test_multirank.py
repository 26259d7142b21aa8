"""The multi-GPU host logic of bench.py on CPU: two ranks over gloo (the same
process-group calls the NCCL run makes).  Every rank reads its place from
the torchrun environment, draws its own batch (rank-dependent seed), and the
step time reported is the maximum over ranks; the reference arm runs on rank
0 only."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import json, os, sys
sys.path.insert(0, os.environ["REPO"])
import torch, torch.distributed as dist
import bench, workloads as W
ws, rank, local = bench.dist_env()
dist.init_process_group("gloo", init_method="env://", rank=rank, world_size=ws)
# per-rank step times: rank r is slower by r ms
mine = [1.0 + rank, 0.25 * (rank + 1)]
red = bench.reduce_max(mine, ws, torch.device("cpu"))
cfg = W.small_dsa(W.TINY, n_seqs=1, rows=1, lens=(256,), topk=16)
inp = W.dsa_inputs(cfg, "cpu", seed=bench.rank_seed(cfg.seed, rank))
dist.barrier()
print(json.dumps({"rank": rank, "ws": ws, "local": local, "red": red,
                  "seed": bench.rank_seed(cfg.seed, rank), "q0": float(inp["q_lat"].float().sum())}))
dist.destroy_process_group()
"""


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_ranks(code: str, n: int = 2, timeout: int = 240):
    port = _free_port()
    procs = []
    for r in range(n):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(n), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), REPO=ROOT, CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", code], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=timeout)
        assert p.returncode == 0, err[-2000:]
        outs.append(out)
    return outs


def test_two_ranks_reduce_max_and_distinct_batches():
    outs = [json.loads(o.strip().splitlines()[-1]) for o in _run_ranks(WORKER)]
    outs.sort(key=lambda d: d["rank"])
    assert [d["rank"] for d in outs] == [0, 1] and all(d["ws"] == 2 for d in outs)
    assert [d["local"] for d in outs] == [0, 1]
    for d in outs:
        assert d["red"] == [2.0, 0.5]          # the maximum over ranks, on every rank
    assert outs[0]["seed"] != outs[1]["seed"]  # weak scaling: every rank draws its own batch
    assert outs[0]["q0"] != outs[1]["q0"]


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the reference arm's other ranks exit at once, silently."""
    code = r"""
import os, sys
sys.path.insert(0, os.environ["REPO"])
import bench
if int(os.environ["RANK"]) != 0:
    bench.main(["--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "0"])
    print("RANK_DONE")
else:
    print("RANK_DONE")
"""
    outs = _run_ranks(code)
    assert all(o.strip().splitlines()[-1] == "RANK_DONE" for o in outs)
    assert all("impl" not in o for o in outs)
