"""The expert-parallel layer on one GPU (NCCL, world size 1): with every expert local, its
candidate exchange, owner-side capacity dispatch (moe_capacity_dispatch), expert FFN on received
rows and combine of returned rows must give moe_forward's routing and outputs bit for bit.
(Two and more ranks are checked on CPU in test_ep_cpu.py; every run here has one GPU.)"""
import math
import os
import socket
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("T,d,F,E,k,C,dtype,flags", [
    (3000, 256, 512, 64, 6, 1.0, "bf16", 0),       # candidate lists + histogram selection
    (64, 2048, 1024, 64, 8, math.inf, "bf16", 0),  # the decode shape: small router and dispatch
    (2000, 128, 256, 8, 2, 0.5, "bf16", 2),        # arrival order
    (2000, 128, 256, 8, 2, 0.75, "bf16", 1),       # renormalised weights
    (3000, 256, 256, 16, 2, 1.0, "bf16", 4),       # gated experts
    (500, 48, 40, 6, 2, 0.75, "f32", 0)])
def test_expert_parallel_world_one_equals_forward(T, d, F, E, k, C, dtype, flags):
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()),
               RANK="0", WORLD_SIZE="1", NCCL_NVLS_ENABLE="0")
    cmd = [sys.executable, os.path.join(ROOT, "tests", "ep_worker.py"), "gpu", str(T), str(d),
           str(F), str(E), str(k), str(C), dtype, str(flags)]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "OK" in r.stdout, (r.stdout[-2000:], r.stderr[-3000:])
