"""The expert-parallel exchange on one GPU with NCCL (one rank): a forward MoE
layer routed through dispatch / give_back equals the purely local path (plan,
permute-quantise, grouped GEMM, combine) bit for bit.  Run in a subprocess
with a deadline so that a stuck process group cannot stall the suite."""
import os
import socket
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import datetime, os, sys
import numpy as np, torch
sys.path.insert(0, os.environ["REPO_ROOT"])
import mxfp8_grouped_gemm_quantize_b200 as mx
from mxfp8_grouped_gemm_quantize_b200 import ep, workloads as wl
torch.cuda.set_device(0)
torch.distributed.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                                     device_id=torch.device("cuda", 0))
try:
    T, k, E, K, N = 300, 2, 8, 256, 128
    rng = np.random.default_rng(5)
    idx = torch.from_numpy(np.argsort(-rng.standard_normal((T, E)), axis=1)[:, :k].astype(np.int32)).cuda()
    w = torch.from_numpy(rng.random((T, k)).astype(np.float32)).cuda()
    x = wl.normal_bf16((T, K), 1.0, 6).cuda()
    wq, ws = mx.mxfp8_quantize_rowwise(wl.normal_bf16((E * N, K), 0.05, 7).cuda())
    work = mx.new_workspace(E, T * k, N, K)

    def layer(rows, ids):
        offs, perm, inv, pw = mx.mxfp8_moe_plan(ids, E)
        q, s, _, _ = mx.mxfp8_permute_quantize_dual(rows, perm, offs)
        y = mx.mxfp8_grouped_gemm_fwd(q, s, wq, ws, offs, N, work=work)
        assert mx.mxfp8_get_status(work) == 0 and mx.mxfp8_get_status(pw) == 0
        return y, inv

    y_grouped, inv = layer(x, idx)                     # local path
    y_a = mx.mxfp8_moe_combine(y_grouped, inv, w)

    rows, le, ex = ep.dispatch(x, idx, E)              # through the exchange
    y_grouped_b, inv_b = layer(rows, le.view(-1, 1))
    ones = torch.ones((rows.shape[0], 1), dtype=torch.float32, device="cuda")
    y_rows = mx.mxfp8_moe_combine(y_grouped_b, inv_b, ones)
    y_pairs = ep.give_back(y_rows, ex)
    pairs = torch.arange(T * k, dtype=torch.int32, device="cuda").view(T, k)
    y_b = mx.mxfp8_moe_combine(y_pairs, pairs, w)
    torch.cuda.synchronize()
    assert torch.equal(y_a.view(torch.int16), y_b.view(torch.int16)), "exchange path differs"
    print("ok")
finally:
    torch.distributed.destroy_process_group()
'''


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_exchange_matches_the_local_layer():
    env = dict(os.environ, REPO_ROOT=ROOT, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()),
               NCCL_NVLS_ENABLE="0")
    r = subprocess.run([sys.executable, "-c", SCRIPT], env=env, capture_output=True, text=True, timeout=240)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:] + r.stderr[-4000:]
