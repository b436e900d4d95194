"""The expert-parallel exchange on one GPU with NCCL (one rank): a forward MoE
layer routed through dispatch (plan, MXFP8 pack, all-to-all), receive (plan,
unpack) and give_back equals the purely local path (plan, permute-quantise,
grouped GEMM, combine) bit for bit.  Run in a subprocess
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

    offs, perm, inv, pw = mx.mxfp8_moe_plan(idx, E)         # local path
    q, s, _, _ = mx.mxfp8_permute_quantize_dual(x, perm, offs)
    y_grouped = mx.mxfp8_grouped_gemm_fwd(q, s, wq, ws, offs, N, work=work)
    assert mx.mxfp8_get_status(work) == 0 and mx.mxfp8_get_status(pw) == 0
    y_a = mx.mxfp8_moe_combine(y_grouped, inv, w)

    d = ep.dispatch(x, idx, E)                               # through the exchange: MXFP8 records
    assert d.records.dtype == torch.uint8 and d.records.shape[1] == mx.mxfp8_ep_record_bytes(K)
    offs_b, perm_b, inv_b, q_b, s_b = ep.receive(d, E)
    assert torch.equal(offs_b, offs) and torch.equal(q_b, q)
    y_grouped_b = mx.mxfp8_grouped_gemm_fwd(q_b, s_b, wq, ws, offs_b, N, work=work)
    y_back = ep.give_back(y_grouped_b, inv_b, d)
    y_b = mx.mxfp8_moe_combine(y_back, d.ret_pos, w)
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
