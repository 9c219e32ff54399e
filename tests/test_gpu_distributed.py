"""The sharded Hessian call on one GPU with a one-rank NCCL group (needs a
B200): the same H as a plain lh_accumulate_hessian call, and a resumed call
adds the new tokens once."""
import os
import socket

import numpy as np
import pytest
import torch

import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_sharded_hessian_one_rank_nccl(cuda_ok):
    import torch.distributed as dist

    import scale_calibration_b200 as lh
    from scale_calibration_b200 import distributed as lhd
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    from datetime import timedelta
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=120))
    try:
        counts = [0, 5, 1, 300, 0, 17, 129, 2100]
        layer = synth.make_layer(8, 128, sum(counts), seed=6, n_mats=len(counts), counts=counts)
        _, X, off = gu.to_device(layer)
        G = len(counts)
        wsb = lh.lh_hessian_workspace_bytes(X.shape[0], 128, G)
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        H1 = torch.zeros(G, 8, 16, 16, device="cuda")
        lh.lh_accumulate_hessian(X, lh.LH_BF16, X.shape[0], 128, X.stride(0), off, G, H1, ws, wsb)
        H2 = torch.zeros_like(H1)
        lhd.accumulate_hessian_sharded(X, X.shape[0], 128, off, G, H2, ws, wsb)
        torch.cuda.synchronize()
        assert torch.equal(H1, H2)
        lhd.accumulate_hessian_sharded(X, X.shape[0], 128, off, G, H2, ws, wsb)  # resumed: adds once
        lh.lh_accumulate_hessian(X, lh.LH_BF16, X.shape[0], 128, X.stride(0), off, G, H1, ws, wsb)
        torch.cuda.synchronize()
        assert torch.equal(H1, H2)
    finally:
        dist.destroy_process_group()
