"""The token-sharded Hessian on one GPU (needs a B200), against the oracle.

"NVIDIA Model Optimizer Local-Hessian: 基于局部 Hessian 的 NVFP4 逐块权重缩放算法实战指南"
(xxmr.cn/news/266017), section "入口 API 与校准流程", Phase 2: H = sum over the
calibration tokens of X^T X; the pages leave the Hessian unsynchronised across
data-parallel ranks, and scale_calibration_b200.distributed is that sync (each
rank's tokens, then a SUM all-reduce).

- one NCCL rank: accumulate_hessian_sharded's H is the oracle's H of all tokens,
  and a resumed call adds the tokens once more;
- two token shares on the one GPU, no second rank: lh_accumulate_hessian on each
  share of token_shard(..., rank, 2, offsets) (groups cut at the share boundary),
  summed in FP32 as a two-rank all-reduce sums, is the oracle's H of all tokens.
"""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

COUNTS = [0, 5, 1, 300, 0, 17, 129, 2100, 64, 1000]


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _assert_hessian(H_gpu: torch.Tensor, H_ref: np.ndarray, scale: float = 1.0):
    per, whole, bad = gu.hessian_rel_errors(H_gpu.cpu().numpy(), scale * H_ref)
    assert per <= gu.HESSIAN_RTOL and whole <= gu.HESSIAN_RTOL and bad == 0, (per, whole, bad)


def test_sharded_hessian_one_rank_nccl_matches_oracle(cuda_ok):
    import torch.distributed as dist

    import scale_calibration_b200 as lh
    from scale_calibration_b200 import distributed as lhd
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    from datetime import timedelta
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=120))
    try:
        layer = synth.make_layer(8, 256, sum(COUNTS), seed=6, n_mats=len(COUNTS), counts=COUNTS)
        _, X, off = gu.to_device(layer)
        G = len(COUNTS)
        Hr = oracle.hessian(layer.X, c_in=256, offsets=layer.offsets)
        wsb = lh.lh_hessian_workspace_bytes(X.shape[0], 256, G)
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        H = torch.zeros(G, 16, 16, 16, device="cuda")
        lhd.accumulate_hessian_sharded(X, X.shape[0], 256, off, G, H, ws, wsb)
        torch.cuda.synchronize()
        _assert_hessian(H, Hr)
        lhd.accumulate_hessian_sharded(X, X.shape[0], 256, off, G, H, ws, wsb)  # resumed: the tokens once more
        torch.cuda.synchronize()
        _assert_hessian(H, Hr, 2.0)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("grouped", [True, False])
def test_two_token_shares_summed_match_oracle(cuda_ok, grouped):
    import scale_calibration_b200 as lh
    from scale_calibration_b200 import distributed as lhd
    if grouped:
        # the share boundary (half of 3616 tokens = 1808) falls inside the 2100-token group
        layer = synth.make_layer(8, 384, sum(COUNTS), seed=9, n_mats=len(COUNTS), counts=COUNTS)
        G = len(COUNTS)
    else:
        layer = synth.make_layer(8, 384, 3001, seed=9)
        G = 1
    Hr = oracle.hessian(layer.X, c_in=384, offsets=layer.offsets)
    J = 384 // 16
    parts = []
    for rank in range(2):
        t0, t1, loc = lhd.token_shard(layer.n_tok, rank, 2, layer.offsets)
        if grouped:
            assert loc[-1] == t1 - t0
        X = torch.from_numpy(np.ascontiguousarray(layer.X[t0:t1]).view(np.int16)).view(torch.bfloat16).cuda()
        off = torch.from_numpy(loc).cuda() if grouped else None
        wsb = lh.lh_hessian_workspace_bytes(t1 - t0, 384, G)
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        Hp = torch.zeros(G, J, 16, 16, device="cuda")
        lh.lh_accumulate_hessian(X, lh.LH_BF16, t1 - t0, 384, X.stride(0), off, G, Hp, ws, wsb)
        assert lh.lh_workspace_status(ws) == 0
        # each share alone is the oracle's H of that share
        _assert_hessian(Hp, oracle.hessian(layer.X[t0:t1], c_in=384, offsets=loc))
        parts.append(Hp)
    H = parts[0] + parts[1]   # what a two-rank SUM all-reduce of FP32 partials computes
    torch.cuda.synchronize()
    _assert_hessian(H, Hr)
