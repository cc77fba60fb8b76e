"""The context-parallel decode exchange with two ranks (world size 2).

Two processes each hold one contiguous half of every sequence's KV cache,
decode their half to per-row softmax states (plx_decode_state), all-gather
the states over a gloo group (through host memory) and merge them
(plx_merge_states).  Both ranks must return the same output, and it must match
the fp64 oracle over the full context.  The two processes share the one GPU of
the test box; no kernel of either waits on the other, so sharing is safe.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))

# B, Hq, Hkv, d, S, lengths (some shorter than the first half), dtype name
CASES = [
    (3, 16, 8, 128, 2048, [2048, 1500, 700], "bfloat16"),
    (2, 4, 2, 64, 300, [300, 151], "float32"),
]


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(case, dev):
    import torch
    B, Hq, Hkv, d, S, lens, dtn = case
    dt = getattr(torch, dtn)
    g = torch.Generator(device=dev).manual_seed(S + B)
    s = d ** -0.25
    q = (torch.randn(B, Hq, d, generator=g, device=dev) * s).to(dt)
    rho = (torch.randn(B, Hq, d, generator=g, device=dev) * 0.3).to(dt)
    k = (torch.randn(B, S, Hkv, d, generator=g, device=dev) * s).to(dt)
    v = (torch.randn(B, S, Hkv, d, generator=g, device=dev) * s).to(dt)
    sl = torch.tensor(lens, dtype=torch.int32, device=dev)
    return q, rho, k, v, sl


def _rank(rank, world, port, case, q_out):
    sys.path[:0] = [ROOT, HERE]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist
    from covariance_corrected_softmax_b200 import plx
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, Hq, Hkv, d, S, lens, _ = case
        q, rho, k, v, _ = _inputs(case, dev)
        a, b = rank * S // world, (rank + 1) * S // world
        kl, vl = k[:, a:b].contiguous(), v[:, a:b].contiguous()
        sll = torch.tensor([min(max(n - a, 0), b - a) for n in lens], dtype=torch.int32,
                           device=dev)
        out = plx.context_parallel_decode(q, rho, kl, vl, sll, softmax_scale=1.0,
                                          out_dtype=torch.float32)
        torch.cuda.synchronize()
        q_out.put((rank, out.cpu().numpy(), plx.device_error()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", CASES, ids=["bf16_gqa", "fp32_d64"])
def test_two_ranks_merge_to_the_full_context(case):
    import torch
    import torch.multiprocessing as mp

    sys.path[:0] = [ROOT, HERE]
    import oracle
    from parity_util import check_out

    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, case, q_out)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted(q_out.get(timeout=300) for _ in range(2))
    finally:
        for p in procs:
            p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    (_, out0, e0), (_, out1, e1) = res
    assert e0 == 0 and e1 == 0
    assert np.array_equal(out0, out1), "the two ranks merged different outputs"
    q, rho, k, v, sl = _inputs(case, torch.device("cuda", 0))
    ref, _ = oracle.decode(q, rho, k, v, sl, 1.0)
    check_out(out0, ref, bf16=case[-1] == "bfloat16", what=f"two-rank merge {case[:5]}")
