"""The head-sharded layer forward: the head split and W_o column blocks, and the
reduction of the ranks' partial outputs with world_size 2 over gloo on CPU (each
rank's local layer is the fp64 oracle on its heads), against the oracle's whole
layer."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from kimi_delta_attention_21_b200.tensor_parallel import head_range, shard, wo_columns  # noqa: E402


@pytest.mark.parametrize("H,world", [(16, 1), (16, 2), (16, 8), (5, 2), (3, 3), (7, 4)])
def test_head_range_partitions_the_heads(H, world):
    spans = [head_range(H, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == H
    assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))          # contiguous, no gaps or overlap
    sizes = [h1 - h0 for h0, h1 in spans]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def test_row_parallel_projection_is_the_head_sum():
    # y = concat_h(x) W_o^T equals the sum over head blocks of x_block W_o[:, cols]^T
    import oracle
    rng = np.random.default_rng(0)
    N, H, Dv, Dm = 7, 6, 4, 5
    x = rng.standard_normal((N, H, Dv))
    W = rng.standard_normal((Dm, H * Dv))
    full = oracle.project(x, W)
    parts = 0
    for r in range(3):
        h0, h1 = head_range(H, 3, r)
        c0, c1 = wo_columns(h0, h1, Dv)
        parts = parts + oracle.project(x[:, h0:h1], W[:, c0:c1])
    np.testing.assert_allclose(parts, full, rtol=1e-12, atol=1e-12)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist

    import kda_inputs as ki
    import oracle
    from kimi_delta_attention_21_b200.tensor_parallel import tp_forward
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = ki.custom("tp", 2, 40, 5, 8, 6, 12, "f32", seed=31, s0_std=0.1)
        inp = ki.make_inputs(w)

        def local(h0, h1, c0, c1):
            sl = lambda a: shard(a, h0, h1)
            o = oracle.forward(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["z"]), sl(inp["beta"]),
                               sl(inp["gate"]), inp["W_o"][:, c0:c1], inp["S0"][:, h0:h1], g_min=w.g_min, eps=w.eps)
            return torch.from_numpy(o["outputs"]), o["final_state"]

        y, s_local, (h0, h1) = tp_forward(local, rank, world, w.H, w.Dv)
        q.put((rank, y.double().numpy(), s_local, h0, h1))
    finally:
        dist.destroy_process_group()


def test_two_rank_head_sharded_layer_matches_the_whole_layer():
    import kda_inputs as ki
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted((q.get(timeout=180) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = ki.custom("tp", 2, 40, 5, 8, 6, 12, "f32", seed=31, s0_std=0.1)
    inp = ki.make_inputs(w)
    want = oracle.forward(inp["q"], inp["k"], inp["v"], inp["z"], inp["beta"], inp["gate"], inp["W_o"], inp["S0"],
                          g_min=w.g_min, eps=w.eps)
    for rank, y, s_local, h0, h1 in out:
        # the reduction sums fp32 partials: within fp32 rounding of the fp64 whole-layer result
        np.testing.assert_allclose(y, want["outputs"], rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(s_local, want["final_state"][:, h0:h1], rtol=1e-12, atol=1e-12)
    assert [(h0, h1) for _, _, _, h0, h1 in out] == [(0, 3), (3, 5)]
