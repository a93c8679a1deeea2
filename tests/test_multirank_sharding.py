"""Head / token sharding of the attention call across ranks, on CPU ranks over gloo.

The all-to-all plumbing of block_sparse_attention_cube_b200.sharding (token shards of all heads ->
all tokens of a rank's heads, and back) is run on 2 and 3 CPU ranks with the fp64 oracle standing in
for the GPU attention; the result on every rank must equal the oracle's whole-sequence output
restricted to that rank's token shard, with zero padding rows.  The GPU path (NCCL, the library's
kernels) is the same code with another backend and the real attention; one GPU runs it as world 1
in tests/test_gpu_prenorm.py.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs(name):
    import synth
    from oracle import vsa_oracle as O
    w = synth.WORKLOADS[name]
    x = synth.make_inputs(w)
    return w, {k: O.bf16_to_f64(v) for k, v in x.items()}


def _attend_oracle(q, k, v, shape, topk_k, scale, gc, gf):
    from oracle import vsa_oracle as O
    r = O.forward(q.numpy(), k.numpy(), v.numpy(), shape.grid, topk_k, scale,
                  None if gc is None else gc.numpy(), None if gf is None else gf.numpy())
    return torch.from_numpy(r["out"])


def _worker(rank, world, port, name, q_out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        import block_sparse_attention_cube_b200 as vsa
        from block_sparse_attention_cube_b200 import sharding as S
        w, f64 = _inputs(name)
        N = w.tokens
        off, n = S.token_shard(N, world, rank)
        def shard(a):
            t = torch.zeros((a.shape[0], n) + a.shape[2:], dtype=torch.float64)
            real = max(0, min(n, N - off))
            t[:, :real] = torch.from_numpy(a[:, off:off + real])
            return t
        s = vsa.Shape(w.batch, w.heads, w.head_dim, w.grid)
        scale = 1.0 / np.sqrt(w.head_dim)
        out = S.sharded_forward(shard(f64["q"]), shard(f64["k"]), shard(f64["v"]), s, w.topk, scale,
                                shard(f64["g_coarse"]), shard(f64["g_fine"]), attend=_attend_oracle)
        q_out.put((rank, off, n, out.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name, world", [("tiny_8x8x8", 2), ("tiny_8x8x8", 3), ("padded_7x15x16", 3)])
def test_token_sharded_call_equals_the_whole(name, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, name, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    from oracle import vsa_oracle as O
    w, f64 = _inputs(name)
    whole = O.forward(f64["q"], f64["k"], f64["v"], w.grid, w.topk, 1.0 / np.sqrt(w.head_dim), f64["g_coarse"],
                      f64["g_fine"])["out"]
    N = w.tokens
    for rank, off, n, out in res:
        real = max(0, min(n, N - off))
        np.testing.assert_allclose(out[:, :real], whole[:, off:off + real], rtol=0, atol=1e-12)
        assert not out[:, real:].any()


def test_partition_helpers():
    sys.path.insert(0, ROOT)
    from block_sparse_attention_cube_b200 import sharding as S
    assert [S.head_range(40, 8, r) for r in (0, 7)] == [(0, 5), (35, 40)]
    assert [S.head_range(4, 3, r) for r in range(3)] == [(0, 2), (2, 3), (3, 4)]
    assert [S.head_range(2, 3, r) for r in range(3)] == [(0, 1), (1, 2), (2, 2)]
    assert S.batch_range(2, 2, 1) == (1, 2)
    assert S.token_shard(32760, 8, 7) == (7 * 4095, 4095)
    assert S.token_shard(512, 3, 2) == (342, 171)   # one padding row
