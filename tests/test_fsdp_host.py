"""Quantized FSDP weight communication on two gloo ranks (CPU): each rank holds a slice of W,
finds the absmax of its rotation, the ranks take the maximum, each quantizes its slice with the
whole tensor's scale, and the codes are all-gathered.  The flow is the binding's
`sharded_quantize_flow`; on CPU its passes are the oracle's (the library's kernels need a GPU),
and the result must equal the oracle's quantization of the whole W bit for bit."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.filterwarnings("ignore")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _weights(fmt_dtype):
    from hadamard_rotated_precision_b200 import synthetic
    w = synthetic.tiny_random((4 * 96, 256), 12, scale=0.02)
    w[:, 7] *= 40.0
    return synthetic.to_bf16_bits(w) if fmt_dtype == "bf16" else w


def _worker(rank, world, port, fmt, dim, k, dtype, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    import oracle
    import hadamard_rotated_precision_b200 as hq
    dist.init_process_group("gloo", rank=rank, world_size=world)
    W = _weights(dtype)
    n = W.shape[0] // world
    shard = W[rank * n:(rank + 1) * n]

    def absmax_pass():
        return torch.tensor([float(oracle.absmax(oracle.rotate(shard, dim, k)))], dtype=torch.float32)

    def reduce_max(a):
        dist.all_reduce(a, op=dist.ReduceOp.MAX)
        return a

    def codes_pass(a):
        return oracle.quantize_rotated(oracle.rotate(shard, dim, k), fmt, absmax_of_whole=np.float32(a.item()))

    codes, scale = hq.sharded_quantize_flow(absmax_pass, reduce_max, codes_pass)
    t = torch.from_numpy(np.ascontiguousarray(codes))
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t)
    full = torch.cat(parts, dim=0 if dim == 1 else 1).numpy()
    out[rank] = (full.tobytes(), full.shape, float(scale))
    dist.destroy_process_group()


@pytest.mark.parametrize("fmt,dim,k,dtype", [(0, 1, 64, "bf16"), (1, 1, 16, "f32"), (0, 0, 32, "f32"),
                                             (2, 0, 16, "bf16")])
def test_sharded_quantization_two_gloo_ranks(oracle_lib, fmt, dim, k, dtype):
    import oracle
    world = 2
    port = _free_port()
    out = mp.Manager().dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, fmt, dim, k, dtype, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    want_codes, want_scale = oracle.quantize(_weights(dtype), dim, k, fmt)
    for r in range(world):
        buf, shape, scale = out[r]
        got = np.frombuffer(buf, dtype=np.uint8).reshape(shape)
        assert np.array_equal(got, want_codes), f"rank {r}"
        assert np.float32(scale) == want_scale
