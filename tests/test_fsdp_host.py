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


# ------------------------------------------------------------------ the layer flow

def _layer_inputs(n_layers, world):
    """Per layer: full X_i [M][K] and W_i [N][K] (N a multiple of world), bf16 bits."""
    from hadamard_rotated_precision_b200 import synthetic
    out = []
    for i in range(n_layers):
        K, N, M = 128 * (i + 1), 64 * world * (i + 2), 96
        X = synthetic.tiny_random((M, K), 300 + i)
        X[:, (5 * i) % K] *= 30.0
        W = synthetic.tiny_random((N, K), 400 + i, scale=0.02)
        out.append((synthetic.to_bf16_bits(X), synthetic.to_bf16_bits(W)))
    return out


def _flow_worker(rank, world, port, fmt, k, n_layers, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    import oracle
    import hadamard_rotated_precision_b200 as hq
    dist.init_process_group("gloo", rank=rank, world_size=world)
    layers = _layer_inputs(n_layers, world)
    log, pending = [], {}

    def start(i):
        log.append(("start", i))
        W = layers[i][1]
        n = W.shape[0] // world
        shard = W[rank * n:(rank + 1) * n]
        a = torch.tensor([float(oracle.absmax(oracle.rotate(shard, 1, k)))], dtype=torch.float32)
        dist.all_reduce(a, op=dist.ReduceOp.MAX)
        codes, scale = oracle.quantize_rotated(oracle.rotate(shard, 1, k), fmt, absmax_of_whole=np.float32(a.item()))
        t = torch.from_numpy(np.ascontiguousarray(codes))
        parts = [torch.empty_like(t) for _ in range(world)]
        work = dist.all_gather(parts, t, async_op=True)  # left in flight while other work runs
        pending[i] = (work, parts, scale)

    def wait(i):
        log.append(("wait", i))
        work, parts, scale = pending.pop(i)
        work.wait()
        return torch.cat(parts, dim=0).numpy(), scale

    def compute(i, g):
        log.append(("compute", i))
        wq, sw = g
        xq, sx = oracle.quantize(layers[i][0], 1, k, fmt)
        _, fast = oracle.epilogue(oracle.gemm(xq, wq, fmt), sx, sw)
        return fast

    ys = hq.fsdp_prefetch_schedule(n_layers, start, wait, compute)
    out[rank] = ([y.tobytes() for y in ys], [y.shape for y in ys], log)
    dist.destroy_process_group()


@pytest.mark.parametrize("fmt,k", [(0, 64), (1, 32)])
def test_fsdp_layer_flow_two_gloo_ranks(oracle_lib, fmt, k):
    """Forward over three layers with quantized FSDP weights on two gloo ranks: layer i + 1's
    gather is issued before layer i computes and waited for only before layer i + 1 computes;
    every layer's output equals the oracle's unsharded forward bit for bit on both ranks."""
    import oracle
    world, n_layers = 2, 3
    port = _free_port()
    out = mp.Manager().dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_flow_worker, args=(r, world, port, fmt, k, n_layers, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    want_log = [("start", 0)]
    for i in range(n_layers):
        want_log.append(("wait", i))
        if i + 1 < n_layers:
            want_log.append(("start", i + 1))
        want_log.append(("compute", i))
    layers = _layer_inputs(n_layers, world)
    for r in range(world):
        bufs, shapes, log = out[r]
        assert list(log) == want_log, f"rank {r}: {log}"
        for i in range(n_layers):
            X, W = layers[i]
            want = oracle.linear_fwd(X, W, k, fmt)["fast"]
            got = np.frombuffer(bufs[i], dtype=np.uint16).reshape(shapes[i])
            assert np.array_equal(got, want), f"rank {r} layer {i}"


def test_fsdp_prefetch_schedule_order_and_empty():
    import hadamard_rotated_precision_b200 as hq
    log = []
    res = hq.fsdp_prefetch_schedule(2, lambda i: log.append(("s", i)), lambda i: log.append(("w", i)) or i * 10,
                                     lambda i, g: (log.append(("c", i)), g + 1)[1])
    assert res == [1, 11]
    assert log == [("s", 0), ("w", 0), ("s", 1), ("c", 0), ("w", 1), ("c", 1)]
    assert hq.fsdp_prefetch_schedule(0, None, None, None) == []
