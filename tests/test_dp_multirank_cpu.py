"""The data-parallel step's host logic on CPU gloo ranks.

``dp_step`` runs S1 + S2, the forward and the backward on each rank's token
shard and sums dW over the ranks. Here its device operations are stood in
for by the oracle (test code only, fp64 outputs unrounded), so that the
exchange can be checked exactly: after the step every rank must hold the
dW of the whole batch (the oracle's, on all ranks' tokens at once), and its
own tokens' y and dX; S1 needs no exchange because every rank ternarises the
same W to the same codes and gamma.
"""

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import bitlinear_ref as ref

M_TOTAL, K, N = 24, 64, 40


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    g = torch.Generator().manual_seed(3)
    x = torch.randn((M_TOTAL, K), generator=g).to(torch.bfloat16)
    w = (torch.randn((N, K), generator=g) * 0.05).to(torch.float32)
    dy = torch.randn((M_TOTAL, N), generator=g).to(torch.bfloat16)
    return x, w, dy


def _shard(world, rank):
    per = M_TOTAL // world
    return slice(rank * per, (rank + 1) * per)


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _oracle_ops():
    from ternary_weight_quantization_b200.dp import DPOps

    def quantize(W, x, w_packed, gamma, xq, sx, ws, stream):
        codes, g = ref.ternarize(W.numpy())
        w_packed.copy_(torch.from_numpy(ref.pack_ternary(codes)))
        gamma[0] = float(g)
        q, s = ref.quantize_activations(ref.bf16_bits_to_f32(_u16(x)))
        xq.copy_(torch.from_numpy(q))
        sx.copy_(torch.from_numpy(s))

    def forward(xq, sx, w_packed, gamma, y, acc, stream):
        codes = ref.unpack_ternary(w_packed.numpy(), xq.shape[1])
        y.copy_(torch.from_numpy(ref.forward_output(ref.forward_accumulate(xq.numpy(), codes), sx.numpy(),
                                                    np.float32(gamma[0].item())).astype(np.float64)))

    def backward(dY, xq, sx, w_packed, gamma, dX, dW, accumulate, stream):
        codes = ref.unpack_ternary(w_packed.numpy(), xq.shape[1])
        dy = ref.bf16_bits_to_f32(_u16(dY))
        xh = ref.bf16_bits_to_f32(ref.round_to_bf16_bits(ref.dequantize_activations(xq.numpy(), sx.numpy())))
        dX.copy_(torch.from_numpy(ref.backward_dx(dy, codes, np.float32(gamma[0].item()))))
        dW.copy_(torch.from_numpy(ref.backward_dw(dy, xh)))

    return DPOps(quantize=quantize, forward=forward, backward=backward)


def _buffers(m):
    from ternary_weight_quantization_b200.bitlinear import StepBuffers
    f64 = torch.float64
    return StepBuffers(w_packed=torch.zeros((N, K // 4), dtype=torch.uint8), gamma=torch.zeros(1),
                       workspace=torch.zeros(16, dtype=torch.uint8), xq=torch.zeros((m, K), dtype=torch.int8),
                       sx=torch.zeros(m), y=torch.zeros((m, N), dtype=f64), dX=torch.zeros((m, K), dtype=f64),
                       dW=torch.zeros((N, K), dtype=f64))


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        from ternary_weight_quantization_b200.dp import dp_step
        x, w, dy = _inputs()
        sl = _shard(world, rank)
        bufs = _buffers(sl.stop - sl.start)
        dp_step(x[sl].contiguous(), w, dy[sl].contiguous(), bufs, ops=_oracle_ops())
        out[rank] = {k: getattr(bufs, k).numpy().copy() for k in ("w_packed", "gamma", "y", "dX", "dW")}
    finally:
        torch.distributed.destroy_process_group()


def _whole_batch():
    x, w, dy = _inputs()
    return ref.bitlinear_step(_u16(x), w.numpy(), _u16(dy), w_is_bf16=False)


@pytest.mark.parametrize("world", [2, 3])
def test_ranks_hold_the_whole_batch_dw(world):
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    whole = _whole_batch()
    for r in range(world):
        o, sl = out[r], _shard(world, r)
        np.testing.assert_array_equal(o["w_packed"], whole["packed"])
        assert o["gamma"][0] == whole["gamma"]
        np.testing.assert_array_equal(o["y"], ref.forward_output(whole["acc"], whole["sx"], whole["gamma"])[sl])
        dy = ref.bf16_bits_to_f32(_u16(_inputs()[2]))
        np.testing.assert_allclose(o["dX"], ref.backward_dx(dy, whole["codes"], whole["gamma"])[sl],
                                   rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(o["dW"], whole["dw_f64"], rtol=1e-12, atol=1e-12)


def test_single_rank_needs_no_process_group():
    from ternary_weight_quantization_b200.dp import dp_step
    x, w, dy = _inputs()
    bufs = _buffers(M_TOTAL)
    dp_step(x, w, dy, bufs, ops=_oracle_ops())
    np.testing.assert_allclose(bufs.dW.numpy(), _whole_batch()["dw_f64"], rtol=1e-12, atol=1e-12)
