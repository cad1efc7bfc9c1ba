"""GPU: the data-parallel step with the library's kernels and a real exchange.

Two ranks (processes, gloo) share the one GPU; each runs ``dp_step`` -- the
library's bl_quantize, bl_forward and bl_backward on its half of the tokens
-- and the all-reduce sums their partial dW. No kernel of one rank waits on
the other's. Bars against the oracle of the whole batch: both ranks hold the
same codes and gamma (bit-exact to the oracle's), each rank's y rows are
bit-exact, its dX rows and the summed dW meet max rel 1e-2 / mean rel 1e-3.
"""

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import bitlinear_ref as ref
from workloads import make_inputs

pytestmark = pytest.mark.gpu

M_TOTAL, K, N, WORLD = 512, 640, 384, 2
MAX_REL, MEAN_REL = 1e-2, 1e-3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _worker(rank, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=WORLD,
                                         timeout=datetime.timedelta(seconds=120))
    try:
        import ternary_weight_quantization_b200 as bl
        from ternary_weight_quantization_b200.dp import dp_step
        bl.load_library()
        torch.cuda.set_device(0)
        x, w, dy = make_inputs(M_TOTAL, K, N, seed=9)
        per = M_TOTAL // WORLD
        sl = slice(rank * per, (rank + 1) * per)
        bufs = bl.StepBuffers.allocate(per, N, K, torch.float32)
        dp_step(x[sl].cuda(), w.cuda(), dy[sl].cuda(), bufs)
        torch.cuda.synchronize()
        if bl.bl_get_last_error() != 0:
            raise RuntimeError("device error word set")
        out[rank] = {"packed": bufs.w_packed.cpu().numpy(), "gamma": float(bufs.gamma.item()),
                     "y": _u16(bufs.y), "dX": _u16(bufs.dX), "dW": bufs.dW.cpu().numpy()}
    finally:
        torch.distributed.destroy_process_group()


def _rel(g, o):
    g, o = np.asarray(g, np.float64), np.asarray(o, np.float64)
    rms = float(np.sqrt(np.mean(o * o)))
    r = np.abs(g - o) / np.maximum(np.abs(o), 1e-3 * rms + 1e-30)
    return float(r.max()), float(r.mean())


def test_two_ranks_sum_dw_over_the_whole_batch():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, out)) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    x, w, dy = make_inputs(M_TOTAL, K, N, seed=9)
    whole = ref.bitlinear_step(_u16(x), _u16(w), _u16(dy), w_is_bf16=True)
    per = M_TOTAL // WORLD
    for r in range(WORLD):
        o, sl = out[r], slice(r * per, (r + 1) * per)
        np.testing.assert_array_equal(o["packed"], whole["packed"])
        assert np.float32(o["gamma"]) == whole["gamma"]
        np.testing.assert_array_equal(o["y"], whole["y_bits"][sl])
        mx, mean = _rel(ref.bf16_bits_to_f32(o["dX"]), ref.bf16_bits_to_f32(whole["dx_bits"][sl]))
        assert mx <= MAX_REL and mean <= MEAN_REL, f"dX rank {r}: {mx:.3e} {mean:.3e}"
        mx, mean = _rel(o["dW"], whole["dw_f32"])
        assert mx <= MAX_REL and mean <= MEAN_REL, f"dW rank {r}: {mx:.3e} {mean:.3e}"
    np.testing.assert_array_equal(out[0]["dW"], out[1]["dW"])
