"""The data-parallel sign-gradient step's host logic on CPU gloo ranks.

``signsgd_dp_step`` decides who packs, who gathers, who votes and updates,
and what is broadcast. Here its device operations are stood in for by the
oracle (test code only), and every rank's final codes and gamma must equal
the single-process oracle chain over all ranks' gradients.
"""

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import bitlinear_ref as ref
from oracle import signsgd_ref as sg

N, K, LR = 16, 96, 2.0 ** -6


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _grad(rank):
    g = torch.Generator().manual_seed(100 + rank)
    return torch.randn((N, K), generator=g).to(torch.bfloat16)


def _master():
    g = torch.Generator().manual_seed(7)
    return (torch.randn((N, K), generator=g) * 0.05).to(torch.float32)


def _oracle_ops(fused=False):
    """The oracle in place of the device calls; fused: the holder's vote,
    update and new codes as one call (the form ``bl_signsgd_apply`` takes)."""
    from ternary_weight_quantization_b200.signsgd import SignOps

    def sign_pack(dW, words):
        words.copy_(torch.from_numpy(sg.sign_bits(dW.float().numpy()).view(np.int32)))

    def sign_vote(gathered, direction):
        per_rank = [w.numpy().view(np.uint32) for w in gathered]
        direction.copy_(torch.from_numpy(ref.pack_ternary(sg.majority_direction(per_rank))))

    def update(W, direction, lr):
        d = ref.unpack_ternary(direction.numpy(), W.shape[1])
        W.copy_(torch.from_numpy(sg.signsgd_update(W.numpy(), d, lr, w_is_bf16=False)))

    def quantize_weight(W, w_packed, gamma, workspace):
        codes, g = ref.ternarize(W.numpy())
        w_packed.copy_(torch.from_numpy(ref.pack_ternary(codes)))
        gamma[0] = float(g)

    def apply(gathered, W, lr, w_packed, gamma, workspace):
        d = sg.majority_direction([w.numpy().view(np.uint32) for w in gathered])
        W.copy_(torch.from_numpy(sg.signsgd_update(W.numpy(), d, lr, w_is_bf16=False)))
        quantize_weight(W, w_packed, gamma, workspace)

    return SignOps(sign_pack=sign_pack, sign_vote=sign_vote, update=update, quantize_weight=quantize_weight,
                   apply=apply if fused else None)


def _expected(world):
    words = [sg.sign_bits(_grad(r).float().numpy()) for r in range(world)]
    w = sg.signsgd_update(_master().numpy(), sg.majority_direction(words), LR, w_is_bf16=False)
    codes, g = ref.ternarize(w)
    return ref.pack_ternary(codes), float(g)


def _words(rank):
    """The rank's sign words as a fused backward would hand them over."""
    return torch.from_numpy(sg.sign_bits(_grad(rank).float().numpy()).view(np.int32).copy())


def _worker(rank, world, port, holder, out, with_words=False, fused=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        from ternary_weight_quantization_b200.signsgd import signsgd_dp_step
        w_packed = torch.zeros((N, K // 4), dtype=torch.uint8)
        gamma = torch.zeros(1, dtype=torch.float32)
        kw = dict(master_W=_master(), workspace=torch.empty(64, dtype=torch.uint8)) if rank == holder else {}
        if with_words:
            signsgd_dp_step(None, w_packed, gamma, LR, holder=holder, ops=_oracle_ops(fused), words=_words(rank), **kw)
        else:
            signsgd_dp_step(_grad(rank), w_packed, gamma, LR, holder=holder, ops=_oracle_ops(fused), **kw)
        out[rank] = (w_packed.numpy().tobytes(), float(gamma[0]))
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.parametrize("world,holder,with_words,fused",
                         [(2, 0, False, False), (3, 1, False, True), (2, 1, True, False), (3, 2, True, True)])
def test_ranks_end_with_the_holders_codes(world, holder, with_words, fused):
    """Every rank ends with the oracle chain's codes and gamma, whether it
    hands over dW (packed here) or the sign words a fused backward made, and
    whether the holder takes the three calls or the fused one."""
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, holder, out, with_words, fused))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    packed, gamma = _expected(world)
    for r in range(world):
        assert out[r][0] == packed.tobytes()
        assert out[r][1] == gamma


def test_single_rank_needs_no_process_group():
    from ternary_weight_quantization_b200.signsgd import signsgd_dp_step
    w_packed = torch.zeros((N, K // 4), dtype=torch.uint8)
    gamma = torch.zeros(1, dtype=torch.float32)
    signsgd_dp_step(_grad(0), w_packed, gamma, LR, master_W=_master(), workspace=torch.empty(64, dtype=torch.uint8),
                    ops=_oracle_ops())
    packed, g = _expected(1)
    assert w_packed.numpy().tobytes() == packed.tobytes() and float(gamma[0]) == g


def test_holder_needs_the_master():
    from ternary_weight_quantization_b200.signsgd import signsgd_dp_step
    with pytest.raises(ValueError):
        signsgd_dp_step(_grad(0), torch.zeros((N, K // 4), dtype=torch.uint8), torch.zeros(1), LR, ops=_oracle_ops())


def test_single_rank_from_sign_words():
    from ternary_weight_quantization_b200.signsgd import signsgd_dp_step
    w_packed = torch.zeros((N, K // 4), dtype=torch.uint8)
    gamma = torch.zeros(1, dtype=torch.float32)
    signsgd_dp_step(None, w_packed, gamma, LR, master_W=_master(), workspace=torch.empty(64, dtype=torch.uint8),
                    ops=_oracle_ops(), words=_words(0))
    packed, g = _expected(1)
    assert w_packed.numpy().tobytes() == packed.tobytes() and float(gamma[0]) == g


def test_exactly_one_gradient_form():
    from ternary_weight_quantization_b200.signsgd import signsgd_dp_step
    kw = dict(master_W=_master(), workspace=torch.empty(64, dtype=torch.uint8), ops=_oracle_ops())
    with pytest.raises(ValueError):
        signsgd_dp_step(_grad(0), torch.zeros((N, K // 4), dtype=torch.uint8), torch.zeros(1), LR, words=_words(0),
                        **kw)
    with pytest.raises(ValueError):
        signsgd_dp_step(None, torch.zeros((N, K // 4), dtype=torch.uint8), torch.zeros(1), LR, **kw)
