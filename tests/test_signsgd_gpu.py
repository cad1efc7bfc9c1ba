"""GPU parity of the sign-gradient kernels against the CPU oracle.

Bar: every output is integer or a once-rounded value the oracle forms in the
same precision, so all comparisons are bit-exact:
  G1  sign words                       bit-exact
  G2  2-bit vote direction             bit-exact
  G3  updated masters (bf16 / f32)     bit-exact
  the whole single-rank step (G1 -> G2 -> G3 -> S1): codes and gamma bit-exact
"""

import numpy as np
import pytest
import torch

from oracle import bitlinear_ref as ref
from oracle import signsgd_ref as sg

pytestmark = pytest.mark.gpu


def _bl():
    import ternary_weight_quantization_b200 as bl
    bl.load_library()
    return bl


def _u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _grad(shape, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    d = torch.randn(shape, generator=g)
    r = torch.rand(shape, generator=g)
    d[r < 0.05] = 0.0
    d[(r >= 0.05) & (r < 0.08)] = -0.0
    d[(r >= 0.08) & (r < 0.09)] = -1e-40  # a subnormal in both dtypes
    return d.to(dtype)


def _as_f32(t):
    return t.float().cpu().numpy()


@pytest.mark.parametrize("shape", [(1, 32), (3, 96), (7, 160), (33, 2560), (6912, 2560)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_sign_pack_matches_oracle(shape, dtype):
    bl = _bl()
    if dtype == torch.float32 and shape[0] * shape[1] > 1 << 22:
        pytest.skip("f32 covered on the smaller shapes")
    d = _grad(shape, dtype, seed=shape[0])
    words = torch.empty((shape[0], shape[1] // 32), dtype=torch.int32, device="cuda")
    bl.bl_sign_pack(d.cuda(), words)
    torch.cuda.synchronize()
    expect = sg.sign_bits(_as_f32(d))  # float() keeps every sign bit
    assert np.array_equal(words.cpu().numpy().view(np.uint32), expect)


@pytest.mark.parametrize("ranks,shape", [(1, (4, 64)), (2, (5, 96)), (3, (8, 128)), (4, (2, 32)),
                                         (7, (16, 256)), (8, (9, 160)), (127, (3, 64)), (2, (6912, 2560))])
def test_sign_vote_matches_oracle(ranks, shape):
    bl = _bl()
    n, k = shape
    g = torch.Generator().manual_seed(1000 + ranks)
    words = torch.randint(-2 ** 31, 2 ** 31, (ranks, n, k // 32), generator=g, dtype=torch.int64).to(torch.int32)
    direction = torch.empty((n, k // 4), dtype=torch.uint8, device="cuda")
    bl.bl_sign_vote(words.cuda(), direction)
    torch.cuda.synchronize()
    expect = ref.pack_ternary(sg.majority_direction([w.numpy().view(np.uint32) for w in words]))
    assert np.array_equal(direction.cpu().numpy(), expect)


def _direction(shape, seed):
    n, k = shape
    g = torch.Generator().manual_seed(seed)
    codes = torch.randint(-1, 2, (n, k), generator=g, dtype=torch.int8).numpy()
    return codes, ref.pack_ternary(codes)


@pytest.mark.parametrize("shape", [(2, 32), (5, 96), (64, 2560), (6912, 2560)])
@pytest.mark.parametrize("lr", [2.0 ** -6, 1e-3, -0.5])
def test_signsgd_update_bf16_matches_oracle(shape, lr):
    bl = _bl()
    g = torch.Generator().manual_seed(shape[0])
    w = (torch.randn(shape, generator=g) * 0.02).to(torch.bfloat16)
    w[0, :4] = torch.tensor([-0.0, 0.0, 1.0, -1.0], dtype=torch.bfloat16)
    codes, packed = _direction(shape, seed=shape[1])
    wd = w.cuda()
    bl.bl_signsgd_update(wd, torch.from_numpy(packed).cuda(), lr)
    torch.cuda.synchronize()
    expect = ref.round_to_bf16_bits(sg.signsgd_update(_as_f32(w), codes, lr, w_is_bf16=True))
    assert np.array_equal(_u16(wd), expect)


@pytest.mark.parametrize("shape", [(2, 32), (7, 160), (128, 2560)])
@pytest.mark.parametrize("lr", [2.0 ** -6, 3e-4])
def test_signsgd_update_f32_matches_oracle(shape, lr):
    bl = _bl()
    g = torch.Generator().manual_seed(7 + shape[0])
    w = torch.randn(shape, generator=g) * 0.02
    w[0, 0] = -0.0
    codes, packed = _direction(shape, seed=3 + shape[1])
    wd = w.cuda()
    bl.bl_signsgd_update(wd, torch.from_numpy(packed).cuda(), lr)
    torch.cuda.synchronize()
    expect = sg.signsgd_update(w.numpy(), codes, lr, w_is_bf16=False)
    assert np.array_equal(wd.cpu().numpy().view(np.uint32), expect.view(np.uint32))


@pytest.mark.parametrize("shape,w_dtype", [((6912, 2560), torch.bfloat16), ((96, 320), torch.float32)])
def test_single_rank_step_matches_oracle_chain(shape, w_dtype):
    bl = _bl()
    from ternary_weight_quantization_b200.signsgd import signsgd_dp_step
    n, k = shape
    g = torch.Generator().manual_seed(11)
    master = (torch.randn(shape, generator=g) * 0.02).to(w_dtype)
    dW = _grad(shape, torch.bfloat16, seed=12)
    lr = 2.0 ** -8
    wd = master.cuda()
    w_packed = torch.empty((n, k // 4), dtype=torch.uint8, device="cuda")
    gamma = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(max(bl.bl_quantize_weight_workspace_size(n, k), 16), dtype=torch.uint8, device="cuda")
    signsgd_dp_step(dW.cuda(), w_packed, gamma, lr, master_W=wd, workspace=ws)
    torch.cuda.synchronize()

    d = sg.majority_direction([sg.sign_bits(_as_f32(dW))])
    w_new = sg.signsgd_update(_as_f32(master), d, lr, w_is_bf16=w_dtype == torch.bfloat16)
    if w_dtype == torch.bfloat16:
        w_new_bits = ref.round_to_bf16_bits(w_new)
        assert np.array_equal(_u16(wd), w_new_bits)
        w_new = ref.bf16_bits_to_f32(w_new_bits)
    else:
        assert np.array_equal(wd.cpu().numpy().view(np.uint32), w_new.view(np.uint32))
    codes, gm = ref.ternarize(w_new)
    assert float(gamma.item()) == float(gm)
    assert np.array_equal(w_packed.cpu().numpy(), ref.pack_ternary(codes))


@pytest.mark.parametrize("M,N,K", [(17, 136, 96), (300, 520, 320), (64, 1000, 160), (257, 392, 544),
                                   (4096, 6912, 2560)])
def test_backward_signs_match_sign_pack_of_dw(M, N, K):
    """bl_backward_signs: dX as bl_backward's and the sign words equal to
    bl_sign_pack of bl_backward's dW (bf16 and f32), bit for bit; against the
    oracle, every element whose dW is clearly away from zero has its sign."""
    bl = _bl()
    from workloads import make_inputs
    x, w, dy = make_inputs(M, K, N, seed=M + N + K)
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device="cuda")
    gamma = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(max(bl.bl_quantize_weight_workspace_size(N, K), 16), dtype=torch.uint8, device="cuda")
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    sx = torch.empty(M, dtype=torch.float32, device="cuda")
    bl.bl_quantize(w.cuda(), x.cuda(), packed, gamma, xq, sx, ws)
    dyd = dy.cuda()
    dx_ref = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    dx = torch.empty_like(dx_ref)
    words_ref = {}
    for dt in (torch.bfloat16, torch.float32):
        dw = torch.empty((N, K), dtype=dt, device="cuda")
        bl.bl_backward(dyd, xq, sx, packed, gamma, dx_ref, dw)
        wr = torch.empty((N, K // 32), dtype=torch.int32, device="cuda")
        bl.bl_sign_pack(dw, wr)
        words_ref[dt] = wr
    words = torch.full((N, K // 32), -1, dtype=torch.int32, device="cuda")
    bl.bl_backward_signs(dyd, xq, sx, packed, gamma, dx, words)
    torch.cuda.synchronize()
    assert bl.bl_get_last_error() == 0
    assert torch.equal(words, words_ref[torch.bfloat16])
    assert torch.equal(words, words_ref[torch.float32])
    assert torch.equal(dx.view(torch.int16), dx_ref.view(torch.int16))
    if M * N * K > 10 ** 9:
        return  # full size: the bit-exact equality above; the oracle's fp64 dW would take minutes
    # signs against the oracle's fp64 dW where |dW| > 1e-2 rms (far above any rounding)
    q, s_x = ref.quantize_activations(ref.bf16_bits_to_f32(_u16(x)))
    x_hat = ref.bf16_bits_to_f32(ref.round_to_bf16_bits(ref.dequantize_activations(q, s_x)))
    dw_o = ref.backward_dw(ref.bf16_bits_to_f32(_u16(dy)), x_hat)
    bits = sg.unpack_sign_bits(words.cpu().numpy().view(np.uint32)).reshape(N, K)
    clear = np.abs(dw_o) > 1e-2 * np.sqrt(np.mean(dw_o ** 2))
    assert np.array_equal(bits[clear], (dw_o[clear] < 0).astype(bits.dtype))


def test_backward_signs_without_tokens():
    """M = 0: dW = +0, so every sign word is zero; dX may be omitted."""
    bl = _bl()
    N, K = 64, 128
    packed = torch.zeros((N, K // 4), dtype=torch.uint8, device="cuda")
    gamma = torch.ones(1, dtype=torch.float32, device="cuda")
    words = torch.full((N, K // 32), -1, dtype=torch.int32, device="cuda")
    bl.bl_backward_signs(torch.empty((0, N), dtype=torch.bfloat16, device="cuda"),
                         torch.empty((0, K), dtype=torch.int8, device="cuda"),
                         torch.empty(0, dtype=torch.float32, device="cuda"), packed, gamma, None, words)
    torch.cuda.synchronize()
    assert int(words.abs().sum()) == 0


def test_single_rank_step_from_fused_sign_words():
    """The whole sign-gradient step fed by bl_backward_signs ends with the same
    master, codes and gamma as the step fed by bl_backward's dW."""
    bl = _bl()
    from ternary_weight_quantization_b200.signsgd import signsgd_dp_step
    from workloads import make_inputs
    M, N, K = 512, 1024, 640
    x, w, dy = make_inputs(M, K, N, seed=5)
    results = []
    for fused in (False, True):
        wd = w.cuda()
        packed = torch.empty((N, K // 4), dtype=torch.uint8, device="cuda")
        gamma = torch.empty(1, dtype=torch.float32, device="cuda")
        ws = torch.empty(max(bl.bl_quantize_weight_workspace_size(N, K), 16), dtype=torch.uint8, device="cuda")
        xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
        sx = torch.empty(M, dtype=torch.float32, device="cuda")
        dx = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
        bl.bl_quantize(wd, x.cuda(), packed, gamma, xq, sx, ws)
        if fused:
            words = torch.empty((N, K // 32), dtype=torch.int32, device="cuda")
            bl.bl_backward_signs(dy.cuda(), xq, sx, packed, gamma, dx, words)
            signsgd_dp_step(None, packed, gamma, 2.0 ** -8, master_W=wd, workspace=ws, words=words)
        else:
            dw = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
            bl.bl_backward(dy.cuda(), xq, sx, packed, gamma, dx, dw)
            signsgd_dp_step(dw, packed, gamma, 2.0 ** -8, master_W=wd, workspace=ws)
        torch.cuda.synchronize()
        results.append((_u16(wd), packed.cpu().numpy(), float(gamma.item())))
    assert np.array_equal(results[0][0], results[1][0])
    assert np.array_equal(results[0][1], results[1][1])
    assert results[0][2] == results[1][2]


def _rank_words(ranks, shape, seed):
    """ranks sign-word arrays [R, N, K/32] int32 of random bits."""
    g = torch.Generator().manual_seed(seed)
    n, k = shape
    return torch.randint(-2 ** 31, 2 ** 31, (ranks, n, k // 32), generator=g, dtype=torch.int64).to(torch.int32)


@pytest.mark.parametrize("ranks,shape,w_dtype", [(1, (3, 96), torch.bfloat16), (3, (33, 2560), torch.bfloat16),
                                                 (8, (1000, 160), torch.bfloat16), (2, (6912, 2560), torch.bfloat16),
                                                 (1, (6912, 2560), torch.bfloat16), (127, (5, 64), torch.float32),
                                                 (3, (96, 320), torch.float32), (4, (2560, 1024), torch.float32)])
def test_apply_matches_the_three_calls_and_the_oracle(ranks, shape, w_dtype):
    """bl_signsgd_apply (vote, update and |W| sums in one sweep, then the code
    launch) leaves W, w_packed and gamma bit for bit as bl_sign_vote,
    bl_signsgd_update and bl_quantize_weight in turn do, and as the oracle
    chain; twice in a row on the same workspace."""
    bl = _bl()
    n, k = shape
    g = torch.Generator().manual_seed(21 + ranks)
    master = (torch.randn(shape, generator=g) * 0.02).to(w_dtype)
    lr = 2.0 ** -9
    ws = torch.empty(bl.bl_quantize_weight_workspace_size(n, k), dtype=torch.uint8, device="cuda")
    ws.fill_(0x5C)
    w_a, w_b = master.cuda(), master.cuda()
    direction = torch.empty((n, k // 4), dtype=torch.uint8, device="cuda")
    outs = []
    for step in range(2):
        words = _rank_words(ranks, shape, seed=100 * step + ranks).cuda()
        pa = torch.full((n, k // 4), 0xAA, dtype=torch.uint8, device="cuda")
        ga = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
        pb, gb = pa.clone(), ga.clone()
        bl.bl_signsgd_apply(words, w_a, lr, pa, ga, ws)
        bl.bl_sign_vote(words, direction)
        bl.bl_signsgd_update(w_b, direction, lr)
        bl.bl_quantize_weight(w_b, pb, gb, ws)
        torch.cuda.synchronize()
        assert bl.bl_get_last_error() == 0
        assert torch.equal(w_a.view(torch.int16 if w_dtype == torch.bfloat16 else torch.int32),
                           w_b.view(torch.int16 if w_dtype == torch.bfloat16 else torch.int32)), step
        assert torch.equal(pa, pb) and ga.cpu().numpy().tobytes() == gb.cpu().numpy().tobytes(), step
        outs.append((words.cpu(), pa.cpu(), ga.cpu()))
    if n * k > 1 << 22:
        return  # the oracle chain runs on the smaller shapes
    w = _as_f32(master)
    for words, pa, ga in outs:
        d = sg.majority_direction([x.numpy().view(np.uint32) for x in words])
        w = sg.signsgd_update(w, d, lr, w_is_bf16=w_dtype == torch.bfloat16)
        if w_dtype == torch.bfloat16:
            w = ref.bf16_bits_to_f32(ref.round_to_bf16_bits(w))
        codes, gm = ref.ternarize(w)
        assert float(ga[0]) == float(gm)
        assert np.array_equal(pa.numpy(), ref.pack_ternary(codes))


@pytest.mark.parametrize("case,expected", [("tie", 1.0), ("above", 1.0 + 2.0 ** -23), ("below", 1.0)])
@pytest.mark.parametrize("w_dtype", [torch.bfloat16, torch.float32])
def test_apply_exact_gamma_at_an_fp32_midpoint(case, expected, w_dtype):
    """Two ranks voting opposite signs everywhere leave W unchanged (a tie
    moves nothing), so on a W whose mean |W| sits on or 2^-44 off the fp32
    midpoint 1 + 2^-24 the code launch must take the exact integer sum after
    the fused sweep's partial sums too: gamma and codes bit-exact."""
    from workloads import gamma_midpoint_weights
    bl = _bl()
    w = gamma_midpoint_weights(case, w_dtype)
    n, k = w.shape
    codes, gm = ref.ternarize(w.float().numpy())
    assert gm == np.float32(expected)
    words = torch.stack([torch.full((n, k // 32), -1, dtype=torch.int32), torch.zeros((n, k // 32), dtype=torch.int32)])
    wd = w.cuda()
    packed = torch.full((n, k // 4), 0xAA, dtype=torch.uint8, device="cuda")
    gamma = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    ws = torch.empty(bl.bl_quantize_weight_workspace_size(n, k), dtype=torch.uint8, device="cuda")
    bl.bl_signsgd_apply(words.cuda(), wd, 2.0 ** -4, packed, gamma, ws)
    torch.cuda.synchronize()
    assert bl.bl_get_last_error() == 0
    assert torch.equal(wd.cpu(), w)
    assert gamma.cpu().numpy()[0].tobytes() == np.float32(expected).tobytes()
    np.testing.assert_array_equal(packed.cpu().numpy(), ref.pack_ternary(codes))
