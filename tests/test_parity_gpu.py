"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bar (per step):
  S1  gamma and the packed 2-bit codes        bit-exact
  S2  xq and sx                               bit-exact
  S3  INT32 accumulators and bf16 y           bit-exact
  S4  dX, dW (bf16 / f32)                     max rel 1e-2, mean rel 1e-3 with
      rel_i = |g_i - o_i| / max(|o_i|, 1e-3 * rms(o)), o the oracle's output
      rounded to the same dtype
"""

import numpy as np
import pytest
import torch

from oracle import bitlinear_ref as ref
from workloads import make_inputs, workload_inputs, WORKLOADS

pytestmark = pytest.mark.gpu

MAX_REL, MEAN_REL = 1e-2, 1e-3


def _bl():
    import ternary_weight_quantization_b200 as bl
    bl.load_library()
    return bl


def bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def rel_err(gpu: np.ndarray, orc: np.ndarray):
    g = np.asarray(gpu, np.float64)
    o = np.asarray(orc, np.float64)
    rms = float(np.sqrt(np.mean(o * o))) if o.size else 0.0
    denom = np.maximum(np.abs(o), 1e-3 * rms + 1e-30)
    r = np.abs(g - o) / denom
    return float(r.max(initial=0.0)), float(r.mean()) if r.size else 0.0


def assert_close(gpu, orc, what):
    mx, mean = rel_err(gpu, orc)
    assert mx <= MAX_REL and mean <= MEAN_REL, f"{what}: max rel {mx:.3e}, mean rel {mean:.3e}"


def run_step(x, w, dy, dw_dtype=torch.bfloat16, debug_acc=True):
    bl = _bl()
    M, K = x.shape
    N = w.shape[0]
    dev = "cuda"
    xd, wd, dyd = x.to(dev), w.to(dev), dy.to(dev)
    bufs = bl.StepBuffers.allocate(M, N, K, dw_dtype)
    acc = torch.empty((M, N), dtype=torch.int32, device=dev) if debug_acc else None
    bl.bl_quantize_weight(wd, bufs.w_packed, bufs.gamma, bufs.workspace)
    bl.bl_quantize_act(xd, bufs.xq, bufs.sx)
    bl.bl_forward(bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, bufs.y, acc)
    if N % 8 == 0:
        bl.bl_backward(dyd, bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, bufs.dX, bufs.dW)
    torch.cuda.synchronize()
    assert bl.bl_get_last_error() == 0
    out = {
        "gamma": bufs.gamma.cpu().numpy(), "packed": bufs.w_packed.cpu().numpy(),
        "q": bufs.xq.cpu().numpy(), "sx": bufs.sx.cpu().numpy(),
        "y_bits": bits(bufs.y), "acc": acc.cpu().numpy() if acc is not None else None,
    }
    if N % 8 == 0:
        out["dx_bits"] = bits(bufs.dX)
        out["dw"] = bufs.dW.float().cpu().numpy()
    return out


def oracle_step(x, w, dy):
    w_is_bf16 = w.dtype == torch.bfloat16
    wn = bits(w) if w_is_bf16 else w.numpy()
    return ref.bitlinear_step(bits(x), wn, bits(dy), w_is_bf16)


def check_all(g, o, N, dw_f32=False):
    assert g["gamma"][0].tobytes() == np.float32(o["gamma"]).tobytes(), (g["gamma"][0], o["gamma"])
    np.testing.assert_array_equal(g["packed"], o["packed"])
    np.testing.assert_array_equal(g["q"], o["q"])
    np.testing.assert_array_equal(g["sx"].view(np.uint32), o["sx"].view(np.uint32))
    if g["acc"] is not None:
        np.testing.assert_array_equal(g["acc"], o["acc"])
    np.testing.assert_array_equal(g["y_bits"], o["y_bits"])
    if N % 8 == 0:
        assert_close(ref.bf16_bits_to_f32(g["dx_bits"]), ref.bf16_bits_to_f32(o["dx_bits"]), "dX")
        want = o["dw_f32"] if dw_f32 else ref.bf16_bits_to_f32(o["dw_bits"])
        assert_close(g["dw"], want, "dW")


# (M, N, K): several tiles, ragged tails in every dimension, K % 128 != 0
SHAPES = [
    (1, 8, 32),
    (17, 136, 96),
    (300, 520, 320),
    (257, 392, 544),
    (64, 1000, 160),
    (513, 264, 1056),
]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("w_dtype", [torch.bfloat16, torch.float32])
def test_step_parity_small(M, N, K, w_dtype):
    x, w, dy = make_inputs(M, K, N, w_dtype=w_dtype, w_init="kaiming", outliers=True, seed=M + N + K)
    check_all(run_step(x, w, dy), oracle_step(x, w, dy), N)


def test_tiny_workload_parity():
    """The tiny BitLinear (M=32, K=128, N=256, f32 masters ~ N(0, 0.02^2))."""
    x, w, dy = workload_inputs("tiny")
    g = run_step(x, w, dy, dw_dtype=torch.float32)
    check_all(g, oracle_step(x, w, dy), 256, dw_f32=True)


@pytest.mark.parametrize("M,N,K", [(33, 130, 64), (5, 7, 32), (200, 301, 256), (8, 64, 33056)])
def test_forward_ragged_n(M, N, K):
    """Forward with N not a multiple of 8 (scalar epilogue stores), and with
    K past the range of the int32 -> fp32 shifter (conversion instruction)."""
    x, w, dy = make_inputs(M, K, N, seed=7)
    check_all(run_step(x, w, dy), oracle_step(x, w, dy), N)


@pytest.mark.parametrize("M,N,K", [(40, 64, 33088), (300, 136, 33024)])
def test_forward_tile_path_shifter_range(M, N, K):
    """The tensor-core forward (more than 16 tokens) at K past the int32 ->
    fp32 shifter's range (33088: conversion instruction, the general kernel
    instance even without the debug output) and at its edge (33024: shifter,
    the lean instance without the debug output): y with and without the
    INT32 output bit for bit equal, and equal to the oracle."""
    bl = _bl()
    x, w, dy = make_inputs(M, K, N, seed=11)
    g = run_step(x, w, dy)
    check_all(g, oracle_step(x, w, dy), N)
    bufs = bl.StepBuffers.allocate(M, N, K)
    bl.bl_quantize_weight(w.cuda(), bufs.w_packed, bufs.gamma, bufs.workspace)
    bl.bl_quantize_act(x.cuda(), bufs.xq, bufs.sx)
    y2 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    bl.bl_forward(bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, y2)
    torch.cuda.synchronize()
    assert bl.bl_get_last_error() == 0
    np.testing.assert_array_equal(bits(y2), g["y_bits"])


def _threshold_probe_weights(N=64, K=128, f32=True, seed=0):
    """Weights whose magnitudes crowd around gamma / 2.

    Half the entries form pairs (p, 0.3 - p) around 0.15 and half form pairs
    (r, 0.9 - r) around 0.45, both differences exact in fp32, so the absmean
    lands near 0.3 and gamma / 2 near 0.15 while the probes p step through
    the fp32 (or bf16) values next to it one unit in the last place at a time.
    """
    rng = np.random.default_rng(seed)
    n = N * K
    dt = np.float32
    base = np.float32(0.15)
    steps = np.arange(-(n // 4) // 2, (n // 4) - (n // 4) // 2)
    if f32:
        probes = (base + steps.astype(np.float64) * float(np.spacing(base))).astype(dt)
    else:
        # bf16 spacing at 0.15 is 2^-10
        probes = (0.15 + steps * 2.0 ** -10 / 8).astype(dt)
        probes = ref.bf16_bits_to_f32(ref.round_to_bf16_bits(probes))
    partners = (np.float32(0.3) - probes).astype(dt)
    r = rng.uniform(0.45, 0.6, n // 4).astype(dt)
    rp = (np.float32(0.9) - r).astype(dt)
    vals = np.concatenate([probes, partners, r, rp])
    vals = vals * np.where(rng.random(n) < 0.5, -1, 1).astype(dt)
    rng.shuffle(vals)
    return torch.from_numpy(vals.reshape(N, K).astype(dt))


@pytest.mark.parametrize("f32", [True, False])
def test_ternary_threshold_probes(f32):
    w = _threshold_probe_weights(f32=f32)
    if not f32:
        w = w.to(torch.bfloat16)
    x, _, dy = make_inputs(8, 128, 64, seed=3)
    o = oracle_step(x, w, dy)
    # the probes really straddle the rounding boundary
    codes = o["codes"]
    assert 0.1 < float(np.mean(codes == 0)) < 0.9
    check_all(run_step(x, w, dy), o, 64)


def test_degenerate_inputs():
    """All-zero masters (gamma = 1e-5, codes 0) and all-zero tokens (q = 0)."""
    M, N, K = 40, 64, 96
    x, w, dy = make_inputs(M, K, N, seed=11)
    x[3] = 0
    x[17] = 0
    w = torch.zeros_like(w)
    g = run_step(x, w, dy)
    o = oracle_step(x, w, dy)
    assert float(g["gamma"][0]) == float(np.float32(1e-5))
    assert not g["packed"].any() and not g["q"][3].any()
    check_all(g, o, N)


def test_quantize_weight_deterministic():
    bl = _bl()
    _, w, _ = make_inputs(4, 2560, 1024, seed=5)
    wd = w.cuda()
    outs = []
    for _ in range(3):
        packed = torch.empty((1024, 640), dtype=torch.uint8, device="cuda")
        gamma = torch.empty(1, dtype=torch.float32, device="cuda")
        ws = torch.empty(bl.bl_quantize_weight_workspace_size(1024, 2560), dtype=torch.uint8, device="cuda")
        ws.fill_(0xAB)  # garbage scratch must not matter
        bl.bl_quantize_weight(wd, packed, gamma, ws)
        outs.append((packed.cpu(), gamma.cpu()))
    for p, g in outs[1:]:
        assert torch.equal(p, outs[0][0]) and torch.equal(g, outs[0][1])


@pytest.mark.parametrize("case,expected", [("tie", 1.0), ("above", 1.0 + 2.0 ** -23), ("below", 1.0)])
@pytest.mark.parametrize("w_dtype", [torch.bfloat16, torch.float32])
def test_gamma_at_an_fp32_midpoint(case, expected, w_dtype):
    """Mean |W| on, 2^-44 above or 2^-44 below the fp32 midpoint 1 + 2^-24
    (the fp64 tree sum's error bound straddles it, so gamma comes from the
    exact integer sum): gamma and the codes bit-exact to the oracle through
    bl_quantize_weight, bl_quantize (with its token rows, also bit-exact) and
    bl_quantize_weight_noalloc, twice."""
    from workloads import gamma_midpoint_weights
    bl = _bl()
    w = gamma_midpoint_weights(case, w_dtype)
    N, K = w.shape
    codes, g = ref.ternarize(w.float().numpy())
    assert g == np.float32(expected)
    expect = ref.pack_ternary(codes)
    wd = w.cuda()
    # 64 tokens all go to the coding launch; 4000 are split between the two launches
    xs = {m: make_inputs(m, K, 8, seed=3 + m)[0] for m in (64, 4000)}
    ws = torch.empty(bl.bl_quantize_weight_workspace_size(N, K), dtype=torch.uint8, device="cuda")
    lib = bl.load_library()
    for rep in range(2):
        for how in ("weight", "fused64", "fused4000", "noalloc"):
            packed = torch.full((N, K // 4), 0xAA, dtype=torch.uint8, device="cuda")
            gamma = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
            if how == "weight":
                bl.bl_quantize_weight(wd, packed, gamma, ws)
            elif how.startswith("fused"):
                m = int(how[5:])
                xq = torch.empty((m, K), dtype=torch.int8, device="cuda")
                sx = torch.empty(m, dtype=torch.float32, device="cuda")
                bl.bl_quantize(wd, xs[m].cuda(), packed, gamma, xq, sx, ws)
                torch.cuda.synchronize()
                q_o, s_o = ref.quantize_activations(ref.bf16_bits_to_f32(bits(xs[m])))
                np.testing.assert_array_equal(xq.cpu().numpy(), q_o, err_msg=how)
                np.testing.assert_array_equal(sx.cpu().numpy().view(np.uint32), s_o.view(np.uint32), err_msg=how)
            else:
                wdt = bl.BL_F32 if w_dtype == torch.float32 else bl.BL_BF16
                import ctypes
                rc = lib.bl_quantize_weight_noalloc(ctypes.c_void_p(wd.data_ptr()), wdt, N, K,
                                                    ctypes.c_void_p(packed.data_ptr()),
                                                    ctypes.c_void_p(gamma.data_ptr()),
                                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
                assert rc == 0
            torch.cuda.synchronize()
            assert bl.bl_get_last_error() == 0
            assert gamma.cpu().numpy()[0].tobytes() == np.float32(expected).tobytes(), (how, rep)
            np.testing.assert_array_equal(packed.cpu().numpy(), expect, err_msg=f"{how} {rep}")


@pytest.mark.parametrize("dw_dtype", [torch.float32, torch.bfloat16])
def test_dw_accumulate(dw_dtype):
    bl = _bl()
    M, N, K = 96, 264, 160
    x, w, dy = make_inputs(M, K, N, seed=13)
    bufs = bl.StepBuffers.allocate(M, N, K, dw_dtype)
    prev = (torch.randn(N, K, generator=torch.Generator().manual_seed(9)) * 3).to(dw_dtype)
    bufs.dW.copy_(prev.cuda())
    xd, wd, dyd = x.cuda(), w.cuda(), dy.cuda()
    bl.bl_quantize_weight(wd, bufs.w_packed, bufs.gamma, bufs.workspace)
    bl.bl_quantize_act(xd, bufs.xq, bufs.sx)
    bl.bl_backward(dyd, bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, None, bufs.dW, accumulate_dW=True)
    torch.cuda.synchronize()
    o = ref.bitlinear_step(bits(x), bits(w), bits(dy), True, dw_prev=prev.float().numpy())
    want = o["dw_f32"] if dw_dtype == torch.float32 else ref.bf16_bits_to_f32(o["dw_bits"])
    assert_close(bufs.dW.float().cpu().numpy(), want, "dW accumulate")


def test_dw_empty_reduction():
    """M = 0 tokens: dW is the empty sum, all zeros."""
    import ctypes
    lib = _bl().load_library()
    N, K = 64, 128
    dW = torch.full((N, K), 5.0, dtype=torch.float32, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.bl_backward(None, None, None, None, None, 0, N, K, None, ctypes.c_void_p(dW.data_ptr()), 1, 0, st)
    assert rc == 0
    torch.cuda.synchronize()
    assert not dW.any()


def test_export_roundtrip():
    bl = _bl()
    x, w, dy = make_inputs(16, 256, 128, seed=21)
    bufs = bl.StepBuffers.allocate(16, 128, 256)
    bl.bl_quantize_weight(w.cuda(), bufs.w_packed, bufs.gamma, bufs.workspace)
    host, gamma = bl.bl_export_weights(bufs.w_packed, bufs.gamma)
    codes, g = ref.ternarize(ref.bf16_bits_to_f32(bits(w)))
    assert gamma == float(g)
    np.testing.assert_array_equal(ref.unpack_ternary(host.numpy(), 256), codes)


# ---------------------------------------------------------------- full size


def _sample(n, k, seed):
    return np.sort(np.random.default_rng(seed).choice(n, size=min(k, n), replace=False))


@pytest.mark.parametrize("name", ["up_proj", "down_proj"])
def test_full_size_parity_sampled(name):
    """The bench workloads at full size, in the bench's launch configuration.

    S1 and S2 are compared in full (bit-exact); S3 on 96 sampled tokens
    (INT32 and y bit-exact); dX on 96 sampled tokens; dW on 96 sampled rows.
    """
    bl = _bl()
    wl = WORKLOADS[name]
    M, K, N = wl.M, wl.K, wl.N
    x, w, dy = workload_inputs(name)
    bufs = bl.StepBuffers.allocate(M, N, K)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    xd, wd, dyd = x.cuda(), w.cuda(), dy.cuda()
    bl.bl_quantize_weight(wd, bufs.w_packed, bufs.gamma, bufs.workspace)
    bl.bl_quantize_act(xd, bufs.xq, bufs.sx)
    bl.bl_forward(bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, bufs.y, acc)
    bl.bl_backward(dyd, bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, bufs.dX, bufs.dW)
    torch.cuda.synchronize()
    assert bl.bl_get_last_error() == 0

    wf = ref.bf16_bits_to_f32(bits(w))
    codes, gamma = ref.ternarize(wf)
    assert bufs.gamma.cpu().numpy()[0].tobytes() == np.float32(gamma).tobytes()
    np.testing.assert_array_equal(bufs.w_packed.cpu().numpy(), ref.pack_ternary(codes))
    q, sx = ref.quantize_activations(ref.bf16_bits_to_f32(bits(x)))
    np.testing.assert_array_equal(bufs.xq.cpu().numpy(), q)
    np.testing.assert_array_equal(bufs.sx.cpu().numpy().view(np.uint32), sx.view(np.uint32))

    rows = _sample(M, 96, 1)
    acc_o = ref.forward_accumulate(q[rows], codes)
    np.testing.assert_array_equal(acc.cpu().numpy()[rows], acc_o)
    y_o = ref.round_to_bf16_bits(ref.forward_output(acc_o, sx[rows], gamma))
    np.testing.assert_array_equal(bits(bufs.y)[rows], y_o)

    dyf = ref.bf16_bits_to_f32(bits(dy))
    dx_o = ref.round_to_bf16_bits(ref.backward_dx(dyf[rows], codes, gamma))
    assert_close(ref.bf16_bits_to_f32(bits(bufs.dX)[rows]), ref.bf16_bits_to_f32(dx_o), "dX")

    nrows = _sample(N, 96, 2)
    xh = ref.bf16_bits_to_f32(ref.round_to_bf16_bits(ref.dequantize_activations(q, sx)))
    dw_o = ref.round_to_bf16_bits(ref.backward_dw(dyf[:, nrows], xh))
    assert_close(ref.bf16_bits_to_f32(bits(bufs.dW)[nrows]), ref.bf16_bits_to_f32(dw_o), "dW")


@pytest.mark.parametrize("w_dtype", [torch.float32, torch.bfloat16])
def test_weight_subnormals_and_zeros(w_dtype):
    """Masters holding zeros and subnormals (the exact widening's rare path)
    next to ordinary values: gamma and codes stay bit-exact."""
    M, N, K = 16, 64, 256
    x, w, dy = make_inputs(M, K, N, w_dtype=torch.float32, w_init="normal0.02", seed=17)
    g = torch.Generator().manual_seed(5)
    pick = torch.rand(N, K, generator=g)
    tiny = torch.full((N, K), 3e-39 if w_dtype == torch.bfloat16 else 7e-42)
    w = torch.where(pick < 0.05, tiny * torch.sign(torch.randn(N, K, generator=g)), w)
    w = torch.where((pick >= 0.05) & (pick < 0.1), torch.zeros_like(w), w)
    w = w.to(w_dtype)
    assert (w.float().abs() < 1.17e-38).any() and (w.float() != 0).any()
    check_all(run_step(x, w, dy), oracle_step(x, w, dy), N)


def test_dx_only_launch():
    """bl_backward with dW = NULL: a launch holding only dX tiles."""
    bl = _bl()
    M, N, K = 300, 264, 352
    x, w, dy = make_inputs(M, K, N, seed=29)
    bufs = bl.StepBuffers.allocate(M, N, K)
    bl.bl_quantize_weight(w.cuda(), bufs.w_packed, bufs.gamma, bufs.workspace)
    bl.bl_quantize_act(x.cuda(), bufs.xq, bufs.sx)
    bl.bl_backward(dy.cuda(), bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, bufs.dX, None)
    torch.cuda.synchronize()
    o = oracle_step(x, w, dy)
    assert_close(ref.bf16_bits_to_f32(bits(bufs.dX)), ref.bf16_bits_to_f32(o["dx_bits"]), "dX")


def test_backward_scheduled_tiles_full_compare():
    """Enough dX + dW tiles (64 + 64) that the launch spreads them over the
    pairs by its precomputed schedule; every output element compared."""
    M = N = K = 2048
    x, w, dy = make_inputs(M, K, N, seed=31)
    g = run_step(x, w, dy, debug_acc=False)
    o = oracle_step(x, w, dy)
    g["acc"] = None
    check_all(g, o, N)


@pytest.mark.parametrize("M,N,K,w_dtype", [
    (4096, 6912, 2560, torch.bfloat16),   # rows read twice in the fused launch
    (300, 520, 320, torch.bfloat16),      # rows in registers
    (64, 264, 1024, torch.float32),
    (17, 136, 96, torch.bfloat16),
    (40, 64, 8448, torch.bfloat16),       # rows past 8192 (read twice)
    (300, 6912, 2560, torch.bfloat16),    # slices past shared memory: a tail read again
    (2048, 2560, 6912, torch.bfloat16),   # the down-projection shape
    (0, 128, 256, torch.bfloat16),        # no tokens: S1 only
])
def test_quantize_fused_matches_separate(M, N, K, w_dtype):
    """bl_quantize gives bit for bit what bl_quantize_weight + bl_quantize_act give."""
    bl = _bl()
    x, w, _ = make_inputs(max(M, 1), K, N, w_dtype=w_dtype, seed=M + N)
    x = x[:M]
    xd, wd = x.cuda(), w.cuda()
    ws = torch.empty(max(bl.bl_quantize_weight_workspace_size(N, K), 16), dtype=torch.uint8, device="cuda")
    outs = []
    for fused in (False, True):
        packed = torch.full((N, K // 4), 0xAA, dtype=torch.uint8, device="cuda")
        gamma = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
        xq = torch.full((M, K), 99, dtype=torch.int8, device="cuda")
        sx = torch.full((M,), -1.0, dtype=torch.float32, device="cuda")
        if fused:
            bl.bl_quantize(wd, xd, packed, gamma, xq, sx, ws)
        else:
            bl.bl_quantize_weight(wd, packed, gamma, ws)
            if M:
                bl.bl_quantize_act(xd, xq, sx)
        torch.cuda.synchronize()
        assert bl.bl_get_last_error() == 0
        outs.append([t.cpu() for t in (packed, gamma, xq, sx)])
    for a, b in zip(*outs):
        assert torch.equal(a, b)
    codes, g = ref.ternarize(ref.bf16_bits_to_f32(bits(w)) if w_dtype == torch.bfloat16 else w.numpy())
    assert outs[1][1].numpy()[0].tobytes() == np.float32(g).tobytes()
    np.testing.assert_array_equal(outs[1][0].numpy(), ref.pack_ternary(codes))
    if M:
        q, s = ref.quantize_activations(ref.bf16_bits_to_f32(bits(x)))
        np.testing.assert_array_equal(outs[1][2].numpy(), q)
        np.testing.assert_array_equal(outs[1][3].numpy().view(np.uint32), s.view(np.uint32))


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 9, 16])
def test_forward_few_tokens(M):
    """Forward with few tokens on the up-projection weight (M <= 16: the
    code-bandwidth kernel, every token-slot count; above: the tile kernel):
    INT32 sums and y bit-exact."""
    bl = _bl()
    N, K = 6912, 2560
    x, w, _ = make_inputs(M, K, 8, seed=40 + M)
    _, w, _ = make_inputs(8, K, N, seed=41)
    bufs = bl.StepBuffers.allocate(M, N, K)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    bl.bl_quantize_weight(w.cuda(), bufs.w_packed, bufs.gamma, bufs.workspace)
    bl.bl_quantize_act(x.cuda(), bufs.xq, bufs.sx)
    bl.bl_forward(bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, bufs.y, acc)
    y2 = torch.empty_like(bufs.y)
    bl.bl_forward(bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, y2)  # without the debug output
    torch.cuda.synchronize()
    assert bl.bl_get_last_error() == 0
    codes, gamma = ref.ternarize(ref.bf16_bits_to_f32(bits(w)))
    q, sx = ref.quantize_activations(ref.bf16_bits_to_f32(bits(x)))
    acc_o = ref.forward_accumulate(q, codes)
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
    y_o = ref.round_to_bf16_bits(ref.forward_output(acc_o, sx, gamma))
    np.testing.assert_array_equal(bits(bufs.y), y_o)
    np.testing.assert_array_equal(bits(y2), y_o)


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K", [(3, 2560, 6912), (16, 2560, 6912), (5, 1000, 96), (16, 333, 160),
                                   (1, 7, 32), (9, 2049, 4096)])
def test_forward_few_tokens_shapes(M, N, K):
    """Few-token forward at other shapes: the down-projection weight (long
    rows), K % 64 != 0 (8-byte code chunks), N not a multiple of the rows a
    warp takes, a single short row: INT32 sums and y bit-exact."""
    bl = _bl()
    x, w, _ = make_inputs(M, K, N, seed=60 + M + K)
    bufs = bl.StepBuffers.allocate(M, N, K)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    bl.bl_quantize_weight(w.cuda(), bufs.w_packed, bufs.gamma, bufs.workspace)
    bl.bl_quantize_act(x.cuda(), bufs.xq, bufs.sx)
    bl.bl_forward(bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, bufs.y, acc)
    torch.cuda.synchronize()
    assert bl.bl_get_last_error() == 0
    codes, gamma = ref.ternarize(ref.bf16_bits_to_f32(bits(w)))
    q, sx = ref.quantize_activations(ref.bf16_bits_to_f32(bits(x)))
    acc_o = ref.forward_accumulate(q, codes)
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_o)
    np.testing.assert_array_equal(bits(bufs.y), ref.round_to_bf16_bits(ref.forward_output(acc_o, sx, gamma)))


@pytest.mark.parametrize("M,N,K", [(2000, 2500, 2560), (2048, 2560, 6912), (2400, 2200, 4096), (2000, 2500, 2592)])
def test_forward_wide_tiles(M, N, K):
    """Shapes with a few more 256-column tiles than CTA pairs take the
    320-column forward tiles (two MMAs per step into one accumulator, tokens
    in five boxes per CTA): INT32 sums and y (through the debug path and
    through the TMA-store path) bit-exact on sampled token rows, ragged
    tokens and features included; K = 2592 (K % 64 != 0) stages the packed
    codes by cp.async and ends on a partial k-block."""
    bl = _bl()
    x, w, _ = make_inputs(M, K, N, seed=70 + M)
    bufs = bl.StepBuffers.allocate(M, N, K)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    y2 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    bl.bl_quantize_weight(w.cuda(), bufs.w_packed, bufs.gamma, bufs.workspace)
    bl.bl_quantize_act(x.cuda(), bufs.xq, bufs.sx)
    bl.bl_forward(bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, bufs.y, acc)
    bl.bl_forward(bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, y2)
    torch.cuda.synchronize()
    assert bl.bl_get_last_error() == 0
    codes, gamma = ref.ternarize(ref.bf16_bits_to_f32(bits(w)))
    q, sx = ref.quantize_activations(ref.bf16_bits_to_f32(bits(x)))
    # every 320-token tile's first and last rows, and a random sample
    rows = np.unique(np.concatenate([np.arange(0, M, 320), np.minimum(np.arange(319, M + 319, 320), M - 1),
                                     _sample(M, 64, 3)]))
    acc_o = ref.forward_accumulate(q[rows], codes)
    np.testing.assert_array_equal(acc.cpu().numpy()[rows], acc_o)
    y_o = ref.round_to_bf16_bits(ref.forward_output(acc_o, sx[rows], gamma))
    np.testing.assert_array_equal(bits(bufs.y)[rows], y_o)
    np.testing.assert_array_equal(bits(y2)[rows], y_o)


@pytest.mark.parametrize("M,N,K,dw_dtype,accumulate", [
    (4096, 6912, 2560, torch.bfloat16, False),   # the up-projection
    (2048, 2560, 6912, torch.bfloat16, False),   # the down-projection
    (300, 2048, 320, torch.float32, False),
    (200, 2040, 256, torch.bfloat16, False),     # N < 2048: workspace left unused
    (257, 3200, 544, torch.bfloat16, True),      # ragged tokens and features, accumulation
    (17, 4096, 96, torch.float32, True),         # K % 64 != 0: a partial x_hat box
    (64, 3080, 1024, torch.bfloat16, False),
])
def test_backward_workspace_matches_rebuild(M, N, K, dw_dtype, accumulate):
    """bl_backward_ws (x_hat made once in the workspace, dW's operand loaded
    by TMA, for N >= 2048) gives dX and dW bit for bit as bl_backward (x_hat
    rebuilt in every dW tile), and the sign-word form the same words; the
    workspace starts as garbage."""
    bl = _bl()
    x, w, dy = make_inputs(M, K, N, seed=80 + M)
    bufs = bl.StepBuffers.allocate(M, N, K, dw_dtype)
    xd, wd, dyd = x.cuda(), w.cuda(), dy.cuda()
    bl.bl_quantize_weight(wd, bufs.w_packed, bufs.gamma, bufs.workspace)
    bl.bl_quantize_act(xd, bufs.xq, bufs.sx)
    ws = torch.full((max(bl.bl_backward_workspace_size(M, N, K), 16),), 0xAB, dtype=torch.uint8, device="cuda")
    prev = (torch.randn(N, K, generator=torch.Generator().manual_seed(5)) * 3).to(dw_dtype).cuda()
    outs = []
    for workspace in (None, ws):
        dX = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
        dW = prev.clone() if accumulate else torch.full((N, K), 7.0, dtype=dw_dtype, device="cuda")
        words = torch.zeros((N, K // 32), dtype=torch.int32, device="cuda")
        dX2 = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
        bl.bl_backward(dyd, bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, dX, dW, accumulate, workspace=workspace)
        bl.bl_backward_signs(dyd, bufs.xq, bufs.sx, bufs.w_packed, bufs.gamma, dX2, words, workspace=workspace)
        torch.cuda.synchronize()
        assert bl.bl_get_last_error() == 0
        outs.append([t.cpu() for t in (dX, dW, words, dX2)])
    for a, b in zip(*outs):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    assert torch.equal(outs[1][0].view(torch.int16), outs[1][3].view(torch.int16))
