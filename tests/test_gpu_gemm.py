"""FP4 GEMM (tcgen05) vs the FP64 oracle.

Exact cases (power-of-two scales, sums exactly representable) must be bit-exact and
pin tile coordinates, nibble order and the scale-factor layout; random cases must
satisfy |D - D_ref| <= 1e-6 * sum_k |a_k b_k| (+ half a BF16 ulp for BF16 output)."""
import numpy as np
import pytest
import torch

import block_scaled_fp4_04_b200 as fp4
import oracle
import workloads
from fp4_testutil import check_gemm, dequant_oracle, gpu_quantize, oracle_quantize, random_input

pytestmark = pytest.mark.gpu


def _gemm(a: fp4.Quantized, b: fp4.Quantized, out_dtype):
    d = fp4.gemm(a, b, out_dtype)
    torch.cuda.synchronize()
    assert fp4.fp4_get_status() == fp4.OK
    return d


def _quantized_from_codes(codes_u4: np.ndarray, scale_byte: int, fmt: int) -> fp4.Quantized:
    """Build an operand directly from 4-bit codes [rows, cols] and one scale byte."""
    rows, cols = codes_u4.shape
    packed = (codes_u4[:, 0::2] | (codes_u4[:, 1::2] << 4)).astype(np.uint8)
    blk = 16 if fmt == fp4.NVFP4 else 32
    sc = oracle.swizzle_scales(np.full((rows, cols // blk), scale_byte, np.uint8))
    return fp4.Quantized(torch.from_numpy(packed).cuda(), torch.from_numpy(sc).cuda(),
                         torch.ones(1, device="cuda"), rows, cols, fmt)


def _hat(codes_u4, scale_val):
    grid = np.array([oracle.e2m1_decode(c) for c in range(16)])
    return grid[codes_u4] * scale_val


@pytest.mark.parametrize("fmt", [fp4.NVFP4, fp4.MXFP4])
@pytest.mark.parametrize("m,n,k", [(128, 128, 256), (130, 256, 512), (16, 384, 256), (1, 128, 64)])
def test_identity_operand_bit_exact(fmt, m, n, k):
    """A = identity (code 1.0 on the diagonal): D = B_hat^T restricted, exactly."""
    a = np.zeros((m, k), np.uint8)
    for i in range(min(m, k)):
        a[i, i] = 2  # 1.0
    rng = np.random.default_rng(m + n + k)
    b = rng.integers(0, 16, (n, k)).astype(np.uint8)
    one = 0x38 if fmt == fp4.NVFP4 else 127
    d = _gemm(_quantized_from_codes(a, one, fmt), _quantized_from_codes(b, one, fmt), torch.float32)
    ref = _hat(a, 1.0) @ _hat(b, 1.0).T
    assert np.array_equal(d.cpu().numpy().astype(np.float64), ref)


@pytest.mark.parametrize("fmt", [fp4.NVFP4, fp4.MXFP4])
@pytest.mark.parametrize("m,n,k", [(256, 256, 512),
                                   # 160 tiles of 128 x 256: 256 x 256 tiles on CTA pairs
                                   (2560, 2048, 512)])
def test_block_scale_placement_bit_exact(fmt, m, n, k):
    """Every block has its own power-of-two scale: pins which scale byte applies to
    which (row, K-block) on both operands (on CTA pairs: the second CTA's A rows and
    scales, and both halves of B's rows and scale row-blocks)."""
    blk = 16 if fmt == fp4.NVFP4 else 32
    rng = np.random.default_rng(7)
    ac = rng.integers(0, 16, (m, k)).astype(np.uint8)
    bc = rng.integers(0, 16, (n, k)).astype(np.uint8)
    # powers of two 2^-1 .. 2^1 on both sides: every product is a multiple of 2^-4 and
    # |sum| < 36 * 4 * 512 < 2^17, so every partial sum needs at most 21 bits
    if fmt == fp4.NVFP4:   # E4M3 exponent field 6..8, mantissa 0
        a_sc = (rng.integers(6, 9, (m, k // blk)) << 3).astype(np.uint8)
        b_sc = (rng.integers(6, 9, (n, k // blk)) << 3).astype(np.uint8)
        val = lambda s: np.vectorize(oracle.e4m3_decode)(s)
    else:
        a_sc = rng.integers(126, 129, (m, k // blk)).astype(np.uint8)
        b_sc = rng.integers(126, 129, (n, k // blk)).astype(np.uint8)
        val = lambda s: np.vectorize(oracle.e8m0_decode)(s)

    def mk(c, s):
        packed = (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
        return fp4.Quantized(torch.from_numpy(packed).cuda(), torch.from_numpy(oracle.swizzle_scales(s)).cuda(),
                             torch.ones(1, device="cuda"), c.shape[0], c.shape[1], fmt)

    d = _gemm(mk(ac, a_sc), mk(bc, b_sc), torch.float32)
    grid = np.array([oracle.e2m1_decode(c) for c in range(16)])
    ah = grid[ac] * np.repeat(val(a_sc), blk, 1)
    bh = grid[bc] * np.repeat(val(b_sc), blk, 1)
    ref = ah @ bh.T
    assert np.array_equal(d.cpu().numpy().astype(np.float64), ref)


def test_rank_one_integer_sums():
    m, n, k = 200, 300, 1024
    a = np.full((m, k), 2, np.uint8)                    # all 1.0
    b = np.random.default_rng(3).integers(0, 16, (n, k)).astype(np.uint8)
    d = _gemm(_quantized_from_codes(a, 0x38, fp4.NVFP4), _quantized_from_codes(b, 0x38, fp4.NVFP4), torch.float32)
    ref = np.tile(_hat(b, 1.0).sum(1), (m, 1))
    assert np.array_equal(d.cpu().numpy().astype(np.float64), ref)


GEMM_CASES = [
    # m, n, k, fmt, out dtype
    (128, 128, 256, fp4.NVFP4, torch.float32),
    (512, 512, 512, fp4.NVFP4, torch.float32),       # the small configuration (glossary-style inputs)
    (200, 600, 1024, fp4.NVFP4, torch.bfloat16),     # ragged M and N
    (256, 256, 96, fp4.NVFP4, torch.float32),        # K tail: half an MMA
    (384, 768, 2880, fp4.MXFP4, torch.bfloat16),     # MoE K
    (96, 256, 64, fp4.MXFP4, torch.float32),
    (1, 256, 512, fp4.NVFP4, torch.bfloat16),        # M = 1 (swapped, split over K)
    (16, 1024, 4096, fp4.NVFP4, torch.bfloat16),     # decode shape, reduced N
    (40, 640, 2048, fp4.NVFP4, torch.float32),       # swapped with N-tile 64
    (64, 384, 8192, fp4.MXFP4, torch.bfloat16),
    (1024, 1024, 1024, fp4.NVFP4, torch.bfloat16),   # training sweep, smallest square
    (256, 256, 8192, fp4.NVFP4, torch.float32),      # few tiles, long K: split over K
    (16, 1000, 2048, fp4.NVFP4, torch.bfloat16),     # decode kernel, ragged last weight tile
    (32, 200, 8192, fp4.NVFP4, torch.float32),       # decode kernel, N-tile 32, few tiles
    (7, 640, 2080, fp4.NVFP4, torch.bfloat16),       # decode kernel, K tail (2080 = 8*256 + 32)
    (130, 384, 4096, fp4.NVFP4, torch.bfloat16),     # split over K with a ragged M tile
    # 256 x 256 tiles on CTA pairs (at least 148 tiles of 128 x 256)
    (4096, 1280, 512, fp4.NVFP4, torch.bfloat16),
    (2560, 2048, 1024, fp4.MXFP4, torch.float32),    # FP32 out: TMEM handed back after the stores
    (2432, 2144, 2080, fp4.NVFP4, torch.bfloat16),   # last M tile: second CTA has no rows; last
                                                     # N tile: 96 columns; K tail of 32
]


@pytest.mark.parametrize("m,n,k,fmt,out_dtype", GEMM_CASES)
def test_gemm_random_within_tolerance(m, n, k, fmt, out_dtype):
    blk = 16 if fmt == fp4.NVFP4 else 32
    xa = random_input(m, k, m * 31 + k, torch.bfloat16)
    xb = random_input(n, k, n * 17 + k + 1, torch.float32, std=0.02, outliers=False)
    qa, qb = gpu_quantize(xa.cuda(), fmt, blk), gpu_quantize(xb.cuda(), fmt, blk)
    d = _gemm(qa, qb, out_dtype)
    oa, ob = oracle_quantize(xa, fmt, blk), oracle_quantize(xb, fmt, blk)
    check_gemm(d, dequant_oracle(oa, fmt), dequant_oracle(ob, fmt), label=f"{m}x{n}x{k}")


def test_gemm_pr1_configuration():
    """512^3 NVFP4 with the seeded fp32 inputs (every 512th element x20), FP32 out."""
    a, b = workloads.pr1_inputs()
    qa, qb = gpu_quantize(a.cuda(), fp4.NVFP4, 16), gpu_quantize(b.cuda(), fp4.NVFP4, 16)
    d = _gemm(qa, qb, torch.float32)
    oa, ob = oracle_quantize(a, fp4.NVFP4, 16), oracle_quantize(b, fp4.NVFP4, 16)
    check_gemm(d, dequant_oracle(oa, fp4.NVFP4), dequant_oracle(ob, fp4.NVFP4), label="pr1")


def test_gemm_repeatable_and_workspace_clean():
    """The split-over-K path leaves its workspace zero-filled; a second call agrees."""
    xa = random_input(16, 2048, 5, torch.bfloat16)
    xb = random_input(512, 2048, 6, torch.float32, std=0.02)
    qa, qb = gpu_quantize(xa.cuda(), fp4.NVFP4, 16), gpu_quantize(xb.cuda(), fp4.NVFP4, 16)
    ws = fp4.Workspace()
    d1 = fp4.gemm(qa, qb, torch.float32, workspace=ws)
    torch.cuda.synchronize()
    assert not ws.buf.any()
    d2 = fp4.gemm(qa, qb, torch.float32, workspace=ws)
    torch.cuda.synchronize()
    # FP32 partial sums meet in a different order: equal to within the tolerance
    oa, ob = oracle_quantize(xa, fp4.NVFP4, 16), oracle_quantize(xb, fp4.NVFP4, 16)
    for d in (d1, d2):
        check_gemm(d, dequant_oracle(oa, fp4.NVFP4), dequant_oracle(ob, fp4.NVFP4))


def test_split_k_counters_reset_between_shapes():
    """The split-over-K path counts each tile's finished K steps in the workspace; the
    pipeline completing a tile writes it and resets its counter, so calls of different
    shapes can share one workspace back to back."""
    shapes = [(16, 1024, 4096), (1, 256, 512), (32, 640, 2048), (16, 1024, 4096)]
    ws = fp4.Workspace()
    for i, (m, n, k) in enumerate(shapes):
        xa = random_input(m, k, 40 + i, torch.bfloat16)
        xb = random_input(n, k, 50 + i, torch.float32, std=0.02)
        qa, qb = gpu_quantize(xa.cuda(), fp4.NVFP4, 16), gpu_quantize(xb.cuda(), fp4.NVFP4, 16)
        d = fp4.gemm(qa, qb, torch.bfloat16, workspace=ws)
        torch.cuda.synchronize()
        assert not ws.buf.any(), f"workspace not clean after {m}x{n}x{k}"
        oa, ob = oracle_quantize(xa, fp4.NVFP4, 16), oracle_quantize(xb, fp4.NVFP4, 16)
        check_gemm(d, dequant_oracle(oa, fp4.NVFP4), dequant_oracle(ob, fp4.NVFP4), label=f"{m}x{n}x{k}")


SMALL_EXPERTS = (0, 130, 130, 300, 301, 560)
LARGE_EXPERTS = (0, 1300, 1300, 4000)   # >= 1280 rows per expert on average: CTA-pair tiles


@pytest.mark.parametrize("offs,N,out", [(SMALL_EXPERTS, 256, "bf16"), (SMALL_EXPERTS, 384, "bf16"),
                                        (SMALL_EXPERTS, 128, "bf16"), (SMALL_EXPERTS, 384, "f32"),
                                        (LARGE_EXPERTS, 256, "bf16"), (LARGE_EXPERTS, 384, "bf16")])
def test_grouped_gemm_moe_small(offs, N, out):
    """Grouped MXFP4 GEMM with an empty expert and ragged expert sizes; N = 384 leaves each
    expert's last 256-wide tile half empty (it reads into the next expert's weights, and
    past the last expert's, without storing those columns).  Small experts run 128-row
    tiles on single CTAs, large ones 256-row tiles on CTA pairs (partly empty last tiles).
    FP32 output takes the epilogue's general path instead of the BF16 row-major one."""
    offsets = np.array(offs, np.int32)
    E, K = len(offsets) - 1, 2880
    rows = int(offsets[-1])
    xa = random_input(rows, K, 41, torch.bfloat16)
    w = workloads.normal((E, N, K), 0.02, 42)
    off_d = torch.from_numpy(offsets).cuda()
    cap = fp4.fp4_scales_bytes_grouped(rows, E, K, fp4.MXFP4)
    codes = torch.empty(rows, K // 2, dtype=torch.uint8, device="cuda")
    scales = torch.empty(cap, dtype=torch.uint8, device="cuda")
    fp4.fp4_quantize_grouped(xa.cuda(), rows, K, fp4.BF16, fp4.MXFP4, E, off_d, codes, scales, None)
    wq = [gpu_quantize(w[e].cuda(), fp4.MXFP4, 32) for e in range(E)]
    B = torch.stack([q.codes for q in wq])
    sB = torch.cat([q.scales for q in wq])
    D = torch.empty(rows, N, dtype=torch.bfloat16 if out == "bf16" else torch.float32, device="cuda")
    fp4.fp4_gemm_grouped(fp4.MXFP4, E, off_d, codes, scales, None, B, sB, None, rows, N, K, D,
                         fp4.BF16 if out == "bf16" else fp4.F32)
    torch.cuda.synchronize()
    assert fp4.fp4_get_status() == fp4.OK
    oa = oracle_quantize(xa, fp4.MXFP4, 32)
    a_hat = dequant_oracle(oa, fp4.MXFP4)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        ob = oracle_quantize(w[e], fp4.MXFP4, 32)
        check_gemm(D[lo:hi], a_hat[lo:hi], dequant_oracle(ob, fp4.MXFP4), label=f"expert {e}")


def test_training_weight_reuse_forward_and_backward():
    """One 16x16 quantization of W serves D = X W^T and dX = dY W (W^T operand)."""
    s = 512
    x, w, dy = workloads.train_inputs(s)
    qw = gpu_quantize(w.cuda(), fp4.NVFP4, 256)
    qx, qdy = gpu_quantize(x.cuda(), fp4.NVFP4, 16), gpu_quantize(dy.cuda(), fp4.NVFP4, 16)
    d = _gemm(qx, qw, torch.bfloat16)
    dx = _gemm(qdy, fp4.transposed(qw), torch.bfloat16)
    ow = oracle_quantize(w, fp4.NVFP4, 256)
    w_hat = oracle.dequantize(ow["codes"], ow["scales"], ow["g"])
    wT_hat = oracle.dequantize(ow["codesT"], ow["scalesT"], ow["g"])
    assert np.array_equal(w_hat.T, wT_hat)
    check_gemm(d, dequant_oracle(oracle_quantize(x, fp4.NVFP4, 16), fp4.NVFP4), w_hat, label="fwd")
    check_gemm(dx, dequant_oracle(oracle_quantize(dy, fp4.NVFP4, 16), fp4.NVFP4), wT_hat, label="bwd")


def test_gemm_ex_weights_ready_decode():
    """Activations quantized by the kernel just before the GEMM; the weights were quantized
    earlier, so the GEMM may stream them before the activation quantize has finished."""
    m, n, k = 16, 4096, 8192
    xa = random_input(m, k, 77, torch.bfloat16)
    xb = random_input(n, k, 78, torch.float32, std=0.02, outliers=False)
    qb = gpu_quantize(xb.cuda(), fp4.NVFP4, 16)
    ws = fp4.Workspace()
    wsn = fp4.fp4_gemm_workspace_size(m, n, k, fp4.NVFP4)
    buf = ws.get(wsn)
    ob = oracle_quantize(xb, fp4.NVFP4, 16)
    for rep in range(3):
        qa = fp4.quantize(xa.cuda(), fp4.NVFP4, 16)   # no synchronization in between
        d = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
        fp4.fp4_gemm_ex(fp4.NVFP4, qa.codes, qa.scales, qa.g, qb.codes, qb.scales, qb.g, m, n, k, d, fp4.BF16,
                        buf, buf.numel(), fp4.GEMM_WEIGHTS_READY)
        torch.cuda.synchronize()
        assert fp4.fp4_get_status() == fp4.OK
        oa = oracle_quantize(xa, fp4.NVFP4, 16)
        check_gemm(d, dequant_oracle(oa, fp4.NVFP4), dequant_oracle(ob, fp4.NVFP4), label=f"rep {rep}")


def _bf16a(xa, qb, n, k, out_dtype=torch.bfloat16, flags=0, ws=None):
    m = xa.shape[0]
    dev = "cuda"
    xq = torch.empty(m, k // 2, dtype=torch.uint8, device=dev)
    xs = torch.empty(fp4.fp4_scales_bytes(m, k, fp4.NVFP4), dtype=torch.uint8, device=dev)
    gx = torch.empty(1, dtype=torch.float32, device=dev)
    d = torch.empty(m, n, dtype=out_dtype, device=dev)
    if ws is None:
        ws = torch.zeros(fp4.fp4_gemm_bf16a_workspace_size(m, n, k), dtype=torch.uint8, device=dev)
    fp4.fp4_gemm_bf16a(xa, qb.codes, qb.scales, qb.g, m, n, k, d, fp4.BF16 if out_dtype == torch.bfloat16 else fp4.F32,
                       xq, xs, gx, ws, ws.numel(), flags)
    torch.cuda.synchronize()
    assert fp4.fp4_get_status() == fp4.OK
    return d, fp4.Quantized(xq, xs, gx, m, k, fp4.NVFP4), ws


@pytest.mark.parametrize("m,n,k,flags", [(16, 1024, 4096, 0), (16, 1024, 4096, 1), (1, 256, 256, 0),
                                         (32, 512, 2048, 1), (5, 384, 96, 0), (200, 256, 512, 1),
                                         (20, 1000, 2080, 1), (16, 384, 16384, 0)])
def test_gemm_bf16a_matches_oracle(m, n, k, flags):
    """Activations quantized inside the call: codes, scales and g bit-exact; D in tolerance."""
    from fp4_testutil import assert_quant_equal
    xa = random_input(m, k, 300 + m, torch.bfloat16).cuda()
    xb = random_input(n, k, 301 + n, torch.float32, std=0.02, outliers=False)
    qb = gpu_quantize(xb.cuda(), fp4.NVFP4, 16)
    ob = oracle_quantize(xb, fp4.NVFP4, 16)
    ws = None
    for rep in range(2):   # the workspace carries state from call to call
        d, qx, ws = _bf16a(xa, qb, n, k, flags=flags, ws=ws)
        ox = oracle_quantize(xa.cpu(), fp4.NVFP4, 16)
        assert_quant_equal(qx, ox, f"activations {m}x{k} rep {rep}")
        check_gemm(d, dequant_oracle(ox, fp4.NVFP4), dequant_oracle(ob, fp4.NVFP4), label=f"{m}x{n}x{k} rep {rep}")


def test_gemm_bf16a_full_decode_shape_sampled():
    """The decode configuration in the bench's launch shape (16 x 28672 x 8192)."""
    x, w = workloads.decode_inputs()
    qb = gpu_quantize(w.cuda(), fp4.NVFP4, 16)
    d, qx, _ = _bf16a(x.cuda(), qb, 28672, 8192, flags=fp4.GEMM_WEIGHTS_READY)
    from fp4_testutil import assert_quant_equal, host_input
    ox = oracle_quantize(x, fp4.NVFP4, 16)
    assert_quant_equal(qx, ox, "decode activations")
    # sampled weight rows (output columns): quantize them with W's global scale
    hw = host_input(w)
    g = oracle.global_scale(oracle.amax(hw))
    cols = np.unique(np.concatenate([[0, 28671], np.random.default_rng(1).integers(0, 28672, 256)]))
    ob = oracle.quantize(hw[cols], oracle.NVFP4, 16, g_in=g)
    b_hat = oracle.dequantize(ob["codes"], ob["scales"], ob["g"])
    d_ref, s = oracle.gemm_reference(dequant_oracle(ox, fp4.NVFP4), b_hat)
    got = d[:, torch.from_numpy(cols).cuda()].float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - d_ref) <= oracle.gemm_tolerance(d_ref, s, True))


def test_bounded_wait_runs_out_and_the_next_call_is_correct():
    """The decode kernel's CTAs wait (bounded) for each other's share of the activations'
    amax.  With one share never published (the test hook), every wait runs out: the call
    latches FP4_ERR_TIMEOUT and returns; the device stays usable, and the next call on a
    zero-filled workspace gives the oracle's result."""
    m, n, k = 16, 2048, 4096
    xa = random_input(m, k, 61, torch.bfloat16).cuda()
    xb = random_input(n, k, 62, torch.float32, std=0.02, outliers=False)
    qb = gpu_quantize(xb.cuda(), fp4.NVFP4, 16)
    ws = torch.zeros(fp4.fp4_gemm_bf16a_workspace_size(m, n, k), dtype=torch.uint8, device="cuda")
    fp4.fp4_debug_stall_next_decode(3)
    xq = torch.empty(m, k // 2, dtype=torch.uint8, device="cuda")
    xs = torch.empty(fp4.fp4_scales_bytes(m, k, fp4.NVFP4), dtype=torch.uint8, device="cuda")
    gx = torch.empty(1, dtype=torch.float32, device="cuda")
    d = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    fp4.fp4_gemm_bf16a(xa, qb.codes, qb.scales, qb.g, m, n, k, d, fp4.BF16, xq, xs, gx, ws, ws.numel())
    assert fp4.fp4_get_status() == fp4.ERR_TIMEOUT
    assert fp4.fp4_get_status() == fp4.OK          # read and cleared
    ws.zero_()
    d2, qx, _ = _bf16a(xa, qb, n, k, ws=ws)
    from fp4_testutil import assert_quant_equal
    ox, ob = oracle_quantize(xa.cpu(), fp4.NVFP4, 16), oracle_quantize(xb, fp4.NVFP4, 16)
    assert_quant_equal(qx, ox, "after the timeout")
    check_gemm(d2, dequant_oracle(ox, fp4.NVFP4), dequant_oracle(ob, fp4.NVFP4), label="after the timeout")
