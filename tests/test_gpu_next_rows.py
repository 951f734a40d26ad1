"""The steps around the hot path against the oracle, through the C ABI:

- stochastic rounding (fp4_quantize_sr): codes and scales bit-exact against
  oracle.quantize_sr on the same random words;
- the Hadamard transform before quantizing (fp4_quantize_rht): bit-exact against
  oracle.quantize of oracle.rht16(x, signs);
- the rounded-down E8M0 scale (fp4_quantize_ex, FP4_QUANT_E8M0_FLOOR): bit-exact;
- a tensor split by rows over ranks (fp4_amax per shard, MAX of the maxima,
  fp4_global_scale): the shards' codes and scales equal the whole tensor's;
- the GEMM epilogue (fp4_gemm_epilogue): bias and ReLU within the epilogue tolerance of
  oracle.epilogue; the NVFP4 copy of the result bit-exact against oracle.quantize of the
  kernel's own FP32 result with the caller's global scale."""
import numpy as np
import pytest
import torch

import block_scaled_fp4_04_b200 as fp4
import oracle
from fp4_testutil import assert_quant_equal, dequant_oracle, gpu_quantize, host_input, oracle_quantize, random_input

pytestmark = pytest.mark.gpu


def _ws():
    return torch.zeros(fp4.fp4_quantize_workspace_size(), dtype=torch.uint8, device="cuda")


def _outs(rows, cols, fmt):
    codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device="cuda")
    scales = torch.full((fp4.fp4_scales_bytes(rows, cols, fmt),), 0xA5, dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    return codes, scales, g


# ---------------------------------------------------------------- stochastic rounding
@pytest.mark.parametrize("rows,cols,dtype", [(130, 256, torch.float32), (512, 1024, torch.bfloat16),
                                             (3, 4096, torch.bfloat16), (257, 2880, torch.float32)])
def test_quantize_sr_bit_exact(rows, cols, dtype):
    x = random_input(rows, cols, rows + cols, dtype)
    bits = np.random.default_rng(rows * cols).integers(0, 2 ** 32, (rows, cols), dtype=np.uint64).astype(np.uint32)
    codes, scales, g = _outs(rows, cols, fp4.NVFP4)
    ws = _ws()
    fp4.fp4_quantize_sr(x.cuda(), rows, cols, fp4.BF16 if dtype == torch.bfloat16 else fp4.F32,
                        torch.from_numpy(bits.view(np.int32)).cuda(), codes, scales, g, None, ws, ws.numel())
    assert fp4.fp4_get_status() == fp4.OK
    oq = oracle.quantize_sr(host_input(x), bits)
    oq["scales_sw"] = oracle.swizzle_scales(oq["scales"])
    assert_quant_equal(fp4.Quantized(codes, scales, g, rows, cols, fp4.NVFP4), oq, f"sr {rows}x{cols}")


def test_quantize_sr_extreme_words_and_global_in():
    """All-zero words round every off-grid magnitude up, all-ones words down (u < frac
    fails for u = 1 - 2^-24 only when frac is smaller); a caller's g is used as given."""
    rows, cols = 64, 512
    x = random_input(rows, cols, 5, torch.float32)
    for word in (0, 0xFFFFFFFF):
        bits = np.full((rows, cols), word, np.uint32)
        codes, scales, g = _outs(rows, cols, fp4.NVFP4)
        gin = torch.tensor([0.0123], dtype=torch.float32, device="cuda")
        fp4.fp4_quantize_sr(x.cuda(), rows, cols, fp4.F32, torch.from_numpy(bits.view(np.int32)).cuda(), codes, scales,
                            g, gin)
        assert fp4.fp4_get_status() == fp4.OK
        oq = oracle.quantize_sr(host_input(x), bits, g_in=np.float32(0.0123))
        oq["scales_sw"] = oracle.swizzle_scales(oq["scales"])
        assert_quant_equal(fp4.Quantized(codes, scales, g, rows, cols, fp4.NVFP4), oq, f"word {word:#x}")


def test_quantize_sr_words_at_the_decision_boundary():
    """Every element's random word is placed at its rounding decision: bits >> 8 either the
    largest value that still rounds up (u just below the fraction) or the one above it.  The
    fractions are worked out here from round-to-nearest block scales (stochastic rounding
    keeps them); whether each word lands exactly on the boundary only sharpens the test: the
    expected codes are the oracle's for those words."""
    rows, cols = 64, 1024
    x = random_input(rows, cols, 21, torch.float32)
    xh = host_input(x)
    oq = oracle.quantize(xh, fp4.NVFP4, 16)
    g = np.float32(oq["g"])
    denom = (np.vectorize(oracle.e4m3_decode)(oq["scales"]).astype(np.float32) * g).astype(np.float32)
    inv = np.zeros_like(denom)
    np.divide(np.float32(1.0), denom, out=inv, where=denom != 0)
    a = np.abs((xh.astype(np.float32) * np.repeat(inv, 16, axis=1)).astype(np.float32))
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    lo = np.clip(np.searchsorted(grid, a, side="right") - 1, 0, 6)
    frac = (a - grid[lo]).astype(np.float64) / (grid[lo + 1] - grid[lo]).astype(np.float64)
    rng = np.random.default_rng(22)
    n = np.ceil(frac * 2 ** 24).astype(np.int64) - 1 + rng.integers(0, 2, a.shape)
    bits = ((np.clip(n, 0, 2 ** 24 - 1) << 8) | rng.integers(0, 256, a.shape)).astype(np.uint32)
    codes, scales, gd = _outs(rows, cols, fp4.NVFP4)
    ws = _ws()
    fp4.fp4_quantize_sr(x.cuda(), rows, cols, fp4.F32, torch.from_numpy(bits.view(np.int32)).cuda(), codes, scales,
                        gd, None, ws, ws.numel())
    assert fp4.fp4_get_status() == fp4.OK
    osr = oracle.quantize_sr(xh, bits)
    osr["scales_sw"] = oracle.swizzle_scales(osr["scales"])
    assert_quant_equal(fp4.Quantized(codes, scales, gd, rows, cols, fp4.NVFP4), osr, "words at the boundary")
    # the placement did reach both sides of the decision: some codes round up, some do not
    assert 0 < np.count_nonzero(osr["codes"] != oq["codes"]) < osr["codes"].size


def test_quantize_sr_is_unbiased_on_the_device():
    """Averaged over many draws, the dequantized value approaches x (the page's reason for
    stochastic rounding).  In units of the block scale, the per-element error of the mean
    of 256 draws is about 1/32 of an E2M1 gap; round-to-nearest would leave a fixed error
    of up to half a gap (about a quarter on average)."""
    rows, cols, reps = 16, 256, 256
    x = random_input(rows, cols, 9, torch.float32, outliers=False)
    rng = np.random.default_rng(10)
    acc = np.zeros((rows, cols))
    ws = _ws()
    for _ in range(reps):
        bits = rng.integers(0, 2 ** 32, (rows, cols), dtype=np.uint64).astype(np.uint32)
        codes, scales, g = _outs(rows, cols, fp4.NVFP4)
        fp4.fp4_quantize_sr(x.cuda(), rows, cols, fp4.F32, torch.from_numpy(bits.view(np.int32)).cuda(), codes,
                            scales, g, None, ws, ws.numel())
        sc = oracle.unswizzle_scales(scales.cpu().numpy(), rows, cols // 16)
        acc += oracle.dequantize(codes.cpu().numpy(), sc, g.item())
    assert fp4.fp4_get_status() == fp4.OK
    scale = np.repeat(np.vectorize(oracle.e4m3_decode)(sc) * g.item(), 16, axis=1)
    err = np.abs(acc / reps - x.numpy().astype(np.float64)) / scale
    assert np.mean(err) < 0.1, np.mean(err)


# ---------------------------------------------------------------- Hadamard transform
@pytest.mark.parametrize("fmt", [fp4.NVFP4, fp4.MXFP4])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("signs", [0x0000, 0xA5C3])
def test_quantize_rht_bit_exact(fmt, dtype, signs):
    rows, cols = 300, 1024
    x = random_input(rows, cols, 77 + signs % 7, dtype)
    codes, scales, g = _outs(rows, cols, fmt)
    ws = _ws()
    fp4.fp4_quantize_rht(x.cuda(), rows, cols, fp4.BF16 if dtype == torch.bfloat16 else fp4.F32, fmt, signs, codes,
                         scales, g, None, ws, ws.numel())
    assert fp4.fp4_get_status() == fp4.OK
    y = oracle.rht16(host_input(x), signs)
    blk = 16 if fmt == fp4.NVFP4 else 32
    oq = oracle.quantize(y, fmt, blk)
    oq["scales_sw"] = oracle.swizzle_scales(oq["scales"])
    assert_quant_equal(fp4.Quantized(codes, scales, g, rows, cols, fmt), oq, f"rht {signs:#x}")


def test_rht_gemm_keeps_the_product():
    """Both operands transformed with the same signs: the GEMM of the quantized
    transforms is within tolerance of the oracle's product of those operands, and close
    to the untransformed product (the transform is orthogonal)."""
    m, n, k, signs = 256, 384, 1024, 0x3C5A
    xa = random_input(m, k, 1, torch.bfloat16)
    xb = random_input(n, k, 2, torch.float32, std=0.02, outliers=False)
    qs = []
    for x, dt in ((xa, fp4.BF16), (xb, fp4.F32)):
        rows = x.shape[0]
        codes, scales, g = _outs(rows, k, fp4.NVFP4)
        fp4.fp4_quantize_rht(x.cuda(), rows, k, dt, fp4.NVFP4, signs, codes, scales, g, None, _ws(),
                             fp4.fp4_quantize_workspace_size())
        qs.append(fp4.Quantized(codes, scales, g, rows, k, fp4.NVFP4))
    d = fp4.gemm(qs[0], qs[1], torch.float32)
    torch.cuda.synchronize()
    assert fp4.fp4_get_status() == fp4.OK
    hats = []
    for x in (xa, xb):
        oq = oracle.quantize(oracle.rht16(host_input(x), signs), fp4.NVFP4, 16)
        hats.append(oracle.dequantize(oq["codes"], oq["scales"], oq["g"]))
    d_ref, s = oracle.gemm_reference(hats[0], hats[1])
    got = d.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - d_ref) <= oracle.gemm_tolerance(d_ref, s, False))
    exact = xa.float().numpy().astype(np.float64) @ xb.numpy().astype(np.float64).T
    assert np.linalg.norm(got - exact) < 0.2 * np.linalg.norm(exact)


# ---------------------------------------------------------------- E8M0 rounded down
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_mx_floor_bit_exact(dtype):
    rows, cols = 257, 2880
    x = random_input(rows, cols, 33, dtype)
    x[3, :64] = 0.0                      # an all-zero block
    x[4, :32] = 2.0 ** -130              # a subnormal block
    codes, scales, g = _outs(rows, cols, fp4.MXFP4)
    fp4.fp4_quantize_ex(x.cuda(), rows, cols, fp4.BF16 if dtype == torch.bfloat16 else fp4.F32, fp4.MXFP4, 32,
                        fp4.QUANT_E8M0_FLOOR, codes, scales, g)
    assert fp4.fp4_get_status() == fp4.OK
    oq = oracle.quantize(host_input(x), fp4.MXFP4, 32, e8m0_floor=True)
    oq["scales_sw"] = oracle.swizzle_scales(oq["scales"])
    assert_quant_equal(fp4.Quantized(codes, scales, g, rows, cols, fp4.MXFP4), oq, "mx floor")


def test_quantize_ex_rejects_floor_for_nvfp4():
    x = torch.zeros(16, 64, device="cuda")
    codes, scales, g = _outs(16, 64, fp4.NVFP4)
    with pytest.raises(fp4.Fp4Error):
        fp4.fp4_quantize_ex(x, 16, 64, fp4.F32, fp4.NVFP4, 16, fp4.QUANT_E8M0_FLOOR, codes, scales, g, None, None,
                            None, _ws(), fp4.fp4_quantize_workspace_size())


# ---------------------------------------------------------------- row shards, one global scale
@pytest.mark.parametrize("splits", [[0, 100, 300], [0, 128, 256, 300]])
def test_row_shards_with_reduced_amax_equal_the_whole_tensor(splits):
    """Each shard's fp4_amax, the maximum over shards (what an all-reduce MAX gives every
    rank), fp4_global_scale, then fp4_quantize of each shard with that g: bit-identical to
    the oracle's whole-tensor quantization."""
    rows, cols = splits[-1], 768
    x = random_input(rows, cols, 55, torch.bfloat16).cuda()
    ws = _ws()
    amaxes = []
    for lo, hi in zip(splits[:-1], splits[1:]):
        a = torch.empty(1, dtype=torch.float32, device="cuda")
        fp4.fp4_amax(x[lo:hi], (hi - lo) * cols, fp4.BF16, a, ws, ws.numel())
        amaxes.append(a)
    amax = torch.stack(amaxes).max().reshape(1).contiguous()
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    fp4.fp4_global_scale(amax, g)
    oq = oracle_quantize(x.cpu(), fp4.NVFP4, 16)
    assert np.float32(g.item()).tobytes() == np.float32(oq["g"]).tobytes()
    for lo, hi in zip(splits[:-1], splits[1:]):
        codes, scales, gout = _outs(hi - lo, cols, fp4.NVFP4)
        fp4.fp4_quantize(x[lo:hi], hi - lo, cols, fp4.BF16, fp4.NVFP4, 16, codes, scales, gout, None, None, g, ws,
                         ws.numel())
        torch.cuda.synchronize()
        assert np.array_equal(codes.cpu().numpy(), oq["codes"][lo:hi])
        sc = oracle.unswizzle_scales(scales.cpu().numpy(), hi - lo, cols // 16)
        assert np.array_equal(sc, oq["scales"][lo:hi])
    assert fp4.fp4_get_status() == fp4.OK


def test_global_scale_of_zero_and_nonfinite():
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    fp4.fp4_global_scale(torch.zeros(1, device="cuda"), g)
    assert g.item() == 1.0 and fp4.fp4_get_status() == fp4.OK
    fp4.fp4_global_scale(torch.tensor([float("inf")], device="cuda"), g)
    assert fp4.fp4_get_status() == fp4.ERR_NONFINITE


# ---------------------------------------------------------------- GEMM epilogue
EPI_CASES = [
    # m, n, k, act, fp4 out, kernel path exercised
    (256, 256, 512, "relu", True),      # whole 128-wide tiles
    (130, 384, 1024, "none", True),     # ragged last M tile
    (2560, 2048, 512, "relu", True),    # 256 x 256 tiles on CTA pairs
    (2560, 2048, 512, "relu", False),   # the same, BF16 tiles handed back before their stores
    (256, 256, 8192, "relu", True),     # few tiles, long K: split over K
    (16, 1024, 2048, "relu", False),    # decode kernel (bias and ReLU at its write-out)
    (48, 640, 2048, "none", False),     # swapped operands, N-tile 64
    (16, 1024, 2048, "relu", True),     # FP4 output of a decode-sized problem: rows kept in place
]


@pytest.mark.parametrize("m,n,k,act,fp4_out", EPI_CASES)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_epilogue(m, n, k, act, fp4_out, out_dtype):
    xa = random_input(m, k, m + 7 * k, torch.bfloat16)
    xb = random_input(n, k, n + 11 * k, torch.float32, std=0.02, outliers=False)
    qa, qb = gpu_quantize(xa.cuda(), fp4.NVFP4, 16), gpu_quantize(xb.cuda(), fp4.NVFP4, 16)
    bias = (np.random.default_rng(n).standard_normal(n) * 3.0).astype(np.float32)
    d = torch.empty(m, n, dtype=out_dtype, device="cuda")
    codes = scales = gD = amax = None
    if fp4_out:
        codes = torch.empty(m, n // 2, dtype=torch.uint8, device="cuda")
        scales = torch.full((fp4.fp4_scales_bytes(m, n, fp4.NVFP4),), 0xA5, dtype=torch.uint8, device="cuda")
        gD = torch.tensor([0.01], dtype=torch.float32, device="cuda")
        amax = torch.full((1,), 123.0, dtype=torch.float32, device="cuda")   # zeroed by the call
    wsn = fp4.fp4_gemm_epilogue_workspace_size(m, n, k, fp4.NVFP4, fp4_out)
    ws = torch.zeros(max(wsn, 16), dtype=torch.uint8, device="cuda")
    fp4.fp4_gemm_epilogue(fp4.NVFP4, qa.codes, qa.scales, qa.g, qb.codes, qb.scales, qb.g, m, n, k,
                          torch.from_numpy(bias).cuda(), fp4.ACT_RELU if act == "relu" else fp4.ACT_NONE, d,
                          fp4.BF16 if out_dtype == torch.bfloat16 else fp4.F32, codes, scales, gD, amax, ws, wsn)
    torch.cuda.synchronize()
    assert fp4.fp4_get_status() == fp4.OK
    assert not ws.any(), "workspace not left zero-filled"
    oa, ob = oracle_quantize(xa, fp4.NVFP4, 16), oracle_quantize(xb, fp4.NVFP4, 16)
    d_ref, s = oracle.gemm_reference(dequant_oracle(oa, fp4.NVFP4), dequant_oracle(ob, fp4.NVFP4))
    t_ref = oracle.epilogue(d_ref, bias.astype(np.float64), act)
    got = d.float().cpu().numpy().astype(np.float64)
    tol = oracle.epilogue_tolerance(t_ref, d_ref, s, bias, out_dtype == torch.bfloat16)
    bad = np.argwhere(~(np.abs(got - t_ref) <= tol))
    assert bad.size == 0, f"{len(bad)} outputs outside tolerance, first {bad[:3].tolist()}"
    if fp4_out:
        # the result's amax: exactly the largest stored FP32 magnitude, or the reference's
        # within the tolerance when the stored copy is BF16
        if out_dtype == torch.float32:
            assert amax.item() == float(np.abs(got).max())
        else:
            i = np.unravel_index(np.argmax(np.abs(t_ref)), t_ref.shape)
            assert abs(amax.item() - abs(t_ref[i])) <= tol[i] + 1e-30
    if fp4_out and out_dtype == torch.float32:
        # the NVFP4 copy quantizes the same FP32 values the kernel stored
        oq = oracle.quantize(d.cpu().numpy(), fp4.NVFP4, 16, g_in=np.float32(0.01))
        oq["scales_sw"] = oracle.swizzle_scales(oq["scales"])
        assert_quant_equal(fp4.Quantized(codes, scales, gD, m, n, fp4.NVFP4), oq, f"fp4 out {m}x{n}x{k}")


def test_gemm_epilogue_fp4_only_output_feeds_the_next_gemm():
    """D in NVFP4 only (no BF16/FP32 copy): it is the A operand of the next GEMM."""
    m, n, k, n2 = 256, 512, 1024, 256
    xa = random_input(m, k, 1, torch.bfloat16)
    xb = random_input(n, k, 2, torch.float32, std=0.02, outliers=False)
    xc = random_input(n2, n, 3, torch.float32, std=0.02, outliers=False)
    qa, qb, qc = (gpu_quantize(t.cuda(), fp4.NVFP4, 16) for t in (xa, xb, xc))
    codes = torch.empty(m, n // 2, dtype=torch.uint8, device="cuda")
    scales = torch.empty(fp4.fp4_scales_bytes(m, n, fp4.NVFP4), dtype=torch.uint8, device="cuda")
    gD = torch.tensor([0.004], dtype=torch.float32, device="cuda")
    d32 = torch.empty(m, n, dtype=torch.float32, device="cuda")
    fp4.fp4_gemm_epilogue(fp4.NVFP4, qa.codes, qa.scales, qa.g, qb.codes, qb.scales, qb.g, m, n, k, None,
                          fp4.ACT_RELU, None, fp4.F32, codes, scales, gD)
    fp4.fp4_gemm_epilogue(fp4.NVFP4, qa.codes, qa.scales, qa.g, qb.codes, qb.scales, qb.g, m, n, k, None,
                          fp4.ACT_RELU, d32, fp4.F32)
    torch.cuda.synchronize()
    assert fp4.fp4_get_status() == fp4.OK
    oq = oracle.quantize(d32.cpu().numpy(), fp4.NVFP4, 16, g_in=np.float32(0.004))
    oq["scales_sw"] = oracle.swizzle_scales(oq["scales"])
    qd = fp4.Quantized(codes, scales, gD, m, n, fp4.NVFP4)
    assert_quant_equal(qd, oq, "fp4-only output")
    e = fp4.gemm(qd, qc, torch.float32)
    torch.cuda.synchronize()
    oc = oracle_quantize(xc, fp4.NVFP4, 16)
    d_ref, s = oracle.gemm_reference(oracle.dequantize(oq["codes"], oq["scales"], oq["g"]), dequant_oracle(oc, fp4.NVFP4))
    assert np.all(np.abs(e.cpu().numpy() - d_ref) <= oracle.gemm_tolerance(d_ref, s, False))


def test_gemm_epilogue_argument_checks():
    q = torch.zeros(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(fp4.Fp4Error):   # no output at all
        fp4.fp4_gemm_epilogue(fp4.NVFP4, q, q, None, q, q, None, 128, 128, 64, None, fp4.ACT_NONE, None, fp4.F32)
    with pytest.raises(fp4.Fp4Error):   # FP4 output needs N % 32 == 0
        fp4.fp4_gemm_epilogue(fp4.NVFP4, q, q, None, q, q, None, 128, 144, 64, None, fp4.ACT_NONE, None, fp4.F32,
                              q, q, torch.ones(1, device="cuda"))
