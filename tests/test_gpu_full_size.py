"""Full-size parity for the tensor-bound configurations, in the launch configurations the
benchmark times, against the oracle on sampled output rows: 64 random rows plus the first
and the last, every column.

- prefill: X [8192, 8192] BF16 (N(0,1), 0.1% outliers x50) quantized inside
  fp4_gemm_bf16a against pre-quantized NVFP4 weights W [8192, 8192]; the activations'
  codes, scales and g bit-exact on the sampled rows; D within tolerance.
- training S = 16384: W quantized once with 16x16 blocks (W and W^T bit-exact on sampled
  16-row bands of each), forward D = X W^T and backward dX = dY W from that one
  quantization, X and dY quantized with 16-element blocks.
- MoE: 32 experts, 4096 tokens routed top-4 (16384 rows), K = 2880, N = 5760, MXFP4:
  every expert's sampled rows (16 random plus its first and last).
- mixed FP4 x FP8: the prefill X quantized to MXFP8 against MXFP4 weights, 8192^3.
The oracle computes global scales over the whole tensors and quantizes only the rows it
needs (1-D blocks are independent per row)."""
import numpy as np
import pytest
import torch

import block_scaled_fp4_04_b200 as fp4
import oracle
import workloads
from fp4_testutil import host_input

pytestmark = pytest.mark.gpu


def _sample(rows: int, seed: int, count: int = 64) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, rows - 1], rng.integers(0, rows, count)]))


def _check_rows(d_gpu: torch.Tensor, rows: np.ndarray, a_hat: np.ndarray, b_hat: np.ndarray, label: str):
    """d_gpu's given rows against the FP64 product of a_hat (those rows) and b_hat."""
    d_ref, s = oracle.gemm_reference(a_hat, b_hat)
    got = d_gpu[torch.from_numpy(rows).to(d_gpu.device)].float().cpu().numpy().astype(np.float64)
    tol = oracle.gemm_tolerance(d_ref, s, d_gpu.dtype == torch.bfloat16)
    bad = np.argwhere(~(np.abs(got - d_ref) <= tol))
    assert bad.size == 0, f"{label}: {len(bad)} outputs outside tolerance, first {bad[:3].tolist()}"


def _oracle_rows_1d(hx: np.ndarray, rows: np.ndarray, fmt: int, blk: int, g=None):
    q = oracle.quantize(np.ascontiguousarray(hx[rows]), fmt, blk, g_in=g)
    return q, oracle.dequantize(q["codes"], q["scales"], q["g"], fmt)


def test_prefill_8192_cubed_bf16_activations():
    m = n = k = 8192
    x, w = workloads.prefill_inputs()
    qw = fp4.quantize(w.cuda(), fp4.NVFP4, 16)
    xq = torch.empty(m, k // 2, dtype=torch.uint8, device="cuda")
    xs = torch.empty(fp4.fp4_scales_bytes(m, k, fp4.NVFP4), dtype=torch.uint8, device="cuda")
    gx = torch.empty(1, dtype=torch.float32, device="cuda")
    d = torch.empty(m, n, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(fp4.fp4_gemm_bf16a_workspace_size(m, n, k), dtype=torch.uint8, device="cuda")
    fp4.fp4_gemm_bf16a(x.cuda(), qw.codes, qw.scales, qw.g, m, n, k, d, fp4.BF16, xq, xs, gx, ws, ws.numel(),
                       fp4.GEMM_WEIGHTS_READY)
    torch.cuda.synchronize()
    assert fp4.fp4_get_status() == fp4.OK
    hx, hw = host_input(x), host_input(w)
    g_x = oracle.global_scale(oracle.amax(hx))
    assert np.float32(gx.item()).tobytes() == np.float32(g_x).tobytes()
    rows = _sample(m, 1)
    qx, x_hat = _oracle_rows_1d(hx, rows, fp4.NVFP4, 16, g_x)
    assert np.array_equal(xq.cpu().numpy()[rows], qx["codes"])
    assert np.array_equal(oracle.unswizzle_scales(xs.cpu().numpy(), m, k // 16)[rows], qx["scales"])
    ow = oracle.quantize(hw, fp4.NVFP4, 16)
    w_hat = oracle.dequantize(ow["codes"], ow["scales"], ow["g"])
    # the weights the GEMM read are the library's quantization of W: bit-exact as well
    assert np.array_equal(qw.codes.cpu().numpy(), ow["codes"])
    _check_rows(d, rows, x_hat, w_hat, "prefill")


def test_training_16384_forward_and_backward_from_one_2d_quantization():
    s = 16384
    x, w, dy = workloads.train_inputs(s)
    qw = fp4.quantize(w.cuda(), fp4.NVFP4, 256)
    wt = fp4.transposed(qw)
    qx = fp4.quantize(x.cuda(), fp4.NVFP4, 16)
    qdy = fp4.quantize(dy.cuda(), fp4.NVFP4, 16)
    d = fp4.gemm(qx, qw, torch.bfloat16)
    dx = fp4.gemm(qdy, wt, torch.bfloat16)
    torch.cuda.synchronize()
    assert fp4.fp4_get_status() == fp4.OK
    hw = host_input(w)
    ow = oracle.quantize(hw, fp4.NVFP4, 256)
    assert np.float32(qw.g.item()).tobytes() == np.float32(ow["g"]).tobytes()
    # W and W^T codes and scales on sampled 16-row bands of each
    bands = np.unique(np.random.default_rng(2).integers(0, s // 16, 8)) * 16
    codes, codes_t = qw.codes.cpu().numpy(), qw.codesT.cpu().numpy()
    sc = oracle.unswizzle_scales(qw.scales.cpu().numpy(), s, s // 16)
    sc_t = oracle.unswizzle_scales(qw.scalesT.cpu().numpy(), s, s // 16)
    for b in bands:
        assert np.array_equal(codes[b:b + 16], ow["codes"][b:b + 16])
        assert np.array_equal(codes_t[b:b + 16], ow["codesT"][b:b + 16])
        assert np.array_equal(sc[b:b + 16], ow["scales"][b:b + 16])
        assert np.array_equal(sc_t[b:b + 16], ow["scalesT"][b:b + 16])
    w_hat = oracle.dequantize(ow["codes"], ow["scales"], ow["g"])
    del ow
    rows = _sample(s, 3)
    hxx, hdy = host_input(x), host_input(dy)
    _, x_hat = _oracle_rows_1d(hxx, rows, fp4.NVFP4, 16, oracle.global_scale(oracle.amax(hxx)))
    _check_rows(d, rows, x_hat, w_hat, "forward X W^T")
    _, dy_hat = _oracle_rows_1d(hdy, rows, fp4.NVFP4, 16, oracle.global_scale(oracle.amax(hdy)))
    # backward: the B operand is W^T, whose dequantization is w_hat transposed (pinned)
    _check_rows(dx, rows, dy_hat, w_hat.T, "backward dY W")


def test_moe_32_experts_16384_rows_mxfp4():
    a, w, offsets, _ = workloads.moe_inputs()
    E, N, K = w.shape
    rows = a.shape[0]
    off = offsets.numpy()
    off_d = offsets.cuda()
    codes = torch.empty(rows, K // 2, dtype=torch.uint8, device="cuda")
    scales = torch.empty(fp4.fp4_scales_bytes_grouped(rows, E, K, fp4.MXFP4), dtype=torch.uint8, device="cuda")
    fp4.fp4_quantize_grouped(a.cuda(), rows, K, fp4.BF16, fp4.MXFP4, E, off_d, codes, scales, None)
    wq = [fp4.quantize(w[e].cuda(), fp4.MXFP4, 32) for e in range(E)]
    B = torch.stack([q.codes for q in wq])
    sB = torch.cat([q.scales for q in wq])
    del wq
    D = torch.empty(rows, N, dtype=torch.bfloat16, device="cuda")
    fp4.fp4_gemm_grouped(fp4.MXFP4, E, off_d, codes, scales, None, B, sB, None, rows, N, K, D, fp4.BF16)
    torch.cuda.synchronize()
    assert fp4.fp4_get_status() == fp4.OK
    ha = host_input(a)
    rng = np.random.default_rng(4)
    for e in range(E):
        lo, hi = int(off[e]), int(off[e + 1])
        if hi == lo:
            continue
        local = np.unique(np.concatenate([[0, hi - lo - 1], rng.integers(0, hi - lo, 16)]))
        qa, a_hat = _oracle_rows_1d(ha, lo + local, fp4.MXFP4, 32)
        assert np.array_equal(codes[lo + torch.from_numpy(local).cuda()].cpu().numpy(), qa["codes"]), f"expert {e}"
        ob = oracle.quantize(w[e].numpy(), fp4.MXFP4, 32)
        b_hat = oracle.dequantize(ob["codes"], ob["scales"], ob["g"], fp4.MXFP4)
        _check_rows(D, lo + local, a_hat, b_hat, f"expert {e}")


def test_mixed_fp4_fp8_8192_cubed():
    """The mixed record's configuration: X [8192, 8192] BF16 quantized to MXFP8, W [8192,
    8192] to MXFP4, D = X W^T through fp4_gemm_mixed; X's codes and scales bit-exact on the
    sampled rows, W's everywhere, D within tolerance on the sampled rows."""
    m = n = k = 8192
    x, w = workloads.prefill_inputs()
    qx = fp4.quantize(x.cuda(), fp4.MXFP8, 32)
    qw = fp4.quantize(w.cuda(), fp4.MXFP4, 32)
    d = fp4.gemm_mixed(qx, qw, torch.bfloat16)
    torch.cuda.synchronize()
    assert fp4.fp4_get_status() == fp4.OK
    rows = _sample(m, 5)
    qx_o, x_hat = _oracle_rows_1d(host_input(x), rows, fp4.MXFP8, 32)
    assert np.array_equal(qx.codes.cpu().numpy()[rows], qx_o["codes"])
    assert np.array_equal(oracle.unswizzle_scales(qx.scales.cpu().numpy(), m, k // 32)[rows], qx_o["scales"])
    ow = oracle.quantize(host_input(w), fp4.MXFP4, 32)
    assert np.array_equal(qw.codes.cpu().numpy(), ow["codes"])
    w_hat = oracle.dequantize(ow["codes"], ow["scales"], ow["g"], fp4.MXFP4)
    _check_rows(d, rows, x_hat, w_hat, "mixed MXFP8 x MXFP4")
