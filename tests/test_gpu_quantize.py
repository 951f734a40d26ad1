"""Quantize kernels vs the oracle: codes, swizzled scales (pads included) and the
global scale must be bit-identical."""
import os

import numpy as np
import pytest
import torch

import block_scaled_fp4_04_b200 as fp4
import oracle
import workloads
from fp4_testutil import assert_quant_equal, gpu_quantize, oracle_quantize, random_input

pytestmark = pytest.mark.gpu

CASES_1D = [
    # rows, cols, dtype, fmt, block
    (1, 32, torch.float32, fp4.NVFP4, 16),
    (1, 4096, torch.float32, fp4.NVFP4, 16),
    (130, 96, torch.bfloat16, fp4.NVFP4, 16),       # ragged rows, scale columns pad 6 -> 8
    (512, 512, torch.float32, fp4.NVFP4, 16),
    (16, 8192, torch.bfloat16, fp4.NVFP4, 16),      # decode activations
    (300, 1056, torch.float32, fp4.NVFP4, 16),
    (64, 32, torch.float32, fp4.MXFP4, 32),
    (257, 2880, torch.bfloat16, fp4.MXFP4, 32),     # MoE K, 90 scale columns pad to 92
    (129, 160, torch.float32, fp4.MXFP4, 32),
]


@pytest.mark.parametrize("rows,cols,dtype,fmt,block", CASES_1D)
def test_quantize_1d_bit_exact(rows, cols, dtype, fmt, block):
    x = random_input(rows, cols, rows * 7 + cols, dtype)
    gq = gpu_quantize(x.cuda(), fmt, block)
    assert fp4.fp4_get_status() == fp4.OK
    assert_quant_equal(gq, oracle_quantize(x, fmt, block), f"{rows}x{cols}")


@pytest.mark.parametrize("rows,cols,dtype", [(32, 32, torch.float32), (64, 96, torch.bfloat16),
                                             (160, 128, torch.float32), (288, 320, torch.bfloat16),
                                             # partial last regions in both directions
                                             (416, 544, torch.float32), (1056, 2080, torch.bfloat16)])
def test_quantize_2d_bit_exact(rows, cols, dtype):
    x = random_input(rows, cols, rows + 3 * cols, dtype, std=0.02)
    gq = gpu_quantize(x.cuda(), fp4.NVFP4, 256)
    assert_quant_equal(gq, oracle_quantize(x, fp4.NVFP4, 256), f"2d {rows}x{cols}")


def test_quantize_2d_nonfinite_with_caller_global_scale():
    # with a caller g there is no amax pass: the 2-D kernel's own patch check reports it
    x = torch.ones(96, 160)
    x[70, 133] = float("inf")
    fp4.fp4_get_status()
    gpu_quantize(x.cuda(), fp4.NVFP4, 256, g_in=0.25)
    assert fp4.fp4_get_status() == fp4.ERR_NONFINITE


def test_quantize_caller_global_scale():
    x = random_input(200, 640, 11)
    for g in (0.5, 1.0 / 3.0, 7.25e-3):
        gq = gpu_quantize(x.cuda(), fp4.NVFP4, 16, g_in=g)
        assert_quant_equal(gq, oracle_quantize(x, fp4.NVFP4, 16, g_in=np.float32(g)), f"g={g}")


def _near_midpoint_maxima(g32: np.float32) -> np.ndarray:
    """Block maxima a whose quotient (a / 6) / g lands within 24 float steps of each point
    where the E4M3 code changes: the midpoints between E4M3 values (subnormal ones too),
    2^-6, and 448 and above (saturation)."""
    vals = sorted({oracle.e4m3_decode(c) for c in range(1, 127)})
    marks = [(a + b) / 2 for a, b in zip(vals, vals[1:])] + [2.0 ** -6, 448.0, 464.0, 480.0, 1e4]
    out = []
    for m in marks:
        a0 = np.float32(np.float64(m) * 6.0 * np.float64(g32))
        if not np.isfinite(a0) or a0 == 0:
            continue
        bits = int(a0.view(np.uint32))
        out.extend(np.array([bits + d for d in range(-24, 25)], np.uint32).view(np.float32))
    return np.array(out, np.float32)


@pytest.mark.parametrize("g", [1.0, 0.37, 3.1e-5, 7.7e4, 2.0 ** -20, 2.0 ** -70, 2.0 ** 70])
def test_nvfp4_block_scale_near_e4m3_midpoints(g):
    """Block maxima on both sides of every point where the E4M3 scale code changes, for
    global scales inside and far outside the usual range: scale bytes and codes equal the
    oracle's (two FP32 divisions, then E4M3 rounding).  The tensor holds more blocks than
    the single-launch path for small tensors takes, so the 1-D encode kernel runs."""
    g32 = np.float32(g)
    amaxes = _near_midpoint_maxima(g32)
    rows, cols = 640, 256
    nb = rows * cols // 16
    assert nb > 8192 and amaxes.size <= nb
    rng = np.random.default_rng(12)
    frac = rng.uniform(-0.999, 0.999, size=(nb, 15)).astype(np.float32)
    a = np.ones(nb, np.float32)
    a[:amaxes.size] = amaxes
    blocks = np.concatenate([a[:, None], (a[:, None] * frac).astype(np.float32)], axis=1)
    x = torch.from_numpy(np.ascontiguousarray(blocks.reshape(rows, cols)))
    gq = gpu_quantize(x.cuda(), fp4.NVFP4, 16, g_in=float(g32))
    torch.cuda.synchronize()
    assert_quant_equal(gq, oracle_quantize(x, fp4.NVFP4, 16, g_in=g32), f"g={g}")


def _golden_blocks():
    path = os.path.join(os.path.dirname(__file__), "golden", "worked_blocks.txt")
    out = []
    with open(path) as f:
        for ln in f:
            if ln.strip() and not ln.startswith("#"):
                parts = ln.split()
                kv = dict(p.split("=") for p in parts[1:])
                out.append((parts[0], float(kv["g"]), [float(v) for v in kv["values"].split(",")],
                            int(kv["scale"], 16), bytes.fromhex(kv["codes"])))
    return out


@pytest.mark.parametrize("idx", range(4))
def test_worked_blocks_on_gpu(idx):
    fmt_name, g, vals, scale, codes = _golden_blocks()[idx]
    x = torch.zeros(1, 32, dtype=torch.float32)    # rows hold a multiple of 32 values
    x[0, :len(vals)] = torch.tensor(vals)
    if fmt_name == "nvfp4":
        q = gpu_quantize(x.cuda(), fp4.NVFP4, 16, g_in=g)
    else:
        q = gpu_quantize(x.cuda(), fp4.MXFP4, 32)
    assert q.codes.cpu().numpy().tobytes()[:len(codes)] == codes
    assert q.scales.cpu().numpy()[0] == scale


# (130, 128) runs the single-launch path for small tensors, (300, 1024) the amax +
# quantize kernels of larger ones
@pytest.mark.parametrize("rows,cols", [(130, 128), (300, 1024)])
@pytest.mark.parametrize("kind", ["zeros", "neg_zeros", "tiny", "huge", "constant", "subnormal"])
def test_quantize_edge_tensors(kind, rows, cols):
    if kind == "zeros":
        x = torch.zeros(rows, cols)
    elif kind == "neg_zeros":
        x = -torch.zeros(rows, cols)
    elif kind == "tiny":
        x = random_input(rows, cols, 1) * 1e-30
    elif kind == "huge":
        x = random_input(rows, cols, 2) * 1e36
    elif kind == "constant":
        x = torch.full((rows, cols), -3.0)
    else:
        x = random_input(rows, cols, 3) * 1e-41
    x = x.float()
    for fmt, block in ((fp4.NVFP4, 16), (fp4.MXFP4, 32)):
        gq = gpu_quantize(x.cuda(), fmt, block)
        assert_quant_equal(gq, oracle_quantize(x, fmt, block), f"{kind} fmt {fmt}")


def test_quantize_block_far_below_tensor_amax():
    x = torch.full((4, 64), 1e-3)
    x[0, 0] = 1e4
    gq = gpu_quantize(x.cuda(), fp4.NVFP4, 16)
    assert_quant_equal(gq, oracle_quantize(x, fp4.NVFP4, 16))


@pytest.mark.parametrize("shape", [(64, 64), (400, 1024)])
@pytest.mark.parametrize("bad", [float("nan"), float("inf"), float("-inf")])
def test_nonfinite_input_latches_status(bad, shape):
    x = torch.ones(*shape)
    x[17, 5] = bad
    fp4.fp4_get_status()
    fp4.quantize(x.cuda(), fp4.NVFP4, 16)
    assert fp4.fp4_get_status() == fp4.ERR_NONFINITE
    fp4.quantize(x.cuda(), fp4.MXFP4, 32)
    assert fp4.fp4_get_status() == fp4.ERR_NONFINITE
    assert fp4.fp4_get_status() == fp4.OK  # reading clears it


def test_amax_entry_point():
    for n, dt in ((1, torch.float32), (1000003, torch.float32), (4097, torch.bfloat16), (16 * 8192, torch.bfloat16)):
        x = random_input(1, n, n % 1000, dt)
        ws = torch.zeros(fp4.fp4_quantize_workspace_size(), dtype=torch.uint8, device="cuda")
        out = torch.empty(1, dtype=torch.float32, device="cuda")
        xc = x.cuda()
        fp4.fp4_amax(xc, n, fp4.BF16 if dt == torch.bfloat16 else fp4.F32, out, ws, ws.numel())
        torch.cuda.synchronize()
        assert out.item() == oracle.amax(__import__("fp4_testutil").host_input(x))
        assert not ws.any()  # the workspace is left zero-filled


def test_grouped_quantize_layout():
    offsets = np.array([0, 3, 3, 200, 201, 460], np.int32)   # empty group, ragged groups
    x = random_input(460, 2880, 21, torch.bfloat16)
    E = len(offsets) - 1
    for fmt in (fp4.MXFP4, fp4.NVFP4):
        blk = 32 if fmt == fp4.MXFP4 else 16
        off_d = torch.from_numpy(offsets).cuda()
        cap = fp4.fp4_scales_bytes_grouped(460, E, 2880, fmt)
        codes = torch.empty(460, 1440, dtype=torch.uint8, device="cuda")
        scales = torch.full((cap,), 0xAB, dtype=torch.uint8, device="cuda")
        g = torch.empty(1, dtype=torch.float32, device="cuda")
        ws = torch.zeros(fp4.fp4_quantize_workspace_size(), dtype=torch.uint8, device="cuda")
        fp4.fp4_quantize_grouped(x.cuda(), 460, 2880, fp4.BF16, fmt, E, off_d, codes, scales, g, None, ws,
                                 ws.numel())
        torch.cuda.synchronize()
        oq = oracle_quantize(x, fmt, blk)
        sw = oracle.swizzle_scales_grouped(oq["scales"], offsets)
        got = scales.cpu().numpy()
        assert np.array_equal(codes.cpu().numpy(), oq["codes"])
        assert np.array_equal(got[:sw.size], sw)
        assert not got[sw.size:].any()   # the rest of the bound is zero pad


GROUP_OFFSETS = [
    # whole 128-row atoms, an empty group, three one-row groups inside one tile, ragged end
    [0, 128, 256, 257, 257, 300, 301, 302, 303, 430, 640, 700],
    # 128 one-row groups (all ending in the first tile), then 6- and 5-row groups
    list(range(0, 129)) + [129 + 5 * k for k in range(1, 40)],
    # leading empty groups, then one group over eight tiles, ending on a tile boundary
    [0, 0, 0, 1024],
    # one group of one row
    [0, 1],
]


@pytest.mark.parametrize("offsets", GROUP_OFFSETS, ids=["atoms", "one_row_groups", "empty_lead", "one_row"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_grouped_quantize_layout_group_patterns(offsets, dtype):
    """Groups that begin and end anywhere in a 128-row tile of x: each row's scale byte goes
    to its group's atom, the lanes past a group's rows and the atoms past the last group's
    are zero, up to the buffer's bound (pre-filled with a marker)."""
    offsets = np.array(offsets, np.int32)
    rows, cols, E = int(offsets[-1]), 320, len(offsets) - 1   # 320: a ragged column tile
    x = random_input(rows, cols, 5 + E, dtype)
    off_d = torch.from_numpy(offsets).cuda()
    dt = fp4.BF16 if dtype == torch.bfloat16 else fp4.F32
    for fmt in (fp4.MXFP4, fp4.NVFP4):
        blk = 32 if fmt == fp4.MXFP4 else 16
        cap = fp4.fp4_scales_bytes_grouped(rows, E, cols, fmt)
        codes = torch.full((rows, cols // 2), 0xCD, dtype=torch.uint8, device="cuda")
        scales = torch.full((cap,), 0xAB, dtype=torch.uint8, device="cuda")
        g = torch.empty(1, dtype=torch.float32, device="cuda")
        ws = torch.zeros(fp4.fp4_quantize_workspace_size(), dtype=torch.uint8, device="cuda")
        fp4.fp4_quantize_grouped(x.cuda(), rows, cols, dt, fmt, E, off_d, codes, scales, g, None, ws, ws.numel())
        torch.cuda.synchronize()
        assert fp4.fp4_get_status() == fp4.OK
        oq = oracle_quantize(x, fmt, blk)
        sw = oracle.swizzle_scales_grouped(oq["scales"], offsets)
        got = scales.cpu().numpy()
        assert np.array_equal(codes.cpu().numpy(), oq["codes"])
        assert np.array_equal(got[:sw.size], sw)
        assert not got[sw.size:].any()
        if fmt == fp4.NVFP4:
            assert np.float32(g.item()).tobytes() == np.float32(oq["g"]).tobytes()


def test_dequantize_matches_oracle():
    x = random_input(130, 256, 31)
    for fmt, blk in ((fp4.NVFP4, 16), (fp4.MXFP4, 32)):
        q = gpu_quantize(x.cuda(), fmt, blk)
        out = torch.empty(130, 256, dtype=torch.float32, device="cuda")
        fp4.fp4_dequantize(q.codes, q.scales, q.g, 130, 256, fmt, out)
        oq = oracle_quantize(x, fmt, blk)
        ref = oracle.dequantize(oq["codes"], oq["scales"], oq["g"], fmt)
        # the device multiplies in FP32: equal to the FP64 value rounded once or twice
        assert np.allclose(out.cpu().numpy(), ref, rtol=2.5e-7, atol=0)


@pytest.mark.parametrize("name", ["decode_w", "prefill_x", "moe_a"])
def test_full_size_quantize_sampled_rows(name):
    """Full-size tensors in the bench's launch configuration; the oracle recomputes
    sampled rows (with the tensor's global scale, which it computes over all rows)."""
    if name == "decode_w":
        x = workloads.normal((28672, 8192), 0.02, 1)
        fmt, blk = fp4.NVFP4, 16
    elif name == "prefill_x":
        x = workloads.prefill_inputs(m=8192, n=16, k=8192)[0]
        fmt, blk = fp4.NVFP4, 16
    else:
        x = workloads.moe_inputs(n=128)[0]
        fmt, blk = fp4.MXFP4, 32
    gq = gpu_quantize(x.cuda(), fmt, blk)
    rows, cols = x.shape
    hx = __import__("fp4_testutil").host_input(x)
    g = None
    if fmt == fp4.NVFP4:
        g = oracle.global_scale(oracle.amax(hx))
        assert np.float32(gq.g.item()) == g
    rng = np.random.default_rng(0)
    sample = np.unique(np.concatenate([[0, rows - 1], rng.integers(0, rows, 64)]))
    oq = oracle.quantize(hx[sample], fmt, blk, g_in=g)
    assert np.array_equal(gq.codes.cpu().numpy()[sample], oq["codes"])
    sc_rm = oracle.unswizzle_scales(gq.scales.cpu().numpy(), rows, cols // blk)
    assert np.array_equal(sc_rm[sample], oq["scales"])
