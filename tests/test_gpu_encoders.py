"""Device encoders vs the oracle, over every float32 bit pattern where that is cheap
(E2M1: all 2^32 patterns against the oracle) and against the oracle-pinned library
conversions elsewhere (E4M3: every non-negative pattern up to 464 vs torch's
float8_e4m3fn; E8M0: every non-negative pattern vs torch's float8_e8m0fnu), plus
direct oracle samples for both scale encoders."""
import numpy as np
import pytest
import torch

import block_scaled_fp4_04_b200 as fp4
import oracle

pytestmark = pytest.mark.gpu

CHUNK = 1 << 28


def _encode_range(start: int, n: int, which: int) -> torch.Tensor:
    bits = torch.arange(start, start + n, dtype=torch.int64, device="cuda")
    bits = torch.where(bits >= 2 ** 31, bits - 2 ** 32, bits).to(torch.int32)
    v = bits.view(torch.float32)
    out = torch.empty(n, dtype=torch.uint8, device="cuda")
    fp4.fp4_debug_encode(v, n, which, out)
    return v, out


def test_e2m1_production_encoder_exhaustive():
    total_bad = 0
    for start in range(0, 1 << 32, CHUNK):
        _, out = _encode_range(start, CHUNK, 0)
        total_bad += oracle.e2m1_count_mismatch(start, out.cpu().numpy())
    assert total_bad == 0


@pytest.mark.parametrize("which", [3, 4])
def test_e2m1_variants_sampled(which):
    rng = np.random.default_rng(which)
    bits = np.concatenate([rng.integers(0, 1 << 32, 1 << 22, dtype=np.uint64),
                           np.arange(0x3E000000, 0x3E000000 + (1 << 22), dtype=np.uint64),
                           np.arange(0xBE800000, 0xBE800000 + (1 << 22), dtype=np.uint64)]).astype(np.uint32)
    v = bits.view(np.float32)
    keep = ~np.isnan(v)
    v = v[keep]
    vt = torch.from_numpy(v.copy()).cuda()
    out = torch.empty(v.size, dtype=torch.uint8, device="cuda")
    fp4.fp4_debug_encode(vt, v.size, which, out)
    assert np.array_equal(out.cpu().numpy(), oracle.e2m1_encode(v))


def _torch_fp8(v: torch.Tensor, dtype) -> torch.Tensor:
    try:
        return v.to(dtype).view(torch.uint8)
    except Exception:  # conversion not available on the device: do it on the CPU
        return v.cpu().to(dtype).view(torch.uint8).cuda()


def test_e4m3_encoder_vs_torch_every_pattern_up_to_464():
    top = int(np.float32(464.0).view(np.uint32))
    for start in range(0, top + 1, CHUNK):
        n = min(CHUNK, top + 1 - start)
        v, out = _encode_range(start, n, 1)
        ref = _torch_fp8(v, torch.float8_e4m3fn)
        assert torch.equal(out, ref), f"chunk at {start:#x}"


def test_e4m3_encoder_saturates_above_464():
    lo = int(np.float32(464.0).view(np.uint32)) + 1
    for start in range(lo, 0x7F800001, CHUNK):        # up to and including +inf
        _, out = _encode_range(start, min(CHUNK, 0x7F800001 - start), 1)
        assert bool((out == 0x7E).all())


def test_e4m3_encoder_vs_oracle_sample():
    rng = np.random.default_rng(5)
    v = np.concatenate([np.exp2(rng.uniform(-16, 10, 1 << 18)), rng.uniform(0, 500, 1 << 18)]).astype(np.float32)
    vt = torch.from_numpy(v).cuda()
    out = torch.empty(v.size, dtype=torch.uint8, device="cuda")
    fp4.fp4_debug_encode(vt, v.size, 1, out)
    assert np.array_equal(out.cpu().numpy(), oracle.e4m3_encode(v))


def test_e8m0_encoder_vs_torch_every_normal_pattern():
    """Normal floats vs torch (pinned to the oracle on normals); torch rounds values of
    1.5 * 2^127 and up to NaN, which the encoder clamps to 2^127."""
    for start in range(0x00800000, 0x7F800001, CHUNK):
        n = min(CHUNK, 0x7F800000 - start)
        v, out = _encode_range(start, n, 2)
        ref = _torch_fp8(v, torch.float8_e8m0fnu)
        ref = torch.where(ref == 255, torch.full_like(ref, 254), ref)
        assert torch.equal(out, ref), f"chunk at {start:#x}"


def test_e8m0_encoder_vs_oracle_every_subnormal_pattern():
    """Zero and the subnormals (torch rounds these differently; the oracle decides)."""
    v, out = _encode_range(0, 0x00800000, 2)
    assert np.array_equal(out.cpu().numpy(), oracle.e8m0_encode(v.cpu().numpy()))


def test_e8m0_encoder_vs_oracle_sample():
    rng = np.random.default_rng(6)
    e = rng.integers(-149, 128, 1 << 16)
    v = np.ldexp(rng.uniform(1, 2, 1 << 16), e).astype(np.float32)
    v = np.concatenate([v, np.ldexp(1.5, np.arange(-140, 127)).astype(np.float32), np.array([0, np.inf], np.float32)])
    vt = torch.from_numpy(v).cuda()
    out = torch.empty(v.size, dtype=torch.uint8, device="cuda")
    fp4.fp4_debug_encode(vt, v.size, 2, out)
    assert np.array_equal(out.cpu().numpy(), oracle.e8m0_encode(v))
