"""fp4_gemm_noalloc: the GEMM entry point for callers that cannot allocate device memory,
such as a host that owns all device memory and gives this library no allocator.  Its
split-K scratch is a fixed array inside the library.

The tests call it twice in a row through the C ABI:
- a decode-shaped problem, which needs that scratch;
- a tile-mode problem, which needs none.
Each result is checked against the oracle's FP64 product at the GEMM tolerance the other
tests use, and against fp4_gemm with a caller workspace at the same tolerance.  The file
is named so that pytest collects it last."""
import numpy as np
import pytest
import torch

import block_scaled_fp4_04_b200 as fp4
import oracle
from fp4_testutil import dequant_oracle, oracle_quantize, random_input

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("m,n,k", [(16, 3072, 4096),    # split over K: uses the built-in scratch
                                   (512, 512, 512)])    # whole tiles: no scratch at all
def test_noalloc_gemm_matches_oracle_and_workspace_gemm_twice(m, n, k):
    need = fp4.fp4_gemm_workspace_size(m, n, k, fp4.NVFP4)
    assert (need > 0) == (m == 16)
    xa = random_input(m, k, 91, torch.bfloat16)
    xb = random_input(n, k, 92, torch.float32, std=0.02, outliers=False)
    qa = fp4.quantize(xa.cuda(), fp4.NVFP4, 16)
    qb = fp4.quantize(xb.cuda(), fp4.NVFP4, 16)
    ref = fp4.gemm(qa, qb, torch.float32).cpu().numpy().astype(np.float64)
    oa, ob = oracle_quantize(xa, fp4.NVFP4, 16), oracle_quantize(xb, fp4.NVFP4, 16)
    d_ref, s = oracle.gemm_reference(dequant_oracle(oa, fp4.NVFP4), dequant_oracle(ob, fp4.NVFP4))
    tol = oracle.gemm_tolerance(d_ref, s, bf16_out=False)
    assert np.all(np.abs(ref - d_ref) <= tol)
    for call in range(2):
        d = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
        fp4.fp4_gemm_noalloc(fp4.NVFP4, qa.codes, qa.scales, qa.g, qb.codes, qb.scales, qb.g, m, n, k, d, fp4.F32)
        torch.cuda.synchronize()
        assert fp4.fp4_get_status() == fp4.OK
        got = d.cpu().numpy().astype(np.float64)
        err = np.abs(got - d_ref)
        assert np.all(err <= tol), f"call {call}: max err / tol {np.max(err / tol)}"
        assert np.all(np.abs(got - ref) <= tol), f"call {call}: differs from fp4_gemm"


def test_noalloc_gemm_rejects_shapes_beyond_its_scratch():
    # 64 x 32768 FP32 partials need 8 MiB > the 4 MiB array
    with pytest.raises(fp4.Fp4Error) as ei:
        fp4.fp4_gemm_noalloc(fp4.NVFP4, 16, 16, None, 16, 16, None, 64, 32768, 4096, 16, fp4.F32)
    assert ei.value.status == fp4.ERR_INVALID_ARG and "4 MiB" in str(ei.value)
