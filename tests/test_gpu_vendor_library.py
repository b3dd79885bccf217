"""Cross-check against the vendor library's MXFP4 GEMM (cuBLASLt, through
torch.nn.functional.scaled_mm): the same E2M1 codes and E8M0 scale bytes, in the
tensor-core scale layout this library writes (the library's 32_4_4 swizzle), go into
both GEMMs. The vendor GEMM is an independent implementation of the same product, so
agreement checks the operand and scale layouts from outside this repository; the
parity proper is against the oracle (tests/test_gpu_gemm.py). The bf16 outputs are
compared: both sides accumulate in fp32, so they must agree within 1 bf16 ulp plus the
GEMM tolerance (2e-5 * S, twice the per-side bound); on random codes and scales they
were bit-identical. (The vendor path's float32 output is not compared: with this torch
its float32 result held bf16-width data -- half of its values bf16-exact, none equal to
its own bf16 result -- while the oracle and this library agree in fp32.) Skipped where
the installed torch offers no MXFP4 scaled_mm.
"""
import numpy as np
import pytest

import oracle
from gpu_helpers import bf16_ulp, to_dev
from test_gpu_gemm import _operand

pytestmark = pytest.mark.gpu


def _vendor_gemm(aq, asf, bq, bsf, M, N, K, out_dtype):
    import torch
    import torch.nn.functional as F
    try:
        from torch.nn.functional import ScalingType, SwizzleType
    except ImportError:
        pytest.skip("torch has no scaled_mm scaling enums")

    def ru(a, b):
        return -(-a // b) * b
    sa = asf[:ru(M, 128) * ru(K // 32, 4)].view(torch.float8_e8m0fnu).view(ru(M, 128), ru(K // 32, 4))
    sb = bsf[:ru(N, 128) * ru(K // 32, 4)].view(torch.float8_e8m0fnu).view(ru(N, 128), ru(K // 32, 4))
    try:
        return F.scaled_mm(aq.view(torch.float4_e2m1fn_x2), bq.view(torch.float4_e2m1fn_x2).t(),
                           sa, ScalingType.BlockWise1x32, sb, ScalingType.BlockWise1x32,
                           SwizzleType.SWIZZLE_32_4_4, SwizzleType.SWIZZLE_32_4_4,
                           output_dtype=out_dtype)
    except (RuntimeError, TypeError, NotImplementedError) as e:
        pytest.skip(f"vendor MXFP4 GEMM unavailable: {str(e).splitlines()[0][:120]}")


# A pair-kernel shape with a last round in column halves, a whole-round one, and a
# few-row one (the vendor GEMM takes any M here).
@pytest.mark.parametrize("M,N,K", [(768, 1024, 8192), (3584, 3072, 3072), (16, 4096, 14336)])
def test_matches_vendor_mxfp4_gemm(M, N, K):
    import torch
    import mxfp4_quantized_linear_block_b200 as mx
    aq, as_ = _operand(M + N + 7, M, K, 40)
    bq, bs = _operand(M + N + 7, N, K, 41)
    dev = [to_dev(aq), to_dev(oracle.sf_to_physical(as_, K)), to_dev(bq),
           to_dev(oracle.sf_to_physical(bs, K))]
    # the exact S = sum |a_i b_i| per element from the oracle, for the tolerance
    mi = np.arange(0, M, max(1, M // 64)).repeat(16)
    ni = np.tile(np.arange(0, N, max(1, N // 16)), mi.size // 16)
    _, S = oracle.gemm_pairs(aq, as_, bq, bs, mi, ni)
    ours_t = mx.gemm(*dev, M, N, K, out_dtype=torch.bfloat16)
    lib_t = _vendor_gemm(*dev, M, N, K, torch.bfloat16)
    ours = ours_t.float().cpu().numpy().astype(np.float64)
    lib = lib_t.float().cpu().numpy().astype(np.float64)
    d = np.abs(ours[mi, ni] - lib[mi, ni])
    bad = d > 2e-5 * S + bf16_ulp(ours[mi, ni])
    assert not bad.any(), (f"{M}x{N}x{K}: {bad.sum()} of {bad.size} sampled bf16 outputs "
                           f"differ from the vendor GEMM beyond tolerance")
    # over every output, the share that is bit-identical (reported, not required)
    same = float((ours_t == lib_t).float().mean())
    print(f"{M}x{N}x{K}: {same:.6f} of the bf16 outputs bit-identical to the vendor GEMM")
