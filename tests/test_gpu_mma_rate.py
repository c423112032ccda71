"""fp4_mma_rate: the tensor-core rate microbenchmark behind the GEMM's
roofline context.  Every variant runs to completion with a clean device
status and reports a finite positive rate; the scale-factor copies cost
tensor-pipe time whichever way they are issued; bad arguments are rejected."""
import math

import pytest

pytestmark = pytest.mark.gpu


def test_every_variant_runs(gpu_lib):
    F = gpu_lib
    rates = {v: F.mma_rate(v, 2000) for v in range(8)}
    for v, r in rates.items():
        assert math.isfinite(r) and r > 0, (v, r)
    # copies into tensor memory share the MMAs' pipe: batched (6, 7) or
    # interleaved (1, 3), they lower the MMA-only rate (0, 2)
    assert rates[6] < rates[0] and rates[1] < rates[0]
    assert rates[7] < rates[2] and rates[3] < rates[2]
    print({v: round(r) for v, r in rates.items()})


@pytest.mark.parametrize("variant,iters", [(-1, 10), (8, 10), (0, 0)])
def test_rejects_bad_arguments(gpu_lib, variant, iters):
    F = gpu_lib
    with pytest.raises(F.Fp4Error) as e:
        F.mma_rate(variant, iters)
    assert e.value.code == 2        # FP4_ERR_SHAPE
