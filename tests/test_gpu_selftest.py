"""The arithmetic shortcuts the kernels use are exact on their whole domain:
every (bf16 numerator, bf16 scale) pair of the division-by-scale domain and every
bf16 amax over the three format maxima, compared with IEEE division on the device."""
import pytest

import kv_cache_quantize_b200 as kvq

pytestmark = pytest.mark.gpu


def test_division_by_scale_used_by_the_kernels_is_exact():
    # the kernels use the two-step form (KVQ_SCALE_DIV = div_scale2)
    assert kvq.selftest(1) == 0


@pytest.mark.parametrize("which", [0, 2, 3, 4])
def test_report_other_shortcuts(which, record_property):
    n = kvq.selftest(which)
    record_property(f"selftest_{which}", n)
    print(f"selftest {which}: {n} mismatches")
