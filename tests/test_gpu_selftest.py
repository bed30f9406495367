"""The arithmetic shortcuts the kernels use, checked on the device over their
whole input domain against IEEE division:
  * division of a code's numerator by the group scale (one-step Markstein form):
    its E4M3 and E2M1 codes equal those of the IEEE quotient for every bf16
    numerator and every bf16 scale in [2^-100, 2^101) with |a| <= 512 s (the
    quotient itself may differ in its last bits for a small share of pairs,
    which is reported, not required);
  * amax / 448, amax / 57344, amax / 6 with constant reciprocals: bit-identical
    for every positive finite bf16 and f16 amax;
  * the dequant kernel's static int8 quantisation through a per-channel
    reciprocal (two-step Markstein form, IEEE division outside its guard):
    the same int8 codes as IEEE division on 2^28 random and near-tie
    (value, scale, offset) triples;
  * the indexer fp8 mode's division by the row scale (two-step Markstein form
    where the row maximum is a finite value >= 2^-60): the same E4M3 and E5M2
    codes as IEEE division on 2^28 random bf16 / f16 (value, maximum) pairs;
  * the rmsnorm kernels' unscaled x / rms (one-step Markstein form inside
    their guard): bit-identical to IEEE division on 2^28 random and near-tie
    pairs, and for every bf16 and f16 numerator mantissa against every
    binary32 divisor mantissa.
Also the failure path of the pipelined kernels' bounded waits: a wait on a
barrier that nothing completes gives up after its limit and reports
FAULT_TIMEOUT through the fault word (no GPU fault, hang or trap)."""
import pytest

import kv_cache_quantize_b200 as kvq

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("which,what", [(2, "E4M3 codes of the one-step quotient"),
                                        (3, "E2M1 codes of the one-step quotient"),
                                        (4, "constant-divisor scale quotients"),
                                        (6, "int8 codes of the reciprocal-based quotient"),
                                        (8, "fp8 row-scale codes of the two-step quotient"),
                                        (9, "unscaled one-step quotient x / rms"),
                                        (10, "one-step quotient, every 16-bit numerator mantissa")])
def test_shortcut_is_exact(which, what):
    assert kvq.selftest(which) == 0, what


def test_report_quotient_bit_differences():
    one, two, normal = kvq.selftest(0), kvq.selftest(1), kvq.selftest(5)
    print(f"quotient bit differences from IEEE: one-step {one} (normal range {normal}), two-step {two}")


def test_bounded_wait_reports_timeout():
    kvq.get_error()                         # clear
    assert kvq.selftest(7) == 1             # the wait gave up, as designed
    assert kvq.get_error() == 0x2           # FAULT_TIMEOUT, then cleared
    assert kvq.get_error() == 0
