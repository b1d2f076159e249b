"""The expansion-rate measurement (qlora_expand_rate): the rate of the library's
NF4 table expansion alone on every SM, the ceiling of the few-token forward."""
import pytest

import bit_nf4_quantized_03_b200 as q
from tests.gpu_util import ensure_built

pytestmark = pytest.mark.gpu


def test_expansion_rate_is_measured_and_plausible():
    ensure_built()
    # positive, and below what the integer pipe could do at the two byte permutes per
    # weight that each lookup needs at least (64 lanes / 2)
    per_clk, per_s = q.qlora_expand_rate(256)
    assert 1.0 < per_clk < 32.0, per_clk
    assert per_s > 1e11, per_s
    q.qlora_check_device_error()


def test_expansion_rate_rejects_bad_arguments():
    ensure_built()
    with pytest.raises(q.QloraError):
        q.qlora_expand_rate(0)
