"""The device error path of the bounded waits, exercised without a fault: a
kernel waits on an mbarrier that nothing arrives on, the wait gives up after a
short limit, the library reports QLORA_DEVERR_TIMEOUT, and the context stays
usable (a quantisation right after is bit-exact with the oracle)."""
import time

import numpy as np
import pytest
import torch

from bit_nf4_quantised_codebook_b200 import inputs
from oracle import nf4
from tests.gpu_util import api, bits, check_dev_err, to_dev

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports():
    a = api()
    err = a.new_error_word()
    gave_up = torch.zeros(1, dtype=torch.int32, device="cuda")
    t = time.perf_counter()
    a.qlora_selftest_bounded_wait(20_000, err, gave_up)  # 20 ms
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t
    assert int(gave_up.item()) == 1
    assert int(err[0].item()) & a.QLORA_DEVERR_TIMEOUT
    assert elapsed < 5.0
    # the context is still usable
    w = inputs.weight_bf16(64, 512, 0.02, 7)
    err2 = a.new_error_word()
    q = a.qlora_quantize(to_dev(w), dev_err=err2)
    check_dev_err(err2)
    assert np.array_equal(bits(a.qlora_dequantize(q)), nf4.dequantize_nf4(nf4.quantize_nf4(w)))


def test_selftest_rejects_bad_arguments():
    a = api()
    err = a.new_error_word()
    with pytest.raises(a.QloraError):
        a.qlora_selftest_bounded_wait(0, err)
