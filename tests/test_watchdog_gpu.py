"""Failure detection without a GPU fault: a load that never arrives makes a bounded
in-kernel wait run out; the kernel drains what it issued and returns, the host reads
PBA_ERR_TIMEOUT from the device watchdog word, and the context stays usable."""
import numpy as np
import pytest

import oracle
import pba_inputs as pi
from pba_testlib import assert_lse_close, assert_out_close, bf16_to_f64_tensor, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pba():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import pair_biased_attention_gated_b200 as p
    return p


def test_watchdog_reports_a_wait_that_ran_out(pba):
    import time
    cfg = pi.custom("wd", B=1, H=1, N=128, c=32, masked=((120, 128),))
    d = pi.make_inputs(cfg, seed=1, with_dout=False)
    t = to_dev(d)
    pba.pba_device_status()                      # nothing pending before the test
    pba.lib.pba_debug_skip_load(0)               # the only step's Q/K load never arrives
    try:
        t0 = time.time()
        pba.attention_fwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"])
        with pytest.raises(pba.PbaError) as ei:
            pba.pba_device_status()
        assert ei.value.status == 4, ei.value
        assert "site" in str(ei.value)
        assert time.time() - t0 < 30
    finally:
        pba.lib.pba_debug_skip_load(-1)
    pba.pba_device_status()                      # the word was cleared by the read
    # the context is intact: the same call now gives the oracle's answer
    out, lse = pba.attention_fwd(t["q"], t["k"], t["v"], t["bias"], t["keep"], t["g"])
    pba.pba_device_status()
    f = {k: (pi.bf16_bits_to_f64(v) if k != "keep" else v) for k, v in d.items()}
    ro, rl = oracle.fwd(f["q"], f["k"], f["v"], f["bias"], f["keep"], f["g"])
    assert_out_close(bf16_to_f64_tensor(out), ro)
    assert_lse_close(lse.cpu().numpy().astype(np.float64), rl)
