"""Failure detection on the GPU without a fault: a kernel waits, with the
same bounded wait the attention kernels use, on a barrier that nothing
arrives on. The wait runs out after a short limit, the kernel records a
timeout in the device status word and returns; the host reads it through
cswattn_sync_status(), and the context stays usable afterwards."""
import numpy as np
import pytest

import causal_sliding_window_rope_b200 as cs
from _helpers import make_inputs, oracle_layer, rel_frob, run_gpu

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_is_reported():
    cs.cswattn_sync_status()  # start from a clear status word
    cs.cswattn_selftest_wait_timeout(2_000_000)  # 2 ms limit
    with pytest.raises(cs.CswattnError) as err:
        cs.cswattn_sync_status()
    assert err.value.status == cs.ERR_TIMEOUT
    cs.cswattn_sync_status()  # reading cleared it

    # The context is still usable: a layer still matches the oracle.
    spec = cs.LayerSpec(1, 200, 4, 2, 128, 64, has_ve=True)
    inp = make_inputs(1, 200, 4, 2, 128, True, "bf16", config=97)
    got, _ = run_gpu(spec, inp)
    _, ref = oracle_layer(spec, inp)
    for key in ("O", "dq", "dk", "dv"):
        assert rel_frob(got[key], ref[key]) <= 2e-2, key
        assert np.isfinite(got[key]).all()
