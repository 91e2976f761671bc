"""Failure detection on the GPU without a fault: a device-side wait that
nothing completes runs out after the library's limit, the kernel returns, the
status word reports XKV_ERR_DEVICE_TIMEOUT (cleared on read), and the context
keeps working (an SR decode afterwards matches the oracle)."""
import time

import numpy as np
import pytest

import oracle
import synth
from gpu_helpers import host, run_sr, sr_inputs_on_device

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_the_context_stays_usable(xkv):
    assert xkv.get_device_status() == xkv.XKV_OK
    t0 = time.monotonic()
    xkv.xkv_selftest_expired_wait()
    status = xkv.get_device_status()
    elapsed = time.monotonic() - t0
    assert status == xkv.XKV_ERR_DEVICE_TIMEOUT
    assert 0.9 < elapsed < 60.0
    assert xkv.get_device_status() == xkv.XKV_OK  # read once, then cleared
    w = synth.WORKLOADS["tiny_f32"]
    inp = synth.compressed_cache(w, 0)
    out, sel = run_sr(xkv, w, sr_inputs_on_device(w, inp))
    assert xkv.get_device_status() == xkv.XKV_OK
    ref, _, _ = oracle.sr_decode(w, sel_in=sel.cpu().numpy(), **inp)
    assert np.abs(host(out) - ref).max() <= 2e-4
