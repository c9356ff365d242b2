"""Failure detection of the tensor-core prefill: a bounded wait between CTAs that
runs out is reported, the kernel returns, and the device stays usable.

Nothing is planted or broken. The waits between the prefill's CTAs (a scan CTA
waiting for its next prepared chunk, a preparing CTA waiting for a free ring
slot) get a 1 microsecond bound through ``kda_set_wait_limit_ns``. Preparing a
chunk takes several microseconds, so the scan's first wait runs out on its own.
The test then checks that the call ended, that ``kda_device_error`` reports
the timeout (code 1, KDA_ERR_TIMEOUT), and that the next call, at the default
bound, matches the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_125_b200 as kda
import kda_inputs as KI
import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    kda.load_library()


def _inputs(lengths, H, seed):
    T = sum(lengths)
    q, k, v, la, beta = KI.token_inputs(T, H, 128, 128, torch.bfloat16, DEV, seed)
    S0 = KI.initial_state(len(lengths), H, 128, 128, 0.1, DEV, seed)
    return q, k, v, la, beta, S0, KI.cu_from_lengths(lengths, DEV)


def test_bounded_wait_runs_out_then_next_call_passes():
    lengths, H = [2048, 700], 4
    q, k, v, la, beta, S0, cu = _inputs(lengths, H, seed=61)
    assert kda.kda_device_error(reset=True) == 0
    prev = kda.kda_set_wait_limit_ns(1000)
    try:
        kda.kda_prefill(q, k, v, la, beta, S0, cu, max_seqlen=max(lengths))
    finally:
        assert kda.kda_set_wait_limit_ns(prev) == 1000
    torch.cuda.synchronize()  # the kernel returned
    assert kda.kda_device_error(reset=False) == 1
    # the status call maps the code to KDA_ERR_TIMEOUT, and reset clears it
    import ctypes
    code = ctypes.c_int32(0)
    assert kda.load_library().kda_device_error(ctypes.byref(code), 1) == kda.KDA_ERR_TIMEOUT
    assert code.value == 1
    assert kda.kda_device_error(reset=True) == 0

    o, S_T = kda.kda_prefill(q, k, v, la, beta, S0, cu, max_seqlen=max(lengths))
    torch.cuda.synchronize()
    assert kda.kda_device_error(reset=True) == 0
    h = lambda x: x.detach().to("cpu", torch.float64).numpy()
    o_ref, S_ref = oracle.recurrent(h(q), h(k), h(v), h(la), h(beta), h(S0), cu.cpu().numpy())
    assert float(np.abs(h(o) - o_ref).max()) <= 2e-2
    assert float(np.linalg.norm(h(S_T) - S_ref) / np.linalg.norm(S_ref)) <= 1e-2


def test_wait_limit_zero_restores_default():
    prev = kda.kda_set_wait_limit_ns(0)
    assert kda.kda_set_wait_limit_ns(prev) == 2_000_000_000
