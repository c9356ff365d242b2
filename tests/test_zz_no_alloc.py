"""kda_prefill_noalloc: the prefill for callers that cannot allocate device memory.

Such callers (a runtime that owns all device memory through its own pool, a
plugin whose host framework hides its allocator, a serving loop that cannot
take a device-synchronising cudaMalloc) get an entry point whose workspace is
a fixed array inside the library. These GPU tests call it through the C ABI
and compare it with kda_prefill (which takes a caller workspace) on two calls
in a row, since every call reuses the same array and must not depend on what
the previous call left there. This file is collected last on purpose.
"""
import pytest
import torch

import gated_delta_rule_125_b200 as kda
import kda_inputs as KI

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    kda.load_library()


def _inputs(lengths, H, d, dtype, seed):
    T = sum(lengths)
    q, k, v, la, beta = KI.token_inputs(T, H, d, d, dtype, DEV, seed)
    S0 = KI.initial_state(len(lengths), H, d, d, 0.1, DEV, seed)
    return q, k, v, la, beta, S0, KI.cu_from_lengths(lengths, DEV), max(lengths)


@pytest.mark.parametrize("lengths,H,d,dtype,atol,stol", [
    ([1500, 64, 130, 1], 8, 128, torch.bfloat16, 2e-2, 1e-2),  # tensor-core path, smaller ring
    ([300, 5, 129], 4, 64, torch.float32, 1e-4, 1e-4),         # fp32 CUDA-core path
])
def test_noalloc_matches_workspace_entry_point(lengths, H, d, dtype, atol, stol):
    q, k, v, la, beta, S0, cu, L = _inputs(lengths, H, d, dtype, seed=21)
    o_ref, S_ref = kda.kda_prefill(q, k, v, la, beta, S0, cu, max_seqlen=L)
    for call in range(2):  # the second call starts from the first call's leftovers
        o = torch.full_like(o_ref, float("nan"))
        S_T = torch.full_like(S_ref, float("nan"))
        kda.kda_prefill_noalloc(q, k, v, la, beta, S0, cu, max_seqlen=L, o=o, S_T=S_T)
        torch.cuda.synchronize()
        err = float((o.float() - o_ref.float()).abs().max())
        rel = float((S_T - S_ref).norm() / S_ref.norm())
        assert err <= atol, (call, err)
        assert rel <= stol, (call, rel)


def test_noalloc_refuses_problems_beyond_its_scratch():
    # fp32 (CUDA-core path) with 512 heads needs more than the fixed array even at
    # one chunk per wave; the call is refused before anything is enqueued (tensors
    # are real and sized right).
    q, k, v, la, beta, S0, cu, L = _inputs([128], 512, 128, torch.float32, seed=22)
    o = torch.empty_like(v)
    S_T = torch.empty_like(S0)
    assert kda.kda_prefill_workspace_min(1, 128, 128, 512, 128, 128, torch.float32) > (32 << 20)
    with pytest.raises(kda.KDAError) as ei:
        kda.kda_prefill_noalloc(q, k, v, la, beta, S0, cu, max_seqlen=L, o=o, S_T=S_T)
    assert ei.value.status == kda.KDA_ERR_WORKSPACE
