"""kda_prefill_noalloc: the prefill for callers that cannot allocate device memory.

Such callers (a runtime that owns all device memory through its own pool, a
plugin whose host framework hides its allocator, a serving loop that cannot
take a device-synchronising cudaMalloc) get an entry point whose workspace is
a fixed array inside the library. These GPU tests call it through the C ABI
and compare it with kda_prefill (which takes a caller workspace) on two calls
in a row after a call on other inputs, since every call reuses the same array
and must not depend on what an earlier call left there: the results must equal
kda_prefill's bit for bit. This file is collected last on purpose.
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


@pytest.mark.parametrize("lengths,other,H,d,dtype", [
    ([1500, 64, 130, 1], [700, 333], 8, 128, torch.bfloat16),  # tensor-core path, smaller ring
    ([300, 5, 129], [77, 200], 4, 64, torch.float32),          # fp32 CUDA-core path
])
def test_noalloc_matches_workspace_entry_point(lengths, other, H, d, dtype):
    q, k, v, la, beta, S0, cu, L = _inputs(lengths, H, d, dtype, seed=21)
    o_ref, S_ref = kda.kda_prefill(q, k, v, la, beta, S0, cu, max_seqlen=L)
    torch.cuda.synchronize()
    assert kda.kda_device_error(reset=True) == 0
    # A first call on other inputs leaves unrelated ring contents and flags in the
    # array; the two calls after it must not see them (results do not depend on the
    # ring size or on earlier calls, so they equal kda_prefill's bit for bit).
    oq, ok_, ov, ola, obeta, oS0, ocu, oL = _inputs(other, H, d, dtype, seed=77)
    kda.kda_prefill_noalloc(oq, ok_, ov, ola, obeta, oS0, ocu, max_seqlen=oL,
                            o=torch.empty_like(ov), S_T=torch.empty_like(oS0))
    torch.cuda.synchronize()
    assert kda.kda_device_error(reset=True) == 0
    for call in range(2):
        o = torch.full_like(o_ref, float("nan"))
        S_T = torch.full_like(S_ref, float("nan"))
        kda.kda_prefill_noalloc(q, k, v, la, beta, S0, cu, max_seqlen=L, o=o, S_T=S_T)
        torch.cuda.synchronize()
        assert kda.kda_device_error(reset=True) == 0, call
        assert torch.equal(o, o_ref), (call, float((o.float() - o_ref.float()).abs().max()))
        assert torch.equal(S_T, S_ref), (call, float((S_T - S_ref).abs().max()))


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
