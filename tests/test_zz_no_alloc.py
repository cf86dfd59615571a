"""psispec_verify_linear_static: psispec_verify_linear with the library-owned scratch array.

The GPU test runs the workspace call once and the static call twice in a row on the same
inputs and requires identical outputs; it passes alone in a fresh process and after the rest
of the suite (the file sorts last). The host check needs no device.
"""
import ctypes

import pytest
import torch

from lossless_speculative_sampling_b200 import build as libbuild
from lossless_speculative_sampling_b200 import psispec, synth

FAKE = ctypes.c_void_p(4096)  # aligned, never dereferenced


def test_static_rejects_oversize_before_any_cuda_call():
    libbuild.build()
    L = psispec.lib()
    # B = 512, K = 16, V = 151936 needs more scratch than the array holds
    assert psispec.workspace_size(psispec.OP_VERIFY_LINEAR, 512, 16, 151936) > psispec.STATIC_WORKSPACE_BYTES
    st = L.psispec_verify_linear_static(FAKE, FAKE, psispec.BF16, 512, 16, 151936, FAKE, None, FAKE, FAKE, FAKE,
                                        FAKE, FAKE, FAKE, None, None, None)
    assert st == psispec.ERR_UNSUPPORTED
    assert L.psispec_verify_linear_static(FAKE, FAKE, psispec.BF16, 0, 16, 151936, FAKE, None, FAKE, FAKE, FAKE,
                                          FAKE, FAKE, FAKE, None, None, None) == psispec.ERR_INVALID_ARG
    # the mid-size workload fits
    assert psispec.workspace_size(psispec.OP_VERIFY_LINEAR, 64, 8, 151936) <= psispec.STATIC_WORKSPACE_BYTES
    # sizes beyond the limits of psispec_verify_linear are unsupported, as they are there
    for B, K, V in ((1, 65, 1000), (1, 4, (1 << 24) + 1)):
        st = L.psispec_verify_linear_static(FAKE, FAKE, psispec.BF16, B, K, V, FAKE, None, FAKE, FAKE, FAKE, FAKE,
                                            FAKE, FAKE, None, None, None)
        assert st == psispec.ERR_UNSUPPORTED, (B, K, V, st)


@pytest.mark.gpu
@pytest.mark.parametrize("use_stats", [True, False])
def test_static_matches_workspace_call_twice(use_stats):
    assert torch.cuda.is_available()
    dev = torch.device("cuda", 0)
    case = synth.LinearCase("static", 16, 8, synth.V_QWEN, torch.bfloat16, 3.0, 1.0, 1.0, 1.0, zipf_bias=8.0,
                            seed=4242)
    B, K, V = case.B, case.K, case.V
    tgt, drf = synth.linear_logits(case, device=dev)
    ud, ua, ur = (t.to(dev) for t in synth.linear_uniforms(case))
    Ts = torch.full((B,), 1.0, device=dev)
    # a mix of requests with and without a top-p cut, and one greedy request
    Ps = torch.tensor([1.0, 0.9, 0.95, 1.0, 0.8, 1.0, 0.99, 1.0] * 2, device=dev)
    Ts[5] = 0.0
    tok, _, stats = psispec.sample_draft(drf, Ts, Ps, ud)
    ds = stats if use_stats else None
    ref = psispec.verify_linear(tgt, drf, tok, ua, ur, Ts, Ps, draft_row_stats=ds)
    outs = []
    for _ in range(2):
        o = {"out_tokens": torch.full((B, K + 1), -7, dtype=torch.int32, device=dev),
             "out_accept_len": torch.full((B,), -7, dtype=torch.int32, device=dev),
             "out_p": torch.full((B, K), -7.0, device=dev), "out_q": torch.full((B, K), -7.0, device=dev)}
        outs.append(o)
    # a first call may load the module and look up the array's address; after it, the device's
    # free memory must not move: the library allocates nothing (torch's allocator would not see
    # a cudaMalloc made by the library, the driver's count does)
    psispec.verify_linear_static(tgt, drf, tok, ua, ur, Ts, Ps, draft_row_stats=ds, **outs[0])
    for t in outs[0].values():
        t.fill_(-7)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info(dev)[0]
    for o in outs:  # two calls in a row, nothing allocated between them
        psispec.verify_linear_static(tgt, drf, tok, ua, ur, Ts, Ps, draft_row_stats=ds, **o)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info(dev)[0] == free0
    for o in outs:
        assert torch.equal(o["out_tokens"], ref["tokens"])
        assert torch.equal(o["out_accept_len"], ref["accept_len"])
        assert torch.equal(o["out_p"], ref["p"])
        assert torch.equal(o["out_q"], ref["q"])
    assert int((ref["accept_len"] >= 0).sum()) == B
