"""ck_w4a4_linear_noalloc: the linear for callers that cannot allocate device memory (a
plugin inside a framework that owns all device memory, or a loop that must not call
cudaMalloc).  It uses the library's built-in 32 MiB scratch array instead of a workspace
and must give the same output as ck_w4a4_linear, call after call.

This file is collected last on purpose, so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process, where its first
call sets up the scratch array's address on the device.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

from rotated_w4a4_quantized_group_b200 import ck
from rotated_w4a4_quantized_group_b200 import workloads as W


def _inputs(case, dev):
    inp = W.make_linear_inputs(case)
    return {k: (None if v is None else v.to(dev)) for k, v in inp.items()}


@pytest.mark.gpu
def test_noalloc_matches_the_workspace_entry_point_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda", 0)
    # the headline shape (8192 x 3840 bf16: 31.5 MB of scratch) and a second, different input
    cases = [W.LINEAR_CASES[W.HEADLINE],
             W.LINEAR_CASES[W.HEADLINE].replace(M=1000, K=1280, N=700, seed=77, rotation="hadamard")]
    for case in cases:
        inp = _inputs(case, dev)
        ref = ck.ck_w4a4_linear(inp["x"], inp["R"], case.g, inp["w_packed"], inp["w_scale"],
                                inp["bias"])
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        outs = []
        for _ in range(2):    # two calls in a row share the scratch array
            out = torch.full_like(ref, float("nan"))
            ck.ck_w4a4_linear_noalloc(inp["x"], inp["R"], case.g, inp["w_packed"], inp["w_scale"],
                                      inp["bias"], out=out, dev_status=status)
            outs.append(out)
        torch.cuda.synchronize()
        assert status.item() == 0
        for out in outs:
            # identical kernels on identical inputs: equal bit for bit (so within any tolerance)
            assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), case.name


def test_noalloc_rejects_scratch_needs_beyond_its_limit():
    """8192 x 10240 activations need 84 MB of scratch: refused on the host, nothing launched."""
    L = ck.lib()
    fake = 1 << 20
    st = L.ck_w4a4_linear_noalloc(fake, ck.CK_F16, 8192, 10240, 10240, 1, fake, 256, None, fake,
                                  3840, 5120, fake, ck.CK_F16, None, fake, ck.CK_F16, 3840, None,
                                  None)
    assert st == ck.CK_ERR_WORKSPACE
    assert "workspace" in ck.status_string(st)
