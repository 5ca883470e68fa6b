"""The decode forward that allocates nothing, moe_forward_decode_noalloc.

It serves callers that cannot allocate device memory for a workspace (memory
pools that forbid cudaMalloc, callbacks that may not allocate, C hosts that
hold only tensor pointers): its scratch is a buffer inside the library. These
checks call it through the C ABI twice in a row, on two different inputs, and
compare each result with moe_forward's on a caller-provided workspace, and
read the call's device status word through moe_noalloc_read_device_status.
The file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

from helpers import assert_bf16_close, bf16_np, device_site, site_inputs, workload

pytestmark = pytest.mark.gpu

capi = pytest.importorskip("routed_nvfp4_expert_b200.capi")


@pytest.mark.parametrize("name,T", [("tiny_t4", 4), ("decode_t1", 1), ("decode_t8", 8)])
def test_noalloc_matches_moe_forward_on_two_calls(name, T):
    from routed_nvfp4_expert_b200 import synthetic as syn
    wl = workload(name, T=T)
    inp = site_inputs(wl)
    site = device_site(wl, inp)
    cfg = capi.config_for(wl)
    xs = [capi.bf16_tensor(inp["x"]), capi.bf16_tensor(syn.random_x(wl, T, seed=77))]
    ws = capi.alloc_workspace(cfg, T, capi.PATH_DECODE)
    for x in xs:                     # two calls in a row, different inputs
        y_ref = torch.empty_like(x)
        capi.moe_forward(cfg, site, x, capi.PATH_DECODE, y_ref, ws)
        y = torch.full_like(x, float("nan"))
        capi.moe_forward_decode_noalloc(cfg, site, x, y)
        capi.moe_noalloc_read_device_status()      # device-side errors of the call: none
        torch.cuda.synchronize()
        assert_bf16_close(bf16_np(y), bf16_np(y_ref), what=f"{name} noalloc vs moe_forward")
        # same kernels, same order: the results agree bit for bit as well
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
