"""The bounded-wait failure path on the GPU, made to happen without a fault:
the BF16 tensor-core GEMM's main-loop waits get a zero limit through the test
hook moe_set_wait_limit, so the first wait for a copy or MMA still in flight
runs out. The kernel must report MOE_ERR_DEVICE_TIMEOUT in the workspace
status word, wind down (it waits with the default limit for everything it
already issued and frees its tensor memory), and leave the device usable: the
same call with the default limit is correct afterwards."""
import numpy as np
import pytest
import torch

from helpers import assert_bf16_close, bf16_np
from oracle import site as OS

pytestmark = pytest.mark.gpu

capi = pytest.importorskip("routed_nvfp4_expert_b200.capi")


def _dense(H, I, T):
    from routed_nvfp4_expert_b200 import synthetic as syn
    wl = syn.Workload("dense", T=T, H=H, I=16, E=1, k=1, Is=0, dense_I=I, sigma_w=0.02)
    return syn.make_dense(wl), syn.make_router_and_x(wl)["x"]


def test_bf16_gemm_wait_timeout_reports_and_the_device_recovers():
    H, I, T = 256, 512, 256          # T >= 128: the two tcgen05 BF16 GEMMs
    d, x = _dense(H, I, T)
    tb = capi.bf16_tensor
    xs, wg, wu, wd = tb(x), tb(d["dense_gate"]), tb(d["dense_up"]), tb(d["dense_down"])
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(capi.dense_ffn_workspace_size(H, I, T), dtype=torch.uint8, device="cuda")
    capi.moe_set_wait_limit(0)
    try:
        capi.dense_ffn_bf16(7.0, xs, wg, wu, wd, y, ws)
        with pytest.raises(capi.MoEError) as ei:
            capi.moe_read_device_status(ws)
        assert ei.value.status == 5          # MOE_ERR_DEVICE_TIMEOUT
    finally:
        capi.moe_set_wait_limit(-1)
    # the same device, default limits: a normal, correct call
    capi.dense_ffn_bf16(7.0, xs, wg, wu, wd, y, ws)
    capi.moe_read_device_status(ws)
    tok = np.array([0, 1, 77, T - 1])
    ref = OS.dense_ffn(x[tok], d["dense_gate"], d["dense_up"], d["dense_down"], 7.0)
    assert_bf16_close(bf16_np(y)[tok], ref, what="dense y after the timeout")
