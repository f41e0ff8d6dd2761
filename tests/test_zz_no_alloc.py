"""gdn_prefill_noalloc: the prefill entry point for callers that cannot
allocate device memory -- e.g. a plugin whose host framework owns all of the
GPU's memory and passes in only inputs and outputs, or a loop that must never
call cudaMalloc/cudaFree because they can synchronise the device.  Its scratch
is one fixed array inside the library, shared by every call, so it must give
the same results as gdn_prefill call after call.

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import pytest
import torch

import linear_attention_layer_causal_b200 as gdn
from linear_attention_layer_causal_b200 import workloads as W
from parity_util import assert_output_close, assert_state_close

pytestmark = pytest.mark.gpu

P = ("conv_w", "A_log", "dt_bias", "norm_w")
LAYER = W.Workload("noalloc", 2, 16, 128, seqlens=(1,), state_std=0.02, seed=1)


def _both(cfg, inp, conv=None):
    ref = gdn.prefill(cfg, inp["qkv"], inp["a"], inp["b"], inp["z"], inp["cu_seqlens"],
                      *[inp[k] for k in P], initial_state=inp["initial_state"],
                      initial_conv=conv, return_final_state=True, return_final_conv=True,
                      return_o_raw=True)
    out = {k: torch.empty_like(v) for k, v in ref.items()}
    gdn.prefill_noalloc(cfg, inp["qkv"], inp["a"], inp["b"], inp["z"], inp["cu_seqlens"],
                        *[inp[k] for k in P], y=out["y"], initial_state=inp["initial_state"],
                        initial_conv=conv, final_state=out["final_state"],
                        final_conv=out["final_conv"], o_raw=out["o_raw"])
    torch.cuda.synchronize()
    return ref, out


def _check(ref, out):
    assert gdn.prefill_noalloc_status() == (gdn.GDN_OK, 0)
    assert_output_close(out["y"], ref["y"])
    assert_output_close(out["o_raw"], ref["o_raw"], "o_raw")
    assert_state_close(out["final_state"], ref["final_state"])
    assert torch.equal(out["final_conv"], ref["final_conv"])


def test_noalloc_matches_prefill_on_consecutive_calls(cuda_device):
    cfg = gdn.Config.of(LAYER)
    # two calls in a row with different inputs and lengths: the second reuses
    # the scratch the first one filled
    for seed, lens in [(11, (77, 130)), (12, (5, 200, 0, 33))]:
        inp = W.make_prefill(LAYER, cuda_device, seed=seed, seqlens=lens)
        g = torch.Generator(device=cuda_device).manual_seed(seed)
        conv = torch.randn((len(lens), 3, LAYER.conv_dim), generator=g,
                           device=cuda_device).to(torch.bfloat16)
        _check(*_both(cfg, inp, conv))


def _limit(cfg):
    """The most tokens one sequence can have within the fixed scratch."""
    n = 1
    while gdn.prefill_workspace_size(cfg, 1, n + 1) <= gdn.NOALLOC_SCRATCH_BYTES:
        n += 1
    return n


def test_noalloc_largest_call_and_limit(cuda_device):
    """At the Qwen3.8 layer shape the fixed scratch holds a few hundred tokens of
    one sequence: the largest such call runs and matches gdn_prefill, one token
    more is rejected before anything is launched."""
    cfg = gdn.Config(16, 128, 128)
    lim = _limit(cfg)
    assert lim >= 512
    wl = W.Workload("noalloc_max", 16, 128, 128, seqlens=(lim,), state_std=0.02, seed=3)
    inp = W.make_prefill(wl, cuda_device)
    _check(*_both(cfg, inp))
    big = W.make_prefill(wl, cuda_device, seqlens=(lim + 1,), seed=4)
    y = torch.empty((lim + 1, 128, 128), dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(gdn.GdnError) as e:
        gdn.prefill_noalloc(cfg, big["qkv"], big["a"], big["b"], big["z"], big["cu_seqlens"],
                            *[big[k] for k in P], y=y)
    assert e.value.status == gdn.GDN_ERR_WORKSPACE
    assert "scratch" in str(e.value)


def test_noalloc_reports_device_status(cuda_device):
    """The device status of a gdn_prefill_noalloc call sits in the library's own
    scratch, out of the caller's reach; gdn_prefill_noalloc_status reads it.  A
    call whose bounded waits are forced to run out reports GDN_ERR_TIMEOUT there,
    and the next call is clean and matches gdn_prefill again."""
    cfg = gdn.Config.of(LAYER)
    inp = W.make_prefill(LAYER, cuda_device, seed=21, seqlens=(150, 40))
    y = torch.empty((190, 16, 128), dtype=torch.bfloat16, device=cuda_device)
    args = (cfg, inp["qkv"], inp["a"], inp["b"], inp["z"], inp["cu_seqlens"],
            *[inp[k] for k in P])
    gdn.wait_limit_next_call(100)
    gdn.prefill_noalloc(*args, y=y, initial_state=inp["initial_state"])
    st, detail = gdn.prefill_noalloc_status()
    assert st == gdn.GDN_ERR_TIMEOUT
    assert detail == 0 or (detail & 0x80000000)
    _check(*_both(cfg, inp))
