"""Failure detection on the GPU without faulting it: a kernel waits on an
mbarrier that nothing will complete, with a 20 ms limit. The bounded wait must
give up, record the timeout in the device error word and return, leaving the
context usable for the next call."""
import pytest
import torch

import compressed_latent_space_cca_b200 as cca
import workloads
from parity import run_gpu, run_oracle, assert_close

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    assert cca.poll_device_status() == cca.CCA_OK
    assert cca.selftest_wait_timeout(20000) == cca.CCA_OK
    assert cca.poll_device_status() == cca.CCA_ERR_DEVICE_TIMEOUT
    assert cca.poll_device_status() == cca.CCA_OK  # the word is cleared by the poll
    sh = workloads.WORKLOADS["tiny_cca_fp32"]
    inp = workloads.make_inputs(sh)
    gpu = run_gpu(sh, inp)
    assert_close("y", gpu["y"], run_oracle(sh, inp)["y"], "f32")


def test_invalid_calls_rejected_before_launch():
    sh = workloads.WORKLOADS["tiny_cca_fp32"]
    cfg = cca.config_from_shape(sh)
    inp = {k: v.cuda() for k, v in workloads.make_inputs(sh).items()}
    out = cca.alloc_outputs(cfg, torch.device("cuda"))
    sentinel = out["y"].fill_(7.0).clone()
    small_ws = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(cca.CcaError) as ei:
        cca.prefill(cfg, inp, out=out, workspace=small_ws)
    assert ei.value.status == cca.CCA_ERR_WORKSPACE
    bad = cca.config_from_shape(sh)
    bad.n_kv_heads = 3
    with pytest.raises(cca.CcaError) as ei:
        cca.alloc_workspace(bad, torch.device("cuda"))
    assert ei.value.status == cca.CCA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.equal(out["y"], sentinel)  # outputs untouched


@pytest.mark.parametrize("path", [cca.CCA_PATH_AUTO, cca.CCA_PATH_SIMT], ids=["auto", "simt"])
@pytest.mark.parametrize("where", ["latents", "channel_mix"])
def test_fp16_range_reported(path, where):
    """bf16 blocks keep their intermediates in fp16. Values beyond fp16's range
    are reported by the next status poll as a numeric-range error, not passed on
    silently: latents that overflow in the down-projection, or q after a channel
    mix whose weights are fine in fp16 but whose outputs are not."""
    sh = workloads.BlockShape("range", 1, 300, 512, 4, 2, 128, 4, "bf16", 5)
    inp = workloads.make_inputs(sh)
    if where == "latents":
        inp["x"] = (inp["x"].float() * 1e5).to(torch.bfloat16)
    else:  # latents below 6 and weights below 43k, but about 4 % of q beyond 65504
        inp["x"] = (inp["x"].float() * 3).to(torch.bfloat16)
        inp["convq_chan"] = (inp["convq_chan"].float() * 1e5).to(torch.bfloat16)
        assert float(inp["convq_chan"].float().abs().max()) < 65504.0
    cfg = cca.config_from_shape(sh)
    assert cca.poll_device_status() == cca.CCA_OK
    cca.prefill(cfg, {k: v.cuda() for k, v in inp.items()}, path=path)
    assert cca.poll_device_status() == cca.CCA_ERR_NUMERIC_RANGE
    assert cca.poll_device_status() == cca.CCA_OK  # cleared by the poll
