"""cca_prefill_noalloc against cca_prefill.

The allocation-free entry point serves callers that must not allocate device
memory while they run (cudaMalloc can synchronize the whole device, and some
host runtimes own every byte of device memory): its intermediates live in a
fixed array inside the library instead of a caller-provided workspace. Two
calls in a row must give what cca_prefill gives on the same inputs, bit for
bit: the kernels are deterministic, so any difference would point at the
workspace (an aliasing or stale-data fault that a tolerance could hide). A
block too large for the array must be rejected with a clear error. This file
sorts last so that a run stopping at the first failure has already run every
other test.
"""
import pytest
import torch

import compressed_latent_space_cca_b200 as cca
import workloads

pytestmark = pytest.mark.gpu


def _shape(seq_len, batch=1):
    return workloads.BlockShape("noalloc", batch, seq_len, 1024, 4, 2, 128, 4, "bf16", 21)


def test_noalloc_matches_prefill_twice():
    sh = _shape(3000, batch=2)
    cfg = cca.config_from_shape(sh)
    assert cca.workspace_size(cfg) <= cca._capi.CCA_NOALLOC_WORKSPACE_BYTES
    inp = {k: v.cuda() for k, v in workloads.make_inputs(sh).items()}
    ref = cca.prefill(cfg, inp)
    for _ in range(2):
        got = cca.prefill_noalloc(cfg, inp)
        assert cca.poll_device_status() == cca.CCA_OK
        for name in ("y", "k_cache", "v_cache"):
            assert torch.equal(got[name], ref[name]), name


def test_noalloc_rejects_blocks_beyond_its_array():
    sh = _shape(16384)
    cfg = cca.config_from_shape(sh)
    assert cca.workspace_size(cfg) > cca._capi.CCA_NOALLOC_WORKSPACE_BYTES
    inp = {k: v.cuda() for k, v in workloads.make_inputs(sh).items()}
    out = cca.alloc_outputs(cfg, torch.device("cuda"))
    out["y"].fill_(3.0)
    with pytest.raises(cca.CcaError) as ei:
        cca.prefill_noalloc(cfg, inp, out=out)
    assert ei.value.status == cca.CCA_ERR_WORKSPACE
    assert "static workspace" in str(ei.value)
    torch.cuda.synchronize()
    assert bool((out["y"] == 3.0).all())  # nothing was launched
