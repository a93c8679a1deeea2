"""The bounded device-side wait gives up, reports VSA_ERR_TIMEOUT through
vsa_device_status, and leaves the context usable (no fault, no hang)."""
import numpy as np
import pytest
import torch

import block_sparse_attention_cube_b200 as vsa
import synth
from tests._util import to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.expects_timeout]


def test_wait_probe_times_out_and_context_survives():
    vsa.device_status()                      # clear any earlier record
    vsa.debug_wait_probe(50_000_000)         # 50 ms on a barrier nothing arrives on
    with pytest.raises(vsa.VsaError) as e:
        vsa.device_status()
    assert e.value.status == 6
    vsa.device_status()                      # the read cleared it
    w = synth.WORKLOADS["tiny_8x8x8"]
    x = synth.make_inputs(w)
    d = {k: to_dev(v) for k, v in x.items()}
    s = vsa.Shape(w.batch, w.heads, w.head_dim, w.grid)
    out = vsa.forward(d["q"], d["k"], d["v"], s, w.topk)
    vsa.device_status()
    assert torch.isfinite(out.float()).all()
