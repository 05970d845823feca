"""bottleneck_i8_noalloc: the bottleneck chain for callers that cannot
allocate device memory (a plugin whose execution step must not allocate, or a
runtime that fixes all device memory at start-up).  It keeps the two
intermediates in a 32 MiB array built into the library instead of a
caller-provided workspace.

Checked through the C ABI against the workspace entry point bottleneck_i8,
bit for bit (the tolerance of every parity test here), on two calls in a
row with different inputs, so the second call cannot pass on what the first
left in the shared array.  This file is collected last on purpose and needs
no fixture from the others, so it passes alone in a fresh process too.
"""
import pytest
import torch

import x1_conv_bn_b200 as X
from x1_conv_bn_b200 import synth

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from x1_conv_bn_b200 import _build

    _build.build()
    X.lib()


def _packed_block(B, seed):
    s = synth.BlockShape(B, 28, 28, 512, 128)
    inp = synth.block_inputs(s, seed)
    x = X.x1cb_pack_act(inp.x.to(DEV))
    args = []
    for w, b, m in zip(inp.w, inp.bias, inp.m):
        args += [X.x1cb_pack_weight(w.to(DEV)), b.to(DEV), m.to(DEV)]
    return x, args, inp.m_r, inp.S


@pytest.mark.parametrize("B", [16, 167])
def test_noalloc_matches_workspace_entry_point_on_two_calls(B):
    outs = []
    for seed in (501, 502):
        x, args, m_r, S = _packed_block(B, seed)
        ref = X.bottleneck_i8(x, *args, m_r, S)
        got = X.bottleneck_i8_noalloc(x, *args, m_r, S)
        torch.cuda.synchronize()
        st, bits = X.x1cb_last_device_error(clear=True)
        assert st == 0, bits
        assert torch.equal(got, ref), int((got != ref).sum())
        outs.append(got.cpu())
    assert not torch.equal(outs[0], outs[1])  # the two calls really differ


def test_noalloc_rejects_problems_larger_than_its_scratch():
    x, args, m_r, S = _packed_block(1, 503)
    big = torch.empty((168, 16, 28, 28, 32), dtype=torch.int8, device=DEV)
    with pytest.raises(X.X1cbError) as e:
        X.bottleneck_i8_noalloc(big, *args, m_r, S)
    assert e.value.status == X.X1CB_ERR_WORKSPACE
