"""nvfp4_quantize_noalloc, the quantizer for callers that cannot allocate device
memory (for example a plugin handed only its input and output buffers by a host
framework that owns every device allocation): it keeps its scratch in the
library's static device array instead of a caller workspace.  Its output must
equal nvfp4_quantize's, byte for byte, on two calls in a row -- the second with a
smaller tensor amax than the first, so scratch left over from the first call
would show up as a wrong tensor scale.  Collected last (file name) so that a run
stopping at the first failure has run every other test before it."""
import numpy as np
import pytest
import torch

from gpu_util import DEV, empty_u8, to_dev_bf16, u8
from nvfp4_bit_quantized_amax_b200 import capi
from nvfp4_bit_quantized_amax_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def buffers(rows, cols):
    return (torch.full((capi.packed_bytes(rows, cols),), 0xA5, dtype=torch.uint8, device=DEV),
            torch.full((capi.scale_bytes(rows, cols),), 0xA5, dtype=torch.uint8, device=DEV),
            torch.full((1,), float("nan"), dtype=torch.float32, device=DEV))


def host(op):
    d, s, g = op
    return u8(d), u8(s), g.cpu().numpy().view(np.uint32)


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    capi.load()
    cases = [
        (syn.normal_bf16((300, 272), 1, outlier_prob=0.01), capi.BLOCK_1X16, capi.ROUND_SR, 31),
        (syn.normal_bf16((256, 512), 2, std=0.02), capi.BLOCK_16X16, capi.ROUND_RNE, 0),
    ]
    xs = [to_dev_bf16(c[0]) for c in cases]
    # two no-alloc calls back to back on the same stream
    got = []
    for x, (xb, bm, rnd, seed) in zip(xs, cases):
        op = buffers(*xb.shape)
        capi.nvfp4_quantize_noalloc(x, bm, rnd, seed, *op)
        got.append(op)
    torch.cuda.synchronize()
    # the same inputs through the entry point that takes a caller workspace
    for x, (xb, bm, rnd, seed), g_op in zip(xs, cases, got):
        ref = buffers(*xb.shape)
        ws = empty_u8(capi.quantize_workspace_bytes())
        capi.nvfp4_quantize(x, bm, rnd, seed, *ref, ws)
        torch.cuda.synchronize()
        assert capi.nvfp4_read_status(ws) == 0
        for a, b in zip(host(g_op), host(ref)):
            assert np.array_equal(a, b)
