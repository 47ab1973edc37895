"""Helpers of the GPU parity tests: move seeded inputs to the device, call the C ABI
through the Python binding, and fetch results.  No arithmetic of the method lives
here; expected values come from the oracle only."""
import numpy as np
import torch

from nvfp4_bit_quantized_amax_b200 import capi

DEV = "cuda:0"


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.to(DEV).view(torch.bfloat16)


def to_dev_u8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(DEV)


def u8(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint8)


def f32_bits(x) -> int:
    return int(np.float32(x).view(np.uint32))


def empty_u8(n):
    return torch.empty(int(n), dtype=torch.uint8, device=DEV)


def new_operand(rows, cols):
    """(data, scales, tensor_scale) device buffers of one quantized operand; the
    buffers start filled with 0xA5 so that unwritten bytes show up in a compare."""
    d = torch.full((int(capi.packed_bytes(rows, cols)),), 0xA5, dtype=torch.uint8, device=DEV)
    s = torch.full((int(capi.scale_bytes(rows, cols)),), 0xA5, dtype=torch.uint8, device=DEV)
    g = torch.full((1,), float("nan"), dtype=torch.float32, device=DEV)
    return d, s, g


def fetch_operand(op, rows, cols):
    d, s, g = op
    torch.cuda.synchronize()
    return u8(d).reshape(rows, cols // 2), u8(s), np.float32(g.item())


def gpu_quantize(x_bits, block_mode, rounding, seed=0):
    rows, cols = x_bits.shape
    x = to_dev_bf16(x_bits)
    op = new_operand(rows, cols)
    ws = empty_u8(capi.quantize_workspace_bytes())
    capi.nvfp4_quantize(x, block_mode, rounding, seed, *op, ws)
    packed, sf, g = fetch_operand(op, rows, cols)
    return packed, sf, g, capi.nvfp4_read_status(ws)


def operand_tensor(view, nbytes_data, nbytes_sf, ws):
    """Copy a workspace operand view (capi.Tensor) into host numpy arrays."""
    base = ws.data_ptr()
    d = ws[view.data - base: view.data - base + nbytes_data]
    s = ws[view.scales - base: view.scales - base + nbytes_sf]
    g = ws[view.tensor_scale - base: view.tensor_scale - base + 4]
    torch.cuda.synchronize()
    return u8(d), u8(s), np.frombuffer(u8(g).tobytes(), dtype=np.float32)[0]
