"""Test-side layout helpers: read libmetis device buffers into the oracle's layout.

These only move bytes (unpack nibbles, undo the 512-byte scale tiling); they
hold none of the method's arithmetic.
"""

import numpy as np
import torch

from oracle import nvfp4


def scales_linear(buf, outer, inner):
    """Tiled E4M3 scale bytes -> (outer x inner/16) array in row-major order."""
    raw = buf.detach().cpu().numpy().astype(np.uint8)
    nb = inner // 16
    o = np.arange(outer)[:, None]
    b = np.arange(nb)[None, :]
    off = ((o >> 7) * (inner // 64) + (b >> 2)) * 512 + (o & 31) * 16 + ((o & 127) >> 5) * 4 + (b & 3)
    return raw[off]


def scales_tiled(lin, outer, inner):
    """Inverse of scales_linear: (outer x inner/16) -> tiled bytes."""
    out = np.zeros(((outer + 127) // 128) * (inner // 64) * 512, dtype=np.uint8)
    nb = inner // 16
    o = np.arange(outer)[:, None]
    b = np.arange(nb)[None, :]
    off = ((o >> 7) * (inner // 64) + (b >> 2)) * 512 + (o & 31) * 16 + ((o & 127) >> 5) * 4 + (b & 3)
    out[off] = lin
    return out


def codes_unpacked(t):
    """Device Nvfp4 -> (codes outer x inner, scale codes outer x inner/16, g)."""
    packed = t.codes.detach().cpu().numpy().reshape(t.outer, t.inner // 2)
    codes = nvfp4.unpack_codes(packed)
    scales = scales_linear(t.scales, t.outer, t.inner)
    g = float(t.tensor_scale[0].item())
    return codes, scales, g


def load_nvfp4(t, codes, scales, g):
    """Write oracle-layout codes/scales/g into a device Nvfp4 (for GeMM inputs)."""
    packed = nvfp4.pack_codes(codes)
    t.codes.copy_(torch.from_numpy(packed.reshape(-1)))
    t.scales.copy_(torch.from_numpy(scales_tiled(scales, t.outer, t.inner)))
    t.tensor_scale.fill_(g)


def dequant(t, rows=None):
    codes, scales, g = codes_unpacked(t)
    if rows is not None:
        codes, scales = codes[:rows], scales[:rows]
    return nvfp4.dequantize_blocks(codes, scales, g)


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def bf16_round(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def hat_select(op, orientation, rows=None, cols=None):
    """Rows or columns of the dense operand hat Q(U) S Q(V)^T + Q(M_R) (oracle layout op).

    orientation "row": the residual quantized along columns (stored rows x cols);
    "col": along rows (stored transposed).  Only the requested slice is decoded.
    """
    from oracle import metis
    codes, scales, g = op[orientation]
    if orientation == "row":
        sel = slice(None) if rows is None else rows
        part = nvfp4.dequantize_blocks(codes[sel], scales[sel], g)
        if cols is not None:
            part = part[:, cols]
    else:
        sel = slice(None) if cols is None else cols
        part = nvfp4.dequantize_blocks(codes[sel], scales[sel], g).T
        if rows is not None:
            part = part[rows]
    if op.get("U") is not None:
        U = metis.dequant_factor(op["Uq"])
        V = metis.dequant_factor(op["Vq"])
        if rows is not None:
            U = U[rows]
        if cols is not None:
            V = V[cols]
        part = part + (U * np.asarray(op["S"], dtype=np.float64)[None, :]) @ V.T
    return part
