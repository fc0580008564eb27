"""Helpers shared by the tests: scale-layout index maps, comparisons and the
CUDA gate.  Nothing here computes any part of the layer."""
import os
import re

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    """Names of every function declared in include/*.h."""
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"NVFP4_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)
    return names


def require_cuda():
    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA device (run it with -m gpu on a B200)")
    major, _ = torch.cuda.get_device_capability()
    if major != 10:
        pytest.fail(f"needs an sm_100 device, found compute capability {major}.x")


def capi():
    from nvfp4_w4a4_quantized_moe_b200 import build
    build.build()
    from nvfp4_w4a4_quantized_moe_b200 import capi as c
    return c


# --- tiled scale layout (the layout the tensor-core MMA reads) ---------------

def tiled_index(rows_padded: int, cols: int) -> np.ndarray:
    """idx[r, b] = byte offset of (row r, 16-element block b) in the tiled layout."""
    nb = cols // 16
    r = np.arange(rows_padded)[:, None]
    b = np.arange(nb)[None, :]
    atom = (r // 128) * (nb // 4) + b // 4
    return atom * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4


def tiled_rows(tiled: np.ndarray, rows_idx, cols: int) -> np.ndarray:
    """Canonical scale rows ``rows_idx`` read out of a tiled scale buffer."""
    r = np.asarray(rows_idx)[:, None]
    nb = cols // 16
    b = np.arange(nb)[None, :]
    idx = ((r // 128) * (nb // 4) + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4
    return np.asarray(tiled).reshape(-1)[idx]


def tiled_to_canonical(tiled: np.ndarray, rows: int, cols: int) -> np.ndarray:
    rp = (rows + 127) // 128 * 128
    return np.asarray(tiled).reshape(-1)[tiled_index(rp, cols)][:rows]


def canonical_to_tiled(canon: np.ndarray) -> np.ndarray:
    rows, nb = canon.shape
    rp = (rows + 127) // 128 * 128
    out = np.zeros(rp * nb, np.uint8)
    out[tiled_index(rows, nb * 16)] = canon
    return out


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    d = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (d if d > 0 else 1.0))


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


# --- staged weight-code layout (one contiguous 16 KiB tile per 128 rows x
# 256 columns, 16-byte chunks swizzled by row; see the library header) --------

def staged_unit_index(rows: int, cols: int) -> np.ndarray:
    """idx[r, b] = index of the 8-byte unit that holds the codes of (row r,
    16-element block b) of one matrix in the staged layout."""
    nb = cols // 16
    r = np.arange(rows)[:, None]
    b = np.arange(nb)[None, :]
    tile = (r // 128) * (nb // 16) + b // 16
    chunk = (b % 16) // 2
    return tile * 2048 + (r % 128) * 16 + (chunk ^ (r % 8)) * 2 + b % 2


def staged_to_canonical(codes, rows: int, cols: int) -> np.ndarray:
    """Row-major codes [rows, cols/2] of one matrix read out of its staged bytes."""
    units = np.asarray(codes).reshape(-1, 8)
    return units[staged_unit_index(rows, cols)].reshape(rows, cols // 2)


def canonical_to_staged(codes, rows: int, cols: int) -> np.ndarray:
    """The staged bytes of one matrix from its row-major codes [rows, cols/2]."""
    out = np.empty((rows * cols // 16, 8), dtype=np.uint8)
    out[staged_unit_index(rows, cols)] = np.asarray(codes, dtype=np.uint8).reshape(rows, cols // 16, 8)
    return out.reshape(rows, cols // 2)
