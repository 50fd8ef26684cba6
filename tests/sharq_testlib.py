"""Test helpers: index permutations between the library's MMA-ready scale
atoms and canonical row-major scale matrices, and numpy/torch glue.  No
method arithmetic lives here."""
import numpy as np

BLOCK = {"nvfp4": 16, "mxfp4": 32, 0: 16, 1: 32}


def atom_index(rows, K, fmt):
    """Byte offsets of canonical scale (r, s) inside the atom buffer,
    [rows, K/B] int64 (the layout stated in include/sharq.h)."""
    nsf = K // BLOCK[fmt]
    r = np.arange(rows, dtype=np.int64)[:, None]
    s = np.arange(nsf, dtype=np.int64)[None, :]
    return (((r // 128) * (nsf // 4) + s // 4) * 512 + (r % 32) * 16
            + ((r % 128) // 32) * 4 + s % 4)


def atoms_to_canonical(buf, rows, K, fmt):
    buf = np.asarray(buf).reshape(-1)
    return buf[atom_index(rows, K, fmt)]


def canonical_to_atoms(scales, K, fmt, rows_pad=None):
    rows = scales.shape[0]
    rp = rows_pad or (rows + 127) // 128 * 128
    out = np.zeros(rp * (K // BLOCK[fmt]), dtype=np.uint8)
    out[atom_index(rows, K, fmt)] = scales
    return out


def to_dev(a_u16_or_u8, dtype="bf16"):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a_u16_or_u8))
    if dtype == "bf16":
        t = t.view(torch.bfloat16)
    return t.cuda()


def to_np(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()
