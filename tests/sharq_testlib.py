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


def meta_atom_index(rows, K):
    """Byte offsets of canonical pair metadata (r, j) ([rows, K/16], group 2j
    of a row in the low nibble of byte j) inside the atom buffer: atom
    (k-block j // 16, row block r // 128) at ((j // 16) * rows_pad / 128 +
    r // 128) * 2048, row r % 128 at 16 bytes a row (layout of include/sharq.h)."""
    rp = (rows + 127) // 128 * 128
    r = np.arange(rows, dtype=np.int64)[:, None]
    j = np.arange(K // 16, dtype=np.int64)[None, :]
    return ((j // 16) * (rp // 128) + r // 128) * 2048 + (r % 128) * 16 + j % 16


def meta_atoms_to_canonical(buf, rows, K):
    return np.asarray(buf).reshape(-1)[meta_atom_index(rows, K)]


def canonical_to_meta_atoms(meta, K):
    rows = meta.shape[0]
    rp = (rows + 127) // 128 * 128
    out = np.full(rp * (K // 16), 0x44, dtype=np.uint8)
    out[meta_atom_index(rows, K)] = meta
    return out
