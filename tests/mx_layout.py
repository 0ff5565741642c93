"""Test-side conversion between the plain [rows, K/32] scale grid and the MMA atom layout
(512-byte atoms of 128 rows x 4 k-blocks; row r is word (r % 32) * 4 + r // 32)."""
import numpy as np

_WORD = np.array([(r % 32) * 4 + r // 32 for r in range(128)])


def plain_to_atoms(plain):
    """[G*128, KS] uint8 -> flat atoms (row group g = row // 128)."""
    plain = np.asarray(plain, dtype=np.uint8)
    rows, ks = plain.shape
    g, kb4 = rows // 128, ks // 4
    src = plain.reshape(g, 128, kb4, 4).transpose(0, 2, 1, 3)          # [g, j, r, byte]
    out = np.empty((g, kb4, 128, 4), dtype=np.uint8)
    out[:, :, _WORD, :] = src
    return out.reshape(-1)


def atoms_to_plain(atoms, groups, ks):
    a = np.asarray(atoms, dtype=np.uint8)[: groups * (ks // 4) * 512].reshape(groups, ks // 4, 128, 4)
    return a[:, :, _WORD, :].transpose(0, 2, 1, 3).reshape(groups * 128, ks)


def tile_atoms_to_plain(atoms, split_sizes, ks):
    """Atoms whose row groups are each expert's 128-row tiles -> plain [R, ks] (tails dropped)."""
    split = [int(n) for n in split_sizes]
    groups = sum((n + 127) // 128 for n in split)
    padded = atoms_to_plain(atoms, groups, ks)
    out, g = [], 0
    for n in split:
        out.append(padded[g * 128: g * 128 + n])
        g += (n + 127) // 128
    return np.concatenate(out) if out else np.zeros((0, ks), np.uint8), padded, groups


def grouped_scales_to_atoms(scales_per_expert, split_sizes, C):
    """Per-expert [ceil(n_e/32), C] scales (blocks along rows) -> the grouped atom layout:
    expert e owns KG_e = ceil(n_e/128) k-groups; atom (cg, kg) of expert e at
    (kgoff_e * C/128 + cg * KG_e + kg); unused block bytes are zero."""
    CG = C // 128
    atoms = []
    for n, s in zip(split_sizes, scales_per_expert):
        n = int(n)
        kg = (n + 127) // 128
        if kg == 0:
            continue
        blocks = np.zeros((kg * 4, C), dtype=np.uint8)
        blocks[: s.shape[0]] = s
        # [kg*4, C] -> per (cg, kg): atom[word(c%128), byte = block % 4]
        b = blocks.reshape(kg, 4, CG, 128).transpose(2, 0, 3, 1)       # [cg, kg, c, byte]
        out = np.empty((CG, kg, 128, 4), dtype=np.uint8)
        out[:, :, _WORD, :] = b
        atoms.append(out.reshape(-1))
    return np.concatenate(atoms) if atoms else np.zeros(0, np.uint8)


def grouped_atoms_to_scales(atoms, split_sizes, C):
    """Inverse of grouped_scales_to_atoms: per-expert [ceil(n_e/32), C] scales."""
    CG = C // 128
    a = np.asarray(atoms, dtype=np.uint8)
    out, base = [], 0
    for n in split_sizes:
        n = int(n)
        kg = (n + 127) // 128
        if kg == 0:
            out.append(np.zeros((0, C), dtype=np.uint8))
            continue
        blk = a[base * 512: (base + CG * kg) * 512].reshape(CG, kg, 128, 4)[:, :, _WORD, :]   # [cg, kg, c, byte]
        scales = blk.transpose(1, 3, 0, 2).reshape(kg * 4, C)
        out.append(scales[: (n + 31) // 32])
        base += CG * kg
    return out
