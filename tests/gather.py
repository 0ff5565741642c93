"""Test-side gathers of the permuted operands (from the library's row_map, whose bits the
routing tests pin): the bf16 rows the permuted tensors hold, without the library writing
them (the MXFP8 layer permutes and quantises in one pass)."""
import numpy as np
import torch


def row_tokens(row_map, k: int) -> np.ndarray:
    """token of every permuted row: row_map[t*k + j] = r  ->  token[r] = t."""
    rm = np.asarray(row_map.cpu() if hasattr(row_map, "cpu") else row_map, dtype=np.int64)
    tok = np.empty(rm.size, dtype=np.int64)
    tok[rm] = np.arange(rm.size) // k
    return tok


def permuted(x, row_map, k: int, rows=None) -> torch.Tensor:
    """x [T, H] (any device) gathered into expert order on the CPU: row r = x[token[r]]
    (only the rows listed in ``rows`` when given)."""
    tok = row_tokens(row_map, k)
    if rows is not None:
        tok = tok[np.asarray(rows)]
    return x.cpu()[torch.from_numpy(tok)]
