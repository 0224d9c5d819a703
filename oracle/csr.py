"""Receiver and sender CSR layouts (oracle side).

Test infrastructure only (see ``oracle/__init__.py``).

FlashCart (arXiv 2610.06409) §4 / App. D: the forward keeps edges sorted by
receiver and sums each receiver's incoming edges locally; ordering edges by
sender makes the sender-feature gradient deterministic.  The plain definition:
    ptr  = [0, cumsum(bincount(keys, minlength=N))]
    perm = stable argsort of keys (ties keep edge order).
"""
from __future__ import annotations

import numpy as np


def csr(keys: np.ndarray, N: int) -> tuple[np.ndarray, np.ndarray]:
    keys = np.asarray(keys)
    if keys.size and (keys.min() < 0 or keys.max() >= N):
        raise ValueError("key out of range")
    counts = np.bincount(keys, minlength=N).astype(np.int64)
    ptr = np.zeros(N + 1, dtype=np.int64)
    np.cumsum(counts, out=ptr[1:])
    perm = np.argsort(keys, kind="stable")
    return ptr.astype(np.int32), perm.astype(np.int32)
