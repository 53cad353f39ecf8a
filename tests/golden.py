"""Reader for the small text fixtures under tests/golden/ (comment lines start with #)."""
import os

import numpy as np

DIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read(name: str) -> dict:
    sections, cur = {}, None
    with open(os.path.join(DIR, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if len(parts) == 1 and not _num(parts[0]):
                cur = parts[0]
                sections[cur] = []
            elif cur is not None and all(_num(p) for p in parts):
                sections[cur].append([float(p) for p in parts])
            else:
                sections[parts[0]] = [float(p) for p in parts[1:]]
                cur = None
    return sections


def _num(s: str) -> bool:
    try:
        float(s)
        return True
    except ValueError:
        return False


def grid_coords(rows: int, cols: int) -> np.ndarray:
    """Unjittered cell centres of a rows x cols grid in raster id order, [1, n, 2] fp32."""
    r, c = np.divmod(np.arange(rows * cols), cols)
    return np.stack([c + 0.5, r + 0.5], axis=1).astype(np.float32)[None]
