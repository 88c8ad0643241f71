"""Plain CPU oracle of the scan-locality measurement: how far apart, in a scanned sequence, the tokens
end up that are neighbours in the 3D latent grid.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the benchmark's CPU-baseline
leg may import this module.  It shares no code with the CUDA library and imports nothing from it.

Source: the LinGen news article ("视频生成模型太贵太慢怎么办"), method section, Rotary Major Scan
paragraphs, and "LinGen：基于Mamba机制的线性复杂度高清长视频生成框架", 功能特色 and 关键算法创新 / RMS: the
four scan orders alternate between layers and bring the average distance, after the scan, between tokens
that were adjacent down to the level of the special Zigzag and Hilbert scans.

Readings (the pages name the quantity but do not define it; each is also listed in the design notes):
  * adjacent = the two tokens differ by one step along exactly one of the axes t, h, w (each unordered
    pair counted once); distance = |position_a - position_b| in the scanned sequence;
  * per index map the measurement is the sum, count and maximum of that distance over all adjacent pairs;
  * the Rotary Major Scan rotation (map 6) takes, per pair, the smallest distance over the four orders, the
    four layers of one rotation cycle;
  * Zigzag (map 4) = the 3D boustrophedon: w fastest, reversing direction on every (t, h) line, h reversing
    on every t plane, t ascending (each step moves to an adjacent token);
  * Hilbert (map 5) = the grid cut into cubes of side H = W (a power of two) stacked along t, each cube
    traversed by the 3D Hilbert curve (Skilling's transposed-index construction), cubes in t order.
Pins: tests/test_oracle_pins.py checks closed forms for the four orders and the rotation, unit steps and
bijectivity of the Zigzag and Hilbert paths, and brute force on small grids.
"""
from __future__ import annotations

import numpy as np

from .mate_oracle import scan_positions

MAP_NAMES = {0: "rms_order0", 1: "rms_order1", 2: "rms_order2", 3: "rms_order3", 4: "zigzag", 5: "hilbert",
             6: "rms_rotation"}


def zigzag_positions(T: int, H: int, W: int) -> np.ndarray:
    """Sequence position of every token [T, H, W] along the 3D boustrophedon path."""
    pos = np.empty((T, H, W), dtype=np.int64)
    k = 0
    for t in range(T):
        hs = range(H) if t % 2 == 0 else range(H - 1, -1, -1)
        for j, h in enumerate(hs):
            line = t * H + j                     # lines visited so far decide the w direction
            ws = range(W) if line % 2 == 0 else range(W - 1, -1, -1)
            for w in ws:
                pos[t, h, w] = k
                k += 1
    return pos


def hilbert_index3(x: int, y: int, z: int, bits: int) -> int:
    """Index of the point (x, y, z) of a 2^bits cube along the 3D Hilbert curve: Skilling's conversion of
    axes to the 'transposed' index (undo the excess work of the Gray-code reflections and exchanges, then
    Gray-encode), followed by interleaving the transposed bits, most significant first."""
    X = [x, y, z]
    n = 3
    M = 1 << (bits - 1)
    Q = M
    while Q > 1:
        P = Q - 1
        for i in range(n):
            if X[i] & Q:
                X[0] ^= P
            else:
                t = (X[0] ^ X[i]) & P
                X[0] ^= t
                X[i] ^= t
        Q >>= 1
    for i in range(1, n):
        X[i] ^= X[i - 1]
    t = 0
    Q = M
    while Q > 1:
        if X[n - 1] & Q:
            t ^= Q - 1
        Q >>= 1
    for i in range(n):
        X[i] ^= t
    idx = 0
    for b in range(bits - 1, -1, -1):
        for i in range(n):
            idx = (idx << 1) | ((X[i] >> b) & 1)
    return idx


def hilbert_positions(T: int, H: int, W: int) -> np.ndarray:
    """Sequence position of every token [T, H, W]: cubes of side H = W along t, Hilbert order inside."""
    if H != W or H & (H - 1) or T % H:
        raise ValueError("Hilbert map needs H = W a power of two dividing T")
    S = H
    bits = max(1, S.bit_length() - 1)
    pos = np.empty((T, H, W), dtype=np.int64)
    for t in range(T):
        cube, tt = divmod(t, S)
        for h in range(H):
            for w in range(W):
                pos[t, h, w] = cube * S ** 3 + hilbert_index3(tt, h, w, bits)
    return pos


def positions(T: int, H: int, W: int, kind: int) -> np.ndarray:
    if 0 <= kind <= 3:
        return scan_positions(T, H, W, kind)
    if kind == 4:
        return zigzag_positions(T, H, W)
    if kind == 5:
        return hilbert_positions(T, H, W)
    raise ValueError(kind)


def _pair_distances(pos: np.ndarray):
    """|position difference| of every axis-adjacent pair, per axis (t, h, w)."""
    return (np.abs(pos[1:, :, :] - pos[:-1, :, :]), np.abs(pos[:, 1:, :] - pos[:, :-1, :]),
            np.abs(pos[:, :, 1:] - pos[:, :, :-1]))


def scan_locality(T: int, H: int, W: int, kind: int):
    """(sum of distances, number of adjacent pairs, largest distance) for index map `kind` (0..6)."""
    if kind == 6:
        per_order = [_pair_distances(scan_positions(T, H, W, o)) for o in range(4)]
        d = [np.minimum.reduce([per_order[o][a] for o in range(4)]) for a in range(3)]
    else:
        d = _pair_distances(positions(T, H, W, kind))
    total = int(sum(int(x.sum()) for x in d))
    pairs = int(sum(x.size for x in d))
    largest = int(max((int(x.max()) for x in d if x.size), default=0))
    return total, pairs, largest
