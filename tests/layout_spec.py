"""The device weight layout as include/fluxbin.h documents it, restated in
numpy for checking fb_pack's output bit for bit.  Plain index arithmetic from
the header text; shares nothing with the library or the oracle."""

import numpy as np


def round_up(a, b):
    return (a + b - 1) // b * b


def pack_reference(signs: np.ndarray) -> np.ndarray:
    """int8 signs [K][M][N] -> uint8 planes in the documented device layout."""
    K, M, N = signs.shape
    assert N % 32 == 0
    M_pad = round_up(M, 32)
    out = np.zeros(K * M_pad * N // 8, dtype=np.uint8)
    bits = np.zeros((K, M_pad, N), dtype=np.uint8)
    bits[:, :M, :] = signs > 0
    # canonical bytes: byte group q of panel p is columns 256p+8q..+7, bit t = column +t
    canon = np.packbits(bits, axis=-1, bitorder="little")      # [K][M_pad][N/8]
    P = (N + 255) // 256
    for k in range(K):
        for p in range(P):
            width = min(256, N - 256 * p)
            Bp = width // 8
            panel = k * M_pad * N // 8 + 32 * p * M_pad
            for c in range(M_pad // 32):
                blk = panel + 32 * Bp * c
                for l in range(32):
                    row = 32 * c + l
                    for u in range(Bp):
                        q = (l + u) % Bp
                        if Bp % 16 == 0:
                            off = (u // 16) * 512 + 16 * l + u % 16
                        else:
                            off = (u // 4) * 128 + 4 * l + u % 4
                        out[blk + off] = canon[k, row, 32 * p + q]
    return out
