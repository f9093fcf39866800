"""Plain-numpy statement of the packed-code layout documented in
``include/ternary_decoder.h`` (the library's own design; the pages fix only
2 bits per weight and 128-weight units).  Used by the tests to check the
bytes the CUDA packer writes; it shares no code with the library.

Layout: code c stored as c+1 in 2 bits; 16-row blocks (N padded with code 0);
tiles of 16 rows x 128 k (512 bytes) stored row-block-major; inside a tile
32-bit word 4*l + j (l = 4g + t) holds row g + 8*(j & 1), k = 64*(j >> 1) +
16*t + 4*s + b at bit 8*b + 2*s.
"""
import numpy as np


def pack(codes: np.ndarray) -> np.ndarray:
    """codes int8 [N, K] in {-1,0,1} -> packed uint8 [ceil(N/16)*16*K/4]."""
    N, K = codes.shape
    assert K % 128 == 0
    Np = -(-N // 16) * 16
    c = np.zeros((Np, K), np.uint32)
    c[:N] = codes.astype(np.int32) + 1
    c[N:] = 1
    KT = K // 128
    # index grids over (rb, kt, g, t, j, s, b)
    rb, kt, g, t, j, s, b = np.meshgrid(np.arange(Np // 16), np.arange(KT), np.arange(8),
                                        np.arange(4), np.arange(4), np.arange(4), np.arange(4),
                                        indexing="ij")
    row = rb * 16 + g + 8 * (j & 1)
    k = kt * 128 + 64 * (j >> 1) + 16 * t + 4 * s + b
    vals = c[row, k] << (8 * b + 2 * s)
    words = vals.sum(axis=(5, 6), dtype=np.uint64).astype(np.uint32)  # disjoint bits
    # word order: tile (rb, kt) -> lane l = 4g + t -> j
    return words.reshape(-1).view(np.uint8).copy()


def unpack(packed: np.ndarray, N: int, K: int) -> np.ndarray:
    words = packed.view(np.uint32)
    Np = -(-N // 16) * 16
    KT = K // 128
    w = words.reshape(Np // 16, KT, 8, 4, 4)
    out = np.empty((Np, K), np.int8)
    for s in range(4):
        for b in range(4):
            f = ((w >> (8 * b + 2 * s)) & 3).astype(np.int8) - 1
            for j in range(4):
                rows = (np.arange(Np // 16)[:, None, None, None] * 16 +
                        np.arange(8)[None, None, :, None] + 8 * (j & 1))
                ks = (np.arange(KT)[None, :, None, None] * 128 + 64 * (j >> 1) +
                      16 * np.arange(4)[None, None, None, :] + 4 * s + b)
                rows_b, ks_b = np.broadcast_arrays(rows, ks)
                out[rows_b, ks_b] = f[..., j]
    return out[:N]


def pack_fast(codes: np.ndarray) -> np.ndarray:
    """The same bytes as ``pack``, computed by reshaping instead of index
    grids (fast enough for full-size matrices).  Rows of a 16-row block
    split as (j & 1, g); k of a 128-k tile as (j >> 1, t, s, b)."""
    N, K = codes.shape
    assert K % 128 == 0
    Np = -(-N // 16) * 16
    c = np.ones((Np, K), np.uint32)
    c[:N] = codes.astype(np.int32) + 1
    # axes: rb, jlo, g, kt, jhi, t, s, b
    c = c.reshape(Np // 16, 2, 8, K // 128, 2, 4, 4, 4)
    shift = (8 * np.arange(4)[None, :] + 2 * np.arange(4)[:, None]).astype(np.uint32)  # [s, b]
    words = np.bitwise_or.reduce((c << shift).reshape(c.shape[:6] + (16,)), axis=-1)
    # word order inside a tile: lane l = 4g + t, then j = 2*jhi + jlo
    words = words.transpose(0, 3, 2, 5, 4, 1)   # rb, kt, g, t, jhi, jlo
    return np.ascontiguousarray(words).reshape(-1).view(np.uint8).copy()
