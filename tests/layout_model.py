"""NumPy model of the MATQ-PL1 plane layout, written from its description in include/matq.h
(test infrastructure: the pack kernel's bytes and the operand builder's lane words are both
checked against it)."""

import numpy as np

PLANE_BITS = [2, 1, 1, 2, 2]
PLANE_LSB = [6, 5, 4, 2, 0]
PLANES_FOR = {2: 1, 3: 2, 4: 3, 6: 4, 8: 5}


def _field_index():
    gid = np.arange(32) // 4
    tg = np.arange(32) % 4
    w = np.arange(8)
    f = np.arange(16)
    L, W, F = np.meshgrid(np.arange(32), w, f, indexing="ij")
    u = F & 7
    hi = F >> 3
    j = u >> 2
    rho = u & 3
    row = gid[L] + 8 * (rho & 1)
    k = 32 * W + 16 * j + 2 * tg[L] + 8 * (rho >> 1) + hi
    return row, k, W, F


def layout_model(q, r_keep):
    N, K = q.shape
    RT, KC = (N + 15) // 16, K // 256
    qp = np.zeros((RT * 16, K), dtype=np.int64)
    qp[:N] = q
    row, k, W, F = _field_index()            # [32, 8, 16]
    out = []
    for p in range(PLANES_FOR[r_keep]):
        b = PLANE_BITS[p]
        vals = (qp >> PLANE_LSB[p]) & ((1 << b) - 1)
        tiles = vals.reshape(RT, 16, KC, 256).transpose(0, 2, 1, 3)   # [RT, KC, 16, 256]
        v = tiles[:, :, row, k]                                     # [RT, KC, 32, 8, 16]
        if b == 2:
            words = (v << (2 * F)).sum(axis=-1).astype(np.uint32)   # [RT, KC, 32, 8]
            mem = words.reshape(RT, KC, 32, 2, 4).transpose(0, 1, 3, 2, 4)  # [.., half, lane, 4]
        else:
            a = W & 1
            pos = 4 * (F >> 1) + 2 * a + (F & 1)
            bits = (v << pos).sum(axis=-1)                          # [RT, KC, 32, 8] per block
            words = (bits[..., 0::2] + bits[..., 1::2]).astype(np.uint32)   # blocks 2v, 2v+1
            mem = words                                             # [RT, KC, lane, 4]
        out.append(np.ascontiguousarray(mem).view(np.uint8).reshape(-1))
    return np.concatenate(out)


def field_coords(gid, tg, w, f):
    """(row within the tile, input within the chunk) of field f of block w held by lane
    (gid, tg)."""
    u, hi = f & 7, f >> 3
    j, rho = u >> 2, u & 3
    return gid + 8 * (rho & 1), 32 * w + 16 * j + 2 * tg + 8 * (rho >> 1) + hi


def tile_lane_words(tile_bytes, lane):
    """p0[8], p1[4], p2[4], p3[8], p4[8] of one lane, read from the bytes of a one-tile pack
    (layout_model of a 16 x 256 code tile with r_keep = 8) at the documented offsets: planes back
    to back (1024, 512, 512, 1024, 1024 bytes); 2-bit planes as two 512-byte halves of 16 bytes a
    lane (words 0-3, then 4-7); 1-bit planes 16 bytes a lane."""
    b = np.asarray(tile_bytes, dtype=np.uint8)
    words = b.view(np.uint32)

    def at(byte_off, n):
        return words[byte_off // 4: byte_off // 4 + n]
    o = [0, 1024, 1536, 2048, 3072]
    p0 = np.concatenate([at(o[0] + 16 * lane, 4), at(o[0] + 512 + 16 * lane, 4)])
    p1 = at(o[1] + 16 * lane, 4)
    p2 = at(o[2] + 16 * lane, 4)
    p3 = np.concatenate([at(o[3] + 16 * lane, 4), at(o[3] + 512 + 16 * lane, 4)])
    p4 = np.concatenate([at(o[4] + 16 * lane, 4), at(o[4] + 512 + 16 * lane, 4)])
    return np.concatenate([p0, p1, p2, p3, p4]).astype(np.uint32)
