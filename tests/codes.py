"""Decoder of the packed INT4 code layout, written from its definition:
a code v in [-7, 7] is a sign-magnitude nibble (bit 3 = sign, bits 0-2 = |v|);
every 8 consecutive elements e0..e7 of the packed axis form one 32-bit
little-endian word whose byte j (0..3) holds e_j (low nibble) and e_{j+4}
(high nibble)."""
import numpy as np


def unpack(packed: np.ndarray) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    b = packed.reshape(*packed.shape[:-1], -1, 4).astype(np.int16)
    nib = np.concatenate([b & 0xF, b >> 4], axis=-1)          # e0..e3, e4..e7
    val = np.where(nib & 8, -(nib & 7), nib & 7)
    return val.reshape(*packed.shape[:-1], packed.shape[-1] * 2).astype(np.int8)
