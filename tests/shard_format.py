"""Independent reader / writer of the shard checkpoint format documented in
include/zr.h (256-byte header, then master, m, v in owned order)."""
import struct

import numpy as np

MAGIC = b"ZRSHARD1"
FNV_OFFSET = 0xcbf29ce484222325
FNV_PRIME = 0x100000001b3
M64 = (1 << 64) - 1
HEADER = struct.Struct("<8sIiiiqqqQQq6fQ")     # 104 bytes, zero padded to 256


def fnv_words(data: bytes, h: int = FNV_OFFSET) -> int:
    """64-bit FNV-1a over little-endian 64-bit words (trailing bytes
    zero-padded to a word)."""
    if len(data) % 8:
        data = data + b"\0" * (8 - len(data) % 8)
    words = np.frombuffer(data, dtype="<u8")
    for w in words.tolist():
        h = ((h ^ w) * FNV_PRIME) & M64
    return h


def shapes_hash(numels) -> int:
    h = fnv_words(struct.pack("<q", len(numels)))
    for n in numels:
        h = fnv_words(struct.pack("<q", int(n)), h)
    return h


def partition_hash(numels, world_size, mode) -> int:
    return fnv_words(struct.pack("<qq", world_size, mode), shapes_hash(numels))


def write_shard(path, numels, world_size, rank, mode, total, padded, master, m, v, step, hp):
    payload = (np.ascontiguousarray(master, np.float32).tobytes() +
               np.ascontiguousarray(m, np.float32).tobytes() +
               np.ascontiguousarray(v, np.float32).tobytes())
    head = HEADER.pack(MAGIC, 1, world_size, rank, mode, total, padded, len(master),
                       shapes_hash(numels), partition_hash(numels, world_size, mode), step,
                       *[float(x) for x in hp], fnv_words(payload))
    with open(path, "wb") as f:
        f.write(head + b"\0" * (256 - len(head)) + payload)


def read_shard(path):
    with open(path, "rb") as f:
        raw = f.read()
    fields = HEADER.unpack(raw[:HEADER.size])
    (magic, version, W, rank, mode, total, padded, owned, sh, ph, step, *rest) = fields
    hp, checksum = rest[:6], rest[6]
    assert magic == MAGIC and version == 1
    payload = raw[256:]
    assert len(payload) == 12 * owned
    assert fnv_words(payload) == checksum
    arr = np.frombuffer(payload, dtype="<f4")
    return {"world_size": W, "rank": rank, "mode": mode, "total": total, "padded": padded,
            "owned": owned, "shapes_hash": sh, "partition_hash": ph, "step": step, "hp": hp,
            "master": arr[:owned].copy(), "m": arr[owned:2 * owned].copy(),
            "v": arr[2 * owned:].copy()}
