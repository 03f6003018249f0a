"""HFQM calibration packages ("hipfire-calib-data" dataset card, ".calib.hfq — HFQM calibration
package"): the container around the Bf16TrilDiagF32 Hessian codec.

Layout, all integers little-endian:

* header, 32 bytes: magic b"HFQM", version u32 (1), arch_id u32, n_entries u32,
  metadata_offset u64, data_offset u64;
* metadata at metadata_offset: one JSON value, self-delimited (it ends where the JSON ends);
* index right after the metadata: n_entries u32, then per entry name_len u16, name (UTF-8),
  quant_type u8, n_dims u8, shape (n_dims x u32), group_size u32, data_size u64;
* payloads from data_offset, concatenated in index order.

Each tensor contributes two entries, "<name>.hessian" (quant_type 130, Bf16TrilDiagF32, shape
[K, K]) and "<name>.imatrix".  Readings where the card is silent: the imatrix payload is K fp32
values with quant_type 0; group_size is 0 for both; the metadata follows the header directly and
the payloads follow the index without padding.

The Hessian payloads are produced and consumed by the library's codec kernels
(hq_hessian_pack_bf16tril / hq_hessian_unpack_bf16tril); this module only frames bytes.
"""

from __future__ import annotations

import dataclasses
import json
import struct

import torch

MAGIC = b"HFQM"
VERSION = 1
HEADER = struct.Struct("<4sIIIQQ")  # 32 bytes
QT_F32 = 0
QT_BF16_TRIL_DIAG_F32 = 130


@dataclasses.dataclass
class Entry:
    name: str
    quant_type: int
    shape: tuple
    group_size: int
    data_size: int
    offset: int = 0  # absolute file offset of the payload (filled in by the reader and writer)


def build_package(arch_id: int, metadata, entries: list, payloads: list) -> bytes:
    """The package bytes for `entries` (Entry, offset ignored) with their payload bytes."""
    if len(entries) != len(payloads):
        raise ValueError("one payload per entry")
    meta = json.dumps(metadata, separators=(",", ":")).encode("utf-8")
    index = bytearray(struct.pack("<I", len(entries)))
    for e, p in zip(entries, payloads):
        if e.data_size != len(p):
            raise ValueError(f"{e.name}: data_size {e.data_size} != payload {len(p)} bytes")
        name = e.name.encode("utf-8")
        index += struct.pack("<H", len(name)) + name
        index += struct.pack("<BB", e.quant_type, len(e.shape))
        index += struct.pack(f"<{len(e.shape)}I", *e.shape)
        index += struct.pack("<IQ", e.group_size, e.data_size)
    metadata_offset = HEADER.size
    data_offset = metadata_offset + len(meta) + len(index)
    head = HEADER.pack(MAGIC, VERSION, arch_id, len(entries), metadata_offset, data_offset)
    return head + meta + bytes(index) + b"".join(bytes(p) for p in payloads)


def parse_package(buf: bytes):
    """(arch_id, metadata, [Entry with offsets]) of package bytes; ValueError if malformed."""
    if len(buf) < HEADER.size:
        raise ValueError("shorter than the header")
    magic, version, arch_id, n, meta_off, data_off = HEADER.unpack_from(buf, 0)
    if magic != MAGIC or version != VERSION:
        raise ValueError("not an HFQM version 1 package")
    dec = json.JSONDecoder()
    # the JSON value's end, found on a byte-preserving (latin-1) view, then decoded as UTF-8
    _, end = dec.raw_decode(buf[meta_off:data_off].decode("latin-1"))
    metadata = json.loads(buf[meta_off:meta_off + end].decode("utf-8"))
    pos = meta_off + end
    (n_index,) = struct.unpack_from("<I", buf, pos)
    pos += 4
    if n_index != n:
        raise ValueError("index count differs from the header")
    entries = []
    off = data_off
    for _ in range(n):
        (ln,) = struct.unpack_from("<H", buf, pos)
        pos += 2
        name = buf[pos:pos + ln].decode("utf-8")
        pos += ln
        qt, nd = struct.unpack_from("<BB", buf, pos)
        pos += 2
        shape = struct.unpack_from(f"<{nd}I", buf, pos)
        pos += 4 * nd
        gs, size = struct.unpack_from("<IQ", buf, pos)
        pos += 12
        entries.append(Entry(name, qt, tuple(shape), gs, size, off))
        off += size
    if pos != data_off:
        raise ValueError("index does not end at data_offset")
    if off > len(buf):
        raise ValueError("payloads run past the end")
    return arch_id, metadata, entries


def write_package(hq, path: str, arch_id: int, metadata, tensors) -> None:
    """tensors: (name, H fp32 [K, K] device (lower triangle and diagonal read), imatrix fp32 [K]).
    Encodes each Hessian with the library's codec and writes the package."""
    entries, payloads = [], []
    for name, H, imp in tensors:
        K = H.shape[0]
        tril = torch.empty(hq.hq_bf16tril_bytes(K), dtype=torch.uint8, device=H.device)
        hq.hq_hessian_pack_bf16tril(H, tril)
        p = tril.cpu().numpy().tobytes()
        entries.append(Entry(f"{name}.hessian", QT_BF16_TRIL_DIAG_F32, (K, K), 0, len(p)))
        payloads.append(p)
        q = imp.detach().to(torch.float32).cpu().numpy().astype("<f4").tobytes()
        entries.append(Entry(f"{name}.imatrix", QT_F32, (K,), 0, len(q)))
        payloads.append(q)
    with open(path, "wb") as f:
        f.write(build_package(arch_id, metadata, entries, payloads))


def read_package(path: str):
    """(arch_id, metadata, entries, bytes) of a package file."""
    with open(path, "rb") as f:
        buf = f.read()
    arch_id, metadata, entries = parse_package(buf)
    return arch_id, metadata, entries, buf


def load_hessian(hq, buf: bytes, entry: Entry, device="cuda", project: bool = False, steps: int = 40):
    """fp32 [K, K] symmetric Hessian of a quant_type 130 entry, decoded on the GPU (and projected
    onto the PSD cone when `project`, as the card requires before a Cholesky)."""
    if entry.quant_type != QT_BF16_TRIL_DIAG_F32 or len(entry.shape) != 2:
        raise ValueError(f"{entry.name} is not a Bf16TrilDiagF32 Hessian")
    K = entry.shape[0]
    if entry.data_size != hq.hq_bf16tril_bytes(K):
        raise ValueError(f"{entry.name}: {entry.data_size} bytes, K = {K} needs {hq.hq_bf16tril_bytes(K)}")
    payload = torch.frombuffer(bytearray(buf[entry.offset:entry.offset + entry.data_size]), dtype=torch.uint8)
    from . import stored_hessian
    return stored_hessian.load_stored_hessian(hq, payload.to(device), K, project=project, steps=steps)


def load_imatrix(buf: bytes, entry: Entry, device="cuda"):
    if entry.quant_type != QT_F32 or len(entry.shape) != 1 or entry.data_size != 4 * entry.shape[0]:
        raise ValueError(f"{entry.name} is not an fp32 vector")
    return torch.frombuffer(bytearray(buf[entry.offset:entry.offset + entry.data_size]), dtype=torch.float32).to(device)
