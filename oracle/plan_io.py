"""Plan file and pool layout, written from the format definition -- oracle side.

TEST INFRASTRUCTURE.  The product library parses the same byte format with
its own code; the two implementations share nothing but the definition
below (also stated in include/stepq.h).

Plan file, little-endian:
  0   8  magic b"STEPQPL1"
  8   4  u32 version (1)
  12  4  u32 mode: 0 = per-head units (GDN), 1 = per-key-row units (KDA)
  16  4  u32 n_layers        20  4  u32 n_heads
  24  4  u32 d_k             28  4  u32 d_v   (d_k == d_v)
  32  4  u32 n_units (mode 0: n_layers*n_heads, mode 1: that times d_k)
  36  4  u32 n_pivots        40  4  u32 bitset (bit b set: width b allowed)
  44  4  f32 nominal bits    48  8  u64 horizon H
  56  4  u32 quantizer: 0 = STEPQuant dual-axis fit, 1 = per-row absmax
         (mode 0 only; every record keeps the codes | r | c layout, c = 1)
  60  4  u32 scale storage: 0 = fp32 r and c, 16 = bfloat16 r and c
  64     u8  width[n_units]  (2, 4, 6, 8, or 16 for an FP16 pivot)
         zero padding to a multiple of 4 bytes
         f32 wbar[n_layers*n_heads*d_k]   row impact omega_i / mean omega
         f32 rho[n_layers*n_heads*d_k]    (wbar)^(-1/4)
         f64 lgate[n_units]               mean log retention gate l_u
         f64 lifetime[n_units]            L_u
  end-4  u32 CRC-32 (IEEE 802.3, as zlib.crc32) of every preceding byte

Pool layout: slot-major.  Slot s starts at s * slot_bytes; inside a slot the
records of the (layer, head) pairs follow in order layer-major.  Record of a
head:
  mode 0, pivot head : binary16 tile, row-major, D*D*2 bytes
  mode 0, width b    : codes (uniform layout, D*D*b/8 bytes) | r[D] | c[D]
  mode 1             : codes (row-major layout) | r[D] | c[D]
r and c are f32, or bf16 in plans with 16-bit scales;
each padded with zeros to a multiple of 128 bytes.
"""
from __future__ import annotations

import struct
import zlib

import numpy as np

MAGIC = b"STEPQPL1"
VERSION = 1
HEADER = struct.Struct("<8sIIIIIIIIIfQII")
PIVOT_BITS = 16


def _align(n: int, a: int) -> int:
    return (n + a - 1) // a * a


def write_plan(path: str, plan: dict) -> bytes:
    mode = int(plan["mode"])
    L, H, D = int(plan["n_layers"]), int(plan["n_heads"]), int(plan["d"])
    n_units = L * H if mode == 0 else L * H * D
    widths = np.asarray(plan["widths"], dtype=np.uint8)
    assert widths.size == n_units
    bitset = 0
    for b in plan["bitset"]:
        bitset |= 1 << int(b)
    head = HEADER.pack(MAGIC, VERSION, mode, L, H, D, D, n_units, int(plan["n_pivots"]),
                       bitset, float(plan["nominal_bits"]), int(plan["horizon"]),
                       int(plan.get("quantizer", 0)), 16 if int(plan.get("scale_bits", 32)) == 16 else 0)
    body = bytearray(head)
    body += widths.tobytes()
    body += b"\0" * (_align(len(body), 4) - len(body))
    body += np.asarray(plan["wbar"], dtype="<f4").reshape(-1).tobytes()
    body += np.asarray(plan["rho"], dtype="<f4").reshape(-1).tobytes()
    body += np.asarray(plan["lgate"], dtype="<f8").reshape(-1).tobytes()
    body += np.asarray(plan["lifetime"], dtype="<f8").reshape(-1).tobytes()
    body += struct.pack("<I", zlib.crc32(bytes(body)) & 0xFFFFFFFF)
    data = bytes(body)
    if path is not None:
        with open(path, "wb") as f:
            f.write(data)
    return data


def read_plan(data: bytes) -> dict:
    (magic, ver, mode, L, H, dk, dv, n_units, n_piv, bitset, nominal, horizon,
     quantizer, sbits) = HEADER.unpack_from(data, 0)
    assert magic == MAGIC and ver == VERSION
    off = HEADER.size
    widths = np.frombuffer(data, dtype=np.uint8, count=n_units, offset=off).copy()
    off = _align(off + n_units, 4)
    nrow = L * H * dk
    wbar = np.frombuffer(data, dtype="<f4", count=nrow, offset=off).copy(); off += 4 * nrow
    rho = np.frombuffer(data, dtype="<f4", count=nrow, offset=off).copy(); off += 4 * nrow
    lgate = np.frombuffer(data, dtype="<f8", count=n_units, offset=off).copy(); off += 8 * n_units
    life = np.frombuffer(data, dtype="<f8", count=n_units, offset=off).copy(); off += 8 * n_units
    crc = struct.unpack_from("<I", data, off)[0]
    assert crc == zlib.crc32(data[:off]) & 0xFFFFFFFF
    return dict(mode=mode, n_layers=L, n_heads=H, d=dk, n_pivots=n_piv,
                bitset=[b for b in range(32) if bitset >> b & 1], nominal_bits=nominal,
                horizon=horizon, widths=widths, wbar=wbar, rho=rho, lgate=lgate, lifetime=life,
                quantizer=quantizer, scale_bits=16 if sbits == 16 else 32)


# --------------------------------------------------------------------------
# pool layout
# --------------------------------------------------------------------------

def head_row_widths(plan: dict, layer: int, head: int) -> np.ndarray:
    D = plan["d"]
    hidx = layer * plan["n_heads"] + head
    if plan["mode"] == 0:
        return np.full(D, int(plan["widths"][hidx]), dtype=np.int32)
    return np.asarray(plan["widths"][hidx * D:(hidx + 1) * D], dtype=np.int32)


def record_bytes(mode: int, D: int, row_widths, scale_bits: int = 32) -> int:
    rw = np.asarray(row_widths)
    sb = 2 * D * (scale_bits // 8)  # r[D] and c[D]
    if mode == 0:
        b = int(rw[0])
        if b == PIVOT_BITS:
            return _align(D * D * 2, 128)
        return _align(D * D * b // 8 + sb, 128)
    return _align(codes_block_bytes(mode, D, rw) + sb, 128)


def codes_block_bytes(mode: int, D: int, row_widths) -> int:
    rw = np.asarray(row_widths)
    if mode == 0:
        b = int(rw[0])
        return D * D * 2 if b == PIVOT_BITS else D * D * b // 8
    # band-tile layout: per band of D/8 rows, D/4 tiles of ceil(4 * sum of the band's widths / 32) words
    RT = D // 8
    words = [-(-4 * int(sum(int(b) for b in rw[g * RT:(g + 1) * RT])) // 32) for g in range(8)]
    return 4 * (D // 4) * int(sum(words))


def pool_layout(plan: dict):
    """(record offsets within a slot [n_layers*n_heads], slot_bytes)."""
    offs = []
    o = 0
    for l in range(plan["n_layers"]):
        for h in range(plan["n_heads"]):
            offs.append(o)
            o += record_bytes(plan["mode"], plan["d"], head_row_widths(plan, l, h), int(plan.get("scale_bits", 32)))
    return np.array(offs, dtype=np.int64), o
