"""Plain Python reader and writer of the .tbin ternary model file -- TEST
INFRASTRUCTURE ONLY: used by the tests to make files and to check the
library's reader, never by the product path.

Layout ("BalancedTernaryEngine" README, ".tbin Format", version 2), every
field little-endian:
  header: magic b"TBN\\0", version u32, num_layers u32, meta_len u32, then
          meta_len bytes of JSON metadata;
  record: kind u8 (0 ternary, 1 raw float16; absent in version 1, where every
          record is ternary), size u32 = payload bytes, payload;
  ternary payload: name_len u16, name, out_feat u32, in_feat u32, delta f32,
          sparsity f32, out_feat float16 scales, 0 or out_feat float16 biases,
          out_feat x ceil(in_feat/10) uint16 base-3 words;
  raw payload: name_len u16, name, ndims u8, ndims x u32 dims, float16 data.
The number of scales (one per output channel) and of biases (0 or one per
channel, whichever the record size leaves room for) are readings: the page
lists the fields without their counts.
"""
import struct

import numpy as np


def write(layers, metadata=b"{}", version=2):
    """layers: dicts with kind 'ternary' (name, out_feat, in_feat, delta, sparsity,
    scales, biases or None, words) or 'raw' (name, dims, data float16)."""
    out = bytearray(b"TBN\0")
    out += struct.pack("<III", version, len(layers), len(metadata)) + metadata
    for L in layers:
        name = L["name"].encode()
        if L["kind"] == "ternary":
            p = struct.pack("<H", len(name)) + name
            p += struct.pack("<IIff", L["out_feat"], L["in_feat"], L["delta"], L["sparsity"])
            p += np.asarray(L["scales"], "<f2").tobytes()
            if L.get("biases") is not None:
                p += np.asarray(L["biases"], "<f2").tobytes()
            p += np.asarray(L["words"], "<u2").tobytes()
            kind = 0
        else:
            assert version == 2
            p = struct.pack("<H", len(name)) + name + struct.pack("<B", len(L["dims"]))
            p += struct.pack("<%dI" % len(L["dims"]), *L["dims"]) + np.asarray(L["data"], "<f2").tobytes()
            kind = 1
        if version == 2:
            out += struct.pack("<B", kind)
        out += struct.pack("<I", len(p)) + p
    return bytes(out)


def read(buf):
    """-> (version, metadata bytes, records); each record a dict with the fields
    above, arrays as numpy (scales/biases float16, words uint16)."""
    if len(buf) < 16 or buf[:4] != b"TBN\0":
        raise ValueError("not a .tbin file")
    version, num, meta_len = struct.unpack_from("<III", buf, 4)
    if version not in (1, 2):
        raise ValueError("unknown version")
    at = 16
    meta = bytes(buf[at:at + meta_len])
    if len(meta) != meta_len:
        raise ValueError("truncated metadata")
    at += meta_len
    recs = []
    for _ in range(num):
        kind = 0
        if version == 2:
            kind = buf[at]
            at += 1
        (size,) = struct.unpack_from("<I", buf, at)
        at += 4
        end = at + size
        if end > len(buf):
            raise ValueError("truncated record")
        (nl,) = struct.unpack_from("<H", buf, at)
        name = bytes(buf[at + 2:at + 2 + nl]).decode()
        q = at + 2 + nl
        if kind == 0:
            out_f, in_f, delta, sparsity = struct.unpack_from("<IIff", buf, q)
            q += 16
            words = out_f * ((in_f + 9) // 10)
            left = end - q - 2 * out_f - 2 * words
            if left not in (0, 2 * out_f):
                raise ValueError("ternary record size does not fit its fields")
            scales = np.frombuffer(buf, "<f2", out_f, q)
            q += 2 * out_f
            biases = None
            if left:
                biases = np.frombuffer(buf, "<f2", out_f, q)
                q += 2 * out_f
            w = np.frombuffer(buf, "<u2", words, q)
            recs.append(dict(kind="ternary", name=name, out_feat=out_f, in_feat=in_f, delta=delta,
                             sparsity=sparsity, scales=scales, biases=biases, words=w))
        elif kind == 1:
            (nd,) = struct.unpack_from("<B", buf, q)
            dims = list(struct.unpack_from("<%dI" % nd, buf, q + 1))
            q += 1 + 4 * nd
            count = int(np.prod(dims)) if nd else 1
            if end - q != 2 * count:
                raise ValueError("raw record size does not fit its dims")
            recs.append(dict(kind="raw", name=name, dims=dims, data=np.frombuffer(buf, "<f2", count, q)))
        else:
            raise ValueError("unknown record kind")
        at = end
    return version, meta, recs
