"""The library's .tbin record-table parser (host code, no GPU) against the
plain oracle reader, on the hand-written golden files and on files the oracle
writer makes; malformed files are rejected."""
import numpy as np
import pytest

from oracle import tbin
from test_oracle_ternary import golden_tbin_files


@pytest.fixture(scope="module")
def bnn():
    from ternary_neural_net_b200 import bnn as mod
    return mod


def _same(bnn, data):
    ver, meta, recs = bnn.bnn_tbin_parse(data)
    over, ometa, orecs = tbin.read(data)
    assert (ver, meta, len(recs)) == (over, ometa, len(orecs))
    raw = np.frombuffer(data, np.uint8)
    for r, o in zip(recs, orecs):
        assert bnn.tbin_record_name(data, r) == o["name"]
        if o["kind"] == "ternary":
            assert r.kind == 0 and (r.out_features, r.in_features) == (o["out_feat"], o["in_feat"])
            assert np.float32(r.delta) == np.float32(o["delta"]) and np.float32(r.sparsity) == np.float32(o["sparsity"])
            sc = raw[r.scales_offset:r.scales_offset + 2 * r.out_features].view("<f2")
            assert np.array_equal(sc.view(np.uint16), o["scales"].view(np.uint16))
            assert r.num_biases == (0 if o["biases"] is None else r.out_features)
            if r.num_biases:
                bi = raw[r.biases_offset:r.biases_offset + 2 * r.num_biases].view("<f2")
                assert np.array_equal(bi.view(np.uint16), o["biases"].view(np.uint16))
            w = raw[r.weights_offset:r.weights_offset + 2 * r.weights_words].view("<u2")
            assert np.array_equal(w, o["words"])
        else:
            assert r.kind == 1 and [r.dims[d] for d in range(r.ndims)] == o["dims"]
            d = raw[r.data_offset:r.data_offset + 2 * r.data_elems].view("<f2")
            assert np.array_equal(d.view(np.uint16), o["data"].view(np.uint16))


def test_golden_files(bnn):
    for data in golden_tbin_files().values():
        _same(bnn, data)


def _random_file(seed, version=2):
    rng = np.random.default_rng(seed)
    layers = []
    for i in range(int(rng.integers(1, 5))):
        if version == 2 and rng.random() < 0.3:
            dims = [int(d) for d in rng.integers(1, 6, int(rng.integers(0, 4)))]
            layers.append(dict(kind="raw", name=f"raw{i}" * int(rng.integers(0, 3)), dims=dims,
                               data=rng.standard_normal(int(np.prod(dims)) if dims else 1).astype(np.float16)))
        else:
            o, k = int(rng.integers(1, 40)), int(rng.integers(1, 90))
            t = rng.integers(-1, 2, (o, k)).astype(np.int8)
            import oracle
            layers.append(dict(kind="ternary", name="layer.%d.weight" % i, out_feat=o, in_feat=k,
                               delta=float(rng.random()), sparsity=float((t == 0).mean()),
                               scales=rng.random(o).astype(np.float16),
                               biases=rng.standard_normal(o).astype(np.float16) if rng.random() < 0.5 else None,
                               words=oracle.base3_pack(t).reshape(-1)))
    return tbin.write(layers, metadata=b'{"arch":"generic"}' if seed % 2 else b"", version=version)


@pytest.mark.parametrize("seed", range(8))
def test_random_files(bnn, seed):
    _same(bnn, _random_file(seed, version=2 if seed % 3 else 1))


def test_malformed_files_are_rejected(bnn):
    good = golden_tbin_files()["v2"]
    bad = [b"XBN\0" + good[4:], good[:-1], good[:15], good[:4] + b"\x03" + good[5:],   # magic, truncation, version
           good[:21] + b"\x19" + good[22:]]                                            # record size one too big
    for data in bad:
        with pytest.raises(bnn.BnnError):
            bnn.bnn_tbin_parse(data)


def test_raw_record_dims_must_match_its_data(bnn):
    """A raw record's dims must multiply to its float16 count: a product larger
    than the file (whatever its wrap-around modulo 2^64) or different from the
    payload is rejected; a matching one parses."""
    import struct

    def raw_file(dims, n_data):
        name = b"t"
        p = struct.pack("<H", len(name)) + name + struct.pack("<B", len(dims))
        p += struct.pack("<%dI" % len(dims), *dims) + b"\0\0" * n_data
        return b"TBN\0" + struct.pack("<III", 2, 1, 0) + struct.pack("<BI", 1, len(p)) + p

    _, _, (rec,) = bnn.bnn_tbin_parse(raw_file([3, 5], 15))
    assert rec.data_elems == 15 and rec.ndims == 2
    for dims, n in (([3, 5], 14), ([65536, 65536, 65536, 65536], 0), ([0xFFFFFFFF, 2], 2), ([2 ** 31, 2], 0)):
        with pytest.raises(bnn.BnnError):
            bnn.bnn_tbin_parse(raw_file(dims, n))


def test_loaders_reject_forged_records(bnn):
    """bnn_tbin_load_ternary / bnn_tbin_load_raw take a record from the caller,
    so they must not trust it: counts whose doubled byte length wraps modulo
    2^64, a word count that is not out_features x ceil(in_features / 10) and
    ranges past the end of the file are rejected on the host, before any CUDA
    call (the file pointer here is a fake, never dereferenced)."""
    import ctypes as C
    lib = bnn.lib()
    fake = C.c_void_p(0x10000)
    length = 4096

    def ternary(**kw):
        r = bnn.TbinRecord()
        r.kind, r.out_features, r.in_features = 0, 4, 20
        r.scales_offset, r.weights_offset, r.weights_words = 16, 64, 8
        for k, v in kw.items():
            setattr(r, k, v)
        return lib.bnn_tbin_load_ternary(fake, length, C.byref(r), fake, fake, fake, None)

    two63 = 1 << 63
    for kw in (dict(weights_words=two63), dict(weights_words=two63 + 8), dict(weights_words=9),
               dict(out_features=0x80000000, in_features=10, weights_words=0x80000000),
               dict(weights_offset=length - 8), dict(scales_offset=length - 4), dict(weights_offset=two63),
               dict(num_biases=4, biases_offset=length - 6), dict(num_biases=3, biases_offset=32)):
        assert ternary(**kw) == bnn.BNN_ERR_INVALID_ARG, kw

    def raw(elems, off=16):
        r = bnn.TbinRecord()
        r.kind, r.data_offset, r.data_elems = 1, off, elems
        return lib.bnn_tbin_load_raw(fake, length, C.byref(r), fake, None)

    for elems, off in ((two63, 16), (two63 + 4, 16), ((1 << 64) - 1, 16), (2041, 16), (1, length)):
        assert raw(elems, off) == bnn.BNN_ERR_INVALID_ARG, (elems, off)
