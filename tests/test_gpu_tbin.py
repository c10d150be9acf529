"""GPU loader of .tbin records: the file's bytes are copied to the device once,
each ternary record is extracted into base-3 words and float32 scales/biases
(bit-exact against the oracle reader's float16 -> float32), and the loaded
layer runs through bnn_ternary_linear against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_bits_equal, assert_ternary_close, host_u16, to_dev_bf16
from oracle import tbin
from test_tbin import _random_file
from ternary_neural_net_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bnn(cuda_device):
    from ternary_neural_net_b200 import bnn as mod
    return mod


@pytest.mark.parametrize("seed", range(6))
def test_load_matches_oracle(bnn, seed):
    data = _random_file(seed, version=2 if seed % 3 else 1)
    _, _, recs = bnn.bnn_tbin_parse(data)
    _, _, orecs = tbin.read(data)
    dev = torch.from_numpy(np.frombuffer(data, np.uint8).copy()).cuda()
    for r, o in zip(recs, orecs):
        if r.kind == 0:
            packed, scale, bias = bnn.bnn_tbin_load_ternary(dev, r)
            kt = (o["in_feat"] + 9) // 10
            assert_bits_equal(host_u16(packed), o["words"].reshape(o["out_feat"], kt), "words")
            assert_bits_equal(scale.cpu().numpy(), o["scales"].astype(np.float32), "scales")
            if o["biases"] is None:
                assert bias is None
            else:
                assert_bits_equal(bias.cpu().numpy(), o["biases"].astype(np.float32), "biases")
        else:
            got = bnn.bnn_tbin_load_raw(dev, r)
            assert_bits_equal(got.cpu().numpy().reshape(-1), o["data"].astype(np.float32), "raw data")


def test_loaded_layer_runs(bnn):
    """A 300 x 4096 TWN layer with biases written to .tbin, loaded on the device
    and run at m = 1 and m = 64."""
    n, k = 300, 4096
    w = synth.normal_f32(5, 1, (n, k))
    trits, scale, delta = oracle.twn_ternarize(w)
    scales16 = scale.astype(np.float16)
    biases16 = synth.normal_f32(5, 2, (n,)).astype(np.float16)
    words = oracle.base3_pack(trits)
    data = tbin.write([dict(kind="ternary", name="ffn.up", out_feat=n, in_feat=k, delta=float(delta),
                            sparsity=float((trits == 0).mean()), scales=scales16, biases=biases16,
                            words=words.reshape(-1))])
    _, _, (rec,) = bnn.bnn_tbin_parse(data)
    dev = torch.from_numpy(np.frombuffer(data, np.uint8).copy()).cuda()
    packed, sc, bi = bnn.bnn_tbin_load_ternary(dev, rec)
    torch.cuda.synchronize()  # weights are complete before a matmul reads them
    for m in (1, 64):
        xb = synth.bf16_bits_from_f32(synth.normal_f32(5 + m, 3, (m, k)))
        got = bnn.bnn_ternary_linear(to_dev_bf16(xb), packed, sc, bi)
        want, mag = oracle.ternary_linear(xb, words, scales16.astype(np.float32), biases16.astype(np.float32), m, n, k)
        assert_ternary_close(got.cpu().numpy(), want, mag, f"loaded layer m={m}")
