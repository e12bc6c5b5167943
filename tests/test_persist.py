"""Persistence of a quantised layer (CB, SCB, bias) as one byte image."""

from __future__ import annotations

import struct

import numpy as np
import pytest
import torch

from oracle import llm_int8 as O
from int8_mixed_precision_column_b200 import build, native, workloads


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    native.lib()


def _layer(N=48, K=80, seed=0):
    g = torch.Generator().manual_seed(seed)
    CB = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8)
    SCB = torch.rand(N, generator=g) * 0.1
    bias = (torch.randn(N, generator=g) * 0.01).half()
    return CB, SCB, bias


@pytest.mark.parametrize("with_bias", [True, False])
def test_round_trip(with_bias):
    CB, SCB, bias = _layer()
    img = native.int8_layer_pack(CB, SCB, bias if with_bias else None)
    cb2, scb2, b2 = native.int8_layer_unpack(img, device="cpu")
    assert torch.equal(cb2, CB) and torch.equal(scb2, SCB)
    assert (b2 is None) == (not with_bias)
    if with_bias:
        assert torch.equal(b2, bias)


def test_byte_layout_is_the_documented_one():
    CB, SCB, bias = _layer(N=16, K=32, seed=1)
    img = native.int8_layer_pack(CB, SCB, bias)
    assert img[:8] == b"I8MPLYR1"
    assert struct.unpack_from("<qqII", img, 8) == (16, 32, 1, 0)
    assert np.array_equal(np.frombuffer(img, np.float32, 16, 32), SCB.numpy())
    assert np.array_equal(np.frombuffer(img, np.float16, 16, 32 + 64), bias.numpy())
    assert np.array_equal(np.frombuffer(img, np.int8, 16 * 32, 32 + 64 + 32).reshape(16, 32), CB.numpy())
    assert len(img) == native.lib().int8_layer_packed_bytes(16, 32, 1) == 32 + 64 + 32 + 512


def test_bf16_bias_round_trip_and_flag():
    CB, SCB, bias = _layer(N=32, K=48, seed=2)
    b16 = bias.float().mul(3.0).to(torch.bfloat16)
    img = native.int8_layer_pack(CB, SCB, b16)
    assert struct.unpack_from("<qqII", img, 8) == (32, 48, 3, 0)     # bias present, bf16
    cb2, scb2, b2 = native.int8_layer_unpack(img, device="cpu")
    assert b2.dtype == torch.bfloat16 and torch.equal(b2, b16)
    assert torch.equal(cb2, CB) and torch.equal(scb2, SCB)
    # the fp16 image of the same layer records no bf16 flag
    assert struct.unpack_from("<I", native.int8_layer_pack(CB, SCB, bias), 24) == (1,)
    for flags in (4, 2 | 4, 8):
        with pytest.raises(native.Int8mpError):
            native.int8_layer_unpack(img[:24] + struct.pack("<I", flags) + img[28:], device="cpu")


def test_malformed_images_are_rejected():
    CB, SCB, bias = _layer()
    img = native.int8_layer_pack(CB, SCB, bias)
    bad = [b"X" + img[1:], img[:-1], img[:20],
           img[:8] + struct.pack("<q", 15) + img[16:],          # N not a multiple of 16
           img[:24] + struct.pack("<I", 2) + img[28:]]           # unknown flag
    for b in bad:
        with pytest.raises(native.Int8mpError):
            native.int8_layer_unpack(b, device="cpu")
    assert native.lib().int8_layer_packed_bytes(15, 32, 0) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("path", [native.PATH_AUTO, native.PATH_DECODE])
def test_loaded_layer_matches_the_oracle(tmp_path, path):
    """A layer saved and loaded back: its CB/SCB equal the oracle's quantisation
    of the fp16 weight bit for bit, and its forward matches the oracle's Y at
    the fp16 tolerance (and the forward of the layer before saving bit for bit)."""
    assert torch.cuda.is_available()
    T = 64 if path == native.PATH_AUTO else 16
    p = workloads.make_problem("persist", T, 1024, 512, n_planted=5, bias_std=0.01, seed=3)
    CB, SCB = native.int8_quantize_weight(p.W.cuda())
    bias = p.bias.cuda()
    f = tmp_path / "layer.i8mp"
    native.save_quantized(str(f), CB, SCB, bias)
    del CB, SCB
    CB2, SCB2, b2 = native.load_quantized(str(f), device="cuda")
    CBo, SCBo = O.quantize_weight(p.W.numpy())
    assert np.array_equal(CB2.cpu().numpy(), CBo) and np.array_equal(SCB2.cpu().numpy(), SCBo)
    assert torch.equal(b2.cpu(), p.bias)
    Y2, idx2, n2, ws = native.int8_linear_forward(p.X.cuda(), CB2, SCB2, b2, 6.0, path=path)
    assert native.int8_check_status(ws)[0] == 0
    r = O.linear_forward(p.X.numpy(), CBo, SCBo, p.bias.numpy(), 6.0)
    n = int(n2.item())
    assert n == r["n_out"] and np.array_equal(idx2[:n].cpu().numpy(), r["idx"])
    err = np.abs(Y2.cpu().numpy().astype(np.float64) - r["Y"]).max()
    assert err <= O.y_tolerance(r["Y"]), err
    Y1, _, _, _ = native.int8_linear_forward(p.X.cuda(), torch.from_numpy(CBo).cuda(), torch.from_numpy(SCBo).cuda(),
                                             bias, 6.0, path=path)
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
