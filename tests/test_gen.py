"""Pins of the seeded input generator (gen/): the Philox known-answer
vectors, the sample statistics, determinism, the checkpoint encoder and the
workload recipes."""
import json
import os

import numpy as np
import torch

import gen
from oracle import moe

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_philox_known_answers():
    # known-answer vectors published with Random123 (philox4x32, 10 rounds)
    assert list(gen.philox4x32_10([0, 0, 0, 0], [0, 0])) == [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]
    assert list(gen.philox4x32_10([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2)) == \
        [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]
    assert list(gen.philox4x32_10([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344],
                                  [0xA4093822, 0x299F31D0])) == [0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]


def test_normal_moments_and_determinism():
    z = gen.normal_f32(7, 1, 2_000_000)
    assert abs(z.mean()) < 5 / np.sqrt(2e6) and abs(z.std() - 1) < 5e-3
    assert abs(((z ** 4).mean()) - 3) < 0.05
    assert np.array_equal(z, gen.normal_f32(7, 1, 2_000_000, nthreads=1))
    assert np.array_equal(z[:1000], gen.normal_f32(7, 1, 1000))
    assert not np.array_equal(z[:1000], gen.normal_f32(7, 2, 1000))


def test_generator_encoder_matches_torch():
    rng = np.random.default_rng(0)
    v = (rng.standard_normal(500_000) * np.exp(rng.uniform(-14, 7, 500_000))).astype(np.float32)
    ref = torch.from_numpy(np.clip(v, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(gen.e4m3_encode_gen(v), ref)


def test_fp8_blocks_checkpoint():
    rows, cols, ld, sigma = 300, 200, 208, 0.05
    codes, scales = gen.fp8_blocks(3, 9, 2, rows, cols, ld, sigma)
    w = gen.normal_f32(3, 9, 2 * rows * cols, sigma).reshape(2, rows, cols)
    assert scales.shape == (2, 3, 2) and not codes[:, :, cols:].any()
    for m in range(2):
        for rb in range(3):
            for cb in range(2):
                blk = w[m, rb * 128:(rb + 1) * 128, cb * 128:(cb + 1) * 128]
                assert scales[m, rb, cb] == np.float32(np.abs(blk).max() / np.float32(448))
        d = moe.dequant_block(codes[m], scales[m], rows, cols)
        s = np.repeat(np.repeat(scales[m], 128, 0), 128, 1)[:rows, :cols]
        assert np.all(np.abs(d - w[m]) <= np.abs(w[m]) * 2 ** -4 + s * 2 ** -10 * 1.0001)


def test_workload_recipes():
    wl, layer, x = gen.workload_inputs("toy")
    assert x.shape == (32, 512) and layer.w_gate.shape == (17, 256, 512) and layer.s_down.shape == (17, 4, 2)
    assert layer.router_w.dtype == np.float32 and abs(layer.router_w.std() - 0.02) < 1e-3
    xs = gen.make_x(16, 5120, 1, outliers=8)
    ch = gen.outlier_channels(1, 5120, 8)
    assert len(set(ch.tolist())) == 8 and 0 not in ch
    xf = gen.bf16_bits_to_f32(xs)
    assert xf[:, ch].std() > 10 and xf[:, np.setdiff1d(np.arange(5120), ch)].std() < 1.1


def test_zipf_alpha_matches_golden_and_skew():
    g = json.load(open(os.path.join(GOLDEN, "zipf_alpha.json")))
    assert gen.ZIPF_ALPHA == g["alpha"]
    assert 9.0 <= g["max_over_mean"] <= 11.0 and g["empty_experts"] >= gen.ZIPF_EMPTY
    b = gen.zipf_bias(1, 256)
    assert (b == np.float32(gen.ZIPF_OFF)).sum() == gen.ZIPF_EMPTY
    finite = np.sort(b[b > gen.ZIPF_OFF])[::-1]
    assert finite[0] == 0.0 and np.allclose(finite, -gen.ZIPF_ALPHA * gen.ZIPF_S * np.log(np.arange(1, 241)), atol=1e-5)
