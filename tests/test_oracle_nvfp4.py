"""The oracle's NVFP4 weight format (oracle/nvfp4.py), pinned on the CPU, with
mistakes planted in copies of it that the pins must catch:

- E4M3 block scales against torch's float8_e4m3fn conversion, over all 256
  codes and at every rounding tie;
- E2M1 elements against the OCP MX table (tests/golden/e2m1_values.json), and
  their rounding against a brute-force nearest search over that table;
- storage (nibble order, block layout) on hand-made cases;
- the quantiser by exact round trips and its error bound."""
import importlib.util
import json
import os

import numpy as np
import pytest
import torch

from oracle import nvfp4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e2m1_values.json")


def _torch_e4m3(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn)


def pin_e4m3_decode_matches_torch_for_every_code(m):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = m.e4m3_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert got[0x7E] == 448.0 and got[1] == 2.0 ** -9


def pin_e4m3_encode_matches_torch_rounding_including_ties(m):
    codes = np.arange(0, 0x7F, dtype=np.uint8)          # every finite non-negative code
    vals = m.e4m3_decode(codes)
    mids = (vals[:-1] + vals[1:]) / 2                   # the ties
    rng = np.random.default_rng(5)
    rand = rng.uniform(0, 448, 4000) * rng.choice([1.0, 2.0 ** -8, 2.0 ** -14], 4000)
    # fp32 values, so that torch's conversion (from fp32) rounds the same numbers
    x = np.concatenate([vals, mids, rand.astype(np.float32).astype(np.float64)])
    ref = _torch_e4m3(x).view(torch.uint8).numpy()
    # fp32 holds every tie exactly, so torch sees the same values
    assert np.array_equal(x.astype(np.float32).astype(np.float64), x)
    assert np.array_equal(m.e4m3_encode(x), ref)


def pin_e4m3_encode_saturates_above_448(m):
    assert m.e4m3_encode(np.array([448.0, 460.0, 1e6])).tolist() == [0x7E] * 3
    with pytest.raises(ValueError):
        m.e4m3_encode(np.array([-1.0]))


def pin_e2m1_decode_matches_the_ocp_table(m):
    with open(GOLDEN) as f:
        table = np.array(json.load(f)["values"])
    got = m.e2m1_decode(np.arange(16))
    assert np.array_equal(got, table)
    assert np.array_equal(np.signbit(got), np.signbit(table))


def _nearest_even(x, table):
    """Brute force: the code of the nearest value, ties to the even code."""
    out = []
    for v in x:
        a = min(abs(v), 6.0)
        d = np.abs(table[:8] - a)
        best = np.flatnonzero(d == d.min())
        c = int(best[0]) if len(best) == 1 else int(best[best % 2 == 0][0])
        out.append(c | (8 if v < 0 and c != 0 else 0))
    return np.array(out, dtype=np.uint8)


def pin_e2m1_encode_is_round_to_nearest_even_with_saturation(m):
    with open(GOLDEN) as f:
        table = np.array(json.load(f)["values"])
    pos = table[:8]
    mids = (pos[:-1] + pos[1:]) / 2
    rng = np.random.default_rng(6)
    x = np.concatenate([pos, -pos, mids, -mids, [6.5, 7.0, 100.0, -9.0],
                        rng.uniform(-7, 7, 5000)])
    assert np.array_equal(m.e2m1_encode(x), _nearest_even(x, table))
    # the ties, spelled out: 0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2,
    # 2.5 -> 2, 3.5 -> 4, 5 -> 4
    ties = m.e2m1_decode(m.e2m1_encode(np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])))
    assert ties.tolist() == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]


def pin_storage_nibble_order_and_block_layout(m):
    # row 0: elements 0..31 in two blocks; element 2i in the low nibble
    codes = np.zeros((1, 32), dtype=np.uint8)
    codes[0, 0] = 2      # 1.0
    codes[0, 1] = 9      # -0.5
    codes[0, 17] = 7     # 6.0, second block
    packed = m.pack_nibbles(codes)
    assert packed.shape == (1, 16) and packed[0, 0] == 0x92 and packed[0, 8] == 0x70
    assert np.array_equal(m.unpack_nibbles(packed), codes)
    scales = np.array([[0x40, 0x28]], dtype=np.uint8)   # E4M3 2.0 and 0.25
    assert m.e4m3_decode(scales).tolist() == [[2.0, 0.25]]
    w = m.nvfp4_dequantize(packed, scales, 0.5)
    expect = np.zeros((1, 32))
    expect[0, 0] = 0.5 * 2.0 * 1.0
    expect[0, 1] = 0.5 * 2.0 * -0.5
    expect[0, 17] = 0.5 * 0.25 * 6.0
    assert np.array_equal(w, expect)


def pin_quantize_round_trips_representable_blocks(m):
    rng = np.random.default_rng(7)
    rows, cols = 8, 64
    codes = rng.integers(0, 16, (rows, cols)).astype(np.uint8)
    codes[:, ::16] = 7                                    # every block reaches 6
    scales = rng.integers(0x08, 0x70, (rows, cols // 16)).astype(np.uint8)  # normal scales
    st = 2.0 ** -7
    w = m.nvfp4_dequantize(m.pack_nibbles(codes), scales, st)
    p2, s2, st2 = m.nvfp4_quantize(w, tensor_scale=st)
    assert st2 == st and np.array_equal(s2, scales)
    assert np.array_equal(m.nvfp4_dequantize(p2, s2, st2), w)


def pin_quantize_error_bound_and_bf16_exactness(m):
    rng = np.random.default_rng(8)
    w = rng.normal(0, 0.02, (16, 256))
    w[3, :16] = 0.0                                       # an all-zero block
    packed, scales, st = m.nvfp4_quantize(w)
    assert st == 2.0 ** np.ceil(np.log2(np.abs(w).max() / (6 * 448)))
    deq = m.nvfp4_dequantize(packed, scales, st)
    sb = np.repeat(m.e4m3_decode(scales), 16, axis=1)
    # half the widest E2M1 gap (between 4 and 6) times the block's scale;
    # a value the rounded-down scale pushes past 6 saturates by less than that
    assert np.all(np.abs(deq - w) <= st * sb * (1.0 + 1e-12))
    assert np.all(deq[3, :16] == 0.0)
    # a power-of-two tensor scale keeps every weight exact in bf16
    as_bf16 = torch.from_numpy(deq).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(as_bf16, deq)


def pin_bf16_bits_are_the_dequantised_weights(m):
    rng = np.random.default_rng(9)
    w = rng.normal(0, 0.02, (4, 64))
    packed, scales, st = m.nvfp4_quantize(w)
    bits = m.nvfp4_to_bf16_bits(packed, scales, st)
    back = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(back, m.nvfp4_dequantize(packed, scales, st))
    # a tensor scale that is not a power of two leaves values bf16 cannot hold
    with pytest.raises(ValueError):
        m.nvfp4_to_bf16_bits(packed, scales, st * 1.1)


def test_seeded_nvfp4_inputs_are_deterministic_and_exact_in_bf16():
    import workloads
    a = workloads.make_nvfp4_experts(2, 8, 64, seed=3)
    b = workloads.make_nvfp4_experts(2, 8, 64, seed=3)
    assert torch.equal(a["packed"], b["packed"]) and torch.equal(a["scales"], b["scales"])
    assert a["packed"].shape == (2, 8, 32) and a["scales"].shape == (2, 8, 4)
    for e in range(2):
        bits = nvfp4.nvfp4_to_bf16_bits(a["packed"][e].numpy(), a["scales"][e].numpy(),
                                        a["tensor_scale"])
        w = nvfp4.nvfp4_dequantize(a["packed"][e].numpy(), a["scales"][e].numpy(),
                                   a["tensor_scale"])
        assert bits.shape == (8, 64) and np.all(np.abs(w) <= 6 * 3.75 * 2.0 ** -7)


PINS = [pin_e4m3_decode_matches_torch_for_every_code,
        pin_e4m3_encode_matches_torch_rounding_including_ties,
        pin_e4m3_encode_saturates_above_448,
        pin_e2m1_decode_matches_the_ocp_table,
        pin_e2m1_encode_is_round_to_nearest_even_with_saturation,
        pin_storage_nibble_order_and_block_layout,
        pin_quantize_round_trips_representable_blocks,
        pin_quantize_error_bound_and_bf16_exactness,
        pin_bf16_bits_are_the_dequantised_weights]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__[4:] for p in PINS])
def test_pin(pin):
    pin(nvfp4)


MUTATIONS = [
    ("E2M1 exponent bias 0", "np.ldexp(1.0 + 0.5 * m, e - 1)", "np.ldexp(1.0 + 0.5 * m, e)"),
    ("E2M1 ties away from zero", "q = np.minimum(np.rint(a / step) * step, E2M1_MAX)",
     "q = np.minimum(np.floor(a / step + 0.5) * step, E2M1_MAX)"),
    ("E2M1 binade edge at 3", "step = np.where(a < 2.0, 0.5, np.where(a < 4.0, 1.0, 2.0))",
     "step = np.where(a < 2.0, 0.5, np.where(a < 3.0, 1.0, 2.0))"),
    ("E2M1 negative zero code", "neg = (x < 0) & (code != 0)", "neg = (x < 0)"),
    ("E4M3 exponent bias 8", "np.ldexp(1.0 + m / 8.0, e - 7)", "np.ldexp(1.0 + m / 8.0, e - 8)"),
    ("E4M3 no NaN code", "mag = np.where((e == 15) & (m == 7), np.nan, mag)", "mag = mag"),
    ("E4M3 subnormal spacing", "np.ldexp(m / 8.0, -6)", "np.ldexp(m / 8.0, -7)"),
    ("E4M3 truncation", "q = np.minimum(np.rint(a / step) * step, E4M3_MAX)",
     "q = np.minimum(np.floor(a / step) * step, E4M3_MAX)"),
    ("nibbles swapped", "return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)",
     "return (c[:, 1::2] | (c[:, 0::2] << 4)).astype(np.uint8)"),
    ("block scales in reverse order", "block = np.repeat(e4m3_decode(s), BLOCK, axis=1)",
     "block = np.repeat(e4m3_decode(s), BLOCK, axis=1)[:, ::-1]"),
    ("tensor scale dropped", "return float(tensor_scale) * block * e2m1_decode(codes)",
     "return block * e2m1_decode(codes)"),
    ("block scale from 4 instead of 6", "scales = e4m3_encode(amax / (E2M1_MAX * st))",
     "scales = e4m3_encode(amax / (4.0 * st))"),
]


def _mutant(tmp_path, old, new):
    src = os.path.join(os.path.dirname(nvfp4.__file__), "nvfp4.py")
    with open(src) as f:
        text = f.read()
    assert text.count(old) == 1, f"mutation site not found once: {old!r}"
    path = os.path.join(tmp_path, "nvfp4_mutant.py")
    with open(path, "w") as f:
        f.write(text.replace(old, new))
    spec = importlib.util.spec_from_file_location("nvfp4_mutant", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("what,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(tmp_path, what, old, new):
    mod = _mutant(tmp_path, old, new)
    caught = []
    for pin in PINS:
        try:
            pin(mod)
        except (AssertionError, ValueError, IndexError, pytest.fail.Exception):
            caught.append(pin.__name__)
    assert caught, f"no pin catches: {what}"
