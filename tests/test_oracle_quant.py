"""Pins for the oracle's reading of the channel-wise 16-bit weight storage
(FlashSchNet paper-curation summary, How: "channel-wise 16-bit quantization"
of the filter network): per output channel o of W[in][out], s_o = max_i |W[i][o]|,
stored value round-to-nearest-even(W / s_o) in fp16 or bf16, effective weight
s_o * stored.

Each check is fixed by the definition itself or by an independent library
conversion, and each fails for one plausible mistake: scales over the input
axis instead of the output axis, rounding by truncation or ties away from zero,
a lost scale, a wrong number of significant bits."""
import numpy as np
import pytest
import torch

from oracle import quant


# ---------------------------------------------------------------------------
# rounding to 16 bits
# ---------------------------------------------------------------------------

def _float32_sweep(n=200_000, seed=3):
    """float32-representable values over many binades, ties and near-powers of two included."""
    rng = np.random.default_rng(seed)
    bits = rng.integers(0x3000_0000, 0x4300_0000, size=n, dtype=np.uint32)   # ~5e-10 .. 128
    x = bits.view(np.float32).astype(np.float64)
    x *= rng.choice([-1.0, 1.0], size=n)
    k = np.arange(-20, 8, dtype=np.float64)
    p2 = np.ldexp(1.0, k.astype(int))
    near = np.concatenate([p2, p2 * (1 + 2.0 ** -23), p2 * (1 - 2.0 ** -24), -p2])
    return np.concatenate([x, near, [0.0, -0.0]])


def test_round_bf16_matches_torch_conversion():
    # torch converts float32 to bfloat16 with round-to-nearest-even; float32 inputs make
    # the float64 -> float32 step exact, so this is a single rounding on both sides
    x = _float32_sweep()
    ref = torch.tensor(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    got = quant._round_bf16(x)
    assert np.array_equal(got, ref)


def test_round_fp16_matches_torch_conversion():
    x = _float32_sweep()
    x = x[np.abs(x) < 60000.0]                   # inside the fp16 range
    x = x[(np.abs(x) >= 2.0 ** -14) | (x == 0)]  # normal fp16 numbers (scaled weights are)
    ref = torch.tensor(x.astype(np.float32)).to(torch.float16).to(torch.float64).numpy()
    got = quant._round_fp16(x)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("fmt,spacing", [("bf16", 2.0 ** -7), ("fp16", 2.0 ** -10)])
def test_ties_go_to_even(fmt, spacing):
    rnd = quant._round_bf16 if fmt == "bf16" else quant._round_fp16
    # halfway between 1 (even mantissa) and 1 + u: to 1; truncation also gives 1
    assert rnd(np.array([1.0 + spacing / 2]))[0] == 1.0
    # halfway between 1 + u (odd) and 1 + 2u (even): to 1 + 2u; truncation gives 1 + u
    assert rnd(np.array([1.0 + 1.5 * spacing]))[0] == 1.0 + 2 * spacing
    # just above a tie goes up, just below goes down (no ties-away rule hides here)
    assert rnd(np.array([1.0 + spacing / 2 + 2.0 ** -30]))[0] == 1.0 + spacing
    assert rnd(np.array([1.0 + 1.5 * spacing - 2.0 ** -30]))[0] == 1.0 + spacing
    # symmetric for negative values (ties away from zero would give -(1 + u) for the first)
    assert rnd(np.array([-(1.0 + spacing / 2)]))[0] == -1.0
    assert rnd(np.array([-(1.0 + 1.5 * spacing)]))[0] == -(1.0 + 2 * spacing)


def test_significant_bits():
    # bf16 keeps 8 significant bits, fp16 11: 1 + 2^-7 and 1 + 2^-10 are representable
    assert quant._round_bf16(np.array([1.0 + 2.0 ** -7]))[0] == 1.0 + 2.0 ** -7
    assert quant._round_fp16(np.array([1.0 + 2.0 ** -10]))[0] == 1.0 + 2.0 ** -10
    # a value needing 9 (resp. 12) bits is not kept
    assert quant._round_bf16(np.array([1.0 + 2.0 ** -8 + 2.0 ** -7]))[0] != 1.0 + 2.0 ** -8 + 2.0 ** -7
    assert quant._round_fp16(np.array([1.0 + 2.0 ** -11 + 2.0 ** -10]))[0] != 1.0 + 2.0 ** -11 + 2.0 ** -10


# ---------------------------------------------------------------------------
# the channel scale
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", ["fp16", "bf16"])
def test_hand_column(fmt):
    # one output column [0.5, -2, 1]: s = 2, stored [0.25, -1, 0.5] (exact in both formats),
    # so the dequantized column equals the input exactly
    W = np.array([[0.5], [-2.0], [1.0]])
    assert np.array_equal(quant.dequantize(W, fmt), W)


@pytest.mark.parametrize("fmt,bits", [("fp16", 11), ("bf16", 8)])
def test_scales_are_per_output_column(fmt, bits):
    # W[in][out]: column 1's max-abs entry is v = 1 + 2^-(bits+2), which needs more bits than
    # the format has.  With s_1 = v (the column's own maximum) it is stored as exactly 1.0 and
    # comes back as v.  Scaled by its row's maximum (3) instead, it would lose its low bit.
    v = 1.0 + 2.0 ** -(bits + 2)
    W = np.array([[3.0, v],
                  [1.0, 0.25]])
    D = quant.dequantize(W, fmt)
    assert D[0, 1] == v
    assert D[0, 0] == 3.0
    # the transposed matrix has v in column 0 under a column maximum of 3: rounded
    Dt = quant.dequantize(W.T.copy(), fmt)
    assert Dt[1, 0] != v
    assert abs(Dt[1, 0] - v) <= 3.0 * 2.0 ** -bits


@pytest.mark.parametrize("fmt", ["fp16", "bf16"])
def test_ties_inside_a_scaled_column(fmt):
    # column with max-abs exactly 1, so the stored values are the column itself rounded
    u = 2.0 ** -7 if fmt == "bf16" else 2.0 ** -10
    W = np.array([[1.0], [(1 + u / 2) / 2], [(1 + 1.5 * u) / 2], [-(1 + 1.5 * u) / 4]])
    D = quant.dequantize(W, fmt)
    assert D[0, 0] == 1.0
    assert D[1, 0] == 0.5                       # tie to even (down)
    assert D[2, 0] == (1 + 2 * u) / 2           # tie to even (up)
    assert D[3, 0] == -(1 + 2 * u) / 4


@pytest.mark.parametrize("fmt,bits", [("fp16", 11), ("bf16", 8)])
def test_random_weights_properties(fmt, bits):
    # layered weights [L][in][out] as the model stores them (Xavier range)
    rng = np.random.default_rng(11)
    W = rng.uniform(-0.18, 0.18, size=(3, 50, 128))
    W[1, :, 5] = 0.0                             # an all-zero column keeps scale 1 and stays zero
    D = quant.dequantize(W, fmt)
    s = np.abs(W).max(axis=1, keepdims=True)
    s = np.where(s > 0, s, 1.0)
    # each column's max-abs entry maps to +-1, which both formats hold exactly
    idx = np.abs(W).argmax(axis=1)
    for l in range(3):
        cols = np.arange(128)
        assert np.array_equal(D[l, idx[l], cols], W[l, idx[l], cols])
    assert np.all(D[1, :, 5] == 0.0)
    # relative error of every stored value within half an ulp of its 16-bit format
    rel = np.abs(D - W) / s
    ulp = np.ldexp(1.0, np.frexp(np.abs(W) / s)[1] - bits)
    assert np.all(np.abs(D - W) / s <= 0.5 * ulp + 1e-300)
    assert rel.max() <= 2.0 ** -bits
    # scaling by the column maximum first: the stored value s * RN(W/s) differs from RN(W)
    # for some entries, so the scale is really applied (and undone)
    direct = quant._round_fp16(W) if fmt == "fp16" else quant._round_bf16(W)
    assert not np.array_equal(D, direct)


def test_dequantized_weights_touches_only_the_filter_network():
    rng = np.random.default_rng(2)
    w = {k: rng.uniform(-0.2, 0.2, size=(2, 8, 8)) for k in ("W1", "W2", "W_in", "Wo1")}
    out = quant.dequantized_weights(w, "bf16")
    assert out["W_in"] is w["W_in"] and out["Wo1"] is w["Wo1"]
    assert not np.array_equal(out["W1"], w["W1"]) and not np.array_equal(out["W2"], w["W2"])
    assert np.array_equal(out["W1"], quant.dequantize(w["W1"], "bf16"))
