"""The oracle against the format facts the pages state (tests/golden/format_facts.txt).

Each fixture line carries its source (page title and section); the checks here
exercise the oracle, not a restatement of its own formulas: shapes of what it
returns, the value set it decodes to, and properties that hold only if the
stated fact does."""
import os

import numpy as np
import pytest

import oracle
import workloads

HERE = os.path.dirname(os.path.abspath(__file__))


def facts():
    out = {}
    with open(os.path.join(HERE, "golden", "format_facts.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            kv, src = line.split("|", 1)
            k, v = (t.strip() for t in kv.split("=", 1))
            assert src.strip(), f"{k}: fixture line without a source"
            out[k] = v
    return out


F = facts()


def test_fixture_has_every_fact():
    assert set(F) == {"nvfp4_block", "nvfp4_element", "higher_precision_block", "mxfp4_scale",
                      "arc_reduction_dim", "arc_residual", "dual_scale"}


def test_nvfp4_scales_one_per_block_of_stated_size():
    B = int(F["nvfp4_block"])
    x = workloads.nvfp4_outliers(8, 256, seed=3)
    y = oracle.bf16_to_f32(x)
    c, s = oracle.nvfp4_quantize(y, oracle.tensor_scale(oracle.amax(y)))
    assert s.shape == (8, 256 // B) and c.shape == (8, 256 // 2)
    # one scale per block: scaling one block of the input rescales exactly one scale byte
    y = oracle.bf16_to_f32(x).astype(np.float32)
    y2 = y.copy()
    y2[0, :B] *= 0.25
    c1, s1 = oracle.nvfp4_quantize(y, np.float32(1.0))
    c2, s2 = oracle.nvfp4_quantize(y2, np.float32(1.0))
    diff = np.argwhere(s1 != s2)
    assert len(diff) >= 1 and set(map(tuple, diff)) <= {(0, 0)}


def test_nvfp4_elements_are_e2m1_values():
    assert F["nvfp4_element"] == "E2M1"
    # every code through the oracle's dequantizer with a unit scale (E8M0 127 = 2^0)
    vals = set()
    for q in range(16):
        d = oracle.dequantize("mxfp4", np.full((1, 16), q | (q << 4), np.uint8), np.array([[127]], np.uint8))
        vals.add(float(d[0, 0]))
    # E2M1: sign, two exponent bits, one mantissa bit
    assert vals == {s * m for s in (1.0, -1.0) for m in (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)}


def test_mxfp4_blocks_and_power_of_two_scales():
    B = int(F["higher_precision_block"])
    assert F["mxfp4_scale"] == "power_of_two"
    x = workloads.mxfp4_student_t(4, 128, seed=5)
    c, s = oracle.mxfp4_quantize(oracle.bf16_to_f32(x))
    assert s.shape == (4, 128 // B)
    # decoded scale of every block: the dequantized value of code 1.0 (0x2) is a power of two
    ones = np.full((4, 64), 0x22, np.uint8)
    d = oracle.dequantize("mxfp4", ones, s)
    m, e = np.frexp(d)
    assert np.all(m == 0.5)


def test_arc_layout_appends_residual_channels_along_k():
    assert F["arc_reduction_dim"] == "K+S"
    M, K, S = 4, 256, 32
    x, g, perm, outl = workloads.arc_activations(M, K, seed=9, S=S)
    c, s, st, y = oracle.arc(x, g, perm, outl, s_t=0.05)
    assert c.shape == (M, (K + S) // 2) and s.shape == (M, (K + S) // 16)


def test_arc_residual_is_original_minus_primary():
    assert F["arc_residual"] == "x - primary"
    M, K, S = 4, 256, 32
    x, g, perm, outl = workloads.arc_activations(M, K, seed=11, S=S)
    st = np.float32(0.05)
    c, s, _, y = oracle.arc(x, g, perm, outl, s_t=st)
    prim = oracle.dequantize("nvfp4", c[:, : K // 2], s[:, : K // 16], st)
    r_true = (y.astype(np.float64) - prim)[:, outl].astype(np.float32)
    # the appended channels are the NVFP4 codes of (original - primary) at the
    # outlier positions, in the order of the outlier list, with the same s_t
    rc, rs = oracle.nvfp4_quantize(r_true, st)
    assert np.array_equal(c[:, K // 2:], rc) and np.array_equal(s[:, K // 16:], rs)
    # and they reconstruct it to NVFP4 accuracy: within one block scale (half
    # the widest E2M1 step, 4 to 6, times amax / 6, plus the E4M3 rounding)
    res = oracle.dequantize("nvfp4", rc, rs, st)
    blk = np.repeat(np.abs(r_true).reshape(M, S // 16, 16).max(axis=2), 16, axis=1)
    assert np.all(np.abs(res - r_true) <= blk / 6 * (1 + 2.0 ** -3) + 1e-12)


def test_dual_format_has_two_scales():
    assert F["dual_scale"] == "group_fp32_and_micro"
    x = workloads.dual_gain(4, 256, seed=13)
    c, s, g = oracle.dual_quantize(oracle.bf16_to_f32(x))
    assert g.dtype == np.float32 and g.shape == (4, 256 // 128)
    assert s.dtype == np.uint8 and s.shape == (4, 256 // int(F["nvfp4_block"]))
