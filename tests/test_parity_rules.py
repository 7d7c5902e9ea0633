"""The GPU acceptance rule itself, checked on the CPU with mistakes planted in oracle results.

The rule lets a GPU code differ from the oracle's by one step only at a rounding tie, and
widens the whole-path output bound by exactly the effect of such codes.  A rule that let a
wrong code through, or that failed a correct one, would make every parity claim meaningless,
so both directions are exercised here on oracle-produced codes (no GPU involved).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from parity_util import (assert_close, compare_stage1, oracle_on_codes, output_widening,
                         tie_distance_bound)
from rotated_w4a4_quantized_group_b200 import workloads as W


def _case(dt="bf16", g=64, M=160, K=4096, seed=3):
    case = W.RotateCase("rules", M=M, K=K, g=g, dtype=dt, seed=seed)
    inp = W.make_rotate_inputs(case)
    oc, os_ = oracle.rotate_quant(inp["x"], inp["R"], g)
    y = oracle.rotate(inp["x"], inp["R"], g)
    return inp, oc, os_, y


def test_identical_codes_pass():
    inp, oc, os_, _ = _case()
    assert compare_stage1(oc.copy(), os_.copy(), oc, os_, torch.bfloat16, "same", 64,
                          x=inp["x"], R=inp["R"]) == 0


@pytest.mark.parametrize("dt", ["bf16", "f16", "f32"])
def test_a_flip_far_from_a_tie_is_rejected(dt):
    inp, oc, os_, y = _case(dt)
    t = y / os_[:, None].astype(np.float64)
    dist = np.abs(t - (np.floor(t) + 0.5))
    r, k = np.argwhere(dist > 0.3)[0]
    gc = oc.copy()
    gc[r, k] += 1 if gc[r, k] < 7 else -1
    with pytest.raises(AssertionError, match="not at a rounding tie"):
        compare_stage1(gc, os_.copy(), oc, os_, W.DTYPES[dt], "far", 64, x=inp["x"], R=inp["R"])


def test_a_flip_without_inputs_is_rejected():
    inp, oc, os_, _ = _case()
    gc = oc.copy()
    gc[0, 0] += 1 if gc[0, 0] < 7 else -1
    with pytest.raises(AssertionError, match="no inputs"):
        compare_stage1(gc, os_.copy(), oc, os_, torch.bfloat16, "bare", 64)


def test_a_flip_at_a_tie_passes():
    """bf16 rows of multiples of 1.5 next to an absmax of 21 (s = 3) with R = I: quotients
    k + 1/2 are exact ties; rounding one of them the other way is an allowed mismatch."""
    M, K, g = 40, 4096, 64
    x = 1.5 * np.random.default_rng(4).integers(-13, 14, size=(M, K))
    x[:, 0] = 21.0
    xt = torch.from_numpy(x).to(torch.bfloat16)
    R = torch.eye(g, dtype=torch.bfloat16)
    oc, os_ = oracle.rotate_quant(xt, R, g)
    t = x / 3.0
    r, k = np.argwhere(np.abs(t - (np.floor(t) + 0.5)) == 0)[0]
    gc = oc.copy()
    gc[r, k] = oc[r, k] + (1 if t[r, k] > oc[r, k] else -1)   # the tie's other neighbour
    assert abs(int(gc[r, k]) - int(oc[r, k])) == 1
    assert compare_stage1(gc, os_.copy(), oc, os_, torch.bfloat16, "tie", g, x=xt, R=R) == 1


def test_too_many_tie_flips_exceed_the_rate():
    M, K, g = 8, 256, 64
    x = 1.5 * np.random.default_rng(5).integers(-13, 14, size=(M, K))
    x[:, 0] = 21.0
    xt = torch.from_numpy(x).to(torch.bfloat16)
    R = torch.eye(g, dtype=torch.bfloat16)
    oc, os_ = oracle.rotate_quant(xt, R, g)
    gc = oc.copy()
    t = x / 3.0
    r, k = np.argwhere(np.abs(t - (np.floor(t) + 0.5)) == 0)[0]
    gc[r, k] = oc[r, k] + (1 if t[r, k] > oc[r, k] else -1)
    with pytest.raises(AssertionError, match="mismatch rate"):
        compare_stage1(gc, os_.copy(), oc, os_, torch.bfloat16, "rate", g, x=xt, R=R)


def test_a_scale_off_by_more_than_its_bound_is_rejected():
    inp, oc, os_, _ = _case("f16")
    gs = os_.copy()
    gs[5] *= 1 + 2.0 ** -9
    with pytest.raises(AssertionError, match="scale relative error"):
        compare_stage1(oc.copy(), gs, oc, os_, torch.float16, "scale", 64, x=inp["x"], R=inp["R"])


def test_tie_bound_for_fp32_uses_the_accumulation_bound():
    """For fp32 inputs the rotated value may move by g 2^-24 sum|x R|: a quotient whose terms
    cancel gets a wider tie window than its own magnitude suggests."""
    y = np.array([1e-3, 1e-3])
    s = np.array([1e-3 / 3.5, 1e-3 / 3.5])
    b = tie_distance_bound(y, s, np.array([1e-3, 10.0]), torch.float32, 16, dynamic=True)
    assert b[1] > 100 * b[0]


@pytest.mark.parametrize("out_dt", [torch.bfloat16, torch.float32])
def test_output_widening_covers_exactly_a_tie_flip(out_dt):
    """A tie flip in one row moves that row's outputs by a*|ws|*|w[n,k]|; the widened bound
    accepts the output computed from the flipped codes, the plain bound does not (fp32)."""
    case = W.LinearCase("wide", M=6, K=256, N=40, g=64, dtype="f32" if out_dt == torch.float32
                        else "bf16", rotation="hadamard", seed=12)
    inp = W.make_linear_inputs(case)
    rows, cols = np.arange(case.M), np.arange(case.N)
    ref, oc, os_ = oracle.linear(inp["x"], inp["R"], case.g, inp["w_packed"], inp["w_scale"],
                                 inp["bias"], rows=rows, cols=cols)
    gc = oc.copy()
    gc[2, 17] += 1 if gc[2, 17] < 7 else -1
    got = oracle_on_codes(gc, os_, inp["w_packed"], case.K, cols, inp["w_scale"], inp["bias"],
                          out_dt)
    extra = output_widening(gc, oc, os_, os_, inp["w_packed"], case.K, cols, inp["w_scale"])
    assert (extra[2] > 0).any() and not extra[[0, 1, 3, 4, 5]].any()
    assert_close(got, ref, out_dt, "widened", extra)
    if out_dt == torch.float32:
        with pytest.raises(AssertionError):
            assert_close(got, ref, out_dt, "plain")


def test_output_widening_covers_a_scale_one_ulp_off():
    """fp32 output with bias: a row scale one fp32 ulp from the oracle's (allowed for fp32
    inputs) moves outputs by |acc| * ulp * |ws|.  Where acc * a * ws cancels against the bias
    that exceeds rtol 1e-5 of |ref|; the widened bound accepts exactly that."""
    case = W.LinearCase("ulp", M=8, K=512, N=300, g=16, dtype="f32", rotation="haar",
                        bias_std=1.0, seed=31)
    inp = W.make_linear_inputs(case)
    rows, cols = np.arange(case.M), np.arange(case.N)
    ref, oc, os_ = oracle.linear(inp["x"], inp["R"], case.g, inp["w_packed"], inp["w_scale"],
                                 inp["bias"], rows=rows, cols=cols)
    gs = os_.copy()
    gs[3] = np.nextafter(gs[3], np.float32(np.inf))
    got = oracle_on_codes(oc, gs, inp["w_packed"], case.K, cols, inp["w_scale"], inp["bias"],
                          torch.float32)
    extra = output_widening(oc, oc, gs, os_, inp["w_packed"], case.K, cols, inp["w_scale"])
    assert not extra[[0, 1, 2, 4, 5, 6, 7]].any() and (extra[3] > 0).all()
    assert_close(got, ref, torch.float32, "scale ulp", extra)
    # the planted difference is real: some outputs of that row moved
    assert (got[3] != ref[3]).any()
