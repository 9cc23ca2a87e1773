"""Pins for the CPU oracle, checked against things other than itself.

Each test names the passage it follows.  Together they are chosen so that a
plausible slip anywhere in the oracle (a dropped term, a wrong sign, a swapped
gate, a transposed operand, a reversed time index, a wrong layer chaining or a
missing bias) fails at least one of them:

* W = 0 closed form (pulsatrix LSTMModule constructor: zero-initialised weights)
* hand-worked steps with rational gates (tests/golden/hand_steps.json)
* invariants |h| < 1, |c_t| - |c_{t-1}| < 1, db_ih == db_hh
* structural identities: batch rows independent, reverse direction = forward
  direction on the time-reversed sequence, two layers = two chained layers,
  seq-first = batch-first transposed
* central finite differences of the BPTT for every input and parameter
* torch.nn.LSTM (CPU, float64) as an independent implementation
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from layer_lstm_b200.workloads import Workload, make_inputs, select_rows

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_steps.json")


def sig(z):
    return 1.0 / (1.0 + np.exp(-z))


# ---------------------------------------------------------------- W = 0 closed form
@pytest.mark.parametrize("L,D", [(1, 1), (2, 1), (1, 2), (2, 2)])
def test_zero_weight_closed_form(L, D):
    """With W_ih = W_hh = 0 the gates are the constants sig(b_i), sig(b_f),
    tanh(b_g), sig(b_o) (b = b_ih + b_hh), so c after n steps is
    f^n c0 + i g (1 - f^n) / (1 - f) and h = o tanh(c).  The reverse
    direction's position t has taken T - t steps."""
    wl = Workload("z", L=L, D=D, I=3, H=5, T=7, B=2, dtype="f32", state_std=0.5, w_k=1.5, seed=7)
    inp = make_inputs(wl, zero_weights=True)
    r = oracle.run_inputs(inp)
    T, H = wl.T, wl.H
    for layer in range(L):
        for d in range(D):
            ld = layer * D + d
            b = inp.b_ih[ld].astype(np.float64) + inp.b_hh[ld].astype(np.float64)
            i, f, g, o = sig(b[:H]), sig(b[H:2 * H]), np.tanh(b[2 * H:3 * H]), sig(b[3 * H:])
            c0 = inp.c0[ld].astype(np.float64)
            for t in range(T):
                n = t + 1 if d == 0 else T - t
                c = f ** n * c0 + i * g * (1 - f ** n) / (1 - f)
                h = o * np.tanh(c)
                if layer == L - 1:
                    np.testing.assert_allclose(r["out"][:, t, d * H:(d + 1) * H], h, rtol=0, atol=1e-14)
                if (d == 0 and t == T - 1) or (d == 1 and t == 0):
                    np.testing.assert_allclose(r["c_n"][ld], c, rtol=0, atol=1e-14)
                    np.testing.assert_allclose(r["h_n"][ld], h, rtol=0, atol=1e-14)


def test_zero_weight_no_bias_halving():
    """No bias and W = 0: every gate is sig(0) = 1/2 or tanh(0) = 0, so
    c_t = c0 / 2^(t+1) and h_t = tanh(c_t) / 2."""
    wl = Workload("z", L=1, D=1, I=2, H=3, T=6, B=3, dtype="f32", state_std=1.0, bias=False, seed=3)
    inp = make_inputs(wl, zero_weights=True)
    r = oracle.run_inputs(inp)
    c0 = inp.c0[0].astype(np.float64)
    for t in range(wl.T):
        c = c0 / 2.0 ** (t + 1)
        np.testing.assert_allclose(r["out"][:, t, :], 0.5 * np.tanh(c), rtol=0, atol=1e-15)
    np.testing.assert_allclose(r["c_n"][0], c0 / 2.0 ** wl.T, rtol=0, atol=1e-15)


def test_zero_weight_backward_closed_form():
    """W = 0: nothing depends on x or h0, so dx = dh0 = 0, and the cell carry
    alone links c0 to every c_t: dL/dc0 = sum_t dL/dh_t o (1 - tanh(c_t)^2) f^(t+1).
    The output-gate bias gradient is sum_{b,t} dL/dh_t tanh(c_t) o (1 - o)."""
    wl = Workload("z", L=1, D=1, I=3, H=4, T=6, B=2, dtype="f32", state_std=0.5, w_k=1.0,
                  train=True, seed=11)
    inp = make_inputs(wl, zero_weights=True)
    r = oracle.run_inputs(inp, backward=True)
    H = wl.H
    b = inp.b_ih[0].astype(np.float64) + inp.b_hh[0].astype(np.float64)
    i, f, g, o = sig(b[:H]), sig(b[H:2 * H]), np.tanh(b[2 * H:3 * H]), sig(b[3 * H:])
    c0 = inp.c0[0].astype(np.float64)
    go = inp.grad_out.astype(np.float64)
    dc0 = np.zeros_like(c0)
    dbo = np.zeros(H)
    for t in range(wl.T):
        n = t + 1
        c = f ** n * c0 + i * g * (1 - f ** n) / (1 - f)
        th = np.tanh(c)
        dc0 += go[:, t, :] * o * (1 - th ** 2) * f ** n
        dbo += (go[:, t, :] * th * o * (1 - o)).sum(axis=0)
    assert np.abs(r["dx"]).max() == 0.0
    assert np.abs(r["dh0"]).max() == 0.0
    np.testing.assert_allclose(r["dc0"][0], dc0, rtol=0, atol=1e-13)
    np.testing.assert_allclose(r["db_ih"][0][3 * H:], dbo, rtol=0, atol=1e-13)


# ------------------------------------------------------------------ hand-worked steps
def _parse(v):
    if isinstance(v, (int, float)):
        return float(v)
    s = v.replace("ln", "math.log(")
    # "2*ln3" -> "2*math.log(3)", "-ln3" -> "-math.log(3)"
    out, k = "", 0
    while k < len(s):
        if s.startswith("math.log(", k):
            j = k + len("math.log(")
            m = j
            while m < len(s) and s[m].isdigit():
                m += 1
            out += "math.log(" + s[j:m] + ")"
            k = m
        else:
            out += s[k]
            k += 1
    return float(eval(out, {"math": math}))


def _expect_h(expr):
    coef, rest = expr.split("*tanh(")
    num, den = rest.rstrip(")").split("/")
    return float(coef) * math.tanh(int(num) / int(den))


def _cases():
    with open(GOLDEN) as fh:
        return json.load(fh)["cases"]


@pytest.mark.parametrize("case", _cases(), ids=lambda c: c["name"])
def test_hand_steps(case):
    I, H, L, D = case["I"], case["H"], case["L"], case["D"]
    LD = L * D
    w_ih = [np.array([_parse(v) for v in w]).reshape(4 * H, -1) for w in case["w_ih"]]
    w_hh = [np.array([_parse(v) for v in w]).reshape(4 * H, H) for w in case["w_hh"]]
    b_ih = [np.array([_parse(v) for v in b]) for b in case["b_ih"]]
    b_hh = [np.array([_parse(v) for v in b]) for b in case["b_hh"]]
    assert len(w_ih) == LD and w_ih[0].shape[1] == I
    out, h_n, c_n = oracle.lstm_forward(np.array(case["x"]), w_ih, w_hh, b_ih, b_hh,
                                        h0=np.array(case["h0"]), c0=np.array(case["c0"]),
                                        num_layers=L, bidirectional=D == 2)
    exp_out = np.vectorize(_expect_h)(np.array(case["expect_out"], dtype=object)).astype(np.float64)
    exp_cn = np.vectorize(lambda s: float(Fraction(s)))(np.array(case["expect_cn"], dtype=object))
    np.testing.assert_allclose(out, exp_out, rtol=0, atol=1e-15)
    np.testing.assert_allclose(c_n, exp_cn.astype(np.float64), rtol=0, atol=1e-15)


# ----------------------------------------------------------------------- invariants
def test_invariants_h_bounded_and_c_growth():
    """|h_t| < 1 since h = o tanh(c) with o in (0,1); |c_t| <= f|c_{t-1}| + i|g|
    < |c_{t-1}| + 1.  c_t is read as c_n of the length-(t+1) prefix."""
    wl = Workload("inv", L=1, D=1, I=4, H=6, T=9, B=3, dtype="f32", state_std=2.0, w_k=3.0, seed=5)
    inp = make_inputs(wl)
    r = oracle.run_inputs(inp)
    assert np.abs(r["out"]).max() < 1.0
    prev = inp.c0[0].astype(np.float64)
    for t in range(1, wl.T + 1):
        _, _, c_n = oracle.lstm_forward(inp.x[:, :t], inp.w_ih, inp.w_hh, inp.b_ih, inp.b_hh,
                                        h0=inp.h0, c0=inp.c0)
        assert np.all(np.abs(c_n[0]) < np.abs(prev) + 1.0)
        prev = c_n[0]


def test_bias_gradients_equal():
    """b_ih and b_hh enter the pre-activation as a plain sum, so their gradients are equal."""
    wl = Workload("bb", L=2, D=2, I=3, H=4, T=5, B=2, dtype="f32", state_std=0.3, train=True, seed=9)
    r = oracle.run_inputs(make_inputs(wl), backward=True)
    for a, b in zip(r["db_ih"], r["db_hh"]):
        assert np.array_equal(a, b)


# ------------------------------------------------------------- structural identities
def test_batch_rows_independent():
    wl = Workload("rows", L=2, D=2, I=3, H=4, T=5, B=5, dtype="f32", state_std=0.4, seed=12)
    inp = make_inputs(wl)
    full = oracle.run_inputs(inp)
    perm = [3, 0, 4]
    sub = oracle.run_inputs(select_rows(inp, perm))
    np.testing.assert_array_equal(sub["out"], full["out"][perm])
    np.testing.assert_array_equal(sub["h_n"], full["h_n"][:, perm])
    np.testing.assert_array_equal(sub["c_n"], full["c_n"][:, perm])


def test_reverse_direction_is_forward_on_reversed_time():
    wl = Workload("rev", L=1, D=2, I=3, H=4, T=6, B=2, dtype="f32", state_std=0.4, seed=13)
    inp = make_inputs(wl)
    bi = oracle.run_inputs(inp)
    out_r, hn_r, cn_r = oracle.lstm_forward(inp.x[:, ::-1], [inp.w_ih[1]], [inp.w_hh[1]],
                                            [inp.b_ih[1]], [inp.b_hh[1]],
                                            h0=inp.h0[1:2], c0=inp.c0[1:2])
    np.testing.assert_allclose(bi["out"][:, :, 4:], out_r[:, ::-1], rtol=0, atol=1e-15)
    np.testing.assert_allclose(bi["h_n"][1], hn_r[0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(bi["c_n"][1], cn_r[0], rtol=0, atol=1e-15)
    out_f, _, _ = oracle.lstm_forward(inp.x, [inp.w_ih[0]], [inp.w_hh[0]], [inp.b_ih[0]],
                                      [inp.b_hh[0]], h0=inp.h0[0:1], c0=inp.c0[0:1])
    np.testing.assert_allclose(bi["out"][:, :, :4], out_f, rtol=0, atol=1e-15)


@pytest.mark.parametrize("D", [1, 2])
def test_two_layers_are_chained_single_layers(D):
    wl = Workload("chain", L=2, D=D, I=3, H=4, T=5, B=2, dtype="f32", state_std=0.4, seed=14)
    inp = make_inputs(wl)
    two = oracle.run_inputs(inp)
    o1, hn1, cn1 = oracle.lstm_forward(inp.x, inp.w_ih[:D], inp.w_hh[:D], inp.b_ih[:D],
                                       inp.b_hh[:D], h0=inp.h0[:D], c0=inp.c0[:D],
                                       bidirectional=D == 2)
    o2, hn2, cn2 = oracle.lstm_forward(o1, inp.w_ih[D:], inp.w_hh[D:], inp.b_ih[D:],
                                       inp.b_hh[D:], h0=inp.h0[D:], c0=inp.c0[D:],
                                       bidirectional=D == 2)
    np.testing.assert_allclose(two["out"], o2, rtol=0, atol=1e-15)
    np.testing.assert_allclose(two["h_n"], np.concatenate([hn1, hn2]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(two["c_n"], np.concatenate([cn1, cn2]), rtol=0, atol=1e-15)


def test_seq_first_layout():
    wl = Workload("sf", L=2, D=2, I=3, H=4, T=5, B=3, dtype="f32", state_std=0.4, train=True, seed=15)
    bf = make_inputs(wl)
    sf = make_inputs(wl.replace(batch_first=False))
    rb = oracle.run_inputs(bf, backward=True)
    rs = oracle.run_inputs(sf, backward=True)
    np.testing.assert_array_equal(rs["out"], rb["out"].transpose(1, 0, 2))
    np.testing.assert_array_equal(rs["dx"], rb["dx"].transpose(1, 0, 2))
    for a, b in zip(rs["dw_hh"], rb["dw_hh"]):
        np.testing.assert_array_equal(a, b)


# ------------------------------------------------------------ central differences
def _loss(inp, gh, gc, **over):
    kw = dict(x=inp.x, w_ih=inp.w_ih, w_hh=inp.w_hh, b_ih=inp.b_ih, b_hh=inp.b_hh,
              h0=inp.h0, c0=inp.c0)
    kw.update(over)
    out, h_n, c_n = oracle.lstm_forward(kw["x"], kw["w_ih"], kw["w_hh"], kw["b_ih"], kw["b_hh"],
                                        h0=kw["h0"], c0=kw["c0"], num_layers=inp.wl.L,
                                        bidirectional=inp.wl.D == 2)
    return (float((out * inp.grad_out).sum()) + float((h_n * gh).sum())
            + float((c_n * gc).sum()))


@pytest.mark.parametrize("D", [1, 2])
def test_bptt_central_differences(D):
    """Every gradient the backward returns against (L(p+e) - L(p-e)) / 2e with
    e = 1e-6, L = <grad_out, out> + <grad_hn, h_n> + <grad_cn, c_n>."""
    wl = Workload("fd", L=2, D=D, I=3, H=2, T=4, B=2, dtype="f32", state_std=0.5, w_k=0.8,
                  train=True, seed=21)
    inp = make_inputs(wl)
    rng = np.random.default_rng(3)
    gh = rng.standard_normal((wl.L * D, wl.B, wl.H))
    gc = rng.standard_normal((wl.L * D, wl.B, wl.H))
    f64 = lambda a: a.astype(np.float64)
    inp.x, inp.h0, inp.c0 = f64(inp.x), f64(inp.h0), f64(inp.c0)
    inp.grad_out = f64(inp.grad_out)
    inp.w_ih = [f64(w) for w in inp.w_ih]
    inp.w_hh = [f64(w) for w in inp.w_hh]
    inp.b_ih = [f64(b) for b in inp.b_ih]
    inp.b_hh = [f64(b) for b in inp.b_hh]
    inp.grad_hn, inp.grad_cn = gh, gc
    g = oracle.run_inputs(inp, backward=True)
    eps = 1e-6

    def fd_check(name, arr, grad, rebuild):
        num = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            orig = arr[idx]
            arr[idx] = orig + eps
            lp = _loss(inp, gh, gc, **rebuild())
            arr[idx] = orig - eps
            lm = _loss(inp, gh, gc, **rebuild())
            arr[idx] = orig
            num[idx] = (lp - lm) / (2 * eps)
        scale = max(np.abs(num).max(), 1e-3)
        err = np.abs(num - grad).max() / scale
        assert err < 1e-6, f"{name}: relative error {err:.3e}"

    fd_check("x", inp.x, g["dx"], lambda: {})
    fd_check("h0", inp.h0, g["dh0"], lambda: {})
    fd_check("c0", inp.c0, g["dc0"], lambda: {})
    for ld in range(wl.L * D):
        fd_check(f"w_ih{ld}", inp.w_ih[ld], g["dw_ih"][ld], lambda: {})
        fd_check(f"w_hh{ld}", inp.w_hh[ld], g["dw_hh"][ld], lambda: {})
        fd_check(f"b_ih{ld}", inp.b_ih[ld], g["db_ih"][ld], lambda: {})
        fd_check(f"b_hh{ld}", inp.b_hh[ld], g["db_hh"][ld], lambda: {})


# ------------------------------------------------ torch.nn.LSTM (float64) as a second opinion
def _torch_lstm(inp):
    import torch
    wl = inp.wl
    m = torch.nn.LSTM(wl.I, wl.H, num_layers=wl.L, bidirectional=wl.D == 2, bias=wl.bias,
                      batch_first=wl.batch_first).double()
    with torch.no_grad():
        for layer in range(wl.L):
            for d in range(wl.D):
                sfx = "_reverse" if d else ""
                ld = layer * wl.D + d
                getattr(m, f"weight_ih_l{layer}{sfx}").copy_(torch.tensor(inp.w_ih[ld], dtype=torch.float64))
                getattr(m, f"weight_hh_l{layer}{sfx}").copy_(torch.tensor(inp.w_hh[ld], dtype=torch.float64))
                if wl.bias:
                    getattr(m, f"bias_ih_l{layer}{sfx}").copy_(torch.tensor(inp.b_ih[ld], dtype=torch.float64))
                    getattr(m, f"bias_hh_l{layer}{sfx}").copy_(torch.tensor(inp.b_hh[ld], dtype=torch.float64))
    x = torch.tensor(inp.x, dtype=torch.float64, requires_grad=True)
    LDBH = (wl.L * wl.D, wl.B, wl.H)
    h0 = torch.tensor(inp.h0 if inp.h0 is not None else np.zeros(LDBH), dtype=torch.float64, requires_grad=True)
    c0 = torch.tensor(inp.c0 if inp.c0 is not None else np.zeros(LDBH), dtype=torch.float64, requires_grad=True)
    if inp.lengths is None:
        out, (hn, cn) = m(x, (h0, c0))
    else:
        # packed sequences (the lstm.data overload); padding back with zeros
        from torch.nn.utils.rnn import pack_padded_sequence, pad_packed_sequence
        packed = pack_padded_sequence(x, torch.tensor(inp.lengths, dtype=torch.int64),
                                      batch_first=wl.batch_first, enforce_sorted=False)
        pout, (hn, cn) = m(packed, (h0, c0))
        out, _ = pad_packed_sequence(pout, batch_first=wl.batch_first, padding_value=0.0,
                                     total_length=wl.T)
    res = dict(out=out.detach().numpy(), h_n=hn.detach().numpy(), c_n=cn.detach().numpy())
    if inp.grad_out is not None:
        loss = (out * torch.tensor(inp.grad_out, dtype=torch.float64)).sum()
        if inp.grad_hn is not None:
            loss = loss + (hn * torch.tensor(inp.grad_hn, dtype=torch.float64)).sum()
        if inp.grad_cn is not None:
            loss = loss + (cn * torch.tensor(inp.grad_cn, dtype=torch.float64)).sum()
        loss.backward()
        res["dx"] = x.grad.numpy()
        res["dh0"] = h0.grad.numpy()
        res["dc0"] = c0.grad.numpy()
        for nm in ("weight_ih", "weight_hh", "bias_ih", "bias_hh"):
            if nm.startswith("bias") and not wl.bias:
                continue
            res[nm] = [getattr(m, f"{nm}_l{ld // wl.D}{'_reverse' if ld % wl.D else ''}").grad.numpy()
                       for ld in range(wl.L * wl.D)]
    return res


@pytest.mark.parametrize("kw", [
    dict(L=1, D=1, I=8, H=16, T=5, B=4, w_k=0.25),
    dict(L=2, D=2, I=5, H=6, T=7, B=3, state_std=0.3),
    dict(L=3, D=1, I=4, H=3, T=6, B=2, state_std=0.2, bias=False),
    dict(L=2, D=2, I=3, H=5, T=4, B=3, state_std=0.2, batch_first=False),
], ids=["c1shape", "bi2", "uni3_nobias", "seqfirst"])
def test_matches_torch_float64(kw):
    wl = Workload("torch", dtype="f32", train=True, seed=31, **kw)
    inp = make_inputs(wl)
    ref = _torch_lstm(inp)
    r = oracle.run_inputs(inp, backward=True)
    for k in ("out", "h_n", "c_n", "dx", "dh0", "dc0"):
        np.testing.assert_allclose(r[k], ref[k], rtol=0, atol=1e-12, err_msg=k)
    for ours, theirs in (("dw_ih", "weight_ih"), ("dw_hh", "weight_hh"),
                         ("db_ih", "bias_ih"), ("db_hh", "bias_hh")):
        if theirs.startswith("bias") and not wl.bias:
            continue
        for a, b in zip(r[ours], ref[theirs]):
            np.testing.assert_allclose(a, b, rtol=0, atol=1e-12, err_msg=ours)


def test_empty_sequence_returns_initial_state():
    """T = 0: no step runs, so h_n = h0 and c_n = c0 (and out is empty)."""
    wl = Workload("t0", L=2, D=2, I=3, H=4, T=0, B=2, dtype="f32", state_std=0.5, seed=41)
    inp = make_inputs(wl)
    r = oracle.run_inputs(inp)
    assert r["out"].shape == (2, 0, 8)
    np.testing.assert_array_equal(r["h_n"], inp.h0)
    np.testing.assert_array_equal(r["c_n"], inp.c0)


# ------------------------------------------------ variable-length batches
def _varlen_inputs(seed, lengths, **kw):
    wl = Workload("vl", dtype="f32", train=True, seed=seed, varlen=True, **kw)
    inp = make_inputs(wl)
    inp.lengths = np.asarray(lengths, dtype=np.int32)
    rng = np.random.default_rng(seed)
    LDBH = (wl.L * wl.D, wl.B, wl.H)
    inp.grad_hn = rng.standard_normal(LDBH).astype(np.float32)
    inp.grad_cn = rng.standard_normal(LDBH).astype(np.float32)
    return inp


@pytest.mark.parametrize("kw,lengths", [
    (dict(L=1, D=1, I=4, H=5, T=6, B=4, state_std=0.3), [6, 1, 3, 5]),
    (dict(L=2, D=2, I=3, H=4, T=7, B=3, state_std=0.3), [2, 7, 4]),
    (dict(L=2, D=2, I=3, H=4, T=5, B=3, state_std=0.2, batch_first=False), [5, 3, 1]),
], ids=["uni", "bi2", "bi_seqfirst"])
def test_varlen_matches_torch_packed_float64(kw, lengths):
    """Per-row lengths against torch's packed-sequence LSTM in float64 (zero
    padding, final states of each row, gradients through the packing)."""
    inp = _varlen_inputs(51, lengths, **kw)
    ref = _torch_lstm(inp)
    r = oracle.run_inputs(inp, backward=True)
    for k in ("out", "h_n", "c_n", "dx", "dh0", "dc0"):
        np.testing.assert_allclose(r[k], ref[k], rtol=0, atol=1e-12, err_msg=k)
    for ours, theirs in (("dw_ih", "weight_ih"), ("dw_hh", "weight_hh"), ("db_ih", "bias_ih")):
        for a, b in zip(r[ours], ref[theirs]):
            np.testing.assert_allclose(a, b, rtol=0, atol=1e-12, err_msg=ours)


def test_varlen_row_is_the_truncated_problem():
    """Row b with n valid steps gives, on its first n steps, exactly the
    fixed-length problem on x[b, :n]; its padded outputs and input
    gradients are zero."""
    inp = _varlen_inputs(52, [5, 2, 4], L=2, D=2, I=3, H=4, T=5, B=3, state_std=0.3)
    r = oracle.run_inputs(inp, backward=True)
    for b, n in enumerate(inp.lengths):
        one = select_rows(inp, [b])
        one.lengths = None
        one.wl = one.wl.replace(T=int(n), varlen=False)
        one.x = np.ascontiguousarray(one.x[:, :n])
        one.grad_out = np.ascontiguousarray(one.grad_out[:, :n])
        ref = oracle.run_inputs(one, backward=True)
        np.testing.assert_array_equal(r["out"][b, :n], ref["out"][0])
        assert not np.any(r["out"][b, n:]) and not np.any(r["dx"][b, n:])
        np.testing.assert_array_equal(r["dx"][b, :n], ref["dx"][0])
        for k in ("h_n", "c_n", "dh0", "dc0"):
            np.testing.assert_array_equal(r[k][:, b], ref[k][:, 0], err_msg=k)


def test_varlen_empty_row_keeps_initial_state():
    """A row of length 0 runs no step: zero outputs, h_n = h0, c_n = c0, and
    the state gradients pass straight through (dh0 = grad_hn, dc0 = grad_cn)."""
    inp = _varlen_inputs(53, [3, 0], L=2, D=2, I=3, H=4, T=3, B=2, state_std=0.5)
    r = oracle.run_inputs(inp, backward=True)
    assert not np.any(r["out"][1]) and not np.any(r["dx"][1])
    np.testing.assert_array_equal(r["h_n"][:, 1], inp.h0[:, 1])
    np.testing.assert_array_equal(r["c_n"][:, 1], inp.c0[:, 1])
    np.testing.assert_array_equal(r["dh0"][:, 1], inp.grad_hn[:, 1])
    np.testing.assert_array_equal(r["dc0"][:, 1], inp.grad_cn[:, 1])


# ------------------------------------------------ inter-layer dropout (training)
def test_philox_matches_numpy():
    """The oracle's Philox4x64-10 against numpy's independent implementation
    of the same published generator (numpy advances its counter by one
    before the first block it returns)."""
    for ctr, key in [([1, 0, 0, 0], [0, 0]), ([2, 0, 0, 0], [0x1234, 5]),
                     ([7, 3, 0, 9], [2 ** 64 - 1, 17]), ([2 ** 40 + 5, 0, 0, 0], [99, 0])]:
        bg = np.random.Philox(key=np.array(key, dtype=np.uint64),
                              counter=np.array([ctr[0] - 1] + ctr[1:], dtype=np.uint64))
        want = [int(v) for v in bg.random_raw(4)]
        assert oracle.philox4x64_10(ctr, key) == want, (ctr, key)


def _numpy_keep_mask(seed, layer, T, B, DH, p):
    """keep[t, b, k] from numpy's Philox: word e mod 4 of the block at counter
    floor(e/4), key (seed, layer), compared as integers with ceil(p * 2^53)."""
    n = T * B * DH
    nblk = (n + 3) // 4
    bg = np.random.Philox(key=np.array([seed, layer], dtype=np.uint64),
                          counter=np.array([2 ** 64 - 1, 2 ** 64 - 1, 2 ** 64 - 1, 2 ** 64 - 1],
                                           dtype=np.uint64))   # +1 wraps to counter 0
    words = bg.random_raw(4 * nblk)[:n]
    thresh = math.ceil(p * 2.0 ** 53)
    return ((words >> np.uint64(11)) >= np.uint64(thresh)).reshape(T, B, DH)


@pytest.mark.parametrize("D", [1, 2])
def test_dropout_equals_chained_layers_with_an_independent_mask(D):
    """A 2-layer training run with inter-layer dropout p equals: layer 0 run
    alone, its output multiplied by a mask drawn with numpy's Philox over
    (1 - p), layer 1 run alone on that; gradients likewise chained through
    the same mask."""
    p, seed = float(np.float32(0.35)), 0xC0FFEE   # the descriptor carries p as a float32
    wl = Workload("dr", L=2, D=D, I=3, H=4, T=5, B=3, dtype="f32", state_std=0.3, train=True,
                  seed=61, dropout=p, dropout_seed=seed)
    inp = make_inputs(wl)
    rng = np.random.default_rng(61)
    inp.grad_hn = rng.standard_normal((2 * D, 3, 4)).astype(np.float32)
    r = oracle.run_inputs(inp, backward=True)
    keep = _numpy_keep_mask(seed, 0, wl.T, wl.B, D * wl.H, p).transpose(1, 0, 2)   # [B][T][DH]
    m = keep / (1.0 - p)
    s0, s1 = slice(0, D), slice(D, 2 * D)
    kw0 = dict(b_ih=inp.b_ih[s0], b_hh=inp.b_hh[s0], h0=inp.h0[s0], c0=inp.c0[s0], bidirectional=D == 2)
    kw1 = dict(b_ih=inp.b_ih[s1], b_hh=inp.b_hh[s1], h0=inp.h0[s1], c0=inp.c0[s1], bidirectional=D == 2)
    out0, _, _ = oracle.lstm_forward(inp.x, inp.w_ih[s0], inp.w_hh[s0], **kw0)
    r1 = oracle.lstm_backward(out0 * m, inp.w_ih[s1], inp.w_hh[s1], inp.grad_out,
                              grad_hn=inp.grad_hn[s1], **kw1)
    r0 = oracle.lstm_backward(inp.x, inp.w_ih[s0], inp.w_hh[s0], r1["dx"] * m,
                              grad_hn=inp.grad_hn[s0], **kw0)
    assert 0 < keep.mean() < 1
    np.testing.assert_allclose(r["out"], r1["out"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(r["h_n"], np.concatenate([r0["h_n"], r1["h_n"]]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(r["dx"], r0["dx"], rtol=0, atol=1e-13)
    np.testing.assert_allclose(r["dh0"], np.concatenate([r0["dh0"], r1["dh0"]]), rtol=0, atol=1e-13)
    for k in ("dw_ih", "dw_hh", "db_ih"):
        for a, b in zip(r[k], r0[k] + r1[k]):
            np.testing.assert_allclose(a, b, rtol=0, atol=1e-13, err_msg=k)


def test_dropout_zero_is_no_dropout():
    wl = Workload("dr0", L=2, D=2, I=3, H=4, T=4, B=2, dtype="f32", state_std=0.3, train=True, seed=62)
    inp = make_inputs(wl)
    a = oracle.run_inputs(inp, backward=True)
    inp.wl = wl.replace(dropout=0.0, dropout_seed=123)
    b = oracle.run_inputs(inp, backward=True)
    for k in ("out", "dx", "dh0"):
        np.testing.assert_array_equal(a[k], b[k])


def test_single_precision_build_agrees_at_float32_rounding():
    """The comparison method of "LSTM Gate Equations > Comparing with
    PyTorch" (Out[20]): two implementations of the cell in float32 agree to
    max-abs 3.22e-08 on h and 6.41e-08 on c (input 8 -> hidden 16).  The
    oracle compiled with every value in float32, against its double build on
    the first workload (I8 H16 T5 B4, five steps), must agree to that order:
    above 1e-9 (the single build really rounds) and below 1e-6."""
    from layer_lstm_b200.workloads import WORKLOADS
    wl = WORKLOADS["c1"]
    inp = make_inputs(wl)
    ref = oracle.run_inputs(inp)
    out, h_n, c_n = oracle.lstm_forward_single(inp.x, inp.w_ih, inp.w_hh, inp.b_ih, inp.b_hh,
                                               inp.h0, inp.c0, wl.L, wl.D == 2)
    err_h = float(np.abs(out.astype(np.float64) - ref["out"]).max())
    err_c = float(np.abs(c_n.astype(np.float64) - ref["c_n"]).max())
    for err in (err_h, err_c, float(np.abs(h_n - ref["h_n"]).max())):
        assert 1e-9 < err < 1e-6, err
