"""Pins for the CPU oracle: each checks it against something other than itself
(a library routine, a closed form, brute force, an invariant) on small inputs,
so that a dropped term, a wrong sign or index, or a transposed operand in the
oracle fails at least one of them.  No GPU."""
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synth
from synth.workloads import Workload

# --------------------------------------------------------------------- codecs


def test_bf16_decode_all_patterns_match_torch():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # the scalar entry point agrees with the vectorised one
    for b in (0x0000, 0x3F80, 0xBF80, 0x0001, 0x7F7F, 0x8001):
        assert oracle.bf16_to_double(b) == ours[b]


def test_bf16_round_matches_torch_on_fp32_values():
    # For inputs that are fp32 values, one rounding double->bf16 equals torch's fp32->bf16 cast.
    rng = np.random.default_rng(1)
    v = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(5000) * 1e-38).astype(np.float32),     # subnormal range
        (rng.standard_normal(5000) * 1e30).astype(np.float32),
        np.float32([3.3895314e38, -3.3895314e38, 1.0 + 2.0**-8, 1.0 + 3 * 2.0**-8]),
    ])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ours = oracle.round_bf16(v.astype(np.float64))
    assert np.array_equal(ours, ref)


@pytest.mark.parametrize("value,bits", [
    (1.0 + 2.0**-8, 0x3F80),                  # tie -> even (1.0)
    (1.0 + 3 * 2.0**-8, 0x3F82),              # tie -> even (1 + 2^-6)
    (1.0 + 2.0**-8 + 2.0**-40, 0x3F81),       # just above the tie: a double-rounding trap via fp32
    (-(1.0 + 2.0**-8 + 2.0**-40), 0xBF81),
    (1.5 * 2.0**-133, 0x0002),                # subnormal tie -> even
    (2.0**-134, 0x0000),                      # half the smallest subnormal -> 0 (even)
    ((2 - 2.0**-8) * 2.0**127, 0x7F80),       # halfway above the largest finite -> inf
    ((2 - 2.0**-7) * 2.0**127, 0x7F7F),       # the largest finite
    (-0.0, 0x8000),
])
def test_bf16_round_closed_forms(value, bits):
    assert oracle.double_to_bf16(value) == bits


def _e4m3_by_definition(code):
    s, e, m = code >> 7, (code >> 3) & 15, code & 7
    if e == 15 and m == 7:
        return math.nan
    mag = (m / 8) * 2.0**-6 if e == 0 else (1 + m / 8) * 2.0**(e - 7)
    return -mag if s else mag


def test_e4m3_decode_all_codes():
    ref_torch = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    for c in range(256):
        ours = oracle.e4m3_to_double(c)
        spec = _e4m3_by_definition(c)
        if math.isnan(spec):
            assert math.isnan(ours) and math.isnan(ref_torch[c])
        else:
            assert ours == spec == ref_torch[c]
    assert oracle.e4m3_to_double(0x7E) == 448.0
    assert oracle.e4m3_to_double(0x08) == 2.0**-6      # smallest normal
    assert oracle.e4m3_to_double(0x01) == 2.0**-9      # smallest subnormal


def test_e4m3_encode_roundtrip_and_rounding():
    for c in range(256):
        v = _e4m3_by_definition(c)
        if math.isnan(v):
            continue
        got = oracle.float_to_e4m3(v)
        assert _e4m3_by_definition(got) == v
    # saturation and NaN
    assert oracle.float_to_e4m3(448.0) == 0x7E
    assert oracle.float_to_e4m3(464.0) == 0x7E      # RNE would give 512: saturate
    assert oracle.float_to_e4m3(1e30) == 0x7E
    assert oracle.float_to_e4m3(-1e30) == 0xFE
    assert oracle.float_to_e4m3(float("nan")) == 0x7F
    # ties to even: 1 + 1/16 lies between 1 (m=0) and 1.125 (m=1) -> 1
    assert oracle.float_to_e4m3(1.0625) == 0x38
    assert oracle.float_to_e4m3(1.1875) == 0x3A      # between 1.125 and 1.25 -> 1.25 (m=2)
    assert oracle.float_to_e4m3(2.0**-10) == 0x00    # half the smallest subnormal -> 0
    assert oracle.float_to_e4m3(3 * 2.0**-10) == 0x02


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.uniform(-448, 448, 20000),
                        rng.standard_normal(20000) * 2.0**-7]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.float_to_e4m3(float(a)) for a in v], dtype=np.uint8)
    # +0 / -0 codes may differ only in sign for values that round to zero
    same = (ours == ref) | ((ours & 0x7F) == 0) & ((ref & 0x7F) == 0)
    assert same.all()


# ---------------------------------------------------------- a1 router logits


def _small(**kw):
    base = dict(name="pin", T=9, H=128, E=6, k=2, I=128, router_sigma=0.05)
    base.update(kw)
    return Workload(**base)


def test_logits_one_hot_columns():
    w = _small()
    inp = synth.make_inputs(w, with_weights=False)
    H = w.H
    for i in (0, 5, H - 1):
        x = torch.zeros(1, H, dtype=torch.bfloat16)
        x[0, i] = 1.0
        l = oracle.router_logits(x, None, inp["router_w"])
        assert np.array_equal(l[0], inp["router_w"][:, i].numpy())
    b = synth.normal_fp32_tensor(0, 77, (w.E,), 1.0)
    x = torch.zeros(1, H, dtype=torch.bfloat16)
    x[0, 3] = 1.0
    l = oracle.router_logits(x, None, inp["router_w"], b)
    expect = (inp["router_w"][:, 3].double() + b.double()).float().numpy()
    assert np.array_equal(l[0], expect)


def test_logits_match_fp64_matmul():
    w = _small(T=33, H=512, E=48)
    inp = synth.make_inputs(w, with_weights=False)
    x = inp["x"].double().numpy()
    Wr = inp["router_w"].double().numpy()
    ref = (x @ Wr.T).astype(np.float32)
    got = oracle.router_logits(inp["x"], None, inp["router_w"])
    ulp = np.abs(got.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert ulp.max() <= 1


def test_logits_padding_rows_are_zero():
    w = _small()
    inp = synth.make_inputs(w, with_weights=False)
    valid = np.ones(w.T, dtype=np.uint8)
    valid[[1, 4]] = 0
    l = oracle.router_logits(inp["x"], valid, inp["router_w"])
    assert (l[[1, 4]] == 0).all()


# ------------------------------------------------------- a2 top-k + weights


def _brute_topk(l, k):
    order = sorted(range(len(l)), key=lambda e: (-float(l[e]), e))
    return order[:k]


@pytest.mark.parametrize("E,k", [(8, 2), (48, 3), (256, 8), (5, 5)])
def test_topk_brute_force(E, k):
    rng = np.random.default_rng(E * 10 + k)
    l = rng.standard_normal((40, E)).astype(np.float32)
    l[3, :] = 0.25                                # all tied
    l[5, 1::2] = l[5, 0::2][: len(l[5, 1::2])]    # pairwise ties
    l[7, :] = np.round(l[7, :], 1)                # many ties
    ids, w = oracle.topk(l, None, k)
    for t in range(l.shape[0]):
        assert list(ids[t]) == _brute_topk(l[t], k)
        sel = l[t, ids[t]].astype(np.float64)
        assert np.allclose(w[t], scipy.special.softmax(sel), rtol=1e-13, atol=0)
        assert abs(w[t].sum() - 1.0) <= 1e-12


def test_topk_duplicated_router_rows_tie_to_lower_index():
    # identical router rows give identical logits: the lower expert index wins
    w = _small(E=8, k=3)
    inp = synth.make_inputs(w, with_weights=False)
    Wr = inp["router_w"].clone()
    Wr[6] = Wr[2]
    Wr[7] = Wr[2] * 10.0     # make 2, 6 the clear top two for some rows
    l = oracle.router_logits(inp["x"], None, Wr)
    ids, _ = oracle.topk(l, None, 3)
    for t in range(w.T):
        row = list(ids[t])
        if 6 in row:
            assert 2 in row and row.index(2) < row.index(6)


def test_topk_zero_router_gives_uniform():
    l = np.zeros((4, 16), dtype=np.float32)
    ids, w = oracle.topk(l, None, 4)
    assert (ids == np.arange(4)).all()
    assert np.allclose(w, 0.25, rtol=0, atol=1e-15)


def test_topk_k_equals_E_is_full_softmax_and_no_renorm_matches_softmax():
    rng = np.random.default_rng(3)
    l = rng.standard_normal((6, 12)).astype(np.float32) * 3
    ids, w = oracle.topk(l, None, 12)
    full = scipy.special.softmax(l.astype(np.float64), axis=1)
    for t in range(6):
        assert np.allclose(w[t], full[t, ids[t]], rtol=1e-13, atol=0)
    ids2, w2 = oracle.topk(l, None, 3, renorm=False)
    for t in range(6):
        assert np.allclose(w2[t], full[t, ids2[t]], rtol=1e-13, atol=0)
        assert w2[t].sum() < 1.0


def test_topk_padding_rows():
    l = np.ones((3, 8), dtype=np.float32)
    ids, w = oracle.topk(l, np.array([1, 0, 1], np.uint8), 2)
    assert (ids[1] == -1).all() and (w[1] == 0).all()


# ---------------------------------------------------------------- a3 permute


@pytest.mark.parametrize("T,E,k,pad", [(16, 8, 2, 0), (33, 48, 3, 5), (64, 256, 8, 11)])
def test_route_against_stable_sort(T, E, k, pad):
    rng = np.random.default_rng(T)
    l = rng.standard_normal((T, E)).astype(np.float32)
    valid = np.ones(T, dtype=np.uint8)
    valid[rng.choice(T, pad, replace=False)] = 0
    ids, _ = oracle.topk(l, valid, k)
    counts, offsets, perm, inv = oracle.route(ids, valid, E)
    pairs = np.array([t * k + j for t in range(T) if valid[t] for j in range(k)], dtype=np.int64)
    experts = ids.reshape(-1)[pairs]
    ref_perm = pairs[np.argsort(experts, kind="stable")]
    assert np.array_equal(perm, ref_perm)
    assert np.array_equal(counts, np.bincount(experts, minlength=E))
    assert offsets[0] == 0 and np.all(np.diff(offsets) >= 0)
    assert offsets[E] == valid.sum() * k
    # every valid token appears exactly k times; inverse is the inverse
    toks = perm // k
    assert np.array_equal(np.bincount(toks, minlength=T), valid.astype(np.int64) * k)
    assert np.array_equal(inv[perm], np.arange(len(perm)))
    assert (inv.reshape(T, k)[valid == 0] == -1).all()
    # within each expert segment tokens ascend
    for e in range(E):
        seg = toks[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)


# ----------------------------------------------------- a4-a6 expert FFN + combine


def _silu(z):
    return z * scipy.special.expit(z)


def _f64(t):
    return oracle.bf16_to_f64(t).reshape(tuple(t.shape))


def _dense_reference(inp, ids, w):
    """Every expert on every token, non-selected weights zero (numpy matmuls)."""
    wl = inp["workload"]
    x = _f64(inp["x"])
    T = x.shape[0]
    gate = np.zeros((T, wl.E))
    for t in range(T):
        for j in range(ids.shape[1]):
            if ids[t, j] >= 0:
                gate[t, ids[t, j]] += w[t, j]
    Wgu, Wd = _f64(inp["w_gate_up"]), _f64(inp["w_down"])
    out = np.zeros((T, wl.H))
    for e in range(wl.E):
        g = x @ Wgu[e, :wl.I].T
        u = x @ Wgu[e, wl.I:].T
        out += gate[:, e:e + 1] * ((_silu(g) * u) @ Wd[e].T)
    if wl.S:
        Ws, Wsd = _f64(inp["ws_gate_up"]), _f64(inp["ws_down"])
        sh = (_silu(x @ Ws[:wl.Is].T) * (x @ Ws[wl.Is:].T)) @ Wsd.T
        out += sh * (ids[:, :1] >= 0)
    return out


@pytest.mark.parametrize("S", [0, 1])
def test_forward_equals_dense_brute_force(S):
    w = Workload("pin", T=12, H=128, E=6, k=2, I=128, S=S, Is=256 if S else 0,
                 router_sigma=0.3, w_sigma=0.05)
    inp = synth.make_inputs(w)
    r = oracle.forward(inp)
    ref = _dense_reference(inp, r["ids"], r["w"])
    assert np.allclose(r["acc"], ref, rtol=1e-11, atol=1e-13)
    assert np.array_equal(r["out"], oracle.round_bf16(r["acc"]))


def test_single_expert_is_textbook_swiglu_mlp():
    w = Workload("pin", T=7, H=128, E=1, k=1, I=256, w_sigma=0.05)
    inp = synth.make_inputs(w)
    r = oracle.forward(inp)
    assert (r["ids"] == 0).all() and (r["w"] == 1.0).all()
    x = _f64(inp["x"])
    Wgu, Wd = _f64(inp["w_gate_up"])[0], _f64(inp["w_down"])[0]
    h = _silu(x @ Wgu[:256].T) * (x @ Wgu[256:].T)
    assert np.allclose(r["acc"], h @ Wd.T, rtol=1e-11, atol=1e-13)


def test_identity_weights_give_silu_x_times_x():
    H = 128
    w = Workload("pin", T=5, H=H, E=1, k=1, I=H)
    inp = synth.make_inputs(w)
    eye = torch.eye(H, dtype=torch.bfloat16)
    inp["w_gate_up"] = torch.cat([eye, eye], 0)[None]
    inp["w_down"] = eye[None].clone()
    r = oracle.forward(inp)
    x = _f64(inp["x"])
    assert np.allclose(r["acc"], _silu(x) * x, rtol=1e-14, atol=0)


def test_gate_and_up_are_not_swapped():
    # with Wg = I and Wu = 2I the expert gives silu(x) * 2x; swapped it would give silu(2x) * x
    H = 128
    w = Workload("pin", T=4, H=H, E=1, k=1, I=H)
    inp = synth.make_inputs(w)
    eye = torch.eye(H, dtype=torch.bfloat16)
    inp["w_gate_up"] = torch.cat([eye, 2 * eye], 0)[None]
    inp["w_down"] = eye[None].clone()
    r = oracle.forward(inp)
    x = _f64(inp["x"])
    assert np.allclose(r["acc"], _silu(x) * 2 * x, rtol=1e-14, atol=0)


def test_down_projection_orientation():
    # Wd[o, i] maps h[i] to y[o]: a permutation matrix permutes the outputs
    H = 128
    w = Workload("pin", T=3, H=H, E=1, k=1, I=H)
    inp = synth.make_inputs(w)
    eye = torch.eye(H, dtype=torch.bfloat16)
    P = torch.roll(eye, 1, dims=0)                # y[o] = h[o-1]
    inp["w_gate_up"] = torch.cat([eye, eye], 0)[None]
    inp["w_down"] = P[None].clone()
    r = oracle.forward(inp)
    x = _f64(inp["x"])
    assert np.allclose(r["acc"], np.roll(_silu(x) * x, 1, axis=1), rtol=1e-14, atol=0)


def test_linearity_in_down_weights():
    w = Workload("pin", T=6, H=128, E=4, k=2, I=128, S=1, Is=128, w_sigma=0.05)
    inp = synth.make_inputs(w)
    r1 = oracle.forward(inp)
    inp2 = dict(inp)
    inp2["w_down"] = inp["w_down"] * 2
    inp2["ws_down"] = inp["ws_down"] * 2
    r2 = oracle.forward(inp2)
    assert np.array_equal(r2["acc"], 2 * r1["acc"])


def test_token_permutation_equivariance():
    w = Workload("pin", T=10, H=128, E=5, k=2, I=128, router_sigma=0.2)
    inp = synth.make_inputs(w)
    r = oracle.forward(inp)
    p = np.random.default_rng(5).permutation(w.T)
    inp2 = dict(inp)
    inp2["x"] = inp["x"][torch.from_numpy(p)]
    r2 = oracle.forward(inp2)
    assert np.array_equal(r2["out"], r["out"][p])
    assert np.array_equal(r2["ids"], r["ids"][p])


def test_padding_rows_ignored_even_if_nan():
    w = Workload("pin", T=16, H=128, E=6, k=2, I=128, S=1, Is=128, mask="dp_padded",
                 dp_rows=(3, 1, 0, 4))
    a = synth.make_inputs(w, masked_fill="normal")
    b = synth.make_inputs(w, masked_fill="nan")
    ra, rb = oracle.forward(a), oracle.forward(b)
    valid = a["valid"].numpy().astype(bool)
    assert np.array_equal(ra["out"][valid], rb["out"][valid])
    assert (rb["out"][~valid] == 0).all()          # +0.0 bit pattern
    assert (rb["ids"][~valid] == -1).all()
    assert np.array_equal(ra["perm"], rb["perm"])


def test_combine_order_is_weighted_sum():
    # with two experts whose outputs are known in closed form the combine is
    # w0 * y0 + w1 * y1: expert e scales its down projection by (e + 1)
    H = 128
    w = Workload("pin", T=6, H=H, E=2, k=2, I=H, router_sigma=0.3)
    inp = synth.make_inputs(w)
    eye = torch.eye(H, dtype=torch.bfloat16)
    inp["w_gate_up"] = torch.stack([torch.cat([eye, eye], 0)] * 2)
    inp["w_down"] = torch.stack([eye, 2 * eye])
    r = oracle.forward(inp)
    x = _f64(inp["x"])
    base = _silu(x) * x
    scale = np.zeros(w.T)
    for t in range(w.T):
        for j in range(2):
            scale[t] += r["w"][t, j] * (r["ids"][t, j] + 1)
    assert np.allclose(r["acc"], base * scale[:, None], rtol=1e-13, atol=1e-300)


# --------------------------------------------------------------- FP8 path


def _torch_quant_rows(v):
    """1x128 quantisation with torch's cast (library), for comparison."""
    v = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
    g = v.view(v.shape[0], -1, 128)
    amax = g.abs().amax(-1)
    s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    q = (g / s[..., None]).to(torch.float8_e4m3fn)
    return q.view(torch.uint8).reshape(v.shape).numpy(), s.numpy()


def test_activation_quant_matches_torch_cast():
    rng = np.random.default_rng(7)
    v = rng.standard_normal((9, 512)).astype(np.float32)
    v[2, :128] = 0.0                              # zero group -> scale 1
    qt, st = _torch_quant_rows(v)
    for r in range(v.shape[0]):
        q, s = oracle.quant_row_e4m3(v[r])
        assert np.array_equal(s, st[r])
        assert np.array_equal(q, qt[r])
    q, s = oracle.quant_row_e4m3(v[2])
    assert s[0] == 1.0 and (q[:128] == 0).all()


def test_activation_quant_exact_on_grid_and_error_bound():
    # values on the e4m3 grid times 2^m with amax = 448 * 2^m quantise losslessly
    grid = np.array([_e4m3_by_definition(c) for c in range(0x7F)], dtype=np.float64)
    rng = np.random.default_rng(8)
    row = rng.choice(grid, 256) * rng.choice([-1, 1], 256)
    row[0], row[200] = 448.0, -448.0
    row = (row * 2.0**-5).astype(np.float32)
    q, s = oracle.quant_row_e4m3(row)
    assert (s == 2.0**-5).all()
    deq = np.array([oracle.e4m3_to_double(c) for c in q]) * np.repeat(s, 128)
    assert np.array_equal(deq, row.astype(np.float64))
    # general rows: relative error at most 2^-4 in the normal range
    v = rng.standard_normal(1024).astype(np.float32)
    q, s = oracle.quant_row_e4m3(v)
    deq = np.array([oracle.e4m3_to_double(c) for c in q]) * np.repeat(s, 128)
    normal = np.abs(v) >= np.repeat(s, 128) * 2.0**-6
    assert np.all(np.abs(deq - v)[normal] <= 2.0**-4 * np.abs(v[normal]))


def test_fp8_expert_equals_dequantised_matmul():
    """Blockwise-scaled GEMMs reduce to a plain matmul of the dequantised
    operands (the scale is constant inside a 128-block); quantisation steps
    use torch's cast."""
    H, I = 256, 256
    w = Workload("pin", T=5, H=H, E=3, k=2, I=I, S=1, Is=128, wtype="fp8", router_sigma=0.3,
                 w_sigma=0.05)
    inp = synth.make_inputs(w)
    r = oracle.forward(inp)

    def deq_w(q, s):
        vals = torch.from_numpy(q.numpy()).view(torch.float8_e4m3fn).double().numpy()
        return vals * np.kron(s.numpy().astype(np.float64), np.ones((128, 128)))

    def deq_act(v):
        q, s = _torch_quant_rows(v)
        vals = torch.from_numpy(q).view(torch.float8_e4m3fn).double().numpy()
        return vals * np.repeat(s.astype(np.float64), 128, axis=1)

    x = _f64(inp["x"]).astype(np.float32)
    xq = deq_act(x)

    def expert(xrow_q, Wgu, Wd, Iexp):
        g = xrow_q @ Wgu[:Iexp].T
        u = xrow_q @ Wgu[Iexp:].T
        h = (_silu(g) * u).astype(np.float32)
        return deq_act(h) @ Wd.T

    ref = np.zeros((w.T, H))
    for e in range(w.E):
        Wgu = deq_w(inp["w_gate_up"][e], inp["s_gate_up"][e])
        Wd = deq_w(inp["w_down"][e], inp["s_down"][e])
        y = expert(xq, Wgu, Wd, I)
        for t in range(w.T):
            for j in range(w.k):
                if r["ids"][t, j] == e:
                    ref[t] += r["w"][t, j] * y[t]
    Ws = deq_w(inp["ws_gate_up"], inp["ss_gate_up"])
    Wsd = deq_w(inp["ws_down"], inp["ss_down"])
    ref += expert(xq, Ws, Wsd, 128)
    assert np.allclose(r["acc"], ref, rtol=1e-10, atol=1e-12)


def test_fp8_weight_scales_enter_linearly():
    # doubling every down-projection scale doubles the output exactly
    w = Workload("pin", T=4, H=128, E=2, k=1, I=128, wtype="fp8", router_sigma=0.3)
    inp = synth.make_inputs(w)
    r1 = oracle.forward(inp)
    inp2 = dict(inp)
    inp2["s_down"] = inp["s_down"] * 2
    r2 = oracle.forward(inp2)
    assert np.array_equal(r2["acc"], 2 * r1["acc"])
