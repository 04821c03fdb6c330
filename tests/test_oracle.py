"""Pins for the FP64 oracle (CPU only).

Every check here compares the oracle with something other than itself:
closed forms derived by hand, torch library routines on a differently written
dense formulation (tests/dense_reference.py), invariants the mathematics fixes,
and finite differences of the oracle's own forward for its backward.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from learned_relative_gqa_b200 import workloads as W
from tests import dense_reference as ref


# --------------------------------------------------------------------------
# helpers
# --------------------------------------------------------------------------
def tiny_workload(name="tiny", B=2, S=24, Hq=4, Hkv=2, D=8, window=0, R=16, docs=(3, 9), pad=(0, 4),
                  seq_k=None, query_offset=0):
    return W.Workload(name, B, S, Hq, Hkv, D, window, R, docs=docs, pad=pad, backward=True,
                      seq_k=seq_k, query_offset=query_offset)


def f64_inputs(w, seed=None):
    x = W.make_inputs(w, "cpu", seed=seed, with_dout=True)
    out = dict(
        q=x["q"].double(), k=x["k"].double(), v=x["v"].double(), profiles=x["profiles"].double(),
        sink=x["sink"].double(), dout=x["dout"].double(),
        valid=x["valid"], key_valid=x["key_valid"], positions=x["positions"],
        key_positions=x["key_positions"], window=x["window"], query_offset=x["query_offset"])
    return out


def run_oracle_fwd(x, **kw):
    return oracle.forward(x["q"].numpy(), x["k"].numpy(), x["v"].numpy(), x["profiles"].numpy(),
                          x["sink"].numpy(), x["valid"].numpy(), x["key_valid"].numpy(),
                          x["positions"].numpy(), x["key_positions"].numpy(),
                          window=kw.get("window", x["window"]), query_offset=x["query_offset"],
                          window_inclusive=kw.get("window_inclusive", False))


def run_oracle_bwd(x, dlse=None):
    return oracle.backward(x["q"].numpy(), x["k"].numpy(), x["v"].numpy(), x["profiles"].numpy(),
                           x["sink"].numpy(), x["valid"].numpy(), x["key_valid"].numpy(),
                           x["positions"].numpy(), x["key_positions"].numpy(),
                           dout=x["dout"].numpy(), dlse=dlse, window=x["window"],
                           query_offset=x["query_offset"])


def mask_of(x):
    return ref.allowed_mask(x["valid"], x["key_valid"], x["positions"], x["key_positions"],
                            window=x["window"], query_offset=x["query_offset"],
                            heads_q=x["q"].shape[2])


GOLDEN = json.load(open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_closed_form.json")))


def tiny_case(R, sink1=None):
    """The hand-worked case: B=1, S=2, H=1, D=1 (scale 1), positions [0,1]."""
    s1 = np.float32(math.log(2.0)) if sink1 is None else sink1
    return dict(
        q=np.array([1.0, 1.0]).reshape(1, 2, 1, 1), k=np.array([1.0, 0.0]).reshape(1, 2, 1, 1),
        v=np.array([2.0, 4.0]).reshape(1, 2, 1, 1),
        profiles=np.array([[0.5, 0.0], [0.0, 1.0]])[:, :R].reshape(1, 1, 2, R),
        sink=np.array([0.0, float(s1)]).reshape(1, 2, 1), valid=np.ones((1, 2), np.uint8))


# --------------------------------------------------------------------------
# 1. closed forms worked by hand
# --------------------------------------------------------------------------
def test_tiny_closed_form_forward():
    c = tiny_case(2)
    out, lse, lsec = oracle.forward(c["q"], c["k"], c["v"], c["profiles"], c["sink"], c["valid"])
    s1 = float(np.float32(math.log(2.0)))
    # row 0 sees key 0 only: z = 1*1 + profiles[0,0]=0.5
    z00 = 1.5
    lse0 = math.log(1.0 + math.exp(z00))
    out0 = 2.0 * math.exp(z00 - lse0)
    # row 1 sees key 0 (d=1: z = 1*1 + profiles[1,1]=1) and key 1 (d=0: z = 0 + profiles[1,0]=0)
    z10, z11 = 2.0, 0.0
    lse1 = math.log(math.exp(s1) + math.exp(z10) + math.exp(z11))
    out1 = (2.0 * math.exp(z10) + 4.0 * math.exp(z11)) / math.exp(lse1)
    np.testing.assert_allclose(out.ravel(), [out0, out1], rtol=1e-13)
    np.testing.assert_allclose(lse.ravel(), [lse0, lse1], rtol=1e-13)
    np.testing.assert_allclose(lsec.ravel(), [z00, math.log(math.exp(z10) + math.exp(z11))], rtol=1e-13)
    # the values quoted in the hand derivation, and the stored fixture of the same case
    np.testing.assert_allclose(out.ravel(), [1.635148952, 1.807489729], atol=2e-9)
    np.testing.assert_allclose(lse.ravel(), [1.701413278, 2.340752954], atol=2e-9)
    np.testing.assert_allclose(out.ravel(), GOLDEN["R2"]["out"], rtol=1e-13)
    np.testing.assert_allclose(lse.ravel(), GOLDEN["R2"]["lse"], rtol=1e-13)


def test_tiny_closed_form_no_bias_beyond_extent():
    c = tiny_case(1)  # R = 1: distance 1 gets no bias
    out, lse, _ = oracle.forward(c["q"], c["k"], c["v"], c["profiles"], c["sink"], c["valid"])
    s1 = float(np.float32(math.log(2.0)))
    z10, z11 = 1.0, 0.0
    lse1 = math.log(math.exp(s1) + math.exp(z10) + math.exp(z11))
    out1 = (2.0 * math.exp(z10) + 4.0 * math.exp(z11)) / math.exp(lse1)
    np.testing.assert_allclose(out.ravel()[1], out1, rtol=1e-13)
    np.testing.assert_allclose(lse.ravel()[1], lse1, rtol=1e-13)
    np.testing.assert_allclose([out.ravel()[1], lse.ravel()[1]], [1.650244591, 1.743668381], atol=2e-9)
    np.testing.assert_allclose([out.ravel()[1], lse.ravel()[1]], [GOLDEN["R1_row1"]["out"], GOLDEN["R1_row1"]["lse"]],
                               rtol=1e-13)


def test_tiny_closed_form_plain_causal_softmax():
    c = tiny_case(2)
    c["profiles"] = np.zeros_like(c["profiles"])
    c["sink"] = np.full_like(c["sink"], -np.inf)
    out, lse, _ = oracle.forward(c["q"], c["k"], c["v"], c["profiles"], c["sink"], c["valid"])
    # row 1: logits 1 and 0 -> weights e/(e+1), 1/(e+1)
    e = math.e
    np.testing.assert_allclose(out.ravel(), [2.0, (2 * e + 4) / (e + 1)], rtol=1e-13)
    np.testing.assert_allclose(lse.ravel(), [1.0, math.log(e + 1)], rtol=1e-13)
    np.testing.assert_allclose(out.ravel(), GOLDEN["plain_causal_zero_profiles_no_sink"]["out"], rtol=1e-13)
    np.testing.assert_allclose(lse.ravel(), GOLDEN["plain_causal_zero_profiles_no_sink"]["lse"], rtol=1e-13)


def test_tiny_closed_form_backward():
    c = tiny_case(2)
    dout = np.ones((1, 2, 1, 1))
    g = oracle.backward(c["q"], c["k"], c["v"], c["profiles"], c["sink"], c["valid"], dout=dout)
    s1 = float(np.float32(math.log(2.0)))
    # row 0
    P00 = math.exp(1.5) / (1 + math.exp(1.5))
    ps0 = 1 / (1 + math.exp(1.5))
    out0 = 2 * P00
    dS00 = P00 * (2.0 - out0)
    # row 1
    Z1 = math.exp(s1) + math.exp(2.0) + 1.0
    P10, P11, ps1 = math.exp(2.0) / Z1, 1.0 / Z1, math.exp(s1) / Z1
    out1 = 2 * P10 + 4 * P11
    dS10, dS11 = P10 * (2.0 - out1), P11 * (4.0 - out1)
    np.testing.assert_allclose(g["dsink"].ravel(), [-ps0 * out0, -ps1 * out1], rtol=1e-12)
    np.testing.assert_allclose(g["dprofiles"].ravel(), [dS00, 0.0, dS11, dS10], rtol=1e-12, atol=1e-15)
    # dq_i = scale * sum_j dS_ij k_j, k = [1, 0]
    np.testing.assert_allclose(g["dq"].ravel(), [dS00, dS10], rtol=1e-12)
    # dk_j = scale * sum_i dS_ij q_i, q = [1, 1]
    np.testing.assert_allclose(g["dk"].ravel(), [dS00 + dS10, dS11], rtol=1e-12)
    # dv_j = sum_i P_ij dout_i
    np.testing.assert_allclose(g["dv"].ravel(), [P00 + P10, P11], rtol=1e-12)
    # the values quoted in the hand derivation
    np.testing.assert_allclose(g["dsink"].ravel(), [-0.298292904, -0.347960337], atol=2e-9)
    # dprofiles[0,0], dprofiles[1,1] (d=1: key 0), dprofiles[1,0] (d=0: key 1)
    dp = g["dprofiles"].reshape(2, 2)
    np.testing.assert_allclose([dp[0, 0], dp[1, 1], dp[1, 0]], [0.298292904, 0.136919964, 0.211040373],
                               atol=2e-9)
    gb = GOLDEN["R2_backward_dout_ones"]
    np.testing.assert_allclose(g["dsink"].ravel(), gb["dsink"], rtol=1e-12)
    np.testing.assert_allclose([dp[0, 0], dp[1, 1], dp[1, 0]], gb["dprofiles_00_11_10"], rtol=1e-12)


def test_empty_row_gives_zero_output_and_sink_lse():
    c = tiny_case(2)
    c["valid"] = np.array([[0, 1]], np.uint8)
    out, lse, lsec = oracle.forward(c["q"], c["k"], c["v"], c["profiles"], c["sink"], c["valid"],
                                    key_valid=np.ones((1, 2), np.uint8))
    assert out.ravel()[0] == 0.0 and lse.ravel()[0] == c["sink"].ravel()[0]
    assert lsec.ravel()[0] == -np.inf
    # row 1 now only sees key 1 (key 0 is a valid key but the row-0 query is invalid; keys stay valid)
    s1 = float(np.float32(math.log(2.0)))
    lse1 = math.log(math.exp(s1) + math.exp(2.0) + 1.0)
    np.testing.assert_allclose(lse.ravel()[1], lse1, rtol=1e-13)


# --------------------------------------------------------------------------
# 2. reductions to library routines on a differently written formulation
# --------------------------------------------------------------------------
SHAPES = [
    dict(B=2, S=24, Hq=4, Hkv=2, D=8, window=0, R=16, docs=(3, 9), pad=(0, 4)),
    dict(B=1, S=33, Hq=6, Hkv=2, D=4, window=7, R=5, docs=(4, 20), pad=(0, 3)),
    dict(B=2, S=17, Hq=2, Hkv=2, D=8, window=0, R=40, docs=None, pad=(0, 6)),
    dict(B=1, S=20, Hq=4, Hkv=1, D=8, window=5, R=8, docs=(5, 8), pad=None),
]


@pytest.mark.parametrize("shape", SHAPES)
def test_matches_sdpa_with_materialised_bias_and_sink(shape):
    x = f64_inputs(tiny_workload(**shape))
    out, lse, _ = run_oracle_fwd(x)
    m = mask_of(x)
    o_sdpa = ref.sdpa_forward(x["q"], x["k"], x["v"], x["profiles"], x["sink"], m)
    o_ref, lse_ref = ref.forward(x["q"], x["k"], x["v"], x["profiles"], x["sink"], m)
    np.testing.assert_allclose(out, o_sdpa.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(out, o_ref.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("shape", SHAPES[:2])
def test_zero_profiles_and_no_sink_is_plain_masked_gqa(shape):
    import torch.nn.functional as F
    x = f64_inputs(tiny_workload(**shape))
    x["profiles"] = torch.zeros_like(x["profiles"])
    x["sink"] = torch.full_like(x["sink"], float("-inf"))
    out, lse, _ = run_oracle_fwd(x)
    m = mask_of(x)
    B, S, Hq, D = x["q"].shape
    G = Hq // x["k"].shape[2]
    rows_with_keys = m.any(-1)                                     # [B,Hq,S]
    qq = x["q"].permute(0, 2, 1, 3)
    kk = x["k"].repeat_interleave(G, 2).permute(0, 2, 1, 3)
    vv = x["v"].repeat_interleave(G, 2).permute(0, 2, 1, 3)
    o = F.scaled_dot_product_attention(qq, kk, vv, attn_mask=m | ~rows_with_keys.unsqueeze(-1))
    o = torch.where(rows_with_keys.unsqueeze(-1), o, torch.zeros((), dtype=o.dtype)).permute(0, 2, 1, 3)
    np.testing.assert_allclose(out, o.numpy(), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("with_dlse", [False, True])
@pytest.mark.parametrize("shape", SHAPES)
def test_backward_matches_autograd(shape, with_dlse):
    x = f64_inputs(tiny_workload(**shape))
    m = mask_of(x)
    leaves = {n: x[n].clone().requires_grad_(True) for n in ("q", "k", "v", "profiles", "sink")}
    o, l = ref.forward(leaves["q"], leaves["k"], leaves["v"], leaves["profiles"], leaves["sink"], m)
    gen = torch.Generator().manual_seed(7)
    dlse = torch.randn(l.shape, generator=gen, dtype=torch.float64) if with_dlse else None
    loss = (o * x["dout"]).sum() + ((l * dlse).sum() if with_dlse else 0.0)
    loss.backward()
    g = run_oracle_bwd(x, dlse=None if dlse is None else dlse.numpy())
    for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("profiles", "dprofiles"), ("sink", "dsink")):
        np.testing.assert_allclose(g[key], leaves[name].grad.numpy(), rtol=1e-10, atol=1e-12,
                                   err_msg=key)


def test_backward_finite_differences():
    w = tiny_workload(B=1, S=10, Hq=2, Hkv=1, D=3, window=6, R=5, docs=(3, 7), pad=(0, 2))
    x = f64_inputs(w)
    gen = torch.Generator().manual_seed(3)
    dlse = torch.randn(x["sink"].shape, generator=gen, dtype=torch.float64).numpy()
    g = run_oracle_bwd(x, dlse=dlse)
    dout = x["dout"].numpy()

    def loss(xx):
        o, l, _ = run_oracle_fwd(xx)
        return float((o * dout).sum() + (l * dlse).sum())

    h = 1e-6
    rng = np.random.default_rng(0)
    for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("profiles", "dprofiles"), ("sink", "dsink")):
        base = x[name]
        flat = base.reshape(-1)
        idxs = rng.choice(flat.numel(), size=min(12, flat.numel()), replace=False)
        for t in idxs:
            plus = {**x, name: base.clone()}
            minus = {**x, name: base.clone()}
            plus[name].view(-1)[t] += h
            minus[name].view(-1)[t] -= h
            fd = (loss(plus) - loss(minus)) / (2 * h)
            an = g[key].reshape(-1)[t]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (key, int(t), fd, an)


# --------------------------------------------------------------------------
# 3. invariants
# --------------------------------------------------------------------------
def test_probabilities_and_sink_mass_sum_to_one():
    x = f64_inputs(tiny_workload(**SHAPES[0]))
    x["v"] = torch.ones_like(x["v"])
    out, lse, _ = run_oracle_fwd(x)
    sink_mass = np.exp(x["sink"].numpy() - lse)                 # [B,S,Hq]
    valid = x["valid"].numpy().astype(bool)
    total = out[..., 0] + sink_mass
    np.testing.assert_allclose(total[valid], 1.0, rtol=1e-12)


def test_gradient_row_sums_vanish():
    # sum_j dz_ij + dsink_i = 0 for each row (softmax Jacobian rows sum to zero); without
    # dlse this shows up in the oracle as sum_d dprofiles + dsink = 0 when R covers every
    # allowed distance
    w = tiny_workload(B=1, S=16, Hq=2, Hkv=1, D=4, window=0, R=16, docs=(4, 12), pad=(0, 2))
    x = f64_inputs(w)
    g = run_oracle_bwd(x)
    rowsum = g["dprofiles"].sum(-1).transpose(0, 2, 1) + g["dsink"]
    np.testing.assert_allclose(rowsum, 0.0, atol=1e-12)


def test_lse_is_logaddexp_of_content_and_sink():
    x = f64_inputs(tiny_workload(**SHAPES[1]))
    _, lse, lsec = run_oracle_fwd(x)
    np.testing.assert_allclose(lse, np.logaddexp(lsec, x["sink"].numpy()), rtol=1e-13)


def test_masked_and_invalid_keys_get_zero_weight():
    x = f64_inputs(tiny_workload(**SHAPES[0]))
    out, lse, _ = run_oracle_fwd(x)
    m = mask_of(x)
    used = m.any(dim=1).any(dim=1)                               # [B,Skv] keys allowed somewhere
    y = dict(x)
    gen = torch.Generator().manual_seed(11)
    noise_k = torch.randn(x["k"].shape, generator=gen, dtype=torch.float64) * 50
    noise_v = torch.randn(x["v"].shape, generator=gen, dtype=torch.float64) * 50
    unused = (~used).view(*used.shape, 1, 1)
    y["k"] = torch.where(unused, x["k"] + noise_k, x["k"])
    y["v"] = torch.where(unused, x["v"] + noise_v, x["v"])
    out2, lse2, _ = run_oracle_fwd(y)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)
    assert (~used).any()


def test_invalid_query_rows_do_not_affect_valid_rows():
    x = f64_inputs(tiny_workload(**SHAPES[0]))
    out, lse, _ = run_oracle_fwd(x)
    inval = ~x["valid"].bool()
    assert inval.any()
    y = dict(x)
    y["q"] = torch.where(inval.view(*inval.shape, 1, 1), x["q"] * -3 + 1, x["q"])
    y["positions"] = torch.where(inval, torch.full_like(x["positions"], 5), x["positions"])
    out2, lse2, _ = run_oracle_fwd(y)
    val = x["valid"].numpy().astype(bool)
    assert np.array_equal(out[val], out2[val]) and np.array_equal(lse[val], lse2[val])
    assert np.all(out2[~val] == 0.0)
    np.testing.assert_array_equal(lse2[~val], x["sink"].numpy()[~val])


def test_packed_documents_are_isolated():
    # one row holding documents A | B equals running A and B as separate rows
    w = tiny_workload(B=1, S=20, Hq=2, Hkv=1, D=4, window=0, R=12, docs=None, pad=None)
    x = f64_inputs(w)
    cut = 8
    pos = torch.cat([torch.arange(cut), torch.arange(20 - cut)]).to(torch.int32).view(1, 20)
    x["positions"] = pos
    x["key_positions"] = pos
    out, lse, _ = run_oracle_fwd(x)
    for lo, hi in ((0, cut), (cut, 20)):
        part = dict(x)
        for n in ("q", "k", "v", "dout"):
            part[n] = x[n][:, lo:hi].contiguous()
        part["profiles"] = x["profiles"][:, :, lo:hi].contiguous()
        part["sink"] = x["sink"][:, lo:hi].contiguous()
        for n in ("valid", "key_valid", "positions", "key_positions"):
            part[n] = x[n][:, lo:hi].contiguous()
        o2, l2, _ = run_oracle_fwd(part)
        np.testing.assert_allclose(out[:, lo:hi], o2, rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(lse[:, lo:hi], l2, rtol=1e-13)


def test_window_at_least_sequence_equals_no_window():
    x = f64_inputs(tiny_workload(**SHAPES[0]))
    S = x["q"].shape[1]
    a = run_oracle_fwd(x, window=0)
    b = run_oracle_fwd(x, window=S)
    c = run_oracle_fwd(x, window=3)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert not np.allclose(a[0], c[0])


def test_window_bound_readings_differ_by_one_key():
    # the oracle's reading admits i_g - j < W; the generic module's "<= W" admits one key more
    x = f64_inputs(tiny_workload(B=1, S=16, Hq=2, Hkv=1, D=4, window=4, R=8, docs=None, pad=None))
    o_lt, _, _ = run_oracle_fwd(x, window=4)
    o_le, _, _ = run_oracle_fwd(x, window=4, window_inclusive=True)
    o_lt5, _, _ = run_oracle_fwd(x, window=5)
    assert np.array_equal(o_le, o_lt5)
    assert not np.allclose(o_lt, o_le)


def test_gqa_equals_mha_with_replicated_kv():
    x = f64_inputs(tiny_workload(**SHAPES[1]))
    G = x["q"].shape[2] // x["k"].shape[2]
    y = dict(x)
    y["k"] = x["k"].repeat_interleave(G, 2).contiguous()
    y["v"] = x["v"].repeat_interleave(G, 2).contiguous()
    a = run_oracle_fwd(x)
    b = run_oracle_fwd(y)
    np.testing.assert_allclose(a[0], b[0], rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(a[1], b[1], rtol=1e-14)


def test_shift_of_profiles_and_sink_moves_only_lse():
    # with R beyond every allowed distance, adding c to a row's profiles and sink adds c
    # to every logit of that row: out is unchanged and lse moves by c
    w = tiny_workload(B=1, S=18, Hq=2, Hkv=1, D=4, window=0, R=18, docs=(4, 10), pad=None)
    x = f64_inputs(w)
    c = 1.75
    y = dict(x)
    y["profiles"] = x["profiles"] + c
    y["sink"] = x["sink"] + c
    a = run_oracle_fwd(x)
    b = run_oracle_fwd(y)
    np.testing.assert_allclose(a[0], b[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(b[1], a[1] + c, rtol=1e-13)


def test_large_sink_drives_output_to_zero():
    x = f64_inputs(tiny_workload(**SHAPES[0]))
    y = dict(x)
    y["sink"] = torch.full_like(x["sink"], 200.0)
    out, lse, _ = run_oracle_fwd(y)
    assert np.max(np.abs(out)) < 1e-60
    np.testing.assert_allclose(lse, 200.0, rtol=1e-14)


def test_query_slice_with_offset_equals_full_rows():
    # a local query slice at query_offset with global keys reproduces the full rows
    w = tiny_workload(B=2, S=30, Hq=4, Hkv=2, D=8, window=9, R=12, docs=(5, 14), pad=(0, 3))
    full = f64_inputs(w)
    o_full, l_full, _ = run_oracle_fwd(full)
    off, S = 11, 13
    part = dict(full)
    for n in ("q", "dout"):
        part[n] = full[n][:, off:off + S].contiguous()
    part["profiles"] = full["profiles"][:, :, off:off + S].contiguous()
    part["sink"] = full["sink"][:, off:off + S].contiguous()
    part["valid"] = full["valid"][:, off:off + S].contiguous()
    part["positions"] = full["positions"][:, off:off + S].contiguous()
    part["query_offset"] = off
    o, l, _ = run_oracle_fwd(part)
    np.testing.assert_allclose(o, o_full[:, off:off + S], rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(l, l_full[:, off:off + S], rtol=1e-14)


def test_document_test_agrees_with_doc_ids():
    # the oracle's same-document test (position difference == column difference) selects
    # exactly the pairs the doc-id formulation selects
    for seed in range(4):
        w = tiny_workload(B=2, S=40, Hq=2, Hkv=1, D=4, window=0, R=64, docs=(1, 9), pad=(0, 5))
        x = f64_inputs(w, seed=seed + 50)
        x["v"] = torch.ones_like(x["v"])
        x["profiles"] = torch.zeros_like(x["profiles"])
        x["q"] = torch.zeros_like(x["q"])
        x["sink"] = torch.full_like(x["sink"], float("-inf"))
        _, _, lsec = run_oracle_fwd(x)
        m = mask_of(x)
        count = m.sum(-1).permute(0, 2, 1).numpy()            # [B,S,Hq]
        with np.errstate(divide="ignore"):
            np.testing.assert_allclose(lsec, np.log(count), rtol=1e-13)


def test_sampled_backward_matches_full():
    w = tiny_workload(B=2, S=20, Hq=4, Hkv=2, D=4, window=6, R=8, docs=(3, 9), pad=(0, 3))
    x = f64_inputs(w)
    full = run_oracle_bwd(x)
    rows = np.array([0, 5, 17, 40, 77, 159])
    keys = np.array([0, 3, 11, 28, 39, 79])
    s = oracle.backward_sampled(x["q"].numpy(), x["k"].numpy(), x["v"].numpy(), x["profiles"].numpy(),
                                x["sink"].numpy(), x["valid"].numpy(), x["key_valid"].numpy(),
                                x["positions"].numpy(), x["key_positions"].numpy(),
                                dout=x["dout"].numpy(), rows=rows, keys=keys, window=x["window"])
    Hq, Hkv = 4, 2
    for r in rows:
        b, i, h = r // (20 * Hq), (r // Hq) % 20, r % Hq
        np.testing.assert_array_equal(s["dq"][b, i, h], full["dq"][b, i, h])
        np.testing.assert_array_equal(s["dprofiles"][b, h, i], full["dprofiles"][b, h, i])
        assert s["dsink"][b, i, h] == full["dsink"][b, i, h]
    for r in keys:
        b, j, g = r // (20 * Hkv), (r // Hkv) % 20, r % Hkv
        np.testing.assert_allclose(s["dk"][b, j, g], full["dk"][b, j, g], rtol=1e-14, atol=1e-16)
        np.testing.assert_allclose(s["dv"][b, j, g], full["dv"][b, j, g], rtol=1e-14, atol=1e-16)


def test_decode_bf16_is_exact():
    t = torch.randn(1000).to(torch.bfloat16)
    dec = oracle.decode_bf16(t.view(torch.int16).numpy())
    np.testing.assert_array_equal(dec, t.double().numpy())
