"""Pins for the oracle's dispatch permute and combine.

Sources: "DODOCO: MoE AlltoAll Traffic Matrices on Real Text", Reading the
counts (payload rows are the hidden states, bf16 on the wire) and
send_matrices.csv (combine returns the same volumes); "Expert Coupling in MoE
Pretraining", Method 1 (a dedup row carries every selected expert of its rank).
Combine = gate-weighted sum, fp32 accumulation in ascending expert order,
rounded to bf16 once.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_warp_top_router_b200 import synth


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _f(bits):
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).float().numpy()


def _case(T, E, k, R, H, seed=0, mode=1):
    lg = synth.group_boost_logits(T, E, 2, 3.0, seed, 1, 5, 6).numpy()
    idx, w = oracle.route_topk(lg, k)
    p = synth.contiguous_placement(E, R).numpy()
    L = oracle.dispatch_layout(idx, E, R, p, mode)
    x = synth.normal_bf16(T, H, seed, 3)
    y = synth.normal_bf16(T * k, H, seed, 4)
    return idx, w, p, L, _bits(x), _bits(y)


@pytest.mark.parametrize("mode", [0, 1])
def test_permute_then_inverse_is_identity(mode):
    T, E, k, R, H = 256, 32, 4, 8, 64
    idx, w, p, L, x, y = _case(T, E, k, R, H, mode=mode)
    out = oracle.dispatch_permute(x, L["row_token"])
    assert out.shape == (L["n_rows"], H)
    for t in range(T):
        for j in range(k):
            assert np.array_equal(out[L["row_of_slot"][t, j]], x[t])


def test_combine_k1_returns_the_expert_row():
    T, E, k, R, H = 128, 16, 1, 4, 32
    idx, w, p, L, x, y = _case(T, E, k, R, H)
    assert np.all(w == 1.0)
    out = oracle.combine(y, L["assign_row"], idx, w)
    assert np.array_equal(out, y[L["assign_row"][:, 0]])


def test_combine_of_copies_with_softmax_gates_is_the_input():
    # every expert returns the token unchanged; the gates sum to 1 within
    # ~1e-7, far below half a bf16 ulp, so the result rounds back to x exactly
    T, E, k, R, H = 200, 32, 6, 8, 48
    idx, w, p, L, x, y = _case(T, E, k, R, H)
    yy = np.zeros((T * k, H), np.uint16)
    for t in range(T):
        for j in range(k):
            yy[L["assign_row"][t, j]] = x[t]
    assert np.array_equal(oracle.combine(yy, L["assign_row"], idx, w), x)


def test_combine_against_float64_sum():
    T, E, k, R, H = 160, 64, 8, 16, 40
    idx, w, p, L, x, y = _case(T, E, k, R, H)
    out = _f(oracle.combine(y, L["assign_row"], idx, w)).astype(np.float64)
    yf = _f(y).astype(np.float64)
    prods = w.astype(np.float64)[:, :, None] * yf[L["assign_row"]]
    ref = prods.sum(1)
    # bound: k fp32 roundings of the running sum + one bf16 rounding
    bound = k * 2.0 ** -24 * np.abs(prods).sum(1) + 2.0 ** -8 * np.abs(ref) + 1e-30
    assert np.all(np.abs(out - ref) <= bound)


def test_combine_order_is_ascending_expert():
    # slot order [5, 1, 3]; expert rows 1.0, -1.0, 2^-30 for experts 1, 3, 5.
    # ascending experts: (1 - 1) + 2^-30 = 2^-30.  slot order would give
    # (2^-30 + 1) - 1 = 0 in float.
    idx = np.array([[5, 1, 3]], np.int32)
    w = np.ones((1, 3), np.float32)
    assign = np.array([[0, 1, 2]], np.int32)
    vals = torch.tensor([2.0 ** -30, 1.0, -1.0]).to(torch.bfloat16)
    y = np.repeat(_bits(vals)[:, None], 4, axis=1)
    out = _f(oracle.combine(y, assign, idx, w))
    assert np.all(out == np.float32(2.0 ** -30))


def test_combine_rounding_matches_torch_bf16():
    # k = 1 with arbitrary gates: out = bf16(fp32(w * y)); torch rounds the same
    # fp32 products to nearest-even, including exact ties
    T, H = 64, 32
    rng = np.random.default_rng(0)
    w = rng.standard_normal((T, 1)).astype(np.float32)
    w[0, 0] = 1.0 + 2.0 ** -8          # tie at 1.0: rounds down to even
    w[1, 0] = 1.0 + 3 * 2.0 ** -8      # tie: rounds up to even 1 + 2^-6
    y = _bits(synth.normal_bf16(T, H, 0, 4))
    y[0:2] = _bits(torch.ones(2, H, dtype=torch.bfloat16))
    idx = np.zeros((T, 1), np.int32)
    assign = np.arange(T, dtype=np.int32)[:, None]
    out = oracle.combine(y, assign, idx, w)
    ref = (torch.from_numpy(w) * torch.from_numpy(_f(y))).to(torch.bfloat16)
    assert np.array_equal(out, _bits(ref))
    assert _f(out)[0, 0] == 1.0 and _f(out)[1, 0] == 1.0 + 2.0 ** -6


def test_wire_with_one_rank_equals_fused():
    T, E, k, R, H = 96, 16, 4, 1, 24
    idx, w, p, L, x, y = _case(T, E, k, R, H)
    fused = oracle.combine(y, L["assign_row"], idx, w)
    wire, z = oracle.combine(y, L["assign_row"], idx, w, oracle.COMBINE_WIRE, p,
                             L["row_of_slot"], L["n_rows"])
    assert np.array_equal(fused, wire)
    assert np.array_equal(z, fused)  # one row per token, in token order


def test_wire_with_one_expert_per_rank():
    # each wire row holds one rounded product; stage 2 adds them in
    # ascending rank (= ascending expert) order in float
    T, E, k, H = 80, 8, 3, 16
    R = E
    idx, w, p, L, x, y = _case(T, E, k, R, H)
    wire, z = oracle.combine(y, L["assign_row"], idx, w, oracle.COMBINE_WIRE, p,
                             L["row_of_slot"], L["n_rows"])
    prod = torch.from_numpy(w)[:, :, None] * torch.from_numpy(_f(y)[L["assign_row"]])
    zb = prod.to(torch.bfloat16)
    for t in range(T):
        for j in range(k):
            assert np.array_equal(z[L["row_of_slot"][t, j]], _bits(zb[t, j]))
    order = np.argsort(idx, axis=1)
    acc = torch.zeros(T, H)
    for i in range(k):
        acc = acc + zb[torch.arange(T), torch.from_numpy(order[:, i])].float()
    assert np.array_equal(wire, _bits(acc.to(torch.bfloat16)))


# ---------------------------------------------------------------- dedup expand
# "Expert Coupling in MoE Pretraining", Method 1: the deduplicating dispatcher
# delivers the same rows as the conventional one, once per (token, rank); the
# receiver copies each into one row per selected expert.  So expanding the
# dedup dispatch buffer must give the conventional dispatch buffer exactly.

@pytest.mark.parametrize("T,E,k,R", [(256, 32, 4, 8), (160, 64, 6, 16), (64, 16, 8, 2), (96, 8, 1, 4)])
def test_expand_of_dedup_dispatch_is_conventional_dispatch(T, E, k, R):
    lg = synth.group_boost_logits(T, E, 2, 3.0, 1, 1, 5, 6).numpy()
    idx, _ = oracle.route_topk(lg, k)
    p = np.random.default_rng(T + E).permutation(synth.contiguous_placement(E, R).numpy()).astype(np.int32)
    Ld = oracle.dispatch_layout(idx, E, R, p, 1)
    Lc = oracle.dispatch_layout(idx, E, R, p, 0)
    x = _bits(synth.normal_bf16(T, 24, 2, 3))
    wire = oracle.dispatch_permute(x, Ld["row_token"])
    conv = oracle.dispatch_permute(x, Lc["row_token"])
    # the dedup layout's assign_row is the conventional position of each slot
    assert np.array_equal(Ld["assign_row"], Lc["row_of_slot"])
    out = oracle.dedup_expand(wire, Ld["row_of_slot"], Ld["assign_row"])
    assert np.array_equal(out, conv)


def test_expand_hand_example():
    # two tokens, k=2; token 0 -> rows (wire 0, wire 0) to conv rows 2, 0;
    # token 1 -> (wire 1, wire 2) to conv rows 1, 3
    wire = np.array([[1, 2], [3, 4], [5, 6]], np.uint16)
    rs = np.array([[0, 0], [1, 2]], np.int32)
    ar = np.array([[2, 0], [1, 3]], np.int32)
    out = oracle.dedup_expand(wire, rs, ar)
    assert out.tolist() == [[1, 2], [3, 4], [1, 2], [5, 6]]


def test_expand_rejects_bad_rows():
    wire = np.zeros((2, 4), np.uint16)
    with pytest.raises(ValueError):
        oracle.dedup_expand(wire, np.array([[0, 2]], np.int32), np.array([[0, 1]], np.int32))
    with pytest.raises(ValueError):
        oracle.dedup_expand(wire, np.array([[0, 1]], np.int32), np.array([[0, 2]], np.int32))
