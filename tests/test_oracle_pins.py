"""Pins of the CPU oracle against things other than itself.

Each test ties one oracle function to a value the pages print, a closed form, a library
routine on a special case, or brute force, chosen so that a dropped term, a wrong sign or
index, or a transposed operand in the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from sparse_fp32_softmax_b200 import inputs
from sparse_fp32_softmax_b200.roofline import moe_parameter_split

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def logits_of(probs):
    """FP32 logits whose softmax is ``probs`` (up to FP32 rounding of the logarithm)."""
    return np.log(np.asarray(probs, np.float64)).astype(np.float32)[None, :]


# ------------------------------------------------------------------ router: pages' values

def test_worked_example(oracle_mod):
    g = golden("worked_example.json")
    l = logits_of(g["probs"])
    idx, w = oracle_mod.select(l, g["k"], norm=True)
    assert idx[0].tolist() == g["experts"]
    assert np.abs(w[0] - np.array(g["weights_renorm"])).max() <= 1e-6
    idx, w = oracle_mod.select(l, g["k"], norm=False)
    assert idx[0].tolist() == g["experts"]
    assert np.abs(w[0] - np.array(g["weights_plain"])).max() <= 1e-6


def test_renorm_example(oracle_mod):
    g = golden("renorm_example.json")
    idx, w = oracle_mod.select(logits_of(g["probs"]), g["k"], norm=True)
    assert idx[0].tolist() == g["experts"]
    assert np.abs(w[0] - np.array(g["weights_renorm"])).max() <= 1e-6
    # the page's printed rounding of the same values
    assert sorted(np.floor(w[0] * 100) / 100) == sorted(g["printed_rounded"])


def test_worked_example_k3_index_tiebreak(oracle_mod):
    # Same probabilities, k = 3: experts 0 and 3 tie at 0.1; the lower index wins.
    idx, w = oracle_mod.select(logits_of([0.1, 0.5, 0.3, 0.1]), 3, norm=True)
    assert idx[0].tolist() == [1, 2, 0]
    assert np.abs(w[0] - np.array([5 / 9, 1 / 3, 1 / 9])).max() <= 1e-6
    assert abs(float(w[0].sum()) - 1.0) <= 1e-6


# ------------------------------------------------------------------ router: closed forms

def test_softmax_closed_form(oracle_mod):
    l = np.array([[0.0, math.log(2.0), math.log(3.0)]], np.float32)
    idx, w = oracle_mod.select(l, 3, norm=False)
    assert idx[0].tolist() == [2, 1, 0]
    assert np.abs(w[0] - np.array([3 / 6, 2 / 6, 1 / 6])).max() <= 1e-7


def test_softmax_matches_library_when_k_equals_E(oracle_mod):
    from scipy.special import softmax
    rng = np.random.default_rng(5)
    l = rng.normal(size=(7, 13)).astype(np.float32)
    for norm in (False, True):
        idx, w = oracle_mod.select(l, 13, norm=norm)
        ref = softmax(l.astype(np.float64), axis=1)
        got = np.zeros_like(ref)
        np.put_along_axis(got, idx.astype(np.int64), w.astype(np.float64), axis=1)
        assert np.abs(got - ref).max() <= 1e-7          # renorm of the full set is a no-op
        order = np.argsort(-l, axis=1, kind="stable")    # library stable sort, lower index first
        assert (idx == order).all()


def test_k1_renorm_is_exactly_one(oracle_mod):
    rng = np.random.default_rng(6)
    l = rng.normal(size=(9, 6)).astype(np.float32)
    idx, w = oracle_mod.select(l, 1, norm=True)
    assert (w == 1.0).all()
    assert (idx[:, 0] == np.argmax(l, axis=1)).all()


def test_renorm_sums_to_one(oracle_mod):
    rng = np.random.default_rng(7)
    l = rng.normal(size=(50, 64)).astype(np.float32)
    _, w = oracle_mod.select(l, 8, norm=True)
    assert np.abs(w.astype(np.float64).sum(1) - 1.0).max() <= 1e-6


@pytest.mark.parametrize("k", [1, 2, 3])
def test_index_tiebreak(oracle_mod, k):
    l = np.array([[1.0, 3.0, 3.0, 0.0, 3.0]], np.float32)
    idx, _ = oracle_mod.select(l, k, norm=True)
    assert idx[0].tolist() == [1, 2, 4][:k]
    z = np.zeros((1, 6), np.float32)
    idx, w = oracle_mod.select(z, 4, norm=True)
    assert idx[0].tolist() == [0, 1, 2, 3]
    assert np.abs(w - 0.25).max() == 0.0
    # -0.0 and +0.0 are the same value: the lower index ranks first
    s = np.array([[-0.0, 0.0, -1.0]], np.float32)
    assert oracle_mod.select(s, 1)[0][0].tolist() == [0]
    s = np.array([[0.0, -0.0, -1.0]], np.float32)
    assert oracle_mod.select(s, 2)[0][0].tolist() == [0, 1]


def test_router_logits_one_hot_rows(oracle_mod):
    rng = np.random.default_rng(8)
    E, D = 10, 64
    W = torch.from_numpy(rng.normal(scale=0.02, size=(E, D)).astype(np.float32)).to(torch.bfloat16)
    x = torch.zeros(D, D, dtype=torch.bfloat16)
    for j in range(D):
        x[j, j] = 1.0
    l = oracle_mod.router_logits(x, W)
    assert np.array_equal(l, W.float().numpy().T)       # l[t=j, e] = W[e, j], exactly
    b = rng.normal(size=E).astype(np.float32)
    lb = oracle_mod.router_logits(x, W, b)
    assert np.array_equal(lb, (W.float().numpy().T + b[None, :]).astype(np.float32))


def test_router_logits_match_library_matmul(oracle_mod):
    g = torch.Generator().manual_seed(9)
    x = torch.randn(33, 96, generator=g).to(torch.bfloat16)
    W = (0.02 * torch.randn(17, 96, generator=g)).to(torch.bfloat16)
    l = oracle_mod.router_logits(x, W)
    ref = (x.double() @ W.double().T).float().numpy()
    # both are the exact dot product rounded once to FP32 (sums of <= 96 exact products in
    # double are exact to far below FP32's last bit, barring a double-rounding tie)
    ulp = np.spacing(np.abs(ref))
    assert (np.abs(l - ref) <= ulp).all()


def test_tiny_tie_rows(oracle_mod):
    cfg = inputs.CONFIGS["tiny"]
    L = inputs.make_layer(cfg)
    logits, idx, w = oracle_mod.route(L["x"], L["W_r"], cfg.k, cfg.norm_topk_prob)
    for row, (_, vals, expect) in inputs.TINY_TIES.items():
        assert tuple(idx[row].tolist()) == expect, row
    for row in (5, 42, 63):
        assert (w[row] == 0.5).all(), row
    y, _, _, _ = oracle_mod.forward_rows(L["x"], L["W_r"], L["W_gate_up"], L["W_down"], cfg.k, [63])
    assert np.abs(y).max() == 0.0                       # zero token -> silu(0) * 0 = 0


# ------------------------------------------------------------------ experts

def _small_layer(T=12, D=64, E=5, I=32, seed=11):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, D, generator=g).to(torch.bfloat16)
    W_r = (0.3 * torch.randn(E, D, generator=g)).to(torch.bfloat16)
    W_gu = (0.1 * torch.randn(E, 2 * I, D, generator=g)).to(torch.bfloat16)
    W_dn = (0.1 * torch.randn(E, D, I, generator=g)).to(torch.bfloat16)
    return x, W_r, W_gu, W_dn


def _swiglu_ffn_library(x, W_gu, W_dn):
    """Textbook SwiGLU FFN with torch.nn.functional in float64."""
    I = W_gu.shape[0] // 2
    gate, up = F.linear(x.double(), W_gu.double()).split(I, dim=-1)
    return F.linear(F.silu(gate) * up, W_dn.double())


def test_single_expert_is_swiglu_ffn(oracle_mod):
    x, W_r, W_gu, W_dn = _small_layer(E=1)
    y, idx, w, _ = oracle_mod.forward_rows(x, W_r, W_gu, W_dn, 1, list(range(x.shape[0])))
    assert (idx == 0).all() and (w == 1.0).all()
    ref = _swiglu_ffn_library(x, W_gu[0], W_dn[0]).numpy()
    assert np.abs(y - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_dense_bruteforce_bmm_formulation(oracle_mod):
    """The all-experts bmm inference path of the HF module (transposed stacked layout
    (E, D, 2I) / (E, I, D), x repeated E times, sum over E of a [T, E] weight matrix that is
    zero off the top-k) equals the sparse per-token oracle."""
    x, W_r, W_gu, W_dn = _small_layer(T=16, E=6)
    k = 2
    T, D = x.shape
    E, I2, _ = W_gu.shape
    I = I2 // 2
    y, idx, w, _ = oracle_mod.forward_rows(x, W_r, W_gu, W_dn, k, list(range(T)))
    dense_w = torch.zeros(T, E, dtype=torch.float64).scatter_(1, torch.from_numpy(idx).long(),
                                                              torch.from_numpy(w).double())
    gate_up_proj = W_gu.double().transpose(1, 2)            # (E, D, 2I)
    down_proj = W_dn.double().transpose(1, 2)               # (E, I, D)
    hs = x.double().repeat(E, 1).view(E, T, D)
    gu = torch.bmm(hs, gate_up_proj)
    gate, up = gu[..., :I], gu[..., I:]
    nxt = torch.bmm(up * F.silu(gate), down_proj)            # (E, T, D)
    ref = (nxt * dense_w.transpose(0, 1)[..., None]).sum(0).numpy()
    assert np.abs(y - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_loop_dispatch_equals_per_token(oracle_mod):
    # the pages' invariant (the loop and grouped dispatches give the same result): the
    # oracle's loop dispatch against its per-token definition
    x, W_r, W_gu, W_dn = _small_layer(T=20, E=7)
    _, idx, w = oracle_mod.route(x, W_r, 3)
    y_loop = oracle_mod.loop_dispatch(x, idx, w, W_gu, W_dn)
    y_tok = oracle_mod.combine_rows(x, idx, w, list(range(20)), W_gu, W_dn)
    assert np.abs(y_loop - y_tok).max() <= 1e-12 * max(1.0, np.abs(y_tok).max())


def test_zero_up_projection_gives_zero(oracle_mod):
    x, W_r, W_gu, W_dn = _small_layer()
    I = W_gu.shape[1] // 2
    W0 = W_gu.clone()
    W0[:, I:, :] = 0
    y, _, _, _ = oracle_mod.forward_rows(x, W_r, W0, W_dn, 2, list(range(x.shape[0])))
    assert np.abs(y).max() == 0.0
    y, _, _, _ = oracle_mod.forward_rows(torch.zeros_like(x), W_r, W_gu, W_dn, 2, [0, 3])
    assert np.abs(y).max() == 0.0


def test_weighted_sum_of_selected_experts(oracle_mod):
    """y = sum_j w_j expert_{e_j}(x), each expert from the library SwiGLU."""
    x, W_r, W_gu, W_dn = _small_layer(T=6, E=5)
    k = 3
    y, idx, w, _ = oracle_mod.forward_rows(x, W_r, W_gu, W_dn, k, list(range(6)), norm=False)
    for t in range(6):
        ref = sum(float(w[t, j]) * _swiglu_ffn_library(x[t:t + 1], W_gu[idx[t, j]], W_dn[idx[t, j]])[0]
                  for j in range(k)).numpy()
        assert np.abs(y[t] - ref).max() <= 1e-12


def test_shared_expert_gate_and_residual(oracle_mod):
    x, W_r, W_gu, W_dn = _small_layer(T=5, E=4)
    g = torch.Generator().manual_seed(12)
    I_s = 16
    sgu = (0.1 * torch.randn(2 * I_s, x.shape[1], generator=g)).to(torch.bfloat16)
    sdn = (0.1 * torch.randn(x.shape[1], I_s, generator=g)).to(torch.bfloat16)
    sg = (0.1 * torch.randn(x.shape[1], generator=g)).to(torch.bfloat16)
    res = torch.randn(x.shape, generator=g).to(torch.bfloat16)
    rows = list(range(5))
    base, _, _, _ = oracle_mod.forward_rows(x, W_r, W_gu, W_dn, 2, rows)
    S = _swiglu_ffn_library(x, sgu, sdn).numpy()
    y, _, _, _ = oracle_mod.forward_rows(x, W_r, W_gu, W_dn, 2, rows, shared_gate_up=sgu, shared_down=sdn)
    assert np.abs(y - (base + S)).max() <= 1e-12           # ungated shared expert
    y, _, _, _ = oracle_mod.forward_rows(x, W_r, W_gu, W_dn, 2, rows, shared_gate_up=sgu,
                                         shared_down=sdn, shared_gate=torch.zeros_like(sg))
    assert np.abs(y - (base + 0.5 * S)).max() <= 1e-12     # sigmoid(0) = 1/2
    y, _, _, _ = oracle_mod.forward_rows(x, W_r, W_gu, W_dn, 2, rows, shared_gate_up=sgu,
                                         shared_down=sdn, shared_gate=sg, residual=res)
    gate = torch.sigmoid(x.double() @ sg.double()).numpy()[:, None]
    assert np.abs(y - (base + gate * S + res.double().numpy())).max() <= 1e-12


# ------------------------------------------------------------------ permute

@pytest.mark.parametrize("tile_m", [1, 4, 16])
def test_permute_matches_library_stable_sort(oracle_mod, tile_m):
    rng = np.random.default_rng(13)
    T, k, E = 37, 3, 9
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, row_token, slot_row = oracle_mod.permute(idx, E, tile_m)
    flat = idx.reshape(-1)
    assert counts.tolist() == np.bincount(flat, minlength=E).tolist()
    assert counts.sum() == T * k
    order = sorted(range(T * k), key=lambda a: flat[a])     # Python's sort is stable
    assert offsets[0] == 0 and all((offsets[1:] - offsets[:-1]) % tile_m == 0)
    assert all(offsets[e + 1] - offsets[e] == -(-counts[e] // tile_m) * tile_m for e in range(E))
    pos = 0
    for e in range(E):
        seg = order[pos:pos + counts[e]]
        pos += counts[e]
        rows = list(range(offsets[e], offsets[e] + counts[e]))
        assert [row_token[r] for r in rows] == [a // k for a in seg]
        assert [slot_row[a] for a in seg] == rows
        assert all(row_token[r] == -1 for r in range(offsets[e] + counts[e], offsets[e + 1]))


# ------------------------------------------------------------------ byte accounting

def test_parameter_split_matches_page():
    g = golden("parameter_split.json")
    s = g["shape"]
    stored, active = moe_parameter_split(s["hidden"], s["layers"], s["experts"], s["top_k"],
                                         s["intermediate"], s["shared_intermediate"])
    p = g["printed"]
    assert round(stored / 1e9, 1) == p["expert_params_stored_B"]
    assert round(active / 1e9, 2) == p["expert_params_active_B"]
    assert round(active / stored, 3) == p["active_fraction"]


# ------------------------------------------------------------------ FP8 weight-only experts

def test_e4m3_values_match_library_decoding(oracle_mod):
    # every code against torch's float8_e4m3fn decoding, and the format's landmarks
    codes = np.arange(256, dtype=np.uint8)
    vals = np.array([oracle_mod.e4m3_value(c) for c in codes])
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(vals), np.isnan(ref))
    assert np.array_equal(vals[~np.isnan(vals)], ref[~np.isnan(ref)])
    assert oracle_mod.e4m3_value(0x7E) == 448.0 and oracle_mod.e4m3_value(0x38) == 1.0
    assert oracle_mod.e4m3_value(0x01) == 2.0 ** -9 and oracle_mod.e4m3_value(0x08) == 2.0 ** -6
    assert np.isnan(oracle_mod.e4m3_value(0x7F)) and oracle_mod.e4m3_value(0xFE) == -448.0


def test_fp8_quantizer_matches_library_rounding(oracle_mod):
    g = torch.Generator().manual_seed(3)
    W = torch.randn(96, 384, generator=g) * 0.02
    W[0] = 0
    W[1, 5] = 50.0                                  # one large value: most of the row underflows
    W[2] *= 1e-3
    W[3, :4] = torch.tensor([448.0, -448.0, 1.0, 2.0 ** -9])
    Wb = W.to(torch.bfloat16)
    q, s = oracle_mod.quantize_fp8_rows(Wb)
    Wf = Wb.float()
    amax = Wf.abs().amax(dim=1)
    s_ref = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))        # FP32 division
    assert np.array_equal(s.view(np.uint32), s_ref.numpy().view(np.uint32))
    quot = (Wf / s_ref[:, None]).clamp(-448.0, 448.0)                           # FP32 quotient
    q_ref = quot.to(torch.float8_e4m3fn).view(torch.uint8).numpy()              # nearest-even
    assert np.array_equal(q, q_ref)


def test_fp8_dequantisation_error_bound(oracle_mod):
    # |w / s - value(q)| is at most half a step of E4M3 at that magnitude: 2^-4 of the value for
    # normal values, 2^-10 in the subnormal range
    g = torch.Generator().manual_seed(4)
    Wb = (torch.randn(64, 256, generator=g) * 0.05).to(torch.bfloat16)
    q, s = oracle_mod.quantize_fp8_rows(Wb)
    table = np.array([oracle_mod.e4m3_value(c) for c in range(256)])
    v = (Wb.float() / torch.from_numpy(s)[:, None]).double().numpy()
    err = np.abs(v - table[q])
    assert (err <= np.maximum(np.abs(v) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-12)).all()


def test_fp8_experts_equal_bf16_experts_on_exact_weights(oracle_mod):
    # weights on the E4M3 grid times a power of two (each row reaching 448 * 2^n), so that
    # the row scale is exactly 2^n and the dequantised weights equal the bf16 weights: the FP8
    # evaluation must then equal the bf16 one bit for bit
    rng = np.random.default_rng(6)
    E, I, D, T, k = 3, 16, 32, 5, 2
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    table = np.array([oracle_mod.e4m3_value(c) for c in range(256)])

    def grid(rows, cols, n):
        c = rng.choice(finite, size=(rows, cols))
        c[:, 0] = 0x7E                               # 448 in every row
        return torch.from_numpy(table[c] * 2.0 ** n).to(torch.bfloat16)

    W_gu = grid(E * 2 * I, D, -12).reshape(E, 2 * I, D)
    W_dn = grid(E * D, I, -11).reshape(E, D, I)
    x = torch.from_numpy(rng.standard_normal((T, D))).to(torch.bfloat16)
    idx = np.array([[0, 2], [1, 0], [2, 1], [0, 1], [2, 0]], np.int32)
    w = np.array([[0.7, 0.3], [0.5, 0.5], [0.25, 0.75], [0.9, 0.1], [0.6, 0.4]], np.float32)
    q_gu, s_gu = oracle_mod.quantize_fp8_rows(W_gu)
    q_dn, s_dn = oracle_mod.quantize_fp8_rows(W_dn)
    assert (s_gu == 2.0 ** -12).all() and (s_dn == 2.0 ** -11).all()
    rows = np.arange(T, dtype=np.int32)
    y8 = oracle_mod.combine_rows_fp8(x, idx, w, rows, q_gu, s_gu, q_dn, s_dn)
    y16 = oracle_mod.combine_rows(x, idx, w, rows, W_gu, W_dn)
    assert np.array_equal(y8, y16)


# ------------------------------------------------------------------ Switch balance loss
# "Qwen3-VL and Mixture of Experts", "An auxiliary balance loss": L = alpha N sum_i f_i P_i;
# the Qwen3-VL MoE walk-through's load_balancing_loss_func: f from the top-k one-hot averaged
# over tokens, P the mean softmax probability, times the number of experts.

def test_aux_loss_uniform_logits_give_alpha_k(oracle_mod):
    """Equal logits make every P_i = 1/N, so L = alpha * sum_i f_i = alpha * k for ANY routing."""
    rng = np.random.default_rng(3)
    T, E, k, alpha = 37, 12, 3, 0.01
    logits = np.full((T, E), 0.75, np.float32)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    loss, _ = oracle_mod.aux_loss(logits, idx, alpha)
    assert abs(loss - alpha * k) <= 1e-15


def test_aux_loss_balanced_routing_gives_alpha_k(oracle_mod):
    """Every expert chosen equally often (f_i = k / N) makes L = alpha * k * sum_i P_i = alpha * k
    for ANY logits."""
    rng = np.random.default_rng(4)
    E, k = 8, 2
    T = E * 5
    logits = rng.normal(0, 3, (T, E)).astype(np.float32)
    idx = np.array([[(t + j) % E for j in range(k)] for t in range(T)], np.int32)   # each expert 2*5 times
    loss, _ = oracle_mod.aux_loss(logits, idx, 0.5)
    assert abs(loss - 0.5 * k) <= 1e-12


def test_aux_loss_collapse_closed_form(oracle_mod):
    """N = 2, k = 1, every token sent to expert 0 with logits (l, 0): f = (1, 0), P_0 =
    sigmoid(l), so L = alpha * 2 * sigmoid(l)."""
    l, T, alpha = 1.25, 9, 0.3
    logits = np.tile(np.array([[l, 0.0]], np.float32), (T, 1))
    idx = np.zeros((T, 1), np.int32)
    loss, d = oracle_mod.aux_loss(logits, idx, alpha)
    sig = 1.0 / (1.0 + math.exp(-float(np.float32(l))))
    assert abs(loss - alpha * 2 * sig) <= 1e-14
    # dL/dl_0 of each token: alpha * 2 / T * sigmoid' (f_0 - f_1 = 1)
    assert np.allclose(d[:, 0], alpha * 2 / T * sig * (1 - sig), rtol=0, atol=1e-15)


def test_aux_loss_gradient_matches_finite_differences(oracle_mod):
    """dL/dlogits (selection held fixed) against central differences of the loss."""
    rng = np.random.default_rng(5)
    T, E, k, alpha = 3, 5, 2, 0.7
    logits = rng.normal(0, 1, (T, E)).astype(np.float32)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    _, d = oracle_mod.aux_loss(logits, idx, alpha)
    h = 2.0 ** -8   # exact in FP32 around values of order 1
    for t in range(T):
        for e in range(E):
            lp, lm = logits.copy(), logits.copy()
            lp[t, e] += h
            lm[t, e] -= h
            fd = (oracle_mod.aux_loss(lp, idx, alpha, False)[0] - oracle_mod.aux_loss(lm, idx, alpha, False)[0]) / (
                float(lp[t, e]) - float(lm[t, e]))
            assert abs(fd - d[t, e]) <= 2e-6, (t, e, fd, d[t, e])
    # each token's gradient sums to zero (a softmax is shift-invariant)
    assert np.abs(d.sum(axis=1)).max() <= 1e-15


# ------------------------------------------------------------------ backward pass
# "Qwen3-VL and Mixture of Experts", "How the router and experts learn", "What gets trained":
# a token's gradient reaches only the experts it chose, and the router learns through the
# gate weights; the selection is held fixed.

def _bwd_problem(seed, T, D, E, k, I, bias=True):
    g = torch.Generator().manual_seed(seed)
    bf = lambda *s, sc=1.0: (torch.randn(*s, generator=g) * sc).to(torch.bfloat16)
    P = dict(x=bf(T, D), W_r=bf(E, D, sc=0.5), W_gu=bf(E, 2 * I, D, sc=0.4), W_dn=bf(E, D, I, sc=0.4),
             dy=bf(T, D), bias=(torch.randn(E, generator=g) * 0.3) if bias else None)
    # any distinct experts per token (not necessarily the top k): the gradient formula holds
    # for a fixed selection whatever it is
    P["idx"] = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    return P


def _block_loss64(P, norm, residual, dl_add=None, over=None):
    """sum_t dy[t] . y[t] (+ sum dl_add * logits) of the block in float64 torch ops, routing fixed.
    `over` replaces some float64 leaves (for finite differences / autograd)."""
    V = {n: P[n].double() for n in ("x", "W_r", "W_gu", "W_dn", "dy")}
    V["bias"] = P["bias"].double() if P["bias"] is not None else None
    V.update(over or {})
    x, W_r, W_gu, W_dn, dy = V["x"], V["W_r"], V["W_gu"], V["W_dn"], V["dy"]
    idx = P["idx"].long()
    I = W_gu.shape[1] // 2
    logits = x @ W_r.T + (V["bias"] if V["bias"] is not None else 0.0)
    p = torch.softmax(logits, dim=-1)
    sel = torch.gather(p, 1, idx)
    w = sel / sel.sum(1, keepdim=True) if norm else sel
    g = torch.einsum("tkid,td->tki", W_gu[idx, :I, :], x)
    u = torch.einsum("tkid,td->tki", W_gu[idx, I:, :], x)
    o = torch.einsum("tkdi,tki->tkd", W_dn[idx], F.silu(g) * u)
    y = (w[..., None] * o).sum(1) + (x if residual else 0.0)
    L = (dy * y).sum()
    if dl_add is not None:
        L = L + (torch.as_tensor(dl_add) * logits).sum()
    return L, logits, w


@pytest.mark.parametrize("norm,residual,with_add", [(True, False, False), (False, True, False), (True, True, True)])
def test_backward_matches_autograd(oracle_mod, norm, residual, with_add):
    """Every gradient of the oracle's backward against float64 autograd of the forward
    definition (x, all weights, the bias, the logits and the routing weights)."""
    T, D, E, k, I = 6, 16, 7, 3, 8
    P = _bwd_problem(11, T, D, E, k, I)
    dl_add = np.random.default_rng(1).normal(0, 0.1, (T, E)) if with_add else None
    leaves = {n: P[n].double().requires_grad_(True) for n in ("x", "W_r", "W_gu", "W_dn")}
    leaves["bias"] = P["bias"].double().requires_grad_(True)
    L, logits, w = _block_loss64(P, norm, residual, dl_add, over=leaves)
    logits.retain_grad()
    w.retain_grad()
    L.backward()
    experts = [0, 3, 5]
    got = oracle_mod.backward(P["x"], P["W_r"], P["W_gu"], P["W_dn"], P["dy"], P["idx"], norm=norm,
                              bias=P["bias"], residual=residual, dlogits_add=dl_add, experts=experts)
    want = dict(dx=leaves["x"].grad, dW_r=leaves["W_r"].grad, db=leaves["bias"].grad, dlogits=logits.grad,
                dw=w.grad, dW_gu=leaves["W_gu"].grad[experts], dW_dn=leaves["W_dn"].grad[experts])
    for name, ref in want.items():
        ref = ref.numpy()
        assert np.abs(got[name] - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max()), name
    # experts nobody chose get no gradient
    unused = sorted(set(range(E)) - set(P["idx"].flatten().tolist()))
    for e in unused:
        assert not leaves["W_gu"].grad[e].any()


def test_backward_finite_differences(oracle_mod):
    """Central differences of the float64 forward (no autograd) on entries of x, W_r, W_gate_up,
    W_down and the bias."""
    T, D, E, k, I = 4, 8, 5, 2, 4
    P = _bwd_problem(12, T, D, E, k, I)
    got = oracle_mod.backward(P["x"], P["W_r"], P["W_gu"], P["W_dn"], P["dy"], P["idx"], norm=True,
                              bias=P["bias"], experts=list(range(E)))
    rng = np.random.default_rng(2)
    cases = [("x", "dx"), ("W_r", "dW_r"), ("W_gu", "dW_gu"), ("W_dn", "dW_dn"), ("bias", "db")]
    h = 1e-6
    for leaf, out in cases:
        base = P[leaf].double()
        for _ in range(4):
            pos = tuple(int(rng.integers(0, n)) for n in base.shape)
            plus, minus = base.clone(), base.clone()
            plus[pos] += h
            minus[pos] -= h
            fd = (_block_loss64(P, True, False, over={leaf: plus})[0] -
                  _block_loss64(P, True, False, over={leaf: minus})[0]).item() / (2 * h)
            assert abs(fd - got[out][pos]) <= 1e-7 * max(1.0, abs(fd)), (leaf, pos, fd, got[out][pos])


def test_backward_one_expert_is_swiglu_mlp(oracle_mod):
    """E = 1, k = 1: the weight is 1 whatever the logits, so the router gets no gradient, and dx,
    dW_gate_up, dW_down are those of a plain SwiGLU MLP y = W_down (silu(W_gate x) * W_up x)
    (torch.nn.functional, autograd)."""
    T, D, I = 5, 12, 6
    P = _bwd_problem(13, T, D, 1, 1, I)
    got = oracle_mod.backward(P["x"], P["W_r"], P["W_gu"], P["W_dn"], P["dy"], P["idx"], norm=True,
                              bias=P["bias"], experts=[0])
    assert not got["dlogits"].any() and not got["dW_r"].any() and not got["db"].any()
    x = P["x"].double().requires_grad_(True)
    Wg = P["W_gu"][0, :I].double().requires_grad_(True)
    Wu = P["W_gu"][0, I:].double().requires_grad_(True)
    Wd = P["W_dn"][0].double().requires_grad_(True)
    y = F.linear(F.silu(F.linear(x, Wg)) * F.linear(x, Wu), Wd)
    (P["dy"].double() * y).sum().backward()
    assert np.allclose(got["dx"], x.grad.numpy(), rtol=0, atol=1e-12)
    assert np.allclose(got["dW_gu"][0], torch.cat([Wg.grad, Wu.grad]).numpy(), rtol=0, atol=1e-12)
    assert np.allclose(got["dW_dn"][0], Wd.grad.numpy(), rtol=0, atol=1e-12)
