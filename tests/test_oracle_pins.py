"""Pins of the CPU oracle against closed forms, invariants and library routines.

Each test is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a wrong scale, a wrong head mapping,
a cache off-by-one) fails at least one of them.  None of these checks uses the
CUDA path.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic as syn

RNG = np.random.default_rng(1234)


def bits(x) -> np.ndarray:
    """bf16 bit patterns of values that are exactly representable (via torch)."""
    t = torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def rand_bf16(shape, scale=1.0):
    return bits(RNG.standard_normal(shape) * scale)


# ----------------------------------------------------------------------------- bf16 rounding

def test_bf16_round_ties_to_even_closed_forms():
    f = oracle.bf16_round
    assert f(1.0) == 0x3F80
    assert f(1.0 + 2 ** -8) == 0x3F80            # tie -> even mantissa (0)
    assert f(1.0 + 3 * 2 ** -8) == 0x3F82        # tie between 0x3F81 and 0x3F82 -> even
    assert f(1.0 + 2 ** -8 + 2 ** -30) == 0x3F81  # just above the tie -> up
    assert f(-1.5) == 0xBFC0
    assert f(2 ** -130) == 0x0008                # subnormal, exact
    assert f(2 ** -134) == 0x0000                # half the smallest subnormal -> even (0)
    assert f(3 * 2 ** -134) == 0x0002            # 1.5 quanta -> 2 (even)
    assert f(0.0) == 0 and f(-0.0) == 0x8000
    assert f(1e39) == 0x7F80 and f(-1e39) == 0xFF80


def test_bf16_round_matches_torch_on_fp32_values():
    x = (RNG.standard_normal(20000) * np.exp(RNG.uniform(-20, 20, 20000))).astype(np.float32)
    ref = torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_round_array(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


# ----------------------------------------------------------------------------- silu

def test_silu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    assert abs(oracle.silu(1.0) - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15
    for z in (-3.0, -0.5, 0.25, 2.0, 7.0):
        # silu(-z) = silu(z) - z
        assert abs(oracle.silu(-z) - (oracle.silu(z) - z)) < 1e-12
    assert abs(oracle.silu(40.0) - 40.0) < 1e-12
    z = RNG.standard_normal(64)
    ref = torch.nn.functional.silu(torch.tensor(z, dtype=torch.float64)).numpy()
    np.testing.assert_allclose([oracle.silu(v) for v in z], ref, rtol=1e-14, atol=1e-15)


# ----------------------------------------------------------------------------- rmsnorm

def test_rmsnorm_constant_vector_closed_form():
    n, eps, c = 256, 1e-5, 0.37
    g = bits(np.ones(n))
    out = oracle.rmsnorm(np.full(n, c), g, eps)
    np.testing.assert_allclose(out, c / math.sqrt(c * c + eps), rtol=1e-14)


def test_rmsnorm_invariants_and_library():
    n, eps = 4096, 1e-5
    x = RNG.standard_normal(n) * 0.3
    ones = bits(np.ones(n))
    h = oracle.rmsnorm(x, ones, eps)
    ms = float(np.mean(x * x))
    assert abs(float(np.mean(h * h)) - ms / (ms + eps)) < 1e-12
    # gains multiply elementwise
    g = rand_bf16(n)
    hg = oracle.rmsnorm(x, g, eps)
    np.testing.assert_allclose(hg, h * oracle.bf16_to_f64(g), rtol=1e-13, atol=1e-15)
    # scale invariance when eps is negligible
    np.testing.assert_allclose(oracle.rmsnorm(x * 1e4, ones, eps), x / math.sqrt(ms), rtol=1e-9)
    # library routine
    ref = torch.nn.functional.rms_norm(torch.tensor(x), (n,), torch.tensor(oracle.bf16_to_f64(g)),
                                       eps=eps).numpy()
    np.testing.assert_allclose(hg, ref, rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------- rope

def test_rope_identity_at_position_zero():
    v = RNG.standard_normal(128)
    np.testing.assert_array_equal(oracle.rope(v, 0, 1e4), v)


def test_rope_rotate_half_pairing_closed_form():
    d, theta = 128, 1e4
    e0 = np.zeros(d); e0[0] = 1.0
    out = oracle.rope(e0, 1, theta)             # inv_freq_0 = 1 -> angle 1
    exp = np.zeros(d); exp[0] = math.cos(1.0); exp[d // 2] = math.sin(1.0)
    np.testing.assert_allclose(out, exp, atol=1e-15)
    # second frequency: pair (1, 1 + d/2), angle p * theta^(-2/d)
    e1 = np.zeros(d); e1[1 + d // 2] = 1.0
    p = 7
    a = p * theta ** (-2.0 / d)
    out = oracle.rope(e1, p, theta)
    exp = np.zeros(d); exp[1] = -math.sin(a); exp[1 + d // 2] = math.cos(a)
    np.testing.assert_allclose(out, exp, atol=1e-15)


def test_rope_norm_preservation_and_relative_position():
    d, theta = 64, 1e4
    q, k = RNG.standard_normal(d), RNG.standard_normal(d)
    for p in (1, 5, 38, 550, 131071):
        r = oracle.rope(q, p, theta)
        h = d // 2
        np.testing.assert_allclose(r[:h] ** 2 + r[h:] ** 2, q[:h] ** 2 + q[h:] ** 2, rtol=1e-12)
    # <R_p q, R_p' k> depends only on p - p'
    base = np.dot(oracle.rope(q, 3, theta), k)
    for p in (10, 100, 1000):
        np.testing.assert_allclose(np.dot(oracle.rope(q, p + 3, theta), oracle.rope(k, p, theta)),
                                   base, rtol=1e-9)
    # complex-number form: (v_i + i v_{i+h}) * exp(i p f_i)
    p = 123
    f = theta ** (-2.0 * np.arange(d // 2) / d)
    z = (q[: d // 2] + 1j * q[d // 2:]) * np.exp(1j * p * f)
    np.testing.assert_allclose(oracle.rope(q, p, theta), np.concatenate([z.real, z.imag]),
                               atol=1e-12)


# ----------------------------------------------------------------------------- gemv

def test_gemv_one_hot_extracts_column():
    W = rand_bf16((48, 80))                      # non-square: a transpose cannot pass
    for j in (0, 17, 79):
        x = np.zeros(80); x[j] = 1.0
        np.testing.assert_array_equal(oracle.gemv(W, x), oracle.bf16_to_f64(W[:, j]))


def test_gemv_integer_exact_and_library():
    Wi = RNG.integers(-8, 9, size=(33, 257))
    xi = RNG.integers(-5, 6, size=257)
    got = oracle.gemv(bits(Wi), xi.astype(np.float64))
    np.testing.assert_array_equal(got, (Wi @ xi).astype(np.float64))
    W = rand_bf16((64, 1000), 0.02)
    x = RNG.standard_normal(1000)
    np.testing.assert_allclose(oracle.gemv(W, x), oracle.bf16_to_f64(W) @ x, rtol=1e-12,
                               atol=1e-14)


# ----------------------------------------------------------------------------- attention

def test_attention_single_token_returns_v0():
    nq, nkv, d = 8, 2, 64
    q = RNG.standard_normal(nq * d)
    K = rand_bf16((1, nkv, d)); V = rand_bf16((1, nkv, d))
    o = oracle.attention(q, K, V, nq, nkv, d)
    for h in range(nq):
        np.testing.assert_array_equal(o[h], oracle.bf16_to_f64(V[0, h * nkv // nq]))


def test_attention_zero_query_is_mean_of_values():
    nq, nkv, d, n = 4, 2, 64, 37
    K = rand_bf16((n, nkv, d)); V = rand_bf16((n, nkv, d))
    o = oracle.attention(np.zeros(nq * d), K, V, nq, nkv, d)
    Vf = oracle.bf16_to_f64(V)
    for h in range(nq):
        np.testing.assert_allclose(o[h], Vf[:, h * nkv // nq].mean(axis=0), rtol=1e-12, atol=1e-14)


def test_attention_gqa_mapping_is_consecutive():
    nq, nkv, d, n = 4, 2, 16, 5
    K = rand_bf16((n, nkv, d))
    V = np.zeros((n, nkv, d), dtype=np.float32); V[:, 0] = 1.0; V[:, 1] = 2.0
    o = oracle.attention(RNG.standard_normal(nq * d), K, bits(V), nq, nkv, d)
    np.testing.assert_allclose(o[:, 0], [1.0, 1.0, 2.0, 2.0], rtol=1e-14)   # heads 0,1 -> kv 0


def test_attention_two_token_closed_form_scale():
    nq, nkv, d = 1, 1, 64
    q = np.zeros(d); q[0] = 2.0
    K = np.zeros((2, 1, d), dtype=np.float32); K[0, 0, 0] = 1.5; K[1, 0, 0] = -0.5
    V = np.zeros((2, 1, d), dtype=np.float32); V[0, 0, 3] = 1.0; V[1, 0, 5] = 1.0
    o = oracle.attention(q, bits(K), bits(V), nq, nkv, d)
    s0, s1 = 2.0 * 1.5 / 8.0, 2.0 * -0.5 / 8.0       # scale 1/sqrt(64)
    a0 = 1.0 / (1.0 + math.exp(s1 - s0))
    assert abs(o[0, 3] - a0) < 1e-15 and abs(o[0, 5] - (1 - a0)) < 1e-15


def test_attention_matches_library_sdpa():
    nq, nkv, d, n = 8, 2, 64, 75
    q = RNG.standard_normal(nq * d)
    K = rand_bf16((n, nkv, d)); V = rand_bf16((n, nkv, d))
    o = oracle.attention(q, K, V, nq, nkv, d)
    qt = torch.tensor(q.reshape(1, nq, 1, d))
    kt = torch.tensor(oracle.bf16_to_f64(K).transpose(1, 0, 2)[None])
    vt = torch.tensor(oracle.bf16_to_f64(V).transpose(1, 0, 2)[None])
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, enable_gqa=True)
    np.testing.assert_allclose(o, ref[0, :, 0].numpy(), rtol=1e-11, atol=1e-13)


def test_argmax_ties_to_lowest():
    assert oracle.argmax([0.0, 3.0, -1.0, 3.0]) == 1
    assert oracle.argmax([5.0, 5.0]) == 0


# ----------------------------------------------------------------------------- ffn / moe

def test_swiglu_ffn_library_composition():
    H, F = 64, 96
    wg, wu, wd = rand_bf16((F, H), 0.2), rand_bf16((F, H), 0.2), rand_bf16((H, F), 0.2)
    h = RNG.standard_normal(H)
    G, U, D = (torch.tensor(oracle.bf16_to_f64(a)) for a in (wg, wu, wd))
    ht = torch.tensor(h)
    ref = (D @ (torch.nn.functional.silu(G @ ht) * (U @ ht))).numpy()
    np.testing.assert_allclose(oracle.swiglu_ffn(wg, wu, wd, h), ref, rtol=1e-11, atol=1e-14)


def test_moe_route_topk_softmax_and_ties():
    E, H, k = 16, 32, 4
    W = rand_bf16((E, H), 0.3)
    W[5] = W[3]                                    # experts 3 and 5 tie exactly
    h = RNG.standard_normal(H)
    sel, wts, probs = oracle.moe_route(W, h, k, renorm=True)
    logits = oracle.bf16_to_f64(W) @ h
    ref_p = torch.softmax(torch.tensor(logits), 0).numpy()
    np.testing.assert_allclose(probs, ref_p, rtol=1e-12)
    order = np.argsort(-probs, kind="stable")      # stable: ties keep the lower index first
    np.testing.assert_array_equal(sel, order[:k])
    np.testing.assert_allclose(wts, probs[sel] / probs[sel].sum(), rtol=1e-13)
    sel2, wts2, _ = oracle.moe_route(W, h, k, renorm=False)
    np.testing.assert_allclose(wts2, probs[sel2], rtol=1e-13)
    # force the tie onto the top-k boundary: expert 3 must win over 5
    Wt = np.zeros((E, H), dtype=np.float32)
    Wt[0, 0], Wt[1, 0], Wt[3, 0], Wt[5, 0] = 3.0, 2.0, 1.0, 1.0
    ht = np.zeros(H); ht[0] = 1.0
    selt, _, _ = oracle.moe_route(bits(Wt), ht, 3, renorm=True)
    np.testing.assert_array_equal(selt, [0, 1, 3])
    selo, _, _ = oracle.moe_route(bits(Wt), ht, 3, renorm=True, override=[0, 1, 5])
    np.testing.assert_array_equal(selo, [0, 1, 5])


# ----------------------------------------------------------------------------- whole step

def _names(cfg):
    return [s.name for s in syn.tensor_specs(cfg)]


def _weights(cfg, seed=7, gain_sigma=0.1):
    return syn.host_weights(cfg, seed, gain_sigma=gain_sigma)


@pytest.mark.parametrize("cfg", [syn.TINY, syn.TINY_MOE], ids=lambda c: c.name)
def test_cached_decode_equals_nocache_recompute(cfg):
    w = _weights(cfg)
    toks = syn.host_tokens(12, 99, cfg.vocab)
    m = oracle.Model(cfg, w, 16, _names(cfg))
    inc = np.stack([m.decode_step(int(t), p)["logits"] for p, t in enumerate(toks)])
    full = oracle.Model(cfg, w, 16, _names(cfg)).forward_nocache(toks)
    np.testing.assert_allclose(inc, full, rtol=1e-10, atol=1e-12)
    # the cache holds exactly the positions written
    assert np.all(m.k[0][12:] == 0) and np.any(m.k[0][11] != 0)


def _zero_like(w):
    return {k: np.zeros_like(v) for k, v in w.items()}


def test_zero_layers_model_is_norm_plus_lm_head():
    cfg = syn.TINY
    w = _weights(cfg)
    z = _zero_like(w)
    z["tok_emb"], z["lm_head"], z["final_norm"] = w["tok_emb"], w["lm_head"], w["final_norm"]
    for l in range(cfg.n_layers):
        z[f"layers.{l}.attn_norm"] = w[f"layers.{l}.attn_norm"]
        z[f"layers.{l}.ffn_norm"] = w[f"layers.{l}.ffn_norm"]
    m = oracle.Model(cfg, z, 8, _names(cfg))
    tok = 321
    out = m.decode_step(tok, 0)["logits"]
    x = oracle.bf16_to_f64(w["tok_emb"][tok])
    g = oracle.bf16_to_f64(w["final_norm"])
    h = x / np.sqrt(np.mean(x * x) + cfg.rms_eps) * g
    np.testing.assert_allclose(out, oracle.bf16_to_f64(w["lm_head"]) @ h, rtol=1e-11, atol=1e-13)


def test_attention_wiring_uniform_average_of_cached_values():
    """W_q = W_k = 0 makes attention uniform over positions 0..p; W_v copies hidden
    dims into v, W_o copies o back, so layer 0's residual update is the mean of
    bf16(v) over the cached positions (including the current one)."""
    cfg = syn.TINY
    H, d, nq, nkv = cfg.hidden, cfg.head_dim, cfg.n_q_heads, cfg.n_kv_heads
    w = _weights(cfg)
    z = _zero_like(w)
    z["tok_emb"] = w["tok_emb"]
    one = bits(np.ones(H))
    for name in list(z):
        if name.endswith("norm"):
            z[name] = one
    Wv = np.zeros((nkv * d, H), dtype=np.float32)
    Wv[np.arange(nkv * d), np.arange(nkv * d)] = 1.0            # v = h[0:nkv*d]
    Wo = np.zeros((H, nq * d), dtype=np.float32)
    Wo[np.arange(nq * d), np.arange(nq * d)] = 1.0              # x += o (flattened)
    z["layers.0.wv"], z["layers.0.wo"] = bits(Wv), bits(Wo)
    m = oracle.Model(cfg, z, 8, _names(cfg))
    toks = [5, 77, 900, 3]
    vs = []
    for p, t in enumerate(toks):
        out = m.decode_step(t, p, want_hidden=True)
        x0 = oracle.bf16_to_f64(w["tok_emb"][t])
        h = x0 / np.sqrt(np.mean(x0 * x0) + cfg.rms_eps)
        vs.append(oracle.bf16_to_f64(oracle.bf16_round_array(h[: nkv * d])).reshape(nkv, d))
        mean_v = np.mean(vs, axis=0)                            # [nkv][d]
        o = np.stack([mean_v[hh * nkv // nq] for hh in range(nq)]).ravel()
        upd = np.zeros(H); upd[: nq * d] = o
        np.testing.assert_allclose(out["hidden"][1] - out["hidden"][0], upd, rtol=1e-12, atol=1e-14)


def _expert_out(w, l, e, h):
    return oracle.swiglu_ffn(w[f"layers.{l}.w_gate"][e], w[f"layers.{l}.w_up"][e],
                             w[f"layers.{l}.w_down"][e], h)


def test_moe_layer_equals_dense_masked_sum():
    cfg = syn.TINY_MOE
    w = _weights(cfg)
    m = oracle.Model(cfg, w, 8, _names(cfg))
    toks = syn.host_tokens(3, 5, cfg.vocab)
    for p, t in enumerate(toks):
        out = m.decode_step(int(t), p, want_hidden=True)
        for l in range(cfg.n_layers):
            x_mid, x_out = out["hidden"][2 * l + 1], out["hidden"][2 * l + 2]
            h = oracle.rmsnorm(x_mid, w[f"layers.{l}.ffn_norm"], cfg.rms_eps)
            logits = oracle.bf16_to_f64(w[f"layers.{l}.w_router"]) @ h
            pi = torch.softmax(torch.tensor(logits), 0).numpy()
            S = np.argsort(-pi, kind="stable")[: cfg.top_k]
            mask = np.zeros(cfg.n_experts)
            mask[S] = pi[S] / pi[S].sum()
            y = sum(mask[e] * _expert_out(w, l, e, h) for e in range(cfg.n_experts))
            np.testing.assert_allclose(x_out - x_mid, y, rtol=1e-10, atol=1e-13)
            np.testing.assert_array_equal(out["moe_sel"][l], S)


def test_moe_all_experts_without_renorm_is_softmax_mixture():
    import dataclasses
    cfg = dataclasses.replace(syn.TINY_MOE, top_k=syn.TINY_MOE.n_experts, moe_renorm=0,
                              name="tiny-moe-all")
    w = _weights(syn.TINY_MOE)
    m = oracle.Model(cfg, w, 4, _names(cfg))
    out = m.decode_step(17, 0, want_hidden=True)
    x_mid, x_out = out["hidden"][1], out["hidden"][2]
    h = oracle.rmsnorm(x_mid, w["layers.0.ffn_norm"], cfg.rms_eps)
    pi = torch.softmax(torch.tensor(oracle.bf16_to_f64(w["layers.0.w_router"]) @ h), 0).numpy()
    y = sum(pi[e] * _expert_out(w, 0, e, h) for e in range(cfg.n_experts))
    np.testing.assert_allclose(x_out - x_mid, y, rtol=1e-10, atol=1e-13)


def test_expert_provider_matches_held_experts():
    cfg = syn.TINY_MOE
    w = _weights(cfg)
    held = oracle.Model(cfg, w, 4, _names(cfg)).decode_step(9, 0)["logits"]
    lazy_w = {k: v for k, v in w.items() if not any(s in k for s in ("w_gate", "w_up", "w_down"))}
    prov = lambda l, e, which: w[f"layers.{l}." + ("w_gate", "w_up", "w_down")[which]][e]
    lazy = oracle.Model(cfg, lazy_w, 4, _names(cfg), expert_provider=prov).decode_step(9, 0)
    np.testing.assert_array_equal(lazy["logits"], held)


def test_dense_ffn_wiring_gate_up_down_closed_form():
    """Layer 0's dense FFN with W_gate = I, W_up = c·I (on the first H rows) and
    W_down = I: the residual update is silu(h_i)·c·h_i, h = rmsnorm(x_mid).  Swapping
    the gate and up slots gives silu(c·h_i)·h_i instead, and a transposed or
    misplaced down matrix moves the update off the diagonal, so either fails."""
    cfg = syn.TINY
    H, F = cfg.hidden, cfg.ffn
    c = 2.0
    w = _weights(cfg)
    z = _zero_like(w)
    z["tok_emb"] = w["tok_emb"]
    for name in list(z):
        if name.endswith("norm"):
            z[name] = w[name]
    Wg = np.zeros((F, H), dtype=np.float32)
    Wg[np.arange(H), np.arange(H)] = 1.0
    Wd = np.zeros((H, F), dtype=np.float32)
    Wd[np.arange(H), np.arange(H)] = 1.0
    z["layers.0.w_gate"], z["layers.0.w_up"], z["layers.0.w_down"] = bits(Wg), bits(c * Wg), bits(Wd)
    m = oracle.Model(cfg, z, 4, _names(cfg))
    out = m.decode_step(123, 0, want_hidden=True)
    x_mid, x_out = out["hidden"][1], out["hidden"][2]
    # attention weights are zero: x_mid is the embedding row
    np.testing.assert_array_equal(x_mid, oracle.bf16_to_f64(w["tok_emb"][123]))
    g = oracle.bf16_to_f64(w["layers.0.ffn_norm"])
    h = x_mid / np.sqrt(np.mean(x_mid * x_mid) + cfg.rms_eps) * g
    silu = h / (1.0 + np.exp(-h))
    np.testing.assert_allclose(x_out - x_mid, silu * c * h, rtol=1e-12, atol=1e-15)
    swapped = c * h / (1.0 + np.exp(-c * h)) * h
    assert np.max(np.abs((x_out - x_mid) - swapped)) > 1e-3


def test_failing_expert_provider_raises():
    """A provider that cannot supply a matrix ends the step with an error: the
    oracle never computes with a partly filled expert buffer."""
    cfg = syn.TINY_MOE
    w = _weights(cfg)
    lazy_w = {k: v for k, v in w.items() if not any(s in k for s in ("w_gate", "w_up", "w_down"))}

    def short(l, e, which):
        return np.zeros(3, dtype=np.uint16)          # wrong size

    m = oracle.Model(cfg, lazy_w, 4, _names(cfg), expert_provider=short)
    with pytest.raises(RuntimeError, match="expert provider failed"):
        m.decode_step(9, 0)

    def boom(l, e, which):
        raise KeyError("no such expert")

    m = oracle.Model(cfg, lazy_w, 4, _names(cfg), expert_provider=boom)
    with pytest.raises(RuntimeError) as ei:
        m.forward_nocache([1, 2])
    assert isinstance(ei.value.__cause__, KeyError)
    # a provider that works afterwards still gives the held-weights result
    prov = lambda l, e, which: w[f"layers.{l}." + ("w_gate", "w_up", "w_down")[which]][e]
    ok = oracle.Model(cfg, lazy_w, 4, _names(cfg), expert_provider=prov).decode_step(9, 0)["logits"]
    np.testing.assert_array_equal(ok, oracle.Model(cfg, w, 4, _names(cfg)).decode_step(9, 0)["logits"])
