"""Full-size parity of the megakernel for the MoE and the long-context workloads.

Both run in the launch configuration that the bench times (same graph shapes,
same synthetic context), and compare every logit of a few steps with the
oracle, element by element.

* MoE 30B-total / 3.3B-active (48 layers, 128 experts, top-8) over an
  8192-token synthetic cache.  The oracle regenerates expert matrices on demand
  (all 128 experts per layer would not fit host memory).  Router choices must
  agree; where they differ, the 8th and 9th router logits must be within 1e-4
  (a near-tie that fp32 and double may break differently).  The oracle then
  takes the GPU's set for that layer, and the case is counted, not failed.
* 8B-class shapes at 131072 tokens of context in shuffled 16-token pages, with
  2 layers (the attention tiles and split counts of the long-context bench; the
  layer count only scales the work).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import persistent_megakernel_decode_03_b200 as mk
import synthetic as syn
from tests.gpu_util import compare_logits, device_weights, fill_kv_context, fill_oracle_kv, make_decoder
from tests.test_gpu_parity import check_counters, names

pytestmark = pytest.mark.gpu

NEAR_TIE = 1e-4


def _router_gap(orc_w, cfg, l, x_mid, sel):
    """Gap between the k-th and (k+1)-th router logit at layer l (oracle arithmetic)."""
    h = oracle.rmsnorm(x_mid, orc_w[f"layers.{l}.ffn_norm"], cfg.rms_eps)
    r = np.sort(oracle.gemv(orc_w[f"layers.{l}.w_router"], h))[::-1]
    return float(r[cfg.top_k - 1] - r[cfg.top_k])


def test_moe30b_full_size_over_8192_token_context():
    cfg = syn.MOE30B
    seed = syn.SEED_WEIGHTS + 3
    n_ctx = 8192
    specs, ts = device_weights(cfg, seed)
    dec = make_decoder(cfg, ts, 1, n_ctx + 256)
    fill_kv_context(dec, cfg, 0, n_ctx, syn.SEED_KV + 3)

    by_name = {s.name: s for s in specs}
    experts = ("w_gate", "w_up", "w_down")
    host_w = {s.name: syn.host_tensor(s, seed) for s in specs
              if not any(s.name.endswith(e) for e in experts)}
    n = cfg.expert_ffn * cfg.hidden

    def prov(l, e, which):
        s = by_name[f"layers.{l}.{experts[which]}"]
        return syn.host_bf16(n, seed, s.tensor_id, s.sigma, s.mean, offset=e * n)

    orc = oracle.Model(cfg, host_w, n_ctx + 4, names(cfg), expert_provider=prov)
    fill_oracle_kv(orc, cfg, 0, n_ctx, syn.SEED_KV + 3)
    toks = syn.host_tokens(2, syn.SEED_PROMPT + 3, cfg.vocab)
    flagged = 0
    for i, t in enumerate(toks):
        p = n_ctx + i
        g = dec.step(torch.tensor([int(t)], dtype=torch.int32, device="cuda"),
                     torch.tensor([p], dtype=torch.int32, device="cuda")).cpu().numpy()[0]
        dec.check()
        sel_g = np.array([mk.mk_state_read_buffer(dec.state, 3, l, cfg.top_k)
                          for l in range(cfg.n_layers)]).astype(np.int32)
        override = -np.ones((cfg.n_layers, cfg.top_k), dtype=np.int32)
        for _ in range(cfg.n_layers):
            out = orc.decode_step(int(t), p, want_hidden=True, moe_override=override)
            bad = [l for l in range(cfg.n_layers) if not np.array_equal(sel_g[l], out["moe_sel"][l])]
            if not bad:
                break
            l = bad[0]
            gap = _router_gap(host_w, cfg, l, out["hidden"][2 * l + 1], out["moe_sel"][l])
            assert gap < NEAR_TIE, f"position {p} layer {l}: router sets differ with gap {gap:.3g}"
            override[l] = sel_g[l]
            flagged += 1
        d, cos, ok = compare_logits(g, out["logits"])
        print(f"MoE step at position {p}: max|diff| {d:.3g} cos {cos:.8f} near-ties {flagged}")
        assert ok, (p, d, cos)
        check_counters(dec)
    dec.close()


def test_long_context_131072_tokens_shuffled_pages():
    cfg = dataclasses.replace(syn.LLAMA8B, n_layers=2)
    seed = syn.SEED_WEIGHTS + 5
    n_ctx = 131072
    max_ctx = n_ctx + 64
    pages = (max_ctx + 15) // 16
    perm = torch.tensor(syn.page_permutation(pages, syn.SEED_KV + 5), dtype=torch.int32,
                        device="cuda").view(1, pages)
    specs, ts = device_weights(cfg, seed)
    dec = make_decoder(cfg, ts, 1, max_ctx, page_table=perm, n_pages=pages)
    fill_kv_context(dec, cfg, 0, n_ctx, syn.SEED_KV + 5)
    orc = oracle.Model(cfg, syn.host_weights(cfg, seed), n_ctx + 2, names(cfg))
    fill_oracle_kv(orc, cfg, 0, n_ctx, syn.SEED_KV + 5)
    toks = syn.host_tokens(2, syn.SEED_PROMPT + 5, cfg.vocab)
    for i, t in enumerate(toks):
        p = n_ctx + i
        g = dec.step(torch.tensor([int(t)], dtype=torch.int32, device="cuda"),
                     torch.tensor([p], dtype=torch.int32, device="cuda")).cpu().numpy()[0]
        dec.check()
        ref = orc.decode_step(int(t), p)["logits"]
        d, cos, ok = compare_logits(g, ref)
        print(f"131072-context step at position {p}: max|diff| {d:.3g} cos {cos:.8f}")
        assert ok, (p, d, cos)
        check_counters(dec)
    # the appended entries landed in the shuffled pages: K of the new positions equals
    # the oracle's (bf16 bits, rare 1-ulp differences from accumulation order)
    k_gpu = dec.k_pages[0].view(torch.int16)
    for i in range(2):
        p = n_ctx + i
        page = int(perm[0, p // 16])
        got = k_gpu[page, :, p % 16, :].cpu().numpy().view(np.uint16).astype(np.int32)
        diff = np.abs(got - orc.k[0][p].astype(np.int32))
        assert diff.max() <= 1, p
    dec.close()
