"""GPU test support: synthetic weights in HBM and a decoder through the C ABI."""
from __future__ import annotations

import numpy as np
import torch

import synthetic as syn
from persistent_megakernel_decode_03_b200.runner import Decoder


def desc_kwargs(cfg, flags: int = 0) -> dict:
    return dict(n_layers=cfg.n_layers, hidden=cfg.hidden, n_q_heads=cfg.n_q_heads,
                n_kv_heads=cfg.n_kv_heads, head_dim=cfg.head_dim, ffn=cfg.ffn, vocab=cfg.vocab,
                rms_eps=cfg.rms_eps, rope_theta=cfg.rope_theta, n_experts=cfg.n_experts,
                top_k=cfg.top_k, expert_ffn=cfg.expert_ffn, moe_renorm=cfg.moe_renorm, flags=flags)


def device_weights(cfg, seed: int, gain_sigma: float = 0.0):
    """bf16 tensors filled on the device by the seeded generator (same bits as the host fill)."""
    specs = syn.tensor_specs(cfg, gain_sigma)
    ts = []
    for s in specs:
        t = torch.empty(s.shape, dtype=torch.bfloat16, device="cuda")
        syn.dev_fill_tensor(t, s, seed)
        ts.append(t)
    torch.cuda.synchronize()
    return specs, ts


def make_decoder(cfg, tensors, max_batch: int, max_ctx: int, flags: int = 0, **kw) -> Decoder:
    return Decoder(desc_kwargs(cfg, flags), [t.data_ptr() for t in tensors], max_batch, max_ctx, **kw)


def fill_kv_context(dec: Decoder, cfg, seq: int, n_ctx: int, seed: int) -> None:
    """Synthetic cache contents for positions [0, n_ctx) of sequence `seq` (all layers)."""
    page_row = dec.page_table[seq]
    for l in range(cfg.n_layers):
        syn.dev_fill_kv_paged(dec.k_pages[l], page_row, seq, 0, n_ctx, cfg, 16, seed,
                              syn.TID_K_BASE + l)
        syn.dev_fill_kv_paged(dec.v_pages[l], page_row, seq, 0, n_ctx, cfg, 16, seed,
                              syn.TID_V_BASE + l)
    torch.cuda.synchronize()


def fill_oracle_kv(model, cfg, seq: int, n_ctx: int, seed: int) -> None:
    for l in range(cfg.n_layers):
        model.k[l][:n_ctx] = syn.host_kv(cfg, seed, l, "k", seq, 0, n_ctx)
        model.v[l][:n_ctx] = syn.host_kv(cfg, seed, l, "v", seq, 0, n_ctx)


def compare_logits(gpu: np.ndarray, ref: np.ndarray, max_abs: float = 0.05, min_cos: float = 0.9999):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = float(np.max(np.abs(gpu - ref)))
    cos = float(np.dot(gpu, ref) / (np.linalg.norm(gpu) * np.linalg.norm(ref)))
    return d, cos, (d <= max_abs and cos >= min_cos)
