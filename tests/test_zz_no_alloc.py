"""The allocation-free decode step against the regular one.

Callers that may not allocate device memory (code running where cudaMalloc is
forbidden, or runtimes with a fixed memory budget) use mk_decode_step_noalloc,
whose scratch is a fixed device array inside the library.  Two decode steps in a
row must give the logits of mk_decode_step on the same inputs, within the
parity tolerance of the other tests.  This file is collected last so that a run
stopping at the first failure has already run everything else; it also passes
when run alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import persistent_megakernel_decode_03_b200 as mk
import synthetic as syn
from tests.gpu_util import compare_logits, desc_kwargs, device_weights, make_decoder

pytestmark = pytest.mark.gpu


def test_noalloc_step_matches_regular_step_twice():
    cfg = syn.TINY
    specs, ts = device_weights(cfg, syn.SEED_WEIGHTS + 1)
    max_ctx = 64
    dec = make_decoder(cfg, ts, 1, max_ctx)             # regular path, its own KV cache
    k2 = torch.zeros_like(dec.k_pages)                  # separate KV cache for the other path
    v2 = torch.zeros_like(dec.v_pages)
    kv2 = mk.make_kv(k2.data_ptr(), v2.data_ptr(), dec.page_table.data_ptr(), dec.n_pages, dec.max_pages)
    desc = mk.make_desc(**desc_kwargs(cfg))
    ptrs = [t.data_ptr() for t in ts]
    out = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    for p, tok in enumerate([17, 401]):
        t = torch.tensor([tok], dtype=torch.int32, device="cuda")
        pos = torch.tensor([p], dtype=torch.int32, device="cuda")
        ref = dec.step(t, pos).clone()
        dec.check()
        mk.mk_decode_step_noalloc(desc, ptrs, max_ctx, t.data_ptr(), pos.data_ptr(), 1, kv2,
                                  out.data_ptr(), torch.cuda.current_stream().cuda_stream)
        d, cos, ok = compare_logits(out.cpu().numpy(), ref.cpu().numpy()[0])
        assert ok, (p, d, cos)
    # the appended KV entries agree too
    np.testing.assert_array_equal(k2.view(torch.int16).cpu().numpy(), dec.k_pages.view(torch.int16).cpu().numpy())
    np.testing.assert_array_equal(v2.view(torch.int16).cpu().numpy(), dec.v_pages.view(torch.int16).cpu().numpy())
    dec.close()


def test_noalloc_rejects_too_large_and_bad_arguments():
    cfg = syn.TINY
    specs, ts = device_weights(cfg, 3)
    desc = mk.make_desc(**desc_kwargs(cfg))
    ptrs = [t.data_ptr() for t in ts]
    kv_t = torch.zeros((cfg.n_layers, 4, cfg.n_kv_heads, 16, cfg.head_dim), dtype=torch.bfloat16, device="cuda")
    pt = torch.arange(4, dtype=torch.int32, device="cuda")
    kv = mk.make_kv(kv_t.data_ptr(), kv_t.data_ptr(), pt.data_ptr(), 4, 4)
    t = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    with pytest.raises(mk.MkError) as e:          # a context whose tables exceed the array
        mk.mk_decode_step_noalloc(desc, ptrs, 1 << 21, t.data_ptr(), t.data_ptr(), 1, kv, out.data_ptr())
    assert e.value.status == mk.MK_ERR_UNSUPPORTED
    with pytest.raises(mk.MkError):                # batch > 1
        mk.mk_decode_step_noalloc(desc, ptrs, 64, t.data_ptr(), t.data_ptr(), 2, kv, out.data_ptr())


def _noalloc_vs_regular(cfg, seed, max_ctx, tokens):
    """Runs `tokens` at positions 0.. through both paths (separate KV caches) and
    compares the logits step by step."""
    specs, ts = device_weights(cfg, seed)
    dec = make_decoder(cfg, ts, 1, max_ctx)
    k2, v2 = torch.zeros_like(dec.k_pages), torch.zeros_like(dec.v_pages)
    kv2 = mk.make_kv(k2.data_ptr(), v2.data_ptr(), dec.page_table.data_ptr(), dec.n_pages, dec.max_pages)
    desc = mk.make_desc(**desc_kwargs(cfg))
    ptrs = [t.data_ptr() for t in ts]
    out = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    for p, tok in enumerate(tokens):
        t = torch.tensor([tok], dtype=torch.int32, device="cuda")
        pos = torch.tensor([p], dtype=torch.int32, device="cuda")
        ref = dec.step(t, pos).clone()
        dec.check()
        mk.mk_decode_step_noalloc(desc, ptrs, max_ctx, t.data_ptr(), pos.data_ptr(), 1, kv2,
                                  out.data_ptr(), torch.cuda.current_stream().cuda_stream)
        d, cos, ok = compare_logits(out.cpu().numpy(), ref.cpu().numpy()[0])
        assert ok, (cfg.name, max_ctx, p, d, cos)
    np.testing.assert_array_equal(k2.view(torch.int16).cpu().numpy(), dec.k_pages.view(torch.int16).cpu().numpy())
    dec.close()


def test_noalloc_replans_for_another_context_and_a_moe_model():
    """The array keeps the last plan: a new context length, a routed-expert model
    (its router, selection and expert buffers live in the array too), and the
    first model again must each be planned afresh and match the regular path."""
    _noalloc_vs_regular(syn.TINY, syn.SEED_WEIGHTS + 1, 64, [17, 401, 5])
    _noalloc_vs_regular(syn.TINY, syn.SEED_WEIGHTS + 1, 200, [9, 33])
    _noalloc_vs_regular(syn.TINY_MOE, syn.SEED_WEIGHTS + 4, 64, [3, 700, 12])
    _noalloc_vs_regular(syn.TINY, syn.SEED_WEIGHTS + 2, 64, [1, 2])
