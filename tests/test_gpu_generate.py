"""Greedy generation on the device (mk_generate): no host round trip per token.

The tokens chosen on the GPU (argmax of each step's logits, ties to the lowest
index) must be the oracle's own greedy sequence, token for token: the tiny
config's prompt and 16 new tokens at batch 1, and ragged synthetic contexts at
batch 4 on the tensor-core path.
"""
import numpy as np
import pytest
import torch

import oracle
import persistent_megakernel_decode_03_b200 as mk
import synthetic as syn
from tests.gpu_util import device_weights, fill_kv_context, fill_oracle_kv, make_decoder
from tests.test_gpu_parity import check_counters, names

pytestmark = pytest.mark.gpu


def test_tiny_prompt_then_16_greedy_tokens_on_device():
    cfg = syn.TINY
    seed = syn.SEED_WEIGHTS + 1
    specs, ts = device_weights(cfg, seed)
    dec = make_decoder(cfg, ts, 1, 64)
    prompt = [int(t) for t in syn.host_tokens(39, syn.SEED_PROMPT + 1, cfg.vocab)]
    last = dec.prefill(torch.tensor(prompt, dtype=torch.int32, device="cuda")).cpu().numpy()
    dec.check()
    orc = oracle.Model(cfg, syn.host_weights(cfg, seed), 64, names(cfg))
    for p, t in enumerate(prompt):
        ref = orc.decode_step(t, p)["logits"]
    first = int(np.argmax(ref))
    assert int(np.argmax(last)) == first
    want = []
    tok = first
    for i in range(16):
        ref = orc.decode_step(tok, 39 + i)["logits"]
        tok = int(np.argmax(ref))
        want.append(tok)
    out = torch.zeros((16, 1), dtype=torch.int32, device="cuda")
    logits = torch.empty((1, cfg.vocab), dtype=torch.float32, device="cuda")
    # (the input tensors are held until the enqueued steps have read them)
    first_d = torch.tensor([first], dtype=torch.int32, device="cuda")
    pos_d = torch.tensor([39], dtype=torch.int32, device="cuda")
    mk.mk_generate(dec.state, first_d.data_ptr(), pos_d.data_ptr(), 1, 16, dec.kv,
                   out.data_ptr(), logits.data_ptr(), dec.stream())
    torch.cuda.synchronize()
    dec.check()
    check_counters(dec)
    assert out[:, 0].cpu().tolist() == want
    dec.close()


def test_batched_greedy_generation_on_device():
    cfg = syn.TINY
    seed = syn.SEED_WEIGHTS + 98
    B, n = 4, 8
    lens = [17, 80, 5, 133]
    specs, ts = device_weights(cfg, seed)
    dec = make_decoder(cfg, ts, B, 160)
    host_w = syn.host_weights(cfg, seed)
    want = []
    firsts = [int(t) for t in syn.host_tokens(B, syn.SEED_PROMPT + 98, cfg.vocab)]
    for b in range(B):
        fill_kv_context(dec, cfg, b, lens[b], syn.SEED_KV + 98)
        o = oracle.Model(cfg, host_w, 160, names(cfg))
        fill_oracle_kv(o, cfg, b, lens[b], syn.SEED_KV + 98)
        tok, seq = firsts[b], []
        for i in range(n):
            tok = int(np.argmax(o.decode_step(tok, lens[b] + i)["logits"]))
            seq.append(tok)
        want.append(seq)
    out = torch.zeros((n, B), dtype=torch.int32, device="cuda")
    logits = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
    firsts_d = torch.tensor(firsts, dtype=torch.int32, device="cuda")
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    mk.mk_generate(dec.state, firsts_d.data_ptr(), lens_d.data_ptr(), B, n, dec.kv,
                   out.data_ptr(), logits.data_ptr(), dec.stream())
    torch.cuda.synchronize()
    dec.check()
    check_counters(dec)
    got = out.cpu().numpy()
    for b in range(B):
        assert got[:, b].tolist() == want[b], b
    dec.close()


@pytest.mark.parametrize("B", [1, 4])
def test_in_step_argmax_over_a_large_vocabulary(B):
    """8B shapes (2 layers, 128256-token vocabulary: thousands of LM-head tiles, many
    argmax groups): after each enqueued step the token written on the device is the
    first index of the largest logit of that step (torch's argmax picks the first
    maximum too), for every sequence."""
    import dataclasses
    cfg = dataclasses.replace(syn.LLAMA8B, n_layers=2)
    specs, ts = device_weights(cfg, syn.SEED_WEIGHTS + 71)
    dec = make_decoder(cfg, ts, B, 64)
    firsts = torch.tensor([int(t) for t in syn.host_tokens(B, 71, cfg.vocab)], dtype=torch.int32, device="cuda")
    pos = torch.tensor([3 * b for b in range(B)], dtype=torch.int32, device="cuda")
    n = 3
    out = torch.full((n, B), -1, dtype=torch.int32, device="cuda")
    logits = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
    for k in range(n):
        # one step at a time, so each step's logits can be checked
        first_k = firsts if k == 0 else out[k - 1].clone()
        pos_k = pos + k                                  # (held until the step has run)
        mk.mk_generate(dec.state, first_k.data_ptr(), pos_k.data_ptr(), B, 1, dec.kv,
                       out[k].data_ptr(), logits.data_ptr(), dec.stream())
        torch.cuda.synchronize()
        dec.check()
        assert out[k].cpu().tolist() == torch.argmax(logits[:B], dim=1).int().cpu().tolist(), k
    check_counters(dec)
    dec.close()
