"""Convenience owner of one model + task graph + state + paged KV cache.

PyTorch only provides device memory and streams here; every decode step is one
launch of the library's megakernel through the C ABI.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import (MK_OK, MkError, make_desc, make_kv, mk_build_taskgraph, mk_decode_step,
               mk_decode_step_host, mk_graph_destroy, mk_graph_get_info, mk_last_error_string,
               mk_load_model, mk_model_destroy, mk_prefill, mk_prefill_seq, mk_state_create,
               mk_state_destroy,
               mk_sync)

PAGE = 16


class Decoder:
    """Decode state for up to ``max_batch`` sequences of up to ``max_ctx`` tokens.

    ``weight_ptrs``: device pointers in the C ABI's order (tensors must outlive
    the decoder).  The KV pools are [L][n_pages][n_kv][16][head_dim] bf16;
    ``page_table`` is int32 [max_batch][max_pages]; by default sequence b owns
    pages b*max_pages .. (b+1)*max_pages-1 in order (contiguous cache).
    """

    def __init__(self, desc_kwargs: dict, weight_ptrs: Sequence[int], max_batch: int, max_ctx: int,
                 page_table: Optional[torch.Tensor] = None, n_pages: Optional[int] = None,
                 device: str = "cuda:0"):
        if not torch.cuda.is_available():
            raise RuntimeError("the megakernel needs a CUDA device; there is no CPU path")
        self.dev = torch.device(device)
        self.desc = make_desc(**desc_kwargs)
        d = self.desc
        self.max_batch, self.max_ctx = max_batch, max_ctx
        self.max_pages = (max_ctx + PAGE - 1) // PAGE
        if page_table is None:
            page_table = torch.arange(max_batch * self.max_pages, dtype=torch.int32,
                                      device=self.dev).view(max_batch, self.max_pages)
            n_pages = max_batch * self.max_pages
        assert page_table.dtype == torch.int32 and page_table.is_cuda
        assert page_table.shape == (max_batch, self.max_pages)
        self.page_table = page_table.contiguous()
        self.n_pages = int(n_pages)
        shape = (d.n_layers, self.n_pages, d.n_kv_heads, PAGE, d.head_dim)
        self.k_pages = torch.zeros(shape, dtype=torch.bfloat16, device=self.dev)
        self.v_pages = torch.zeros(shape, dtype=torch.bfloat16, device=self.dev)
        self.kv = make_kv(self.k_pages.data_ptr(), self.v_pages.data_ptr(),
                          self.page_table.data_ptr(), self.n_pages, self.max_pages)
        self.model = mk_load_model(self.desc, list(weight_ptrs))
        self.graph = mk_build_taskgraph(self.model, max_batch, max_ctx)
        self.state = mk_state_create(self.graph)
        self.info = mk_graph_get_info(self.graph)
        self.logits = torch.empty((max_batch, d.vocab), dtype=torch.float32, device=self.dev)

    def stream(self) -> int:
        return torch.cuda.current_stream(self.dev).cuda_stream

    def step(self, tokens: torch.Tensor, positions: torch.Tensor) -> torch.Tensor:
        """tokens, positions: int32 device [batch]; returns logits [batch][vocab] (a view)."""
        b = tokens.numel()
        mk_decode_step(self.state, tokens.data_ptr(), positions.data_ptr(), b, self.kv,
                       self.logits.data_ptr(), self.stream())
        return self.logits[:b]

    def step_host(self, tokens_host, positions_host, logits_host) -> None:
        """Host int32 arrays in, host fp32 logits out (numpy arrays or pinned tensors)."""
        def ptr(a):
            return a.data_ptr() if isinstance(a, torch.Tensor) else a.ctypes.data
        mk_decode_step_host(self.state, ptr(tokens_host), ptr(positions_host), len(tokens_host),
                            self.kv, ptr(logits_host), self.stream())

    def prefill(self, tokens: torch.Tensor, pos0: int = 0, seq: int = 0) -> torch.Tensor:
        """Prompt of sequence `seq` (a page-table row) at positions pos0 .. pos0 + n - 1;
        returns the last token's logits [vocab]."""
        out = self.logits[seq]
        if pos0 == 0:
            mk_prefill(self.state, tokens.data_ptr(), tokens.numel(), seq, self.kv, out.data_ptr(),
                       self.stream())
        else:
            mk_prefill_seq(self.state, tokens.data_ptr(), tokens.numel(), pos0, seq, self.kv,
                           out.data_ptr(), self.stream())
        return out

    def sync(self) -> int:
        return mk_sync(self.state, self.stream())

    def check(self) -> None:
        st = self.sync()
        if st != MK_OK:
            raise MkError(st, mk_last_error_string())

    def close(self) -> None:
        if getattr(self, "state", None):
            mk_state_destroy(self.state)
            self.state = None
        if getattr(self, "graph", None):
            mk_graph_destroy(self.graph)
            self.graph = None
        if getattr(self, "model", None):
            mk_model_destroy(self.model)
            self.model = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
