"""Tensor-parallel decode: a dense model split over ranks, one megakernel per rank.

The model is cut the usual Megatron way: rank r holds q heads
[r*nq/tp, (r+1)*nq/tp) with their KV heads (so each rank's attention is
self-contained), the O-projection's matching columns, FFN rows
[r*F/tp, (r+1)*F/tp) of gate/up and the matching columns of down, and rows
[r*V/tp, (r+1)*V/tp) of the LM head; the embedding and the norms are whole on
every rank.  Inside the megakernel each O- and down-projection tile pushes its
partial sums of its residual rows into every rank's receive buffer and raises
that tile's arrival flag; reduce tasks add the ranks' parts as soon as their own
rows are complete (MPK digest, "Part 1. Compiler": the all-reduce after a matmul
starts on the finished parts of the product).

PyTorch is plumbing here (device memory, the rank group's handle exchange);
every step is one megakernel launch per rank through the C ABI.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import torch

from . import (MK_OK, MkError, make_desc, make_kv, mk_build_taskgraph, mk_decode_step,
               mk_decode_step_tp_emulated, mk_graph_destroy, mk_last_error_string, mk_load_model_tp,
               mk_model_destroy, mk_state_create, mk_state_destroy, mk_state_tp_buffer,
               mk_state_tp_ipc_handle, mk_state_tp_open_peer, mk_state_tp_set_peer, mk_sync)

PAGE = 16
DENSE_SLOTS = 9      # attn_norm, wq, wk, wv, wo, ffn_norm, w_gate, w_up, w_down


def shard_weights(desc_kwargs: dict, tensors: Sequence[torch.Tensor], tp: int, rank: int) -> List[torch.Tensor]:
    """Rank `rank`'s shard of a dense model's weights (the C ABI's order), as
    contiguous tensors on the tensors' device.  Row slices are views made
    contiguous; column slices (wo, w_down) are copies."""
    L, H = desc_kwargs["n_layers"], desc_kwargs["hidden"]
    nq, nkv, hd = desc_kwargs["n_q_heads"], desc_kwargs["n_kv_heads"], desc_kwargs["head_dim"]
    F, V = desc_kwargs["ffn"], desc_kwargs["vocab"]
    if desc_kwargs.get("n_experts", 0):
        raise ValueError("tensor parallelism covers dense models")
    if nkv % tp or F % tp or V % tp or (F // tp) % 8:
        raise ValueError("the model does not divide evenly over the ranks")
    if len(tensors) != 1 + L * DENSE_SLOTS + 2:
        raise ValueError("expected the dense model's weight list")
    qs, ks, fs, vs = nq // tp * hd, nkv // tp * hd, F // tp, V // tp
    out = [tensors[0].contiguous()]
    for l in range(L):
        an, wq, wk, wv, wo, fn, wg, wu, wd = tensors[1 + l * DENSE_SLOTS: 1 + (l + 1) * DENSE_SLOTS]
        out += [an.contiguous(),
                wq[rank * qs:(rank + 1) * qs].contiguous(),
                wk[rank * ks:(rank + 1) * ks].contiguous(),
                wv[rank * ks:(rank + 1) * ks].contiguous(),
                wo[:, rank * qs:(rank + 1) * qs].contiguous(),
                fn.contiguous(),
                wg[rank * fs:(rank + 1) * fs].contiguous(),
                wu[rank * fs:(rank + 1) * fs].contiguous(),
                wd[:, rank * fs:(rank + 1) * fs].contiguous()]
    out.append(tensors[1 + L * DENSE_SLOTS].contiguous())
    out.append(tensors[2 + L * DENSE_SLOTS][rank * vs:(rank + 1) * vs].contiguous())
    return out


def kv_heads_of(desc_kwargs: dict, tp: int, rank: int) -> range:
    """The KV heads rank `rank` holds (its KV cache holds exactly these)."""
    n = desc_kwargs["n_kv_heads"] // tp
    return range(rank * n, (rank + 1) * n)


def exchange_handles(local: bytes, group=None) -> List[bytes]:
    """Every rank's IPC handle, in rank order, through the process group (any
    backend: the handles are host bytes)."""
    import torch.distributed as dist
    out: List[Optional[bytes]] = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, bytes(local), group=group)
    if any(h is None or len(h) != len(local) for h in out):
        raise RuntimeError("tensor parallelism: a rank sent no handle")
    return [bytes(h) for h in out]


class _RankState:
    """One rank's model shard, batch-1 graph, state and KV cache (this device)."""

    def __init__(self, desc_kwargs: dict, shard: Sequence[torch.Tensor], tp: int, rank: int, max_ctx: int,
                 device: torch.device):
        self.dev = device
        self.desc = make_desc(**desc_kwargs)
        self.tp, self.rank = tp, rank
        self.max_ctx = max_ctx
        self.max_pages = (max_ctx + PAGE - 1) // PAGE
        nkv = desc_kwargs["n_kv_heads"] // tp
        shape = (desc_kwargs["n_layers"], self.max_pages, nkv, PAGE, desc_kwargs["head_dim"])
        self.k_pages = torch.zeros(shape, dtype=torch.bfloat16, device=device)
        self.v_pages = torch.zeros(shape, dtype=torch.bfloat16, device=device)
        self.page_table = torch.arange(self.max_pages, dtype=torch.int32, device=device).view(1, -1)
        self.kv = make_kv(self.k_pages.data_ptr(), self.v_pages.data_ptr(), self.page_table.data_ptr(),
                          self.max_pages, self.max_pages)
        self.shard = list(shard)        # kept alive: the library borrows the weights
        self.model = mk_load_model_tp(self.desc, tp, rank, [t.data_ptr() for t in self.shard])
        self.graph = mk_build_taskgraph(self.model, 1, max_ctx)
        self.state = mk_state_create(self.graph)
        self.logits = torch.empty(desc_kwargs["vocab"] // tp, dtype=torch.float32, device=device)

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


class TPRank(_RankState):
    """This process's rank of a tensor-parallel decoder (one process per GPU,
    torch.distributed initialised).  The receive buffers are shared through CUDA
    IPC handles exchanged over the process group; every rank must call step()
    with the same token and position, in the same order."""

    def __init__(self, desc_kwargs: dict, shard: Sequence[torch.Tensor], max_ctx: int, group=None):
        import torch.distributed as dist
        tp, rank = dist.get_world_size(group), dist.get_rank(group)
        super().__init__(desc_kwargs, shard, tp, rank, max_ctx, torch.device("cuda", torch.cuda.current_device()))
        handles = exchange_handles(mk_state_tp_ipc_handle(self.state), group)
        for q, h in enumerate(handles):
            if q != rank:
                mk_state_tp_open_peer(self.state, q, h)

    def step(self, token: torch.Tensor, position: torch.Tensor) -> torch.Tensor:
        """token, position: int32 device [1]; returns this rank's logits shard."""
        mk_decode_step(self.state, token.data_ptr(), position.data_ptr(), 1, self.kv, self.logits.data_ptr(),
                       torch.cuda.current_stream(self.dev).cuda_stream)
        return self.logits

    def check(self) -> None:
        st = mk_sync(self.state, torch.cuda.current_stream(self.dev).cuda_stream)
        if st != MK_OK:
            raise MkError(st, mk_last_error_string())


class EmulatedTP:
    """n ranks (2..4) of a tensor-parallel decoder on ONE GPU: each rank's state
    points at the others' buffers on the same device, and a step runs all ranks
    in one cooperative launch (each on n_sm/n SMs), since ranks whose kernels wait
    on one another must never be separate launches on one GPU."""

    def __init__(self, desc_kwargs: dict, tensors: Sequence[torch.Tensor], tp: int, max_ctx: int,
                 device: str = "cuda:0"):
        if not torch.cuda.is_available():
            raise RuntimeError("the megakernel needs a CUDA device; there is no CPU path")
        dev = torch.device(device)
        self.tp = tp
        self.vocab = desc_kwargs["vocab"]
        self.ranks = [_RankState(desc_kwargs, shard_weights(desc_kwargs, tensors, tp, r), tp, r, max_ctx, dev)
                      for r in range(tp)]
        bases = [mk_state_tp_buffer(r.state)[0] for r in self.ranks]
        for r in self.ranks:
            for q, b in enumerate(bases):
                if q != r.rank:
                    mk_state_tp_set_peer(r.state, q, b)
        self.dev = dev

    def step(self, token: torch.Tensor, position: torch.Tensor) -> torch.Tensor:
        """token, position: int32 device [1]; returns the whole logits row [vocab]
        (the ranks' shards concatenated)."""
        mk_decode_step_tp_emulated([r.state for r in self.ranks], token.data_ptr(), position.data_ptr(),
                                   [r.kv for r in self.ranks], [r.logits.data_ptr() for r in self.ranks],
                                   torch.cuda.current_stream(self.dev).cuda_stream)
        return torch.cat([r.logits for r in self.ranks])

    def check(self) -> None:
        s = torch.cuda.current_stream(self.dev).cuda_stream
        for r in self.ranks:
            st = mk_sync(r.state, s)
            if st != MK_OK:
                raise MkError(st, mk_last_error_string())

    def close(self) -> None:
        for r in self.ranks:
            r.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
