"""Python binding of libmk.so, the persistent decode megakernel for B200 (sm_100a).

Argument marshalling only: every step of the decode path runs in the library's
CUDA kernels.  The functions carry the names of the C ABI in ``include/mk.h``
and take raw integers for pointers (``tensor.data_ptr()``) and streams
(``torch.cuda.current_stream().cuda_stream``).  Errors raise ``MkError``.

There is no CPU path: importing works without a GPU (for inspecting task
graphs built on the host), but every call that needs the device fails loudly
when the CUDA library or a GPU is missing.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
# MK_LIBRARY may name another build of the same C ABI (e.g. an experimental one).
LIB_PATH = os.environ.get("MK_LIBRARY") or os.path.join(_HERE, "libmk.so")

MK_OK = 0
MK_ERR_INVALID_ARG = 1
MK_ERR_CUDA = 2
MK_ERR_OOM = 3
MK_ERR_UNSUPPORTED = 4
MK_ERR_TIMEOUT = 5
MK_ERR_DEVICE_FAULT = 6
MK_FLAG_TRACE = 0x1
MK_NO_EVENT = 0xFFFFFFFF

MK_OP_QKV, MK_OP_ATTN, MK_OP_OPROJ, MK_OP_GATEUP, MK_OP_DOWN, MK_OP_LMHEAD = 1, 2, 3, 4, 5, 6
MK_OP_ROUTER, MK_OP_EXP_GATEUP, MK_OP_EXP_DOWN = 7, 8, 9
MK_OP_NORM, MK_OP_MM_QKV, MK_OP_MM_OPROJ, MK_OP_MM_GATEUP, MK_OP_MM_DOWN, MK_OP_MM_LMHEAD = (
    10, 11, 12, 13, 14, 15)
MM_OPS = (MK_OP_MM_QKV, MK_OP_MM_OPROJ, MK_OP_MM_GATEUP, MK_OP_MM_DOWN, MK_OP_MM_LMHEAD)
MK_OP_KVAPPEND = 16
MK_OP_ATTN_MERGE = 17
MK_OP_TP_REDUCE = 18
MK_TP_IPC_HANDLE_BYTES = 64
OP_NAMES = {1: "qkv", 2: "attn", 3: "oproj", 4: "gateup", 5: "down", 6: "lmhead", 7: "router",
            8: "exp_gateup", 9: "exp_down", 10: "norm", 11: "mm_qkv", 12: "mm_oproj", 13: "mm_gateup",
            14: "mm_down", 15: "mm_lmhead", 16: "kvappend", 17: "attn_merge", 18: "tp_reduce"}

# Exported symbols (declared in include/mk.h).
SYMBOLS = (
    "mk_load_model", "mk_model_destroy", "mk_build_taskgraph", "mk_build_taskgraph_solo",
    "mk_plan_taskgraph",
    "mk_graph_destroy", "mk_graph_get_info", "mk_graph_export_tasks", "mk_graph_export_thresholds",
    "mk_wave_stats", "mk_state_create", "mk_state_destroy", "mk_state_set_timeout",
    "mk_state_debug_wait_offset", "mk_state_set_prefetch",
    "mk_decode_step", "mk_decode_step_host", "mk_decode_step_per_op", "mk_generate", "mk_prefill", "mk_prefill_seq", "mk_decode_step_noalloc", "mk_sync",
    "mk_state_read_counters",
    "mk_state_read_buffer", "mk_state_read_trace", "mk_state_read_stats", "mk_last_error_string",
    "mk_version",
    "mk_load_model_tp", "mk_plan_taskgraph_tp", "mk_state_tp_buffer", "mk_state_tp_set_peer", "mk_state_tp_ipc_handle",
    "mk_state_tp_open_peer", "mk_decode_step_tp_emulated",
)


class MkError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"mk status {status}: {msg}")
        self.status = status


class mk_model_desc(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("hidden", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("ffn", ctypes.c_int),
                ("vocab", ctypes.c_int), ("rms_eps", ctypes.c_float), ("rope_theta", ctypes.c_float),
                ("n_experts", ctypes.c_int), ("top_k", ctypes.c_int), ("expert_ffn", ctypes.c_int),
                ("moe_renorm", ctypes.c_int), ("dtype", ctypes.c_int), ("flags", ctypes.c_uint)]


class mk_paged_kv(ctypes.Structure):
    _fields_ = [("k_pages", ctypes.c_void_p), ("v_pages", ctypes.c_void_p),
                ("page_table", ctypes.c_void_p), ("n_pages", ctypes.c_int),
                ("page_size", ctypes.c_int), ("max_pages_per_seq", ctypes.c_int)]


class mk_graph_info(ctypes.Structure):
    _fields_ = [("n_tasks", ctypes.c_int), ("n_events", ctypes.c_int), ("n_sm", ctypes.c_int),
                ("max_batch", ctypes.c_int), ("max_ctx", ctypes.c_int), ("attn_splits", ctypes.c_int),
                ("n_ops", ctypes.c_int), ("weight_bytes_per_step", ctypes.c_int64)]


class mk_task_info(ctypes.Structure):
    _fields_ = [("op", ctypes.c_int), ("layer", ctypes.c_int), ("b", ctypes.c_int),
                ("aux", ctypes.c_int), ("r0", ctypes.c_uint32), ("r1", ctypes.c_uint32),
                ("wait", ctypes.c_uint32 * 2), ("signal", ctypes.c_uint32),
                ("pointer_wait", ctypes.c_uint32)]


class mk_state_counters(ctypes.Structure):
    _fields_ = [("epoch", ctypes.c_uint32), ("done", ctypes.c_uint32),
                ("queue_head", ctypes.c_uint64), ("error", ctypes.c_int32),
                ("error_info", ctypes.c_int32 * 4)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libmk.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python persistent_megakernel_decode_03_b200/build.py` "
                               "(there is no fallback implementation)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_int
        P = ctypes.POINTER
        sig = {
            "mk_load_model": ([P(mk_model_desc), vp, i32, P(vp)], st),
            "mk_model_destroy": ([vp], None),
            "mk_build_taskgraph": ([vp, i32, i32, P(vp)], st),
            "mk_plan_taskgraph": ([P(mk_model_desc), i32, i32, i32, P(vp)], st),
            "mk_build_taskgraph_solo": ([vp, i32, i32, i32, P(vp)], st),
            "mk_graph_destroy": ([vp], None),
            "mk_graph_get_info": ([vp, P(mk_graph_info)], st),
            "mk_graph_export_tasks": ([vp, P(mk_task_info), i32, P(i32)], st),
            "mk_graph_export_thresholds": ([vp, P(ctypes.c_uint32), i32, P(i32)], st),
            "mk_wave_stats": ([i32, i32, P(i32), P(i32)], st),
            "mk_state_create": ([vp, P(vp)], st),
            "mk_state_destroy": ([vp], None),
            "mk_state_set_timeout": ([vp, ctypes.c_int64], st),
            "mk_state_debug_wait_offset": ([vp, ctypes.c_uint32], st),
            "mk_state_set_prefetch": ([vp, i32], st),
            "mk_decode_step": ([vp, vp, vp, i32, P(mk_paged_kv), vp, vp], st),
            "mk_decode_step_host": ([vp, vp, vp, i32, P(mk_paged_kv), vp, vp], st),
            "mk_prefill": ([vp, vp, i32, i32, P(mk_paged_kv), vp, vp], st),
            "mk_decode_step_per_op": ([vp, vp, vp, i32, P(mk_paged_kv), vp, vp, P(ctypes.c_int)], st),
            "mk_generate": ([vp, vp, vp, i32, i32, P(mk_paged_kv), vp, vp, vp], st),
            "mk_prefill_seq": ([vp, vp, i32, i32, i32, P(mk_paged_kv), vp, vp], st),
            "mk_decode_step_noalloc": ([P(mk_model_desc), vp, i32, i32, vp, vp, i32, P(mk_paged_kv),
                                        vp, vp], st),
            "mk_sync": ([vp, vp], st),
            "mk_state_read_counters": ([vp, vp, P(mk_state_counters), vp, i32], st),
            "mk_state_read_buffer": ([vp, i32, i32, vp, ctypes.c_size_t, vp], st),
            "mk_state_read_trace": ([vp, vp, i32, vp], st),
            "mk_state_read_stats": ([vp, vp, i32, vp], st),
            "mk_last_error_string": ([], ctypes.c_char_p),
            "mk_version": ([], ctypes.c_char_p),
            "mk_load_model_tp": ([P(mk_model_desc), i32, i32, vp, i32, P(vp)], st),
            "mk_plan_taskgraph_tp": ([P(mk_model_desc), i32, i32, i32, i32, P(vp)], st),
            "mk_state_tp_buffer": ([vp, P(vp), P(ctypes.c_size_t)], st),
            "mk_state_tp_set_peer": ([vp, i32, vp], st),
            "mk_state_tp_ipc_handle": ([vp, vp], st),
            "mk_state_tp_open_peer": ([vp, i32, vp], st),
            "mk_decode_step_tp_emulated": ([vp, i32, vp, vp, vp, vp, vp], st),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _check(status: int) -> None:
    if status != MK_OK:
        raise MkError(status, lib().mk_last_error_string().decode())


# ----------------------------------------------------------------------------- same-name wrappers

def mk_version() -> str:
    return lib().mk_version().decode()


def mk_last_error_string() -> str:
    return lib().mk_last_error_string().decode()


def mk_load_model(desc: mk_model_desc, weight_ptrs: Sequence[int]) -> int:
    arr = (ctypes.c_void_p * len(weight_ptrs))(*weight_ptrs)
    out = ctypes.c_void_p()
    _check(lib().mk_load_model(ctypes.byref(desc), arr, len(weight_ptrs), ctypes.byref(out)))
    return out.value


def mk_model_destroy(model: int) -> None:
    lib().mk_model_destroy(model)


def mk_build_taskgraph(model: int, max_batch: int, max_ctx: int) -> int:
    out = ctypes.c_void_p()
    _check(lib().mk_build_taskgraph(model, max_batch, max_ctx, ctypes.byref(out)))
    return out.value


def mk_build_taskgraph_solo(model: int, max_batch: int, max_ctx: int, op: int) -> int:
    out = ctypes.c_void_p()
    _check(lib().mk_build_taskgraph_solo(model, max_batch, max_ctx, op, ctypes.byref(out)))
    return out.value


def mk_plan_taskgraph(desc: mk_model_desc, max_batch: int, max_ctx: int, n_sm: int) -> int:
    out = ctypes.c_void_p()
    _check(lib().mk_plan_taskgraph(ctypes.byref(desc), max_batch, max_ctx, n_sm, ctypes.byref(out)))
    return out.value


def mk_graph_destroy(graph: int) -> None:
    lib().mk_graph_destroy(graph)


def mk_graph_get_info(graph: int) -> mk_graph_info:
    info = mk_graph_info()
    _check(lib().mk_graph_get_info(graph, ctypes.byref(info)))
    return info


def mk_graph_export_tasks(graph: int) -> List[mk_task_info]:
    n_tasks = mk_graph_get_info(graph).n_tasks
    arr = (mk_task_info * n_tasks)()
    n = ctypes.c_int()
    _check(lib().mk_graph_export_tasks(graph, arr, n_tasks, ctypes.byref(n)))
    return list(arr[: n.value])


def mk_graph_export_thresholds(graph: int) -> List[int]:
    n_ev = mk_graph_get_info(graph).n_events
    arr = (ctypes.c_uint32 * max(1, n_ev))()
    n = ctypes.c_int()
    _check(lib().mk_graph_export_thresholds(graph, arr, n_ev, ctypes.byref(n)))
    return list(arr[: n.value])


def mk_wave_stats(n_tiles: int, n_sm: int) -> Tuple[int, int]:
    w, i = ctypes.c_int(), ctypes.c_int()
    _check(lib().mk_wave_stats(n_tiles, n_sm, ctypes.byref(w), ctypes.byref(i)))
    return w.value, i.value


def mk_state_create(graph: int) -> int:
    out = ctypes.c_void_p()
    _check(lib().mk_state_create(graph, ctypes.byref(out)))
    return out.value


def mk_state_destroy(state: int) -> None:
    lib().mk_state_destroy(state)


def mk_state_set_timeout(state: int, timeout_ns: int) -> None:
    _check(lib().mk_state_set_timeout(state, int(timeout_ns)))


def mk_state_debug_wait_offset(state: int, offset: int) -> None:
    _check(lib().mk_state_debug_wait_offset(state, int(offset)))


def mk_state_set_prefetch(state: int, tasks_ahead: int) -> None:
    _check(lib().mk_state_set_prefetch(state, int(tasks_ahead)))


def mk_decode_step(state: int, token_ids: int, positions: int, batch: int, kv: mk_paged_kv,
                   logits_out: int, stream: int = 0) -> None:
    _check(lib().mk_decode_step(state, token_ids, positions, batch, ctypes.byref(kv), logits_out,
                                stream))


def mk_decode_step_host(state: int, token_ids: int, positions: int, batch: int, kv: mk_paged_kv,
                        logits_host: int, stream: int = 0) -> None:
    _check(lib().mk_decode_step_host(state, token_ids, positions, batch, ctypes.byref(kv),
                                     logits_host, stream))


def mk_prefill(state: int, tokens: int, n_tokens: int, seq_slot: int, kv: mk_paged_kv,
               last_logits: int, stream: int = 0) -> None:
    _check(lib().mk_prefill(state, tokens, n_tokens, seq_slot, ctypes.byref(kv), last_logits, stream))


def mk_decode_step_per_op(state: int, token_ids: int, positions: int, batch: int, kv: mk_paged_kv,
                          logits_out: int, stream: int = 0) -> int:
    """Kernel-per-operator baseline of one step; returns the number of launches."""
    n = ctypes.c_int(0)
    _check(lib().mk_decode_step_per_op(state, token_ids, positions, batch, ctypes.byref(kv), logits_out,
                                       stream, ctypes.byref(n)))
    return n.value


def mk_generate(state: int, first_tokens: int, positions: int, batch: int, n_steps: int, kv: mk_paged_kv,
                tokens_out: int, logits_out: int, stream: int = 0) -> None:
    _check(lib().mk_generate(state, first_tokens, positions, batch, n_steps, ctypes.byref(kv), tokens_out,
                             logits_out, stream))


def mk_prefill_seq(state: int, tokens: int, n_tokens: int, pos0: int, seq_slot: int, kv: mk_paged_kv,
                   last_logits: int, stream: int = 0) -> None:
    _check(lib().mk_prefill_seq(state, tokens, n_tokens, pos0, seq_slot, ctypes.byref(kv), last_logits,
                                stream))


def mk_decode_step_noalloc(desc: mk_model_desc, weight_ptrs: Sequence[int], max_ctx: int,
                           token_ids: int, positions: int, batch: int, kv: mk_paged_kv,
                           logits_out: int, stream: int = 0) -> None:
    """The allocation-free decode step (see include/mk.h); waits for the step."""
    arr = (ctypes.c_void_p * len(weight_ptrs))(*weight_ptrs)
    _check(lib().mk_decode_step_noalloc(ctypes.byref(desc), arr, len(weight_ptrs), max_ctx, token_ids,
                                        positions, batch, ctypes.byref(kv), logits_out, stream))


def mk_load_model_tp(desc: mk_model_desc, tp_size: int, tp_rank: int, weight_ptrs: Sequence[int]) -> int:
    """Rank tp_rank's shard of the model `desc` describes (weights: the shard's, in
    mk_load_model's order)."""
    arr = (ctypes.c_void_p * len(weight_ptrs))(*weight_ptrs)
    out = ctypes.c_void_p()
    _check(lib().mk_load_model_tp(ctypes.byref(desc), int(tp_size), int(tp_rank), arr, len(weight_ptrs),
                                  ctypes.byref(out)))
    return out.value


def mk_plan_taskgraph_tp(desc: mk_model_desc, tp_size: int, tp_rank: int, max_ctx: int, n_sm: int) -> int:
    """Host-only plan of one rank's tensor-parallel graph (no device needed)."""
    out = ctypes.c_void_p()
    _check(lib().mk_plan_taskgraph_tp(ctypes.byref(desc), int(tp_size), int(tp_rank), int(max_ctx), int(n_sm),
                                      ctypes.byref(out)))
    return out.value


def mk_state_tp_buffer(state: int) -> Tuple[int, int]:
    """(device address, bytes) of the state's receive buffer and arrival flags."""
    base, n = ctypes.c_void_p(), ctypes.c_size_t()
    _check(lib().mk_state_tp_buffer(state, ctypes.byref(base), ctypes.byref(n)))
    return base.value, n.value


def mk_state_tp_set_peer(state: int, rank: int, peer_base: int) -> None:
    _check(lib().mk_state_tp_set_peer(state, int(rank), peer_base))


def mk_state_tp_ipc_handle(state: int) -> bytes:
    buf = ctypes.create_string_buffer(MK_TP_IPC_HANDLE_BYTES)
    _check(lib().mk_state_tp_ipc_handle(state, buf))
    return buf.raw


def mk_state_tp_open_peer(state: int, rank: int, handle: bytes) -> None:
    if len(handle) != MK_TP_IPC_HANDLE_BYTES:
        raise ValueError("an IPC handle is 64 bytes")
    buf = ctypes.create_string_buffer(bytes(handle), MK_TP_IPC_HANDLE_BYTES)
    _check(lib().mk_state_tp_open_peer(state, int(rank), buf))


def mk_decode_step_tp_emulated(states: Sequence[int], token_ids: int, positions: int,
                               kvs: Sequence[mk_paged_kv], logits_out: Sequence[int], stream: int = 0) -> None:
    """len(states) ranks of one tensor-parallel model in one launch on this GPU."""
    n = len(states)
    st = (ctypes.c_void_p * n)(*states)
    kp = (ctypes.POINTER(mk_paged_kv) * n)(*[ctypes.pointer(k) for k in kvs])
    lo = (ctypes.c_void_p * n)(*logits_out)
    _check(lib().mk_decode_step_tp_emulated(st, n, token_ids, positions, kp, lo, stream))


def mk_sync(state: int, stream: int = 0) -> int:
    """Returns the device status (MK_OK or an error code) without raising."""
    return int(lib().mk_sync(state, stream))


def mk_state_read_counters(state: int, n_events: int = 0, stream: int = 0):
    c = mk_state_counters()
    ev = (ctypes.c_uint32 * max(1, n_events))()
    _check(lib().mk_state_read_counters(state, stream, ctypes.byref(c), ev if n_events else None,
                                        n_events))
    return c, list(ev[:n_events])


def mk_state_read_buffer(state: int, which: int, layer: int, n: int, stream: int = 0):
    buf = (ctypes.c_float * n)()
    _check(lib().mk_state_read_buffer(state, which, layer, buf, n, stream))
    return list(buf)


def mk_state_read_stats(state: int, n_sm: int, stream: int = 0):
    buf = (ctypes.c_uint64 * (8 * n_sm))()
    _check(lib().mk_state_read_stats(state, buf, 8 * n_sm, stream))
    return list(buf)


def mk_state_read_trace(state: int, n_tasks: int, stream: int = 0):
    buf = (ctypes.c_uint64 * (4 * n_tasks))()
    _check(lib().mk_state_read_trace(state, buf, n_tasks, stream))
    return list(buf)


# ----------------------------------------------------------------------------- helpers

def make_desc(n_layers: int, hidden: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
              ffn: int, vocab: int, rms_eps: float = 1e-5, rope_theta: float = 1e4,
              n_experts: int = 0, top_k: int = 0, expert_ffn: int = 0, moe_renorm: int = 1,
              flags: int = 0) -> mk_model_desc:
    d = mk_model_desc()
    d.n_layers, d.hidden, d.n_q_heads, d.n_kv_heads = n_layers, hidden, n_q_heads, n_kv_heads
    d.head_dim, d.ffn, d.vocab = head_dim, ffn, vocab
    d.rms_eps, d.rope_theta = rms_eps, rope_theta
    d.n_experts, d.top_k, d.expert_ffn, d.moe_renorm = n_experts, top_k, expert_ffn, moe_renorm
    d.dtype, d.flags = 0, flags
    return d


def make_kv(k_pages: int, v_pages: int, page_table: int, n_pages: int, max_pages_per_seq: int,
            page_size: int = 16) -> mk_paged_kv:
    kv = mk_paged_kv()
    kv.k_pages, kv.v_pages, kv.page_table = k_pages, v_pages, page_table
    kv.n_pages, kv.page_size, kv.max_pages_per_seq = n_pages, page_size, max_pages_per_seq
    return kv
