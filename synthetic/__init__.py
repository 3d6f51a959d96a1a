"""Seeded synthetic inputs for the decode step: model shapes, weights, KV, tokens.

This module is the only code that both the CPU oracle side and the CUDA side of
the tests use.  It draws random numbers and describes tensor shapes; it holds
none of the decode step's arithmetic.  Every value comes from the counter-based
generator defined in ``gen.h`` (SplitMix64 output function + Irwin-Hall sum of
12 uniforms), implemented once for the host (``synthetic.c``) and once for the
device (``synthetic_fill.cu``); the two give identical bits.

Workload shapes follow the pages' examples: an 8B-class dense decoder at batch
1 with a 39-token prompt (MPK digest, section "MPK का मुख्य मूल्य"), and a
30B-total / 3.3B-active MoE with 8K context (Cohere page, section "A szűk
keresztmetszet a memória-sávszélesség").
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import subprocess
from typing import Dict, List, Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_LIB = os.path.join(_HERE, "libsynthetic_host.so")
DEV_LIB = os.path.join(_HERE, "libsynthetic_dev.so")

# Seeds: weights 1000+cfg, prompt 2000+cfg, KV context 3000+cfg.
SEED_WEIGHTS = 1000
SEED_PROMPT = 2000
SEED_KV = 3000

# Tensor ids inside one seed's stream.
TID_TOK_EMB = 0
TID_FINAL_NORM = 8
TID_LM_HEAD = 9
TID_LAYER_BASE = 16          # layer l, slot s  ->  16 + 16*l + s
TID_K_BASE = 1 << 24         # K of layer l     ->  TID_K_BASE + l
TID_V_BASE = 2 << 24         # V of layer l     ->  TID_V_BASE + l
TID_TOKENS = 3 << 24         # token stream of sequence b -> TID_TOKENS + b
TID_LENS = 4 << 24           # ragged sequence lengths
TID_PAGES = 5 << 24          # page-permutation words

KV_SEQ_SHIFT = 20            # logical KV index = ((seq << 20) + pos) * n_kv*d + ...

WEIGHT_SIGMA = 0.02


@dataclasses.dataclass(frozen=True)
class ModelConfig:
    name: str
    n_layers: int
    hidden: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    rms_eps: float = 1e-5
    rope_theta: float = 1e4
    n_experts: int = 0
    top_k: int = 0
    expert_ffn: int = 0
    moe_renorm: int = 1

    @property
    def is_moe(self) -> bool:
        return self.n_experts > 0

    @property
    def q_dim(self) -> int:
        return self.n_q_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim


# The workloads (shapes only).
TINY = ModelConfig("tiny-2L-h256", 2, 256, 4, 2, 64, 688, 1024)
LLAMA8B = ModelConfig("llama-8b-class", 32, 4096, 32, 8, 128, 14336, 128256)
MOE30B = ModelConfig("moe-30b-a3b", 48, 2048, 32, 4, 128, 0, 151936,
                     n_experts=128, top_k=8, expert_ffn=768)
# Small shapes used only by tests (MoE and GQA structure at oracle-friendly size).
TINY_MOE = ModelConfig("tiny-moe-2L", 2, 256, 4, 2, 64, 0, 1024,
                       n_experts=16, top_k=4, expert_ffn=96)

CONFIGS = {c.name: c for c in (TINY, LLAMA8B, MOE30B, TINY_MOE)}


@dataclasses.dataclass(frozen=True)
class TensorSpec:
    name: str
    shape: Tuple[int, ...]
    tensor_id: int
    sigma: float
    mean: float

    @property
    def numel(self) -> int:
        return int(np.prod(self.shape))


DENSE_LAYER_SLOTS = ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_gate", "w_up", "w_down")
MOE_LAYER_SLOTS = ("attn_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w_router", "w_gate", "w_up",
                   "w_down")


def tensor_specs(cfg: ModelConfig, gain_sigma: float = 0.0) -> List[TensorSpec]:
    """All weight tensors of ``cfg`` in the C ABI's pointer order.

    Matrices and the embedding are ~N(0, 0.02^2); the router is ~N(0, 1/hidden)
    so that its logits are ~N(0, 1) for a unit-RMS input; norm gains are
    1 + N(0, gain_sigma^2) (exactly 1 when gain_sigma == 0).
    """
    H, V = cfg.hidden, cfg.vocab
    specs = [TensorSpec("tok_emb", (V, H), TID_TOK_EMB, WEIGHT_SIGMA, 0.0)]
    for l in range(cfg.n_layers):
        base = TID_LAYER_BASE + 16 * l

        def add(slot: int, name: str, shape, sigma=WEIGHT_SIGMA, mean=0.0):
            specs.append(TensorSpec(f"layers.{l}.{name}", tuple(shape), base + slot, sigma, mean))

        add(0, "attn_norm", (H,), gain_sigma, 1.0)
        add(1, "wq", (cfg.q_dim, H))
        add(2, "wk", (cfg.kv_dim, H))
        add(3, "wv", (cfg.kv_dim, H))
        add(4, "wo", (H, cfg.q_dim))
        add(5, "ffn_norm", (H,), gain_sigma, 1.0)
        if cfg.is_moe:
            E, Fe = cfg.n_experts, cfg.expert_ffn
            add(6, "w_router", (E, H), 1.0 / math.sqrt(H))
            add(7, "w_gate", (E, Fe, H))
            add(8, "w_up", (E, Fe, H))
            add(9, "w_down", (E, H, Fe))
        else:
            add(7, "w_gate", (cfg.ffn, H))
            add(8, "w_up", (cfg.ffn, H))
            add(9, "w_down", (H, cfg.ffn))
    specs.append(TensorSpec("final_norm", (H,), TID_FINAL_NORM, gain_sigma, 1.0))
    specs.append(TensorSpec("lm_head", (V, H), TID_LM_HEAD, WEIGHT_SIGMA, 0.0))
    return specs


def weight_bytes(cfg: ModelConfig) -> int:
    return sum(2 * s.numel for s in tensor_specs(cfg))


# ----------------------------------------------------------------------------- build / load

def build(verbose: bool = False) -> None:
    """Compile the host and device fill libraries in place."""
    host_cmd = ["gcc", "-O3", "-march=x86-64-v3", "-fopenmp", "-fPIC", "-shared",
                os.path.join(_HERE, "synthetic.c"), "-o", HOST_LIB]
    dev_cmd = ["nvcc", "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "-Xcompiler", "-fPIC",
               "-shared", os.path.join(_HERE, "synthetic_fill.cu"), "-o", DEV_LIB]
    for cmd in (host_cmd, dev_cmd):
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)


_host = None
_dev = None


def _src_newer(lib: str, srcs) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(os.path.join(_HERE, s)) > t for s in srcs)


def host_lib() -> ctypes.CDLL:
    global _host
    if _host is None:
        if _src_newer(HOST_LIB, ("synthetic.c", "gen.h")):
            subprocess.run(["gcc", "-O3", "-march=x86-64-v3", "-fopenmp", "-fPIC", "-shared",
                            os.path.join(_HERE, "synthetic.c"), "-o", HOST_LIB], check=True)
        lib = ctypes.CDLL(HOST_LIB)
        u64, f32, vp = ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p
        lib.syn_fill_bf16.argtypes = [vp, u64, u64, u64, u64, f32, f32]
        lib.syn_fill_int32.argtypes = [vp, u64, u64, u64, u64, ctypes.c_int64, u64]
        lib.syn_fill_words.argtypes = [vp, u64, u64, u64, u64]
        lib.syn_fill_kv_contig.argtypes = [vp, u64, u64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, f32]
        for f in (lib.syn_fill_bf16, lib.syn_fill_int32, lib.syn_fill_words, lib.syn_fill_kv_contig):
            f.restype = None
        _host = lib
    return _host


def dev_lib() -> ctypes.CDLL:
    global _dev
    if _dev is None:
        if not os.path.exists(DEV_LIB):
            raise RuntimeError(f"{DEV_LIB} is missing: run synthetic.build()")
        lib = ctypes.CDLL(DEV_LIB)
        u64, f32, vp, i32 = ctypes.c_uint64, ctypes.c_float, ctypes.c_void_p, ctypes.c_int
        lib.syn_dev_fill_bf16.argtypes = [vp, u64, u64, u64, u64, f32, f32, vp]
        lib.syn_dev_fill_int32.argtypes = [vp, u64, u64, u64, u64, ctypes.c_int64, u64, vp]
        lib.syn_dev_fill_kv_paged.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, u64, u64, f32, vp]
        for f in (lib.syn_dev_fill_bf16, lib.syn_dev_fill_int32, lib.syn_dev_fill_kv_paged):
            f.restype = ctypes.c_int
        _dev = lib
    return _dev


# ----------------------------------------------------------------------------- host fills

def host_bf16(n: int, seed: int, tensor_id: int, sigma: float, mean: float = 0.0,
              offset: int = 0) -> np.ndarray:
    """uint16 array holding bf16 bits of elements [offset, offset+n)."""
    out = np.empty(n, dtype=np.uint16)
    host_lib().syn_fill_bf16(out.ctypes.data, n, seed, tensor_id, offset, sigma, mean)
    return out


def host_tensor(spec: TensorSpec, seed: int) -> np.ndarray:
    return host_bf16(spec.numel, seed, spec.tensor_id, spec.sigma, spec.mean).reshape(spec.shape)


def host_weights(cfg: ModelConfig, seed: int, gain_sigma: float = 0.0) -> Dict[str, np.ndarray]:
    return {s.name: host_tensor(s, seed) for s in tensor_specs(cfg, gain_sigma)}


def host_tokens(n: int, seed: int, vocab: int, seq: int = 0, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    host_lib().syn_fill_int32(out.ctypes.data, n, seed, TID_TOKENS + seq, offset, 0, vocab)
    return out


def host_uniform_ints(n: int, seed: int, tensor_id: int, lo: int, hi_inclusive: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    host_lib().syn_fill_int32(out.ctypes.data, n, seed, tensor_id, 0, lo, hi_inclusive - lo + 1)
    return out


def host_words(n: int, seed: int, tensor_id: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    host_lib().syn_fill_words(out.ctypes.data, n, seed, tensor_id, 0)
    return out


def host_kv(cfg: ModelConfig, seed: int, layer: int, which: str, seq: int, pos0: int,
            pos1: int, sigma: float = 1.0) -> np.ndarray:
    """Synthetic cache contents [pos1-pos0][n_kv][head_dim] (bf16 bits)."""
    tid = (TID_K_BASE if which == "k" else TID_V_BASE) + layer
    out = np.empty((max(pos1 - pos0, 0), cfg.n_kv_heads, cfg.head_dim), dtype=np.uint16)
    if pos1 > pos0:
        host_lib().syn_fill_kv_contig(out.ctypes.data, seed, tid, seq, pos0, pos1,
                                      cfg.n_kv_heads, cfg.head_dim, sigma)
    return out


def page_permutation(n_pages: int, seed: int) -> np.ndarray:
    """A seeded random permutation of range(n_pages) (Fisher-Yates on generator words)."""
    w = host_words(n_pages, seed, TID_PAGES)
    perm = np.arange(n_pages, dtype=np.int64)
    for i in range(n_pages - 1, 0, -1):
        j = int(w[i] % np.uint64(i + 1))
        perm[i], perm[j] = perm[j], perm[i]
    return perm.astype(np.int32)


def ragged_lengths(batch: int, seed: int, lo: int = 512, hi: int = 8192) -> np.ndarray:
    """Sequence lengths drawn uniformly from [lo, hi]."""
    return host_uniform_ints(batch, seed, TID_LENS, lo, hi)


# ----------------------------------------------------------------------------- bf16 helpers

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32 (a format view, no rounding)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------- device fills

def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise RuntimeError(f"{what} failed with CUDA error {rc}")


def dev_fill_tensor(t, spec: TensorSpec, seed: int, stream_ptr: int = 0) -> None:
    """Fill torch CUDA tensor ``t`` (dtype bfloat16, ``spec.numel`` elements)."""
    assert t.is_cuda and t.numel() == spec.numel
    _check(dev_lib().syn_dev_fill_bf16(t.data_ptr(), spec.numel, seed, spec.tensor_id, 0,
                                       spec.sigma, spec.mean, stream_ptr), spec.name)


def dev_fill_kv_paged(pool_layer, page_row_dev, seq: int, pos0: int, pos1: int,
                      cfg: ModelConfig, page_size: int, seed: int, tensor_id: int,
                      sigma: float = 1.0, stream_ptr: int = 0) -> None:
    _check(dev_lib().syn_dev_fill_kv_paged(pool_layer.data_ptr(), page_row_dev.data_ptr(), seq,
                                           pos0, pos1, cfg.n_kv_heads, page_size, cfg.head_dim,
                                           seed, tensor_id, sigma, stream_ptr), "kv fill")
