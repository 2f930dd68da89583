"""Synthetic workloads and seeded input generators.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests.  It holds shapes, head policies and random numbers only: none
of the method's arithmetic (visible sets, stored sets, page layout, softmax,
the retrieval heads' block choice) lives here.  Head policies are plain
tuples ``(kind, sink, window)`` with ``kind`` one of the strings
``"global"``, ``"local"`` or ``"dense"``, or ``("retrieval", sink, window,
top_p)``; each side maps the strings to its own codes.  A retrieval head's
importance per page-size block is a seeded synthetic draw (``block_mass``)
that both sides receive as an input.

The shapes follow the synthetic layers of the SegPagedAttention write-ups
(head-aware paged KV cache; "RedKnot SegPagedAttention runtime design", §2 head
kinds and §5 H200 operator results at 8K and 32K context; "RedKnot head
classification", the Llama-3.3-70B and DeepSeek-V4-Flash frozen policies).
The pages measure on RAG datasets (HotpotQA, LongBench) with trained weights;
those are not available here, so i.i.d. N(0, 1) Q/K/V of the same shapes stand
in for them.

Random numbers: every (tensor, sequence, head, block of 1024 rows) draws its
own ``torch.Generator`` seeded from a 64-bit mix of those indices, so that any
slice can be regenerated without materialising the whole tensor.  Values
depend on the generator's device: a run uses one device throughout, and the
oracle always receives host copies of exactly the tensors the GPU path used.
"""
from __future__ import annotations

import math
import random
from dataclasses import dataclass
from typing import Sequence

import torch

BLOCK_ROWS = 1024
_TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "mass": 4}
_MASK64 = (1 << 64) - 1


def _mix64(x: int) -> int:
    """splitmix64 finaliser (Steele, Lea, Flood 2014): a bijective 64-bit mixer."""
    x = (x + 0x9E3779B97F4A7C15) & _MASK64
    x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & _MASK64
    return x ^ (x >> 31)


def block_seed(cfg_seed: int, tensor: str, b: int, head: int, block: int) -> int:
    """Seed of one 1024-row block of one (tensor, sequence, head) stream."""
    h = _mix64(cfg_seed)
    for part in (_TENSOR_IDS[tensor], b, head, block):
        h = _mix64(h ^ part)
    return h & ((1 << 63) - 1)


def normal_rows(cfg_seed: int, tensor: str, b: int, head: int, r0: int, r1: int,
                d: int, device: str | torch.device = "cpu") -> torch.Tensor:
    """Rows [r0, r1) of the N(0, 1) fp32 stream of (tensor, b, head), shape [r1-r0, d]."""
    if r1 <= r0:
        return torch.empty(0, d, dtype=torch.float32, device=device)
    out = []
    for blk in range(r0 // BLOCK_ROWS, (r1 - 1) // BLOCK_ROWS + 1):
        g = torch.Generator(device=device)
        g.manual_seed(block_seed(cfg_seed, tensor, b, head, blk))
        rows = torch.randn(BLOCK_ROWS, d, generator=g, device=device, dtype=torch.float32)
        lo = max(r0, blk * BLOCK_ROWS) - blk * BLOCK_ROWS
        hi = min(r1, (blk + 1) * BLOCK_ROWS) - blk * BLOCK_ROWS
        out.append(rows[lo:hi])
    return torch.cat(out, 0)


def block_mass(cfg_seed: int, b: int, kv: int, n_blocks: int) -> list[float]:
    """Synthetic importance of the first n_blocks page-size blocks of (sequence b, kv-head kv).

    Heavy-tailed and seeded: exp(2 z) with z ~ N(0, 1) i.i.d. per block (a
    lognormal stand-in for a head's attention mass per page, which is
    concentrated on a few pages), rounded to float32.  The stream of a head
    does not depend on n_blocks: a longer context extends it.
    """
    if n_blocks <= 0:
        return []
    z = normal_rows(cfg_seed, "mass", b, kv, 0, -(-n_blocks // 64), 64).flatten()[:n_blocks]
    return [float(x) for x in torch.exp(2.0 * z.double()).float()]


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


@dataclass(frozen=True)
class Workload:
    """One synthetic attention layer.

    ``ctx_lens[b]`` is the length of sequence b's token stream; ``policy`` has
    ``batch * num_kv_heads`` entries in (b, kv) order.  A decode problem puts
    one query at the last position of each sequence; a prefill problem puts
    ``chunk`` queries at the end of each sequence (``chunk == ctx`` is a full
    prefill).
    """

    name: str
    seed: int
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str
    page_size: int
    ctx_lens: tuple[int, ...]
    policy: tuple[tuple, ...]
    prefill_chunk: int | None = None
    prefill_ctx_lens: tuple[int, ...] | None = None
    note: str = ""

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def has_retrieval(self) -> bool:
        return any(p[0] == "retrieval" for p in self.policy)

    def decode_problem(self) -> "Problem":
        return Problem(self, tuple(self.ctx_lens), tuple(L - 1 for L in self.ctx_lens))

    def prefill_problem(self) -> "Problem":
        assert self.prefill_chunk is not None, f"{self.name} has no prefill chunk"
        lens = self.prefill_ctx_lens or self.ctx_lens
        return Problem(self, tuple(lens), tuple(L - min(self.prefill_chunk, L) for L in lens))


@dataclass(frozen=True)
class Problem:
    """A workload with concrete per-sequence context lengths and first query positions."""

    wl: Workload
    ctx_lens: tuple[int, ...]
    q_starts: tuple[int, ...]

    @property
    def q_counts(self) -> tuple[int, ...]:
        return tuple(L - q0 for L, q0 in zip(self.ctx_lens, self.q_starts))

    @property
    def q_offsets(self) -> list[int]:
        off = [0]
        for c in self.q_counts:
            off.append(off[-1] + c)
        return off

    @property
    def total_queries(self) -> int:
        return sum(self.q_counts)

    def block_masses(self) -> list[list[float] | None]:
        """Per (sequence, kv-head): the importance of each page-size block for a retrieval head, else None."""
        wl = self.wl
        out = []
        for b, L in enumerate(self.ctx_lens):
            for kv in range(wl.num_kv_heads):
                pol = wl.policy[b * wl.num_kv_heads + kv]
                out.append(block_mass(wl.seed, b, kv, -(-L // wl.page_size)) if pol[0] == "retrieval" else None)
        return out


# --------------------------------------------------------------------------
# Tensors of a problem
# --------------------------------------------------------------------------

def dense_kv(prob: Problem, device="cpu", gen_device=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Dense K and V, padded layout [B, Hkv, Lmax, d] in the workload dtype.

    Rows beyond ctx_lens[b] are zero (they are never read).  The stream of
    (b, kv) is shared between a workload's decode and prefill problems.
    """
    wl = prob.wl
    gen_device = gen_device or device
    Lmax = max(prob.ctx_lens)
    dt = torch_dtype(wl.dtype)
    out = []
    for name in ("k", "v"):
        t = torch.zeros(wl.batch, wl.num_kv_heads, Lmax, wl.head_dim, dtype=dt, device=device)
        for b, L in enumerate(prob.ctx_lens):
            for h in range(wl.num_kv_heads):
                t[b, h, :L] = normal_rows(wl.seed, name, b, h, 0, L, wl.head_dim, gen_device).to(dt).to(device)
        out.append(t)
    return out[0], out[1]


def queries(prob: Problem, device="cpu", gen_device=None) -> torch.Tensor:
    """Queries, varlen layout [sum_b C_b, Hq, d]; row i of sequence b is position q_starts[b] + i."""
    wl = prob.wl
    gen_device = gen_device or device
    dt = torch_dtype(wl.dtype)
    q = torch.empty(prob.total_queries, wl.num_q_heads, wl.head_dim, dtype=dt, device=device)
    off = prob.q_offsets
    for b, (L, q0) in enumerate(zip(prob.ctx_lens, prob.q_starts)):
        for h in range(wl.num_q_heads):
            q[off[b]:off[b + 1], h] = normal_rows(wl.seed, "q", b, h, q0, L, wl.head_dim, gen_device).to(dt).to(device)
    return q


# --------------------------------------------------------------------------
# The five synthetic layers
# --------------------------------------------------------------------------

def _local(s: int, w: int) -> tuple[str, int, int]:
    return ("local", s, w)


GLOBAL = ("global", 0, 0)


def tiny() -> Workload:
    """1 layer, B1, 4 q-heads / 2 kv-heads, d64, fp32, page 16; kv0 global, kv1 local s4 w32.

    Full causal prefill of 256 queries (context 256) plus one decode query at
    position 256 (context 257, the same token stream extended by one token).
    """
    return Workload("tiny", 0, 1, 4, 2, 64, "f32", 16, (257,),
                    (GLOBAL, _local(4, 32)), prefill_chunk=256, prefill_ctx_lens=(256,))


def mistral() -> Workload:
    """Mistral-7B-shaped layer: B4, 32/8 heads, d128, bf16, 8K context, page 64; 2 of 8 kv-heads global."""
    rnd = random.Random(1)
    glob = set(rnd.sample(range(8), 2))
    layer = tuple(GLOBAL if h in glob else _local(4, 512) for h in range(8))
    return Workload("mistral", 1, 4, 32, 8, 128, "bf16", 64, (8192,) * 4, layer * 4,
                    prefill_chunk=2048)


def llama_layer_globals(n_layers: int = 80) -> list[int]:
    """The global kv-head of each of 80 layers (one of 8 per layer, seeded)."""
    rnd = random.Random(2)
    return [rnd.randrange(8) for _ in range(n_layers)]


def llama(layer: int = 0, batch: int = 8) -> Workload:
    """Llama-70B-shaped layer: B8, 64/8 heads, d128, bf16, 32K context, page 64; 1 of 8 kv-heads global.

    ``batch=1`` keeps sequence 0 only: the same per-sequence work at one eighth
    of the memory (used for detailed profiles).
    """
    g = llama_layer_globals()[layer]
    row = tuple(GLOBAL if h == g else _local(4, 8192) for h in range(8))
    name = f"llama_l{layer}" if batch == 8 else f"llama_l{layer}_b{batch}"
    return Workload(name, 2 + 1000 * layer, batch, 64, 8, 128, "bf16", 64, (32768,) * batch,
                    row * batch, prefill_chunk=4096)


def ragged() -> Workload:
    """Ragged decode: 32 sequences, L log-uniform in [1024, 65536], 32/8 heads, d128, bf16, page 64.

    Per sequence, exactly 2 of 8 kv-heads are global (drawn without replacement).
    """
    rnd = random.Random(3)
    lens, pol = [], []
    for _ in range(32):
        lens.append(int(math.floor(math.exp(rnd.uniform(math.log(1024), math.log(65536))))))
        glob = set(rnd.sample(range(8), 2))
        pol.extend(GLOBAL if h in glob else _local(4, 512) for h in range(8))
    return Workload("ragged", 3, 32, 32, 8, 128, "bf16", 64, tuple(lens), tuple(pol))


def mha() -> Workload:
    """Long-context MHA-style layer: B4, 64/64 heads, d128, bf16, 128K context, page 64; heads 0,8,...,56 global."""
    row = tuple(GLOBAL if h % 8 == 0 else _local(4, 128) for h in range(64))
    return Workload("mha", 4, 4, 64, 64, 128, "bf16", 64, (131072,) * 4, row * 4,
                    prefill_chunk=4096)


def llama_retrieval(batch: int = 8, top_p: float = 0.5) -> Workload:
    """The Llama-70B-shaped 32K layer with retrieval heads: per sequence the layer's global
    kv-head, two retrieval kv-heads (sink 4, window 512, top_p) and five local ones (sink 4,
    window 8192).  The pages give no retrieval share for this model; two of eight is this
    workload's choice.  Block importance: ``block_mass`` draws."""
    g = llama_layer_globals()[0]
    rest = [h for h in range(8) if h != g]
    retr = set(rest[:2])
    row = tuple(GLOBAL if h == g else ("retrieval", 4, 512, top_p) if h in retr else _local(4, 8192)
                for h in range(8))
    name = "llama_retrieval" if batch == 8 else f"llama_retrieval_b{batch}"
    return Workload(name, 5, batch, 64, 8, 128, "bf16", 64, (32768,) * batch, row * batch, prefill_chunk=4096)


def tiny_retrieval() -> Workload:
    """The tiny layer (fp32, page 16) with kv-head 1 a retrieval head (sink 4, window 32, top_p 0.6)."""
    return Workload("tiny_retrieval", 6, 1, 4, 2, 64, "f32", 16, (257,),
                    (GLOBAL, ("retrieval", 4, 32, 0.6)), prefill_chunk=256, prefill_ctx_lens=(256,))


ALL = {"tiny": tiny, "mistral": mistral, "llama": llama, "ragged": ragged, "mha": mha,
       "llama_b1": lambda: llama(batch=1), "llama_retrieval": llama_retrieval,
       "tiny_retrieval": tiny_retrieval}


def custom(name: str, seed: int, batch: int, hq: int, hkv: int, d: int, dtype: str, page: int,
           ctx_lens: Sequence[int], policy: Sequence[tuple],
           chunk: int | None = None) -> Workload:
    """A hand-made workload for edge-case tests."""
    assert len(policy) == batch * hkv
    return Workload(name, seed, batch, hq, hkv, d, dtype, page, tuple(ctx_lens), tuple(policy),
                    prefill_chunk=chunk)
