"""Task graph of a Qwen3-style decoder built on the PersistentKernel API.

The pages name Qwen3-8B as the demo model ("Mirage Persistent Kernel: Fusing
Multi-GPU LLM Inference into One Kernel Launch", "Getting Started") and the
fused rmsnorm_linear layer as the building block ("The API").  One decoding
iteration is: embedding, then per layer [RMSNorm+QKV, QK-norm+RoPE+attention,
o_proj+residual, RMSNorm+gate/up+SiLU*up, down_proj+residual], then final
RMSNorm + LM head + greedy argmax, which advances `step` and writes `tokens`.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Optional, Tuple

import torch

from . import _lib
from .kernel import FP32_TAGGED, PersistentKernel


FUSED_ATTENTION_MAX_SEQ = 4096


def reduction_split(K: int, max_k: int = _lib.MAX_GEMV_K) -> int:
    """Segments a residual projection of reduction length K is split into (the
    rule of MPK_OP_LINEAR_RESIDUAL): the fewest equal segments of at most max_k
    whose length is a multiple of 256."""
    ks = -(-K // max_k)
    while ks <= K // 256 and (K % ks or (K // ks) % 256):
        ks += 1
    return ks


# Tensor-core projections over several requests (the rule of the batched path
# in mpk.h): row blocks of BATCH_BM rows, K blocks of BATCH_BK elements, at most
# BATCH_MAX_KBLOCKS K blocks per reduction segment; grid_dim = (tasks per
# segment, segments).
BATCH_BM, BATCH_BK, BATCH_MAX_KBLOCKS = 128, 64, 24
# Task-size model used to choose the grid: a worker streams weights at about
# its share of HBM bandwidth and pays a fixed cost per task, per extra pass
# over the input rows, and (split reductions) per partial sum that the
# finishing task gathers and adds (measured on the 8B shape with 8 requests:
# the o and down projections at 4 segments beat 9, 5.46 vs 5.89 ms/step).
_WORKER_BYTES_PER_S = 43e9
_TASK_OVERHEAD_S = 3e-6
_PASS_OVERHEAD_S = 4e-6
_SPLIT_PARTIAL_S = 1.5e-6
BATCH_SLOTS = 16  # accumulator slots: row blocks a task may hold across passes
# Graphs of 9..16 requests run every contraction 16 requests wide: the input
# rows of a K block take twice the shared memory and an accumulator twice the
# tensor-memory columns, so a pass holds half the K blocks and half the slots.
MAX_BATCH = 16
BATCH_WIDE_MAX_KBLOCKS, BATCH_WIDE_SLOTS = 12, 8


def batch_limits(requests: int) -> Tuple[int, int]:
    """(K blocks per pass, accumulator slots) of a contraction over `requests`."""
    return (BATCH_WIDE_MAX_KBLOCKS, BATCH_WIDE_SLOTS) if requests > 8 else (BATCH_MAX_KBLOCKS, BATCH_SLOTS)


def batched_grid(rows: int, K: int, workers: int, pair: bool = False, requests: int = 8) -> Tuple[int, int]:
    """grid_dim (tasks per reduction segment, segments) of a projection over
    several requests: among segment counts s and, per number of rounds k of
    the workers, the largest run split gx <= row blocks with gx * s <= k *
    workers, the one with the least rounds x (largest task's weight bytes /
    bandwidth + task, pass and per-partial split costs); fewer segments on ties.  A task
    longer than the input rows (passes) holds at most the accumulator slots'
    row blocks (batch_limits)."""
    max_kblocks, slots = batch_limits(requests)
    # a partial sum holds one value per request of the batch width (8 or 16):
    # at width 16 it costs twice as much (measured on the 8B shape with 16
    # requests: o and down projections in 3 and 4 segments, 8.18 ms/step,
    # against 4 and 9 at the width-8 cost, 8.62)
    partial_s = _SPLIT_PARTIAL_S * (2 if requests > 8 else 1)
    nb = -(-rows // BATCH_BM)
    nkb = K // BATCH_BK
    block_bytes = BATCH_BM * K * 2 * (2 if pair else 1)
    best = None
    for s in range(1, min(nkb, 16) + 1):
        npass = -(-(-(-nkb // s)) // max_kblocks)
        for k in range(1, 5):
            gx = max(1, min(nb, (k * workers) // s))
            most = -(-nb // gx)
            if npass > 1 and most > slots:
                continue
            rounds = -(-(gx * s) // workers)
            t = rounds * (most * block_bytes / s / _WORKER_BYTES_PER_S + _TASK_OVERHEAD_S +
                          (npass - 1) * _PASS_OVERHEAD_S) + (s * partial_s if s > 1 else 0.0)
            if best is None or t < best[0] * (1 - 1e-2):
                best = (t, gx, s)
    return best[1], best[2]


def lm_head_grid(rows: int, K: int, workers: int, requests: int = 8) -> Tuple[int, int]:
    """grid_dim of the LM head over several requests: no split of the
    reduction (the argmax needs whole logits, and a split's last arrival runs
    the epilogue late) and tasks for about five sixths of the workers, so the
    workers that finish the last layer late claim none (measured on the 8B
    shape with 8 requests: (120, 1) at 5.43 ms/step against 5.49 for the
    batched_grid rule's (48, 3)).  When a task would hold more row blocks
    than the accumulator slots, the fewest tasks that fit them (up to two per
    worker), else batched_grid."""
    max_kblocks, slots = batch_limits(requests)
    nb = -(-rows // BATCH_BM)
    gx = max(1, min(nb, (workers * 5) // 6))
    if -(-(K // BATCH_BK) // max_kblocks) > 1 and -(-nb // gx) > slots:
        # a task whose reduction runs in passes holds at most `slots` row
        # blocks: the fewest whole-reduction tasks that fit (measured on the 8B
        # shape with 16 requests: 160 such tasks at 8.63 ms/step against 8.76
        # for batched_grid's six-way split)
        gx = -(-nb // slots)
        if gx <= 2 * workers:
            return gx, 1
        return batched_grid(rows, K, workers, requests=requests)
    return gx, 1


def batched_layer_plan(shape, requests: int, plan_workers: int, attn_chunks: int, block_dim: int = 0,
                       tied: Optional[bool] = None) -> List[dict]:
    """The fused-layer list for several requests: projections on the tensor
    cores (grids from batched_grid for plan_workers workers), attention as its
    own split-K operation."""
    s = shape
    W = plan_workers
    tied = s.tied if tied is None else tied
    plan: List[dict] = [dict(method="embed_layer", embedding="embed_tokens", output="x", grid_dim=requests,
                             block_dim=block_dim, capture_slot=0)]
    for l in range(s.layers):
        p = f"layers.{l}."
        plan.append(dict(method="rmsnorm_linear_layer", input="x", weight_norm=p + "input_layernorm",
                         weight_linear=[p + "q_proj", p + "k_proj", p + "v_proj"], output=["q", "k", "v"],
                         grid_dim=batched_grid(s.q_dim + 2 * s.kv_dim, s.hidden, W, requests=requests), block_dim=block_dim, eps=s.eps))
        plan.append(dict(method="attention_layer", q="q", k="k", v="v", q_norm=p + "q_norm",
                         k_norm=p + "k_norm", k_cache="k_cache", v_cache="v_cache", output="o", layer=l,
                         grid_dim=(s.kv_heads, attn_chunks, requests), block_dim=block_dim, eps=s.eps,
                         rope_theta=s.rope_theta))
        plan.append(dict(method="linear_residual_layer", input="o", weight=p + "o_proj", residual="x",
                         grid_dim=batched_grid(s.hidden, s.q_dim, W, requests=requests), block_dim=block_dim))
        plan.append(dict(method="rmsnorm_linear_silu_mul_layer", input="x",
                         weight_norm=p + "post_attention_layernorm", weight_gate=p + "gate_proj",
                         weight_up=p + "up_proj", output="a",
                         grid_dim=batched_grid(s.intermediate, s.hidden, W, pair=True, requests=requests), block_dim=block_dim,
                         eps=s.eps))
        plan.append(dict(method="linear_residual_layer", input="a", weight=p + "down_proj", residual="x",
                         grid_dim=batched_grid(s.hidden, s.intermediate, W, requests=requests), block_dim=block_dim,
                         capture_slot=l + 1))
    plan.append(dict(method="rmsnorm_lmhead_argmax_layer", input="x", weight_norm="norm",
                     weight_lm="embed_tokens" if tied else "lm_head", pred="pred",
                     grid_dim=lm_head_grid(s.vocab, s.hidden, W, requests=requests), block_dim=block_dim, eps=s.eps))
    return plan


def layer_plan(shape, requests: int, num_workers: int, attn_chunks: int, gemv_tasks: Optional[int] = None,
               block_dim: int = 0, tied: Optional[bool] = None, fused_attention: bool = False,
               tasks_per_worker: int = 2) -> List[dict]:
    """The fused-layer list (pure host logic, no GPU): one dict per operation with
    the method name and its keyword arguments.  With ``fused_attention`` the q/k/v
    projections and the attention are one operation (tasks grouped per kv head,
    the last task of a group runs its attention); otherwise attention is its own
    split-K operation with ``attn_chunks`` chunks.  Several requests take
    batched_layer_plan."""
    if requests >= 2:
        return batched_layer_plan(shape, requests, gemv_tasks or num_workers, attn_chunks, block_dim, tied)
    s = shape
    gt = gemv_tasks or num_workers                       # fused projections+attention: one task per worker
    dt = gemv_tasks or num_workers * tasks_per_worker    # claimed GEMV ops: more, smaller tasks
    tied = s.tied if tied is None else tied
    plan: List[dict] = [dict(method="embed_layer", embedding="embed_tokens", output="x", grid_dim=requests,
                             block_dim=block_dim, capture_slot=0)]
    rows_per_group = (s.q_heads // s.kv_heads + 2) * s.head_dim
    for l in range(s.layers):
        p = f"layers.{l}."
        if fused_attention:
            tpg = max(1, min(rows_per_group, gt // (s.kv_heads * requests)))
            plan.append(dict(method="rmsnorm_qkv_attention_layer", input="x", weight_norm=p + "input_layernorm",
                             wq=p + "q_proj", wk=p + "k_proj", wv=p + "v_proj", q_norm=p + "q_norm",
                             k_norm=p + "k_norm", k_cache="k_cache", v_cache="v_cache", q="q", k="k", v="v",
                             output="o", layer=l, grid_dim=(tpg, s.kv_heads, requests), block_dim=block_dim,
                             eps=s.eps, rope_theta=s.rope_theta))
        else:
            plan.append(dict(method="rmsnorm_linear_layer", input="x", weight_norm=p + "input_layernorm",
                             weight_linear=[p + "q_proj", p + "k_proj", p + "v_proj"], output=["q", "k", "v"],
                             grid_dim=min(dt, s.q_dim + 2 * s.kv_dim), block_dim=block_dim, eps=s.eps))
            plan.append(dict(method="attention_layer", q="q", k="k", v="v", q_norm=p + "q_norm",
                             k_norm=p + "k_norm", k_cache="k_cache", v_cache="v_cache", output="o", layer=l,
                             grid_dim=(s.kv_heads, attn_chunks, requests), block_dim=block_dim, eps=s.eps,
                             rope_theta=s.rope_theta))
        plan.append(dict(method="linear_residual_layer", input="o", weight=p + "o_proj", residual="x",
                         grid_dim=min(dt, s.hidden), block_dim=block_dim))
        plan.append(dict(method="rmsnorm_linear_silu_mul_layer", input="x",
                         weight_norm=p + "post_attention_layernorm", weight_gate=p + "gate_proj",
                         weight_up=p + "up_proj", output="a", grid_dim=min(dt, s.intermediate), block_dim=block_dim,
                         eps=s.eps))
        plan.append(dict(method="linear_residual_layer", input="a", weight=p + "down_proj", residual="x",
                         grid_dim=min(dt, s.hidden * reduction_split(s.intermediate)), block_dim=block_dim,
                         capture_slot=l + 1))
    plan.append(dict(method="rmsnorm_lmhead_argmax_layer", input="x", weight_norm="norm",
                     weight_lm="embed_tokens" if tied else "lm_head", pred="pred", grid_dim=min(dt, s.vocab),
                     block_dim=block_dim, eps=s.eps))
    return plan


def default_attn_chunks(shape, requests: int, num_workers: int, max_seq: int) -> int:
    """Split-K chunks per (request, kv head): enough tasks to cover the workers for
    long contexts, about 64 positions per chunk for short ones."""
    by_workers = max(1, num_workers // (shape.kv_heads * requests))
    by_length = max(1, -(-max_seq // 64))
    return max(1, min(by_workers, by_length))


@dataclass
class Decoder:
    """A compiled decoder: the kernel plus the tensors a caller reads or writes."""
    kernel: PersistentKernel
    shape: object
    requests: int
    max_seq: int
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    pred: torch.Tensor
    buffers: Dict[str, torch.Tensor]
    kv_pages: Optional[torch.Tensor] = None  # paged caches: the page table

    def run(self, step, tokens, step_end=None, stream=None):
        self.kernel(step, tokens, step_end, stream)

    def run_op_by_op(self, step, tokens, step_end=None, stream=None):
        self.kernel.run_op_by_op(step, tokens, step_end, stream)


def build_decoder(shape, weights: Dict[str, torch.Tensor], requests: int, max_seq: int,
                  num_workers: Optional[int] = None, num_local_schedulers: int = 16,
                  attn_chunks: Optional[int] = None, gemv_tasks: Optional[int] = None, block_dim: int = 0,
                  k_cache: Optional[torch.Tensor] = None, v_cache: Optional[torch.Tensor] = None,
                  profiling: bool = False, sched_lookahead: int = 0, timeout_s: float = 0.0,
                  prefetch_kb: int = 0, fused_attention: Optional[bool] = None,
                  debug_stall_op: int = 0, dynamic_tasks: bool = False, tasks_per_worker: int = 2,
                  poll_inputs: bool = False, prefill_tokens: int = 0, kv_page_size: int = 0,
                  kv_pages: Optional[torch.Tensor] = None, num_pages: Optional[int] = None) -> Decoder:
    """Attach the weights (bf16 CUDA tensors keyed as in synth.qwen3), allocate the
    activations and compile the task graph.  max_seq = KV-cache positions = the
    tokens' row length (seq_length).  fused_attention: None picks the fused
    projection+attention operation for one request with up to
    FUSED_ATTENTION_MAX_SEQ positions, split-K attention otherwise.

    prefill_tokens = T in 2..8 builds a prefill graph: every iteration ingests
    T consecutive prompt positions of one request as the T columns of the
    tensor-core projections (mpk_options.prefill_tokens), the requests one
    after another.  Pass the decode graph's caches as k_cache / v_cache (and
    the same `requests`) to continue decoding from the prefilled state.

    kv_page_size = P > 0 (a multiple of 128) makes the KV caches paged
    (mpk_options.kv_page_size): k_cache / v_cache are [L, num_pages, Hkv, P, d]
    and kv_pages (int32 [requests, ceil(max_seq / P)], default: request r's
    pages r * max_pages ..) maps each request's logical pages to cache pages;
    the attention is then the split-K operation."""
    from . import _lib

    s = shape
    cols = requests
    if prefill_tokens > 1:
        cols = prefill_tokens
    if num_workers is None:
        num_workers = _lib.load().mpk_device_sm_count() - num_local_schedulers // 4
    mk = PersistentKernel(num_workers, num_local_schedulers, 0)
    for name, t in weights.items():
        mk.attach_input(t, name)
    dev = next(iter(weights.values())).device
    kv_shape = (s.layers, requests, s.kv_heads, max_seq, s.head_dim)
    if kv_page_size > 0:
        if fused_attention:
            raise ValueError("paged KV caches take the split-K attention operation")
        fused_attention = False
        max_pages = -(-max_seq // kv_page_size)
        if kv_pages is None:
            kv_pages = torch.arange(requests * max_pages, dtype=torch.int32, device=dev).view(requests, max_pages)
        if num_pages is None:
            num_pages = requests * max_pages
        kv_shape = (s.layers, num_pages, s.kv_heads, kv_page_size, s.head_dim)
        mk.attach_input(kv_pages, "kv_pages")
    if k_cache is None:
        k_cache = torch.zeros(kv_shape, dtype=torch.bfloat16, device=dev)
    if v_cache is None:
        v_cache = torch.zeros(kv_shape, dtype=torch.bfloat16, device=dev)
    mk.attach_input(k_cache, "k_cache")
    mk.attach_input(v_cache, "v_cache")
    pred = torch.full((requests, max_seq), -1, dtype=torch.int64, device=dev)
    mk.attach_input(pred, "pred")
    bufs = {
        "x": mk.new_tensor((cols, s.hidden), FP32_TAGGED, "x"),
        "q": mk.new_tensor((cols, s.q_dim), FP32_TAGGED, "q"),
        "k": mk.new_tensor((cols, s.kv_dim), FP32_TAGGED, "k"),
        "v": mk.new_tensor((cols, s.kv_dim), FP32_TAGGED, "v"),
        "o": mk.new_tensor((cols, s.q_dim), FP32_TAGGED, "o"),
        "a": mk.new_tensor((cols, s.intermediate), FP32_TAGGED, "a"),
    }
    if attn_chunks is None:
        attn_chunks = default_attn_chunks(s, cols, num_workers, max_seq)
    if fused_attention is None:
        fused_attention = cols == 1 and max_seq <= FUSED_ATTENTION_MAX_SEQ
    for op in layer_plan(s, cols, num_workers, attn_chunks, gemv_tasks, block_dim,
                         fused_attention=fused_attention, tasks_per_worker=tasks_per_worker if dynamic_tasks else 1):
        op = dict(op)
        getattr(mk, op.pop("method"))(**op)
    mk.compile(profiling=profiling, sched_lookahead=sched_lookahead, timeout_s=timeout_s, prefetch_kb=prefetch_kb,
               debug_stall_op=debug_stall_op, dynamic_tasks=dynamic_tasks, poll_inputs=poll_inputs,
               prefill_tokens=prefill_tokens if prefill_tokens > 1 else 0, kv_page_size=max(0, kv_page_size))
    return Decoder(mk, s, requests, max_seq, k_cache, v_cache, pred, bufs, kv_pages)
