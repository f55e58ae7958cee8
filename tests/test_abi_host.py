"""Host-only checks of the C ABI (no GPU needed): the library loads, exports every
symbol the header declares, and validates the worker/scheduler split."""
import ctypes
import json
import os
import re

import pytest

from persistent_megakernel_decode_02_b200 import _lib, layer_plan, default_attn_chunks
from synth import qwen3 as sq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    txt = open(os.path.join(ROOT, "include", "mpk.h")).read()
    return sorted(set(re.findall(r"^MPK_API [^(]*?\b(mpk_\w+)\(", txt, flags=re.M)))


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    names = _header_functions()
    assert len(names) >= 18
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, f"binding lacks {n}"
    txt = open(os.path.join(ROOT, "include", "mpk.h")).read()
    assert lib.mpk_abi_version() == int(re.search(r"#define MPK_ABI_VERSION (\d+)", txt).group(1))
    assert lib.mpk_worker_threads() == 256


def _header_struct_fields(name):
    """Member names, in order, of `typedef struct { ... } name;` in the header."""
    txt = open(os.path.join(ROOT, "include", "mpk.h")).read()
    body = re.search(r"typedef struct \{([^}]*)\}\s*" + name + ";", txt).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    names = []
    for decl in body.split(";"):
        for part in decl.split(","):
            part = re.sub(r"\[\w*\]", "", part).strip()
            if part:
                names.append(re.findall(r"\w+", part)[-1])
    return names


@pytest.mark.parametrize("cname,pyname", [("mpk_options", "Options"), ("mpk_layer", "Layer"), ("mpk_dim3", "Dim3")])
def test_binding_structs_mirror_the_header(cname, pyname):
    """The ctypes structures passed through the C ABI list the header's members
    in the header's order (a missing or reordered member shifts every later one)."""
    fields = [f[0] for f in getattr(_lib, pyname)._fields_]
    assert fields == _header_struct_fields(cname)


GOLDEN = json.load(open(os.path.join(ROOT, "tests", "golden", "sm_split.json")))


@pytest.mark.parametrize("case", GOLDEN["cases"], ids=lambda c: c["id"])
def test_sm_formula_cases(case):
    lib = _lib.load()
    rc = lib.mpk_validate_split(case["sms"], case["workers"], case["local"], case["remote"])
    assert _lib.ERRORS.get(rc, "OK") == case["expect"], lib.mpk_last_error(None)


def test_create_without_device_reports_cuda_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("host without a GPU only")
    lib = _lib.load()
    ctx = ctypes.c_void_p()
    rc = lib.mpk_create(144, 16, 0, ctypes.byref(ctx))
    assert _lib.ERRORS[rc] == "CUDA" and not ctx.value


def test_layer_plan_structure():
    s = sq.QWEN3_8B
    plan = layer_plan(s, requests=1, num_workers=144, attn_chunks=9)
    assert plan[0]["method"] == "embed_layer" and plan[-1]["method"] == "rmsnorm_lmhead_argmax_layer"
    assert len(plan) == 2 + 5 * s.layers
    kinds = [p["method"] for p in plan[1:6]]
    assert kinds == ["rmsnorm_linear_layer", "attention_layer", "linear_residual_layer",
                     "rmsnorm_linear_silu_mul_layer", "linear_residual_layer"]
    assert plan[2]["grid_dim"] == (8, 9, 1)
    # claimed GEMV ops get two tasks per worker
    assert all(p["grid_dim"] == 288 for p in plan[1:-1] if p["method"] != "attention_layer")
    assert all(p["grid_dim"] == 144 for p in layer_plan(s, 1, 144, 9, tasks_per_worker=1)[1:-1]
               if p["method"] != "attention_layer")
    assert plan[-1]["weight_lm"] == "lm_head"
    assert layer_plan(sq.QWEN3_0_6B, 1, 144, 4)[-1]["weight_lm"] == "embed_tokens"
    # the down projection of layer l captures residual slot l+1
    assert [p.get("capture_slot") for p in plan if p.get("weight", "").endswith("down_proj")] == \
        list(range(1, s.layers + 1))


def test_layer_plan_fused_attention():
    s = sq.QWEN3_8B
    plan = layer_plan(s, requests=1, num_workers=144, attn_chunks=9, fused_attention=True)
    assert len(plan) == 2 + 4 * s.layers
    op = plan[1]
    assert op["method"] == "rmsnorm_qkv_attention_layer"
    assert op["grid_dim"] == (18, 8, 1)      # 18 tasks per kv head, 8 kv heads
    assert [p["method"] for p in plan[1:5]] == ["rmsnorm_qkv_attention_layer", "linear_residual_layer",
                                                "rmsnorm_linear_silu_mul_layer", "linear_residual_layer"]


def test_reduction_split_rule():
    from persistent_megakernel_decode_02_b200.qwen3 import reduction_split
    txt = open(os.path.join(ROOT, "include", "mpk.h")).read()
    assert int(re.search(r"#define MPK_MAX_GEMV_K (\d+)", txt).group(1)) == _lib.MAX_GEMV_K
    assert [reduction_split(k) for k in (256, 3072, 4096, 4352, 8192, 12288, 17408)] == [1, 1, 1, 17, 2, 3, 17]
    plan = layer_plan(sq.QWEN3_8B, requests=1, num_workers=144, attn_chunks=9)
    assert plan[5]["grid_dim"] == 288 and plan[5]["weight"].endswith("down_proj")


def test_default_attention_chunks():
    assert default_attn_chunks(sq.QWEN3_8B, 1, 144, 551) == 9
    assert default_attn_chunks(sq.QWEN3_8B, 1, 144, 32897) == 18
    assert default_attn_chunks(sq.TINY, 1, 144, 24) == 1


def _header_define(name):
    import re
    txt = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "mpk.h")).read()
    m = re.search(rf"#define {name} (\d+)", txt)
    return int(m.group(1))


def test_batched_grid_rule():
    """The batched projections' grid (tasks per segment, segments) obeys the
    header's geometry for every model shape and worker count: at most one task
    per row block and segment, at most one segment per K block, and a task
    whose segment needs passes holds at most the accumulator slots."""
    from persistent_megakernel_decode_02_b200.qwen3 import (BATCH_BM, BATCH_MAX_KBLOCKS, BATCH_SLOTS, batched_grid,
                                                            lm_head_grid)
    assert BATCH_BM == _header_define("MPK_BATCH_BM")
    assert BATCH_MAX_KBLOCKS * 64 == _header_define("MPK_BATCH_MAX_PASS_K")
    assert BATCH_SLOTS == _header_define("MPK_BATCH_SLOTS")
    for shape in (sq.TINY, sq.QWEN3_0_6B, sq.QWEN3_8B):
        cases = [(shape.q_dim + 2 * shape.kv_dim, shape.hidden, False), (shape.hidden, shape.q_dim, False),
                 (shape.intermediate, shape.hidden, True), (shape.hidden, shape.intermediate, False),
                 (shape.vocab, shape.hidden, False)]
        for rows, K, pair in cases:
            for W in (1, 7, 100, 144, 300):
                gx, gy = batched_grid(rows, K, W, pair)
                nb, nkb = -(-rows // BATCH_BM), K // 64
                assert 1 <= gx <= nb and 1 <= gy <= nkb
                if -(-nkb // gy) > BATCH_MAX_KBLOCKS:
                    assert -(-nb // gx) <= BATCH_SLOTS
        for W in (1, 7, 100, 144, 300):
            gx, gy = lm_head_grid(shape.vocab, shape.hidden, W)
            nb, nkb = -(-shape.vocab // BATCH_BM), shape.hidden // 64
            assert 1 <= gx <= nb and 1 <= gy <= nkb
            if -(-nkb // gy) > BATCH_MAX_KBLOCKS:
                assert -(-nb // gx) <= BATCH_SLOTS
    # the LM head: whole reductions, tasks for five sixths of the workers
    assert lm_head_grid(151936, 4096, 144) == (120, 1)
    # 9..16 requests: contractions 16 wide, half the K blocks per pass and
    # half the accumulator slots
    from persistent_megakernel_decode_02_b200.qwen3 import (BATCH_WIDE_MAX_KBLOCKS, BATCH_WIDE_SLOTS, MAX_BATCH,
                                                            batch_limits)
    assert MAX_BATCH == _header_define("MPK_MAX_BATCH")
    assert BATCH_WIDE_MAX_KBLOCKS * 64 == _header_define("MPK_BATCH_WIDE_MAX_PASS_K")
    assert BATCH_WIDE_SLOTS == _header_define("MPK_BATCH_WIDE_SLOTS")
    assert batch_limits(8) == (BATCH_MAX_KBLOCKS, BATCH_SLOTS) and batch_limits(9) == (12, 8)
    for shape in (sq.TINY, sq.QWEN3_0_6B, sq.QWEN3_8B):
        for rows, K, pair in [(shape.intermediate, shape.hidden, True), (shape.hidden, shape.intermediate, False),
                              (shape.vocab, shape.hidden, False)]:
            for W in (1, 7, 144):
                for gx, gy in (batched_grid(rows, K, W, pair, requests=16), lm_head_grid(rows, K, W, requests=16)):
                    nb, nkb = -(-rows // BATCH_BM), K // 64
                    assert 1 <= gx <= nb and 1 <= gy <= nkb
                    if -(-nkb // gy) > BATCH_WIDE_MAX_KBLOCKS:
                        assert -(-nb // gx) <= BATCH_WIDE_SLOTS
    # the 8B plan for 144 workers: one round of tasks for the projections, the
    # reductions split three or four ways
    assert batched_grid(6144, 4096, 144) == (48, 3)
    assert batched_grid(12288, 4096, 144, True) == (48, 3)
    assert batched_grid(4096, 4096, 144) == (32, 4)
    assert batched_grid(4096, 12288, 144) == (32, 4)
    # 16 requests: partial sums of 16 values cost twice as much, fewer segments
    assert batched_grid(4096, 4096, 144, requests=16) == (32, 3)
    assert batched_grid(4096, 12288, 144, requests=16) == (32, 4)
    assert lm_head_grid(151936, 4096, 144, requests=16) == (149, 1)


def test_batched_layer_plan():
    """Several requests: split-K attention (no fused projections+attention op)
    and two-dimensional grids for every projection."""
    s = sq.QWEN3_8B
    plan = layer_plan(s, requests=8, num_workers=144, attn_chunks=2)
    methods = [p["method"] for p in plan]
    assert "rmsnorm_qkv_attention_layer" not in methods
    assert methods.count("attention_layer") == s.layers
    assert plan[0]["grid_dim"] == 8
    for p in plan[1:]:
        if p["method"] == "attention_layer":
            assert p["grid_dim"] == (s.kv_heads, 2, 8)
        else:
            assert isinstance(p["grid_dim"], tuple) and len(p["grid_dim"]) == 2


def test_wide_batched_layer_plan():
    """16 requests: the projections' grids follow the 16-wide limits (a task
    whose segment exceeds 12 K blocks holds at most 8 row blocks), the LM head
    runs whole reductions in tasks that fit the slots, the embedding and the
    attention grids carry the 16 requests."""
    from persistent_megakernel_decode_02_b200.qwen3 import BATCH_WIDE_MAX_KBLOCKS, BATCH_WIDE_SLOTS
    s = sq.QWEN3_8B
    plan = layer_plan(s, requests=16, num_workers=144, attn_chunks=1)
    assert plan[0]["grid_dim"] == 16
    rows_k = {"rmsnorm_linear_layer": (s.q_dim + 2 * s.kv_dim, s.hidden),
              "rmsnorm_linear_silu_mul_layer": (s.intermediate, s.hidden),
              "rmsnorm_lmhead_argmax_layer": (s.vocab, s.hidden)}
    for p in plan[1:]:
        m = p["method"]
        if m == "attention_layer":
            assert p["grid_dim"] == (s.kv_heads, 1, 16)
            continue
        gx, gy = p["grid_dim"]
        rows, K = rows_k.get(m) or ((s.hidden, s.q_dim) if p["input"] == "o" else (s.hidden, s.intermediate))
        nb, nkb = -(-rows // 128), K // 64
        assert 1 <= gx <= nb and 1 <= gy <= nkb
        if -(-nkb // gy) > BATCH_WIDE_MAX_KBLOCKS:
            assert -(-nb // gx) <= BATCH_WIDE_SLOTS
        if m == "rmsnorm_lmhead_argmax_layer":
            assert (gx, gy) == (-(-nb // BATCH_WIDE_SLOTS), 1)
