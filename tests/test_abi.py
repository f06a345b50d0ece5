"""C-ABI checks that need no GPU: the library loads, exports every function
include/pa.h declares, plans on the host, and rejects bad arguments before
queuing any GPU work."""
import ctypes
import os
import re

import numpy as np
import pytest

import paged_kv_attention_token_b200 as pa
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(pa_[a-z_0-9]+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from paged_kv_attention_token_b200 import build
    build.build()
    return pa.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = header_functions()
    assert "pa_reshape_and_cache" in names and "pa_attention_varlen" in names
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_library_is_built_for_sm100a(lib):
    # the build passes -gencode arch=compute_100a,code=sm_100a; check the
    # flags the build module uses rather than reading the binary
    from paged_kv_attention_token_b200 import build
    assert build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert os.path.exists(pa.library_path())


def dims_for(lay):
    return pa.Dims(lay.num_tokens, lay.num_seqs, lay.num_q_heads, lay.num_kv_heads,
                   lay.head_dim, lay.num_blocks, lay.max_blocks_per_seq, 16)


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_plan_invariants(lib, name):
    lay = W.layout(name)
    plan = pa.Plan(lay.cu_seqlens_q, lay.seq_lens, dims_for(lay), device=-1)
    info = plan.info()
    ql = lay.q_lens.astype(np.int64)
    sl = lay.seq_lens.astype(np.int64)
    dec = ql <= 16
    prefill_on_tensor_cores = info["num_prefill_tiles"] > 0
    if not prefill_on_tensor_cores:
        dec = ql > 0
    # one row per (decode query, kv head); its keys are its causal prefix
    rows = int(ql[dec].sum()) * lay.num_kv_heads
    assert info["num_decode_rows"] == rows
    blocks = keys = 0
    for L, n in zip(ql[dec], sl[dec]):
        for j in range(L):
            blocks += -(-(n - L + j + 1) // 16)
            keys += n - L + j + 1
    assert info["decode_kv_blocks"] == blocks * lay.num_kv_heads
    assert info["decode_kv_keys"] == keys * lay.num_kv_heads
    # one wave of warps at most (12 per SM at D=64, 8 at D=128), each with a
    # fair share of at least 4 blocks
    warps_per_sm = 12 if lay.head_dim == 64 else 8
    if blocks == 0:
        assert info["num_decode_units"] == 0 and info["num_partials"] == 0
    else:
        assert 1 <= info["num_decode_units"] <= 148 * warps_per_sm
    assert info["num_decode_units"] <= max(1, -(-info["decode_kv_blocks"] // 4))
    # every split row has at least two partials; rows and partials fit the workspace
    assert info["num_partials"] >= 2 * info["num_combine_rows"]
    assert info["num_partials"] <= info["num_combine_rows"] + info["num_decode_units"] * 2
    G = lay.num_q_heads // lay.num_kv_heads
    # the workspace holds the status word, one ticket per split row and the
    # partials; the plan's own tables live in device memory the plan owns
    assert info["table_bytes"] > 0
    assert info["workspace_bytes"] >= 256 + info["num_partials"] * G * lay.head_dim * 4
    assert info["table_bytes"] >= 4 * info["num_combine_rows"]
    assert plan.workspace_bytes == info["workspace_bytes"]
    # prefill tiles are dealt to at most one persistent CTA per SM; K/V of
    # every prefill segment are staged per kv head in 128-key tiles
    # (when decode rows exist too, the planner may give the prefill kernel a
    # share of the SMs to run beside the decode kernel, sized for the rest)
    # (the pair kernel takes a tile's two heads on a cluster of two CTAs:
    # head_dim 128, an even group, two CTAs per tile slot)
    if info["prefill_pair"]:
        assert lay.head_dim == 128 and G % 2 == 0 and info["num_prefill_ctas"] % 2 == 0
    slots = info["num_sms"] // 2 if info["prefill_pair"] else info["num_sms"]
    per_slot = 2 if info["prefill_pair"] else 1
    if info["num_decode_units"] == 0:
        assert info["overlap_sms"] == 0
        assert info["num_prefill_ctas"] == per_slot * min(info["num_prefill_tiles"], slots)
    else:
        assert 0 <= info["num_prefill_ctas"] <= per_slot * min(info["num_prefill_tiles"], (info["num_sms"] - 8) // per_slot)
        if info["overlap_sms"] > 0:
            assert info["num_prefill_ctas"] <= info["overlap_sms"] <= info["num_sms"] - 8
            assert info["num_decode_units"] <= (info["num_sms"] - info["overlap_sms"]) * warps_per_sm
    pre = ql > 16 if prefill_on_tensor_cores else np.zeros_like(ql, dtype=bool)
    staged = int(sum(-(-n // 128) for n in sl[pre])) * lay.num_kv_heads
    assert info["num_staged_kv_tiles"] == staged
    assert info["workspace_bytes"] >= staged * 2 * 128 * lay.head_dim * 2


def test_plan_rebuild_in_place(lib):
    a = W.layout("decode_tinyllama_b64")
    b = W.layout("tiny_mixed")
    plan = pa.Plan(a.cu_seqlens_q, a.seq_lens, dims_for(a), device=-1)
    h0 = plan.handle.value
    ia = plan.info()
    plan.rebuild(b.cu_seqlens_q, b.seq_lens, dims_for(b))
    assert plan.handle.value == h0
    ib = plan.info()
    assert ib == pa.Plan(b.cu_seqlens_q, b.seq_lens, dims_for(b), device=-1).info()
    plan.rebuild(a.cu_seqlens_q, a.seq_lens, dims_for(a))
    assert plan.info() == ia
    # a plan cannot move to another device
    h = plan.handle
    d = dims_for(a)
    assert lib.pa_plan_build(a.cu_seqlens_q.ctypes.data_as(ctypes.c_void_p),
                             a.seq_lens.ctypes.data_as(ctypes.c_void_p), None, ctypes.byref(d), 0,
                             ctypes.byref(h)) == pa.PA_ERR_PLAN


def test_plan_is_deterministic(lib):
    lay = W.layout("decode_llama3_8b_b256")
    a = pa.Plan(lay.cu_seqlens_q, lay.seq_lens, dims_for(lay), device=-1).info()
    b = pa.Plan(lay.cu_seqlens_q, lay.seq_lens, dims_for(lay), device=-1).info()
    assert a == b


def _status(fn, *args):
    return fn(*args)


def test_plan_rejects_bad_arguments(lib):
    lay = W.layout("tiny_mixed")
    cu, sl = lay.cu_seqlens_q.copy(), lay.seq_lens.copy()

    def build(cu, sl, d):
        h = ctypes.c_void_p()          # NULL: ask for a new plan
        st = lib.pa_plan_build(cu.ctypes.data_as(ctypes.c_void_p), sl.ctypes.data_as(ctypes.c_void_p), None,
                               ctypes.byref(d), -1, ctypes.byref(h))
        assert st == pa.PA_OK or not h.value
        lib.pa_plan_destroy(h)
        return st

    h = ctypes.c_void_p()
    assert build(cu, sl, dims_for(lay)) == pa.PA_OK
    bad = cu.copy(); bad[-1] += 1
    assert build(bad, sl, dims_for(lay)) == pa.PA_ERR_SHAPE          # does not end at T
    bad = cu.copy(); bad[1], bad[2] = bad[2], bad[1]
    assert build(bad, sl, dims_for(lay)) == pa.PA_ERR_SHAPE          # not monotone
    bad = sl.copy(); bad[2] = 5
    assert build(cu, bad, dims_for(lay)) == pa.PA_ERR_SHAPE          # q_len > seq_len
    d = dims_for(lay); d.head_dim = 96
    assert build(cu, sl, d) == pa.PA_ERR_UNSUPPORTED
    d = dims_for(lay); d.block_size = 32
    assert build(cu, sl, d) == pa.PA_ERR_UNSUPPORTED
    d = dims_for(lay); d.num_q_heads = 3
    assert build(cu, sl, d) == pa.PA_ERR_SHAPE                       # Hq % Hkv != 0
    d = dims_for(lay); d.num_q_heads, d.num_kv_heads = 34, 2
    assert build(cu, sl, d) == pa.PA_ERR_UNSUPPORTED                 # group 17
    d = dims_for(lay); d.max_blocks_per_seq = 2
    assert build(cu, sl, d) == pa.PA_ERR_SHAPE                       # table too narrow
    assert lib.pa_plan_build(None, None, None, ctypes.byref(dims_for(lay)), -1, ctypes.byref(h)) == pa.PA_ERR_NULL
    assert lib.pa_plan_build(cu.ctypes.data_as(ctypes.c_void_p), sl.ctypes.data_as(ctypes.c_void_p), None,
                             ctypes.byref(dims_for(lay)), -1, None) == pa.PA_ERR_NULL


def test_compute_calls_reject_bad_arguments_before_any_launch(lib):
    lay = W.layout("tiny_mixed")
    d = dims_for(lay)
    fake = ctypes.c_void_p(0x10000)          # never dereferenced: checks fail first
    odd = ctypes.c_void_p(0x10008)
    S = None
    # reshape_and_cache
    assert lib.pa_reshape_and_cache(S, S, S, S, S, ctypes.byref(d), S) == pa.PA_ERR_NULL
    assert lib.pa_reshape_and_cache(odd, fake, fake, fake, fake, ctypes.byref(d), S) == pa.PA_ERR_ALIGN
    d0 = dims_for(lay); d0.num_tokens = 0
    assert lib.pa_reshape_and_cache(S, S, S, S, S, ctypes.byref(d0), S) == pa.PA_OK
    d2 = dims_for(lay); d2.head_dim = 80
    assert lib.pa_reshape_and_cache(fake, fake, fake, fake, fake, ctypes.byref(d2), S) == pa.PA_ERR_UNSUPPORTED
    # attention: no plan, plan of other dims, missing or misaligned workspace
    args = [fake] * 6 + [ctypes.c_float(0.125), fake, ctypes.byref(d)]
    assert lib.pa_attention_varlen(*args, None, fake, 1 << 20, S) == pa.PA_ERR_NULL
    plan = pa.Plan(lay.cu_seqlens_q, lay.seq_lens, d, device=-1)
    other = dims_for(lay); other.num_q_heads = 8
    args_other = [fake] * 6 + [ctypes.c_float(0.125), fake, ctypes.byref(other)]
    assert lib.pa_attention_varlen(*args_other, plan.handle, fake, 1 << 20, S) == pa.PA_ERR_PLAN
    assert lib.pa_attention_varlen(*args, plan.handle, None, 0, S) == pa.PA_ERR_WORKSPACE
    assert lib.pa_attention_varlen(*args, plan.handle, fake, 16, S) == pa.PA_ERR_WORKSPACE
    assert lib.pa_attention_varlen(*args, plan.handle, ctypes.c_void_p(0x10010), 1 << 20, S) == pa.PA_ERR_WORKSPACE
    args_odd = [odd] + [fake] * 5 + [ctypes.c_float(0.125), fake, ctypes.byref(d)]
    assert lib.pa_attention_varlen(*args_odd, plan.handle, fake, 1 << 20, S) == pa.PA_ERR_ALIGN
    # fused scatter + attention: its own pointers are checked before anything else
    fused = lambda *a: lib.pa_reshape_and_attention(*a)
    tail = [fake, fake, fake, fake, fake, fake, ctypes.c_float(0.125), fake, ctypes.byref(d), plan.handle, fake,
            ctypes.c_size_t(1 << 20), S]
    assert fused(None, fake, fake, fake, *tail[1:]) == pa.PA_ERR_NULL
    assert fused(odd, fake, fake, fake, *tail[1:]) == pa.PA_ERR_ALIGN
    assert fused(fake, fake, ctypes.c_void_p(0x10004), fake, *tail[1:]) == pa.PA_ERR_ALIGN  # slots: 8-byte aligned
    assert fused(fake, fake, fake, fake, *tail[1:9], None, *tail[10:]) == pa.PA_ERR_NULL  # no plan
    assert fused(S, S, S, S, S, S, S, S, S, ctypes.c_float(0.125), S, ctypes.byref(d0), plan.handle, S, 0, S) \
        in (pa.PA_OK, pa.PA_ERR_PLAN)                                   # T = 0: nothing to check or queue
    # KV export / import
    for name in ("pa_kv_export", "pa_kv_import"):
        fn = getattr(lib, name)
        dk = dims_for(lay)
        assert fn(S, S, S, S, S, S, None, S) == pa.PA_ERR_NULL
        assert fn(None, fake, fake, fake, fake, fake, ctypes.byref(dk), S) == pa.PA_ERR_NULL
        assert fn(odd, fake, fake, fake, fake, fake, ctypes.byref(dk), S) == pa.PA_ERR_ALIGN
        assert fn(fake, fake, fake, ctypes.c_void_p(0x10002), fake, fake, ctypes.byref(dk), S) == pa.PA_ERR_ALIGN
        dk.head_dim = 96
        assert fn(fake, fake, fake, fake, fake, fake, ctypes.byref(dk), S) == pa.PA_ERR_UNSUPPORTED
        dk = dims_for(lay); dk.num_tokens = 0
        assert fn(S, S, S, S, S, S, ctypes.byref(dk), S) == pa.PA_OK          # nothing to move
        dk = dims_for(lay); dk.num_seqs = 0
        assert fn(fake, fake, fake, fake, fake, fake, ctypes.byref(dk), S) == pa.PA_ERR_SHAPE  # rows, no requests
    # validate: scratch too small
    assert lib.pa_validate_inputs(fake, fake, fake, fake, ctypes.byref(d), fake, 8, S) == pa.PA_ERR_WORKSPACE
    # bounded-wait self-test: status word missing or misaligned, limit out of range
    assert lib.pa_selftest_wait_timeout(None, 1000, S) == pa.PA_ERR_NULL
    assert lib.pa_selftest_wait_timeout(ctypes.c_void_p(0x10010), 1000, S) == pa.PA_ERR_WORKSPACE
    assert lib.pa_selftest_wait_timeout(fake, 0, S) == pa.PA_ERR_SHAPE
    assert lib.pa_selftest_wait_timeout(fake, 3 * 10 ** 9, S) == pa.PA_ERR_SHAPE
    # no-alloc status word: nowhere to put it
    assert lib.pa_noalloc_status(None, 0, S) == pa.PA_ERR_NULL


def test_status_strings(lib):
    for s in range(-9, 1):
        assert pa.status_string(s)
    assert pa.status_string(-100) == "unknown status"


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_attention_launch_count(lib, name):
    # decode kernel; staging (when tiles are staged: the pair kernel reads a
    # shared prefix from the paged cache) + prefill; the merge kernel only
    # when shared-prefix tiles run beside the decode kernel
    lay = W.layout(name)
    info = pa.Plan(lay.cu_seqlens_q, lay.seq_lens, dims_for(lay), device=-1,
                   block_tables=lay.block_tables).info()
    per_prefill = 1 + (info["num_staged_kv_tiles"] > 0)
    base = (info["num_decode_units"] > 0) + per_prefill * (info["num_prefill_tiles"] > 0)
    assert base <= info["attention_launches"] <= base + (info["num_prefix_groups"] > 0)
    if name == "prefix_llama3_70b_b128":
        # 128 decodes on a 4096-token prefix: prefix tiles (pair kernel) beside
        # the suffix decode, then the merge kernel
        assert info["num_prefix_groups"] == 1 and info["prefill_pair"] == 1 and info["attention_launches"] == 3


@pytest.mark.parametrize("seed", range(40))
def test_plan_invariants_on_random_batches(lib, seed):
    # random mixes of decodes, speculative-decode rows, chunks and fresh
    # prompts, head counts and head_dims: the planner's accounting holds
    rng = np.random.default_rng(9000 + seed)
    S = int(rng.integers(1, 200))
    seq = rng.integers(1, 6000, S)
    kind = rng.integers(0, 4, S)
    q = np.where(kind == 0, 1, np.where(kind == 1, rng.integers(2, 17, S),
                                        np.where(kind == 2, rng.integers(17, 700, S), seq)))
    q = np.minimum(q, seq).astype(np.int32)
    seq = seq.astype(np.int32)
    cu = np.concatenate([[0], np.cumsum(q)]).astype(np.int32)
    Hkv = int(2 ** rng.integers(0, 4))
    G = int(rng.integers(1, 17))
    D = int(rng.choice([64, 128]))
    MB = int(-(-seq.max() // 16))
    d = pa.Dims(int(cu[-1]), S, Hkv * G, Hkv, D, 1 << 20, MB, 16)
    info = pa.Plan(cu, seq, d, device=-1).info()
    dec = q <= 16
    rows = int(q[dec].sum()) * Hkv
    assert info["num_decode_rows"] == rows
    blocks = sum(-(-(int(n) - int(L) + j + 1) // 16) for L, n in zip(q[dec], seq[dec]) for j in range(int(L)))
    assert info["decode_kv_blocks"] == blocks * Hkv
    warps_per_sm = 12 if D == 64 else 8
    assert (info["num_decode_units"] == 0) == (blocks == 0)
    assert info["num_decode_units"] <= 148 * warps_per_sm
    assert info["num_partials"] >= 2 * info["num_combine_rows"]
    assert info["num_partials"] <= info["num_combine_rows"] + info["num_decode_units"] * 2
    # prefill: one tile per (128-query chunk, kv head, query-head pair)
    tiles = sum(-(-int(L) // 128) for L in q[~dec]) * Hkv * (-(-G // 2))
    assert info["num_prefill_tiles"] == tiles
    pairs = sum(int(n) - int(L) + j + 1 for L, n in zip(q[~dec], seq[~dec]) for j in range(int(L)))
    assert info["prefill_causal_pairs"] == pairs
    assert info["num_staged_kv_tiles"] == sum(-(-int(n) // 128) for n in seq[~dec]) * Hkv
    base = (info["num_decode_units"] > 0) + 2 * (info["num_prefill_tiles"] > 0)
    assert info["attention_launches"] == base            # no shared prefixes without host tables
    assert info["workspace_bytes"] >= 256 + info["num_partials"] * G * D * 4


def test_shared_prefix_detection_on_constructed_tables(lib):
    # runs of >= 4 consecutive single-token segments whose tables agree on
    # >= 16 leading blocks (blocks wholly before each query's own key) form
    # a group; the decode rows then read only the blocks after the prefix
    rng = np.random.default_rng(77)
    pool = rng.permutation(100000).astype(np.int32)
    nxt = [0]

    def fresh(n):
        ids = pool[nxt[0]:nxt[0] + n]
        nxt[0] += n
        return list(ids)

    segs = []   # (q_len, seq_len, table, shared blocks expected)
    pa_ = fresh(20)
    for s in (5, 40, 77, 3, 16, 90):           # 6 decodes on a 20-block prefix
        n = 20 * 16 + s
        segs.append((1, n, pa_ + fresh(-(-n // 16) - 20), 20))
    pb = fresh(18)
    for s in (7, 9, 11):                        # only 3: no group
        n = 18 * 16 + s
        segs.append((1, n, pb + fresh(-(-n // 16) - 18), 0))
    segs.append((300, 900, fresh(-(-900 // 16)), 0))   # a prefill segment breaks runs
    pc = fresh(16)
    for s in (1, 2, 30, 60, 17):                # 5 decodes on a 16-block prefix
        n = 16 * 16 + s
        segs.append((1, n, pc + fresh(-(-n // 16) - 16), 16))
    q = np.array([a for a, _, _, _ in segs], np.int32)
    sl = np.array([b for _, b, _, _ in segs], np.int32)
    MB = max(len(t) for _, _, t, _ in segs)
    bt = np.zeros((len(segs), MB), np.int32)
    for i, (_, _, t, _) in enumerate(segs):
        bt[i, :len(t)] = t
    cu = np.concatenate([[0], np.cumsum(q)]).astype(np.int32)
    Hkv, G, D = 2, 4, 128
    d = pa.Dims(int(cu[-1]), len(segs), Hkv * G, Hkv, D, 100000, MB, 16)
    with_tables = pa.Plan(cu, sl, d, device=-1, block_tables=bt).info()
    without = pa.Plan(cu, sl, d, device=-1).info()
    assert with_tables["num_prefix_groups"] == 2 and without["num_prefix_groups"] == 0
    dec = [(n, sh) for L, n, _, sh in segs if L == 1]
    assert without["decode_kv_blocks"] == sum(-(-n // 16) for n, _ in dec) * Hkv
    assert with_tables["decode_kv_blocks"] == sum(-(-n // 16) - sh for n, sh in dec) * Hkv
    assert without["decode_kv_keys"] == sum(n for n, _ in dec) * Hkv
    assert with_tables["decode_kv_keys"] == sum(n - 16 * sh for n, sh in dec) * Hkv
    # the prefix tiles join the prefill segment's tiles and pairs
    assert with_tables["num_prefill_tiles"] > without["num_prefill_tiles"]
    extra_pairs = (6 * 20 + 5 * 16) * 16
    assert with_tables["prefill_causal_pairs"] == without["prefill_causal_pairs"] + extra_pairs
    assert with_tables["attention_launches"] in (2, 3, 4)
