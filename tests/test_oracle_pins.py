"""Pins of the CPU oracle to things other than itself (CPU only).

Each test is chosen so that a plausible mistake in the oracle (a dropped
block, an off-by-one causal edge, a wrong kv-head mapping, a transposed
index, a missing scale, top-left instead of bottom-right alignment) fails at
least one of them:

* a hand-worked example whose outputs follow in closed form
  (tests/golden/handworked_mixed.json);
* special cases that reduce to torch's fp64 scaled_dot_product_attention on
  dense (non-paged) K/V: fresh prefill (causal), decode (no mask), chunked
  prefill (explicit bottom-right mask), with GQA;
* closed forms: seq_len 1, constant V, zero q, a sharply peaked q;
* invariants: relabelling the pool, deleting or reordering other segments,
  perturbing keys a query must not see, NaN in every unread slot;
* the scatter round trip, checked by flattening the pool with numpy;
* power of the parity tolerance: a wrong block or a causal edge off by one
  must fail the tolerance on peaked inputs.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from tests.parity import within, errors

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits(x) -> np.ndarray:
    return W.bf16_bits(torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16))


def from_bits(b: np.ndarray) -> np.ndarray:
    return torch.from_numpy(b.view(np.int16).copy()).view(torch.bfloat16).double().numpy()


def dense_problem(q_lens, seq_lens, Hq, Hkv, D, seed, num_blocks=None, q_gain=1.0):
    """Random dense per-request K/V (bf16-exact) and a paged pool built from
    them by block (logical block b of request i holds positions 16b..16b+15 in
    physical block block_tables[i][b]).  Unread pool rows are NaN."""
    rng = np.random.default_rng(seed)
    nb_total = sum(-(-n // 16) for n in seq_lens)
    lay = W.custom_layout(q_lens, seq_lens, Hq, Hkv, D, num_blocks or nb_total + 4, seed)
    Kd = [from_bits(bits(rng.standard_normal((n, Hkv, D)))) for n in seq_lens]
    Vd = [from_bits(bits(rng.standard_normal((n, Hkv, D)))) for n in seq_lens]
    T = int(sum(q_lens))
    q = from_bits(bits(q_gain * rng.standard_normal((T, Hq, D))))
    kc = np.full((lay.num_blocks, 16, Hkv, D), np.nan, dtype=np.float32)
    vc = kc.copy()
    for i, n in enumerate(seq_lens):
        for b in range(-(-n // 16)):
            rows = min(16, n - 16 * b)
            kc[lay.block_tables[i, b], :rows] = Kd[i][16 * b:16 * b + rows]
            vc[lay.block_tables[i, b], :rows] = Vd[i][16 * b:16 * b + rows]
    return lay, q, Kd, Vd, bits(kc), bits(vc)


def scattered(b):
    """Pool of a generated batch after the oracle writes the scheduled tokens."""
    kc, vc = W.bf16_bits(b.k_cache).copy(), W.bf16_bits(b.v_cache).copy()
    O.reshape_and_cache(W.bf16_bits(b.k), W.bf16_bits(b.v), b.layout.slot_mapping, kc, vc)
    return kc, vc


def run_oracle(lay, q, kc, vc, scale=None, **kw):
    scale = 1.0 / math.sqrt(lay.head_dim) if scale is None else scale
    return O.attention_varlen(bits(q) if q.dtype != np.uint16 else q, kc, vc,
                              lay.block_tables, lay.cu_seqlens_q, lay.seq_lens, scale, **kw)


def sdpa_segment(q_seg, Kd, Vd, G, scale, mask):
    """torch fp64 SDPA on dense K/V for one segment. q_seg [L,Hq,D]."""
    qt = torch.from_numpy(q_seg).permute(1, 0, 2).unsqueeze(0)            # [1,Hq,L,D]
    kt = torch.from_numpy(Kd).permute(1, 0, 2).unsqueeze(0).repeat_interleave(G, dim=1)
    vt = torch.from_numpy(Vd).permute(1, 0, 2).unsqueeze(0).repeat_interleave(G, dim=1)
    if isinstance(mask, str) and mask == "causal":
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    elif mask is None:
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    else:
        o = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, attn_mask=torch.from_numpy(mask), scale=scale)
    return o.squeeze(0).permute(1, 0, 2).numpy()


# --------------------------------------------------------------------------
# hand-worked golden example
# --------------------------------------------------------------------------

def test_golden_handworked_mixed_batch():
    g = json.load(open(os.path.join(GOLDEN, "handworked_mixed.json")))
    Hq, Hkv, D, B, NB = g["num_q_heads"], g["num_kv_heads"], g["head_dim"], g["block_size"], g["num_blocks"]
    kc = np.full((NB, B, Hkv, D), np.nan, np.float32)
    vc = kc.copy()
    for s, val in g["history"]["k"].items():
        kc.reshape(-1, Hkv, D)[int(s)] = val
    for s, val in g["history"]["v"].items():
        vc.reshape(-1, Hkv, D)[int(s)] = val
    kc, vc = bits(kc), bits(vc)
    O.reshape_and_cache(bits(g["k"]), bits(g["v"]), np.array(g["slot_mapping"]), kc, vc)
    out = O.attention_varlen(bits(g["q"]), kc, vc, np.array(g["block_tables"], np.int32),
                             np.array(g["cu_seqlens_q"], np.int32), np.array(g["seq_lens"], np.int32),
                             math.log(3.0))
    np.testing.assert_allclose(out, np.array(g["expected_out"]), rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# scatter
# --------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny_mixed", "custom"])
def test_scatter_round_trip(name):
    if name == "tiny_mixed":
        lay = W.layout("tiny_mixed")
    else:
        lay = W.custom_layout([1, 5, 17, 0, 3], [33, 5, 40, 9, 16], 6, 3, 64, 40, seed=5)
    b = W.make_batch(lay)
    kc0, vc0 = W.bf16_bits(b.k_cache), W.bf16_bits(b.v_cache)
    kc, vc = kc0.copy(), vc0.copy()
    k, v = W.bf16_bits(b.k), W.bf16_bits(b.v)
    slots = lay.slot_mapping
    O.reshape_and_cache(k, v, slots, kc, vc)
    Hkv, D = lay.num_kv_heads, lay.head_dim
    flat_k, flat_v = kc.reshape(-1, Hkv, D), vc.reshape(-1, Hkv, D)
    # written rows hold exactly k[t], v[t]
    assert np.array_equal(flat_k[slots], k) and np.array_equal(flat_v[slots], v)
    # every other row is unchanged, bit for bit (NaN payloads included)
    keep = np.ones(flat_k.shape[0], bool)
    keep[slots] = False
    assert np.array_equal(flat_k[keep], kc0.reshape(-1, Hkv, D)[keep])
    assert np.array_equal(flat_v[keep], vc0.reshape(-1, Hkv, D)[keep])
    # the token at logical position p of request i is found in logical block
    # p // 16 of its block table, at row p % 16 of that physical block
    cu = lay.cu_seqlens_q
    for i in range(lay.num_seqs):
        n, L = int(lay.seq_lens[i]), int(lay.q_lens[i])
        for j in range(L):
            p = n - L + j
            blk = lay.block_tables[i, p // 16]
            assert np.array_equal(kc[blk, p % 16], k[cu[i] + j])
            assert np.array_equal(vc[blk, p % 16], v[cu[i] + j])


def test_scatter_skips_negative_slots_and_rejects_out_of_pool():
    lay = W.layout("tiny_mixed")
    b = W.make_batch(lay)
    kc0 = W.bf16_bits(b.k_cache)
    kc, vc = kc0.copy(), W.bf16_bits(b.v_cache).copy()
    slots = lay.slot_mapping.copy()
    slots[:] = -1
    O.reshape_and_cache(W.bf16_bits(b.k), W.bf16_bits(b.v), slots, kc, vc)
    assert np.array_equal(kc, kc0)
    slots[0] = lay.num_blocks * 16
    with pytest.raises(O.OracleError):
        O.reshape_and_cache(W.bf16_bits(b.k), W.bf16_bits(b.v), slots, kc, vc)


# --------------------------------------------------------------------------
# reductions to torch SDPA on dense K/V
# --------------------------------------------------------------------------

@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (8, 1), (6, 6), (12, 2)])
def test_against_sdpa_mixed_segments(Hq, Hkv):
    # decode (q 1 on 53), fresh prefill (q = seq = 37), chunk (q 11 on 70),
    # decode on a 1-token history, chunk whose start is not block aligned
    q_lens = [1, 37, 11, 1, 20]
    seq_lens = [53, 37, 70, 2, 45]
    D = 64
    lay, q, Kd, Vd, kc, vc = dense_problem(q_lens, seq_lens, Hq, Hkv, D, seed=Hq * 10 + Hkv)
    scale = 0.7 / math.sqrt(D)       # not 1/sqrt(D): pins that the scale is applied once
    out = run_oracle(lay, q, kc, vc, scale)
    cu = lay.cu_seqlens_q
    G = Hq // Hkv
    for i, (L, n) in enumerate(zip(q_lens, seq_lens)):
        qs = q[cu[i]:cu[i + 1]]
        if L == 1:
            want = sdpa_segment(qs, Kd[i], Vd[i], G, scale, None)
        elif L == n:
            want = sdpa_segment(qs, Kd[i], Vd[i], G, scale, "causal")
        else:
            mask = np.arange(n)[None, :] <= (n - L + np.arange(L))[:, None]
            want = sdpa_segment(qs, Kd[i], Vd[i], G, scale, mask)
        np.testing.assert_allclose(out[cu[i]:cu[i + 1]], want, rtol=1e-10, atol=1e-12)


def test_head_dim_128_and_long_history_against_sdpa():
    lay, q, Kd, Vd, kc, vc = dense_problem([1, 3], [700, 260], 16, 2, 128, seed=3)
    out = run_oracle(lay, q, kc, vc)
    cu = lay.cu_seqlens_q
    want0 = sdpa_segment(q[0:1], Kd[0], Vd[0], 8, 1 / math.sqrt(128), None)
    mask = np.arange(260)[None, :] <= (257 + np.arange(3))[:, None]
    want1 = sdpa_segment(q[1:4], Kd[1], Vd[1], 8, 1 / math.sqrt(128), mask)
    np.testing.assert_allclose(out[cu[0]:cu[1]], want0, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(out[cu[1]:cu[2]], want1, rtol=1e-10, atol=1e-12)


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------

def test_seq_len_one_returns_v0_exactly():
    lay, q, Kd, Vd, kc, vc = dense_problem([1, 1], [1, 1], 4, 2, 64, seed=7)
    out = run_oracle(lay, q, kc, vc)
    for i in range(2):
        for h in range(4):
            assert np.array_equal(out[i, h], Vd[i][0, h // 2])


def test_constant_v_gives_constant():
    lay, q, Kd, Vd, kc, vc = dense_problem([1, 9], [300, 41], 4, 2, 64, seed=8)
    vc_const = bits(np.full(from_bits(vc).shape, 1.5, np.float32))
    out = run_oracle(lay, q, kc, vc_const)
    np.testing.assert_allclose(out, 1.5, rtol=0, atol=1e-13)


def test_zero_query_averages_visible_values():
    q_lens, seq_lens = [1, 4], [77, 30]
    lay, q, Kd, Vd, kc, vc = dense_problem(q_lens, seq_lens, 4, 2, 64, seed=9)
    out = run_oracle(lay, np.zeros_like(q), kc, vc)
    np.testing.assert_allclose(out[0], np.repeat(Vd[0].mean(axis=0), 2, axis=0), atol=1e-12)
    for j in range(4):
        p = 30 - 4 + j
        np.testing.assert_allclose(out[1 + j], np.repeat(Vd[1][:p + 1].mean(axis=0), 2, axis=0),
                                   atol=1e-12)


def test_peaked_query_selects_one_value():
    # q = 50 * K[tau*] makes the score at tau* exceed every other by far more
    # than the log of the number of keys, so the output is V[tau*].
    lay, q, Kd, Vd, kc, vc = dense_problem([1], [200], 2, 1, 64, seed=10)
    tau = 137
    qpk = np.zeros_like(q)
    qpk[0, :] = 50 * Kd[0][tau, 0] / np.linalg.norm(Kd[0][tau, 0])
    out = run_oracle(lay, from_bits(bits(qpk)), kc, vc, scale=1.0)
    np.testing.assert_allclose(out[0, 0], Vd[0][tau, 0], atol=1e-6)


# --------------------------------------------------------------------------
# invariants
# --------------------------------------------------------------------------

def test_pool_relabelling_leaves_output_bit_identical():
    lay = W.custom_layout([1, 6, 1], [39, 23, 64], 4, 2, 64, 30, seed=11)
    b = W.make_batch(lay)
    kc, vc = scattered(b)
    out = O.attention_varlen(W.bf16_bits(b.q), kc, vc, lay.block_tables, lay.cu_seqlens_q,
                             lay.seq_lens, b.scale)
    assert not np.isnan(out).any()
    perm = np.random.default_rng(0).permutation(lay.num_blocks)
    inv = np.argsort(perm)
    kc2, vc2 = kc[perm], vc[perm]           # new block j holds old block perm[j]
    bt2 = inv[lay.block_tables].astype(np.int32)
    out2 = O.attention_varlen(W.bf16_bits(b.q), kc2, vc2, bt2, lay.cu_seqlens_q, lay.seq_lens, b.scale)
    assert np.array_equal(out, out2)


def test_segments_isolated_and_order_free():
    lay = W.custom_layout([1, 7, 1, 3], [50, 7, 18, 33], 4, 2, 64, 40, seed=12)
    b = W.make_batch(lay)
    kc, vc = scattered(b)
    full = O.attention_varlen(W.bf16_bits(b.q), kc, vc,
                              lay.block_tables, lay.cu_seqlens_q, lay.seq_lens, b.scale)
    assert not np.isnan(full).any()
    cu = lay.cu_seqlens_q
    qb = W.bf16_bits(b.q)
    for order in ([3, 1, 0, 2], [2], [1, 3]):
        ql = lay.q_lens[order]
        cu2 = np.concatenate([[0], np.cumsum(ql)]).astype(np.int32)
        q2 = np.concatenate([qb[cu[i]:cu[i + 1]] for i in order])
        out = O.attention_varlen(q2, kc, vc,
                                 lay.block_tables[order], cu2, lay.seq_lens[order], b.scale)
        for r, i in enumerate(order):
            assert np.array_equal(out[cu2[r]:cu2[r + 1]], full[cu[i]:cu[i + 1]])


def test_causality_future_keys_and_other_segments_do_not_matter():
    q_lens, seq_lens = [5, 1], [21, 30]
    lay, q, Kd, Vd, kc, vc = dense_problem(q_lens, seq_lens, 4, 2, 64, seed=13)
    base = run_oracle(lay, q, kc, vc)
    # perturb positions 18.. of segment 0 (query j=2 sits at position 18 and
    # must not see 19, 20), and all of segment 1's history
    kf, vf = from_bits(kc), from_bits(vc)
    for p in (19, 20):
        blk = lay.block_tables[0, p // 16]
        kf[blk, p % 16] += 3.0
        vf[blk, p % 16] -= 5.0
    for p in range(30):
        blk = lay.block_tables[1, p // 16]
        kf[blk, p % 16] *= -1
    out = run_oracle(lay, q, bits(kf), bits(vf))
    assert np.array_equal(out[0:3], base[0:3])      # queries at positions 16, 17, 18
    assert not np.allclose(out[3:5], base[3:5])     # positions 19, 20 see the change
    assert not np.allclose(out[5], base[5])         # segment 1 reads its own history


def test_unread_slots_are_nan_and_never_reach_the_output():
    for name in ("tiny_mixed",):
        lay = W.layout(name)
        b = W.make_batch(lay)
        kc, vc = scattered(b)
        assert np.isnan(from_bits(kc)).any()
        out = O.attention_varlen(W.bf16_bits(b.q), kc, vc, lay.block_tables, lay.cu_seqlens_q,
                                 lay.seq_lens, b.scale)
        assert not np.isnan(out).any()


def test_sampled_rows_match_full_output():
    lay = W.custom_layout([1, 6, 1], [39, 23, 64], 4, 2, 64, 30, seed=14)
    b = W.make_batch(lay)
    kc, vc = scattered(b)
    args = (W.bf16_bits(b.q), kc, vc, lay.block_tables,
            lay.cu_seqlens_q, lay.seq_lens, b.scale)
    full = O.attention_varlen(*args)
    rows = np.array([0, 5, 13, 31, 7], np.int64)
    part = O.attention_varlen(*args, rows=rows)
    assert np.array_equal(part, full.reshape(-1, lay.head_dim)[rows])


def test_empty_segments_and_empty_batch():
    lay, q, Kd, Vd, kc, vc = dense_problem([0, 2, 0], [5, 9, 16], 4, 2, 64, seed=15)
    out = run_oracle(lay, q, kc, vc)
    assert out.shape == (2, 4, 64)
    mask = np.arange(9)[None, :] <= (7 + np.arange(2))[:, None]
    want = sdpa_segment(q, Kd[1], Vd[1], 2, 1 / 8, mask)
    np.testing.assert_allclose(out, want, rtol=1e-10, atol=1e-12)
    e = O.attention_varlen(np.zeros((0, 4, 64), np.uint16), kc, vc, np.zeros((0, 1), np.int32),
                           np.zeros(1, np.int32), np.zeros(0, np.int32), 0.125)
    assert e.shape == (0, 4, 64)


def test_invalid_inputs_are_rejected():
    lay, q, Kd, Vd, kc, vc = dense_problem([2], [9], 4, 2, 64, seed=16)
    with pytest.raises(O.OracleError):      # q_len > seq_len
        O.attention_varlen(bits(q), kc, vc, lay.block_tables, lay.cu_seqlens_q,
                           np.array([1], np.int32), 0.1)
    bt = lay.block_tables.copy()
    bt[0, 0] = lay.num_blocks               # block id outside the pool
    with pytest.raises(O.OracleError):
        O.attention_varlen(bits(q), kc, vc, bt, lay.cu_seqlens_q, lay.seq_lens, 0.1)


# --------------------------------------------------------------------------
# power of the parity tolerance
# --------------------------------------------------------------------------

def _peaked(lay_name):
    lay = W.layout(lay_name)
    b = W.make_batch(lay, q_gain=8.0)
    kc, vc = scattered(b)
    return lay, b, kc, vc


def test_tolerance_catches_a_wrong_block():
    lay, b, kc, vc = _peaked("tiny_mixed")
    args = (W.bf16_bits(b.q), kc, vc)
    good = O.attention_varlen(*args, lay.block_tables, lay.cu_seqlens_q, lay.seq_lens, b.scale)
    # request 1 (seq 40) reads its middle block from another request's block
    bt = lay.block_tables.copy()
    bt[1, 1] = lay.block_tables[0, 0]
    bad = O.attention_varlen(*args, bt, lay.cu_seqlens_q, lay.seq_lens, b.scale)
    assert not within(bad.astype(np.float32), good), errors(bad, good)


def test_tolerance_catches_a_causal_edge_off_by_one():
    lay, b, kc, vc = _peaked("tiny_mixed")
    args = (W.bf16_bits(b.q), kc, vc, lay.block_tables, lay.cu_seqlens_q)
    good = O.attention_varlen(*args, lay.seq_lens, b.scale)
    # emulate "query j also sees key j+1" for the 6-token prefill (seq 6):
    # its first five queries asked as a 5-query chunk on the same 6 keys sit
    # at positions j+1
    sl = lay.seq_lens.copy()
    cu = lay.cu_seqlens_q.copy()
    cu2 = cu.copy()
    cu2[3] = cu[3] - 1
    q2 = W.bf16_bits(b.q)[:cu2[3]]
    bad = O.attention_varlen(q2, kc, vc, lay.block_tables, cu2, sl, b.scale)
    # bad row for prefill query j (j=0..4) sees keys 0..j+1; good sees 0..j
    assert not within(bad[cu[2]:cu2[3]].astype(np.float32), good[cu[2]:cu[3] - 1])


def test_tolerance_catches_a_wrong_kv_head_mapping():
    lay, b, kc, vc = _peaked("tiny_mixed")
    q = W.bf16_bits(b.q)
    good = O.attention_varlen(q, kc, vc, lay.block_tables, lay.cu_seqlens_q, lay.seq_lens, b.scale)
    # h -> h % Hkv instead of h // G: swap query heads 1 and 2 (Hq 4, Hkv 2)
    q2 = q[:, [0, 2, 1, 3]]
    bad = O.attention_varlen(q2, kc, vc, lay.block_tables, lay.cu_seqlens_q, lay.seq_lens, b.scale)[:, [0, 2, 1, 3]]
    assert not within(bad.astype(np.float32), good)


# --------------------------------------------------------------------------
# KV export / import ("vLLM 学习笔记 01" §2.5: a request's KV cache moved
# between instances; the local half is a gather to / scatter from a
# contiguous buffer through the block table)
# --------------------------------------------------------------------------

def _cu_tokens(seq_lens):
    return np.concatenate([[0], np.cumsum(seq_lens)]).astype(np.int32)


def test_kv_export_returns_each_requests_dense_history():
    # the pool is built block by block from dense per-request K/V (numpy
    # slicing); export must give those dense arrays back, concatenated
    seq_lens = [33, 1, 16, 70, 0, 17]
    lay, _, Kd, Vd, kc, vc = dense_problem([1, 1, 1, 1, 0, 1], seq_lens, 4, 2, 64, seed=21)
    k_out, v_out = O.kv_export(kc, vc, lay.block_tables, _cu_tokens(seq_lens))
    assert np.array_equal(k_out, bits(np.concatenate(Kd)))
    assert np.array_equal(v_out, bits(np.concatenate(Vd)))


def test_kv_export_after_scatter_returns_the_written_tokens():
    # a step's new tokens, written by the scatter, come back from export at
    # their positions n - L .. n - 1
    lay = W.custom_layout([1, 5, 17, 3], [33, 5, 40, 16], 6, 3, 64, 40, seed=5)
    b = W.make_batch(lay)
    kc, vc = scattered(b)
    k_out, v_out = O.kv_export(kc, vc, lay.block_tables, _cu_tokens(lay.seq_lens))
    k, v = W.bf16_bits(b.k), W.bf16_bits(b.v)
    cu_t = _cu_tokens(lay.seq_lens)
    for i in range(lay.num_seqs):
        n, L = int(lay.seq_lens[i]), int(lay.q_lens[i])
        rows = np.arange(cu_t[i] + n - L, cu_t[i] + n)
        tok = np.arange(lay.cu_seqlens_q[i], lay.cu_seqlens_q[i + 1])
        assert np.array_equal(k_out[rows], k[tok]) and np.array_equal(v_out[rows], v[tok])


def test_kv_import_into_another_pool_gives_the_same_attention():
    # export from one pool, import into an empty pool with other block ids:
    # attention over the new pool is bit-identical, and only the slots the
    # requests use are written
    lay = W.custom_layout([1, 6, 1, 2], [39, 23, 64, 100], 8, 2, 64, 40, seed=13)
    b = W.make_batch(lay)
    kc, vc = scattered(b)
    cu_t = _cu_tokens(lay.seq_lens)
    k_buf, v_buf = O.kv_export(kc, vc, lay.block_tables, cu_t)
    NB2 = lay.num_blocks + 25
    used = int(sum(-(-int(n) // 16) for n in lay.seq_lens))
    ids = np.random.default_rng(3).permutation(NB2)[:used].astype(np.int32)
    bt2 = np.zeros_like(lay.block_tables)
    o = 0
    for i, n in enumerate(lay.seq_lens):
        nb = -(-int(n) // 16)
        bt2[i, :nb] = ids[o:o + nb]
        o += nb
    kc2 = np.full((NB2,) + kc.shape[1:], 0x7fc1, dtype=np.uint16)   # a NaN payload
    vc2 = kc2.copy()
    O.kv_import(k_buf, v_buf, bt2, cu_t, kc2, vc2)
    q = W.bf16_bits(b.q)
    out = O.attention_varlen(q, kc, vc, lay.block_tables, lay.cu_seqlens_q, lay.seq_lens, b.scale)
    out2 = O.attention_varlen(q, kc2, vc2, bt2, lay.cu_seqlens_q, lay.seq_lens, b.scale)
    assert not np.isnan(out).any() and np.array_equal(out, out2)
    written = np.zeros(kc2.shape[:2], bool)
    for i, n in enumerate(lay.seq_lens):
        for p in range(int(n)):
            written[bt2[i, p // 16], p % 16] = True
    assert np.all(kc2[~written] == 0x7fc1) and np.all(vc2[~written] == 0x7fc1)
    # and the round trip returns the buffers
    k3, v3 = O.kv_export(kc2, vc2, bt2, cu_t)
    assert np.array_equal(k3, k_buf) and np.array_equal(v3, v_buf)


def test_kv_transfer_rejects_blocks_outside_the_pool_and_overlong_requests():
    lay, _, _, _, kc, vc = dense_problem([1, 1], [20, 5], 4, 2, 64, seed=2)
    bt = lay.block_tables.copy()
    bt[0, 1] = lay.num_blocks
    with pytest.raises(O.OracleError):
        O.kv_export(kc, vc, bt, _cu_tokens([20, 5]))
    with pytest.raises(O.OracleError):
        O.kv_export(kc, vc, lay.block_tables, _cu_tokens([20, 16 * lay.max_blocks_per_seq + 1]))
