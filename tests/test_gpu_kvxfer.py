"""KV export / import (pa_kv_export, pa_kv_import) on the GPU against the
oracle, bit for bit, and a round trip through another pool that attention
cannot tell apart from the original."""
import numpy as np
import pytest
import torch

import oracle as O
import paged_kv_attention_token_b200 as pa
import workloads as W
from tests.test_gpu_parity import dims_for

pytestmark = pytest.mark.gpu

CASES = ["tiny_mixed", "decode_tinyllama_b64", "prefix_llama3_70b_b128",
         ([1, 5, 17, 0, 3], [33, 5, 40, 9, 16], 6, 3, 64),
         ([1, 1, 130, 1], [700, 2100, 3000, 16], 12, 2, 128)]


def batch_for(case):
    if isinstance(case, str):
        return W.make_batch(W.layout(case), device="cuda")
    q_lens, seq_lens, Hq, Hkv, D = case
    nb = sum(-(-s // 16) for s in seq_lens) + 64
    return W.make_batch(W.custom_layout(q_lens, seq_lens, Hq, Hkv, D, nb, seed=77), device="cuda")


def cu_tokens(seq_lens):
    return np.concatenate([[0], np.cumsum(seq_lens)]).astype(np.int32)


def scattered_pool(b):
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    _, _, _, slots = b.device_ints("cuda")
    pa.reshape_and_cache(b.k, b.v, slots, kc, vc)
    return kc, vc


def other_tables(lay, extra=37, seed=5):
    """Block tables over a larger pool whose requests own disjoint blocks."""
    nb2 = int(sum(-(-int(n) // 16) for n in lay.seq_lens)) + extra
    ids = np.random.default_rng(seed).permutation(nb2).astype(np.int32)
    bt2 = np.zeros_like(lay.block_tables)
    o = 0
    for i, n in enumerate(lay.seq_lens):
        k = -(-int(n) // 16)
        bt2[i, :k] = ids[o:o + k]
        o += k
    return nb2, bt2


@pytest.mark.parametrize("case", range(len(CASES)))
def test_kv_export_matches_oracle(cuda_lib, case):
    b = batch_for(CASES[case])
    lay = b.layout
    kc, vc = scattered_pool(b)
    cu_t = cu_tokens(lay.seq_lens)
    N = int(cu_t[-1])
    k_out = torch.empty((N, lay.num_kv_heads, lay.head_dim), dtype=torch.bfloat16, device="cuda")
    v_out = torch.empty_like(k_out)
    bt = torch.from_numpy(lay.block_tables).cuda()
    pa.kv_export(kc, vc, bt, torch.from_numpy(cu_t).cuda(), k_out, v_out)
    torch.cuda.synchronize()
    want_k, want_v = O.kv_export(W.bf16_bits(kc), W.bf16_bits(vc), lay.block_tables, cu_t)
    assert np.array_equal(W.bf16_bits(k_out), want_k) and np.array_equal(W.bf16_bits(v_out), want_v)


@pytest.mark.parametrize("case", [0, 1, 3, 4])   # (the shared-prefix case imports into shared slots)
def test_kv_import_matches_oracle_and_attention_cannot_tell_the_pools_apart(cuda_lib, case):
    b = batch_for(CASES[case])
    lay = b.layout
    kc, vc = scattered_pool(b)
    cu_t = cu_tokens(lay.seq_lens)
    cu_d = torch.from_numpy(cu_t).cuda()
    N = int(cu_t[-1])
    k_buf = torch.empty((N, lay.num_kv_heads, lay.head_dim), dtype=torch.bfloat16, device="cuda")
    v_buf = torch.empty_like(k_buf)
    pa.kv_export(kc, vc, torch.from_numpy(lay.block_tables).cuda(), cu_d, k_buf, v_buf)
    nb2, bt2 = other_tables(lay)
    kc2 = torch.full((nb2,) + tuple(kc.shape[1:]), float("nan"), dtype=torch.bfloat16, device="cuda")
    vc2 = kc2.clone()
    want_k, want_v = W.bf16_bits(kc2).copy(), W.bf16_bits(vc2).copy()
    bt2_d = torch.from_numpy(bt2).cuda()
    pa.kv_import(k_buf, v_buf, bt2_d, cu_d, kc2, vc2)
    torch.cuda.synchronize()
    O.kv_import(W.bf16_bits(k_buf), W.bf16_bits(v_buf), bt2, cu_t, want_k, want_v)
    assert np.array_equal(W.bf16_bits(kc2), want_k) and np.array_equal(W.bf16_bits(vc2), want_v)
    # attention over the imported pool (same plan inputs, other block ids)
    dims = dims_for(lay)
    _, cu, sl, _ = b.device_ints("cuda")
    outs = []
    for kcx, vcx, btx, nbx in ((kc, vc, torch.from_numpy(lay.block_tables).cuda(), lay.num_blocks),
                               (kc2, vc2, bt2_d, nb2)):
        dims.num_blocks = nbx
        plan = pa.Plan(lay.cu_seqlens_q, lay.seq_lens, dims)
        ws = pa.workspace_for(plan)
        out = torch.full_like(b.q, float("nan"))
        pa.attention_varlen(b.q, kcx, vcx, btx, cu, sl, b.scale, out, plan, ws)
        torch.cuda.synchronize()
        outs.append(out)
    assert not torch.isnan(outs[0].float()).any()
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
