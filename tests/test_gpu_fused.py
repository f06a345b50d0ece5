"""The fused step (pa_reshape_and_attention) against the two calls it
replaces: caches and output bit for bit, on every workload and the custom
shapes, plus oracle parity on speculative-decode shapes (q_len 2..16), whose
rows see several keys of their own step.

The pool holds NaN in every slot a step writes until its scatter lands, so
a key of the step read from the cache before the scatter wrote it would
show up as NaN in the output."""
import pytest
import torch

import paged_kv_attention_token_b200 as pa
import workloads as W
from tests.parity import assert_parity
from tests.test_gpu_parity import CUSTOM, PREFILL, dims_for, gpu_rows, oracle_subset, run_step

pytestmark = pytest.mark.gpu


def run_fused(batch, with_tables=True, stream=None, repeats=1):
    lay = batch.layout
    kc, vc = batch.k_cache.clone(), batch.v_cache.clone()
    bt, cu, sl, slots = batch.device_ints("cuda")
    plan = pa.Plan(lay.cu_seqlens_q, lay.seq_lens, dims_for(lay),
                   block_tables=lay.block_tables if with_tables else None)
    ws = pa.workspace_for(plan)
    out = torch.full_like(batch.q, float("nan"))
    for _ in range(repeats):
        pa.reshape_and_attention(batch.k, batch.v, slots, batch.q, kc, vc, bt, cu, sl, batch.scale, out, plan,
                                 ws, stream=stream)
    torch.cuda.synchronize()
    assert pa.workspace_status(ws) == 0
    return kc, vc, out, plan


def same_bits(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


def check_against_two_calls(b, **kw):
    kc1, vc1, out1, _ = run_step(b, with_tables=kw.get("with_tables", True))
    kc2, vc2, out2, plan = run_fused(b, **kw)
    assert same_bits(kc1, kc2) and same_bits(vc1, vc2), "caches differ"
    assert not torch.isnan(out2.float()).any(), f"NaN in the fused output: plan={plan.info()}"
    assert same_bits(out1, out2), f"outputs differ: plan={plan.info()}"


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_fused_matches_two_calls_on_workloads(cuda_lib, name):
    check_against_two_calls(W.make_batch(W.layout(name), device="cuda"))


@pytest.mark.parametrize("case", range(len(CUSTOM)))
def test_fused_matches_two_calls_on_custom_shapes(cuda_lib, case):
    q_lens, seq_lens, Hq, Hkv, D = CUSTOM[case]
    nb = sum(-(-s // 16) for s in seq_lens) + 64
    lay = W.custom_layout(q_lens, seq_lens, Hq, Hkv, D, nb, seed=100 + case)
    check_against_two_calls(W.make_batch(lay, device="cuda"))


SPEC = [
    # (q_lens, seq_lens, Hq, Hkv, D): verification of 2..16 drafted tokens on
    # a long paged history; a row's step keys can straddle a block edge
    ([2, 4, 8, 16, 3], [1000, 515, 33, 2048, 17], 32, 4, 64),
    ([16, 5, 9, 1, 12], [1700, 129, 2100, 64, 300], 12, 2, 128),
]


@pytest.mark.parametrize("case", range(len(SPEC)))
@pytest.mark.parametrize("q_gain", [1.0, 8.0])
def test_fused_spec_decode_against_oracle(cuda_lib, case, q_gain):
    q_lens, seq_lens, Hq, Hkv, D = SPEC[case]
    nb = sum(-(-s // 16) for s in seq_lens) + 64
    lay = W.custom_layout(q_lens, seq_lens, Hq, Hkv, D, nb, seed=400 + case)
    b = W.make_batch(lay, device="cuda", q_gain=q_gain)
    _, _, out, plan = run_fused(b)
    assert plan.info()["num_prefill_tiles"] == 0  # every row on the decode kernel
    tok, want = oracle_subset(b, range(lay.num_seqs))
    assert_parity(gpu_rows(out, tok), want, f"spec case {case} q_gain={q_gain} plan={plan.info()}")
    check_against_two_calls(b)


@pytest.mark.parametrize("case", range(len(PREFILL)))
@pytest.mark.parametrize("q_gain", [1.0, 8.0])
def test_fused_prefill_shapes_against_oracle(cuda_lib, case, q_gain):
    # the prefill shapes through the fused call: with the two-SM kernel, key
    # tiles of only the step's own tokens come straight from the K/V input
    # (ragged last tiles included), chunks stage their earlier keys, and a
    # plan with nothing left to stage starts the prefill kernel behind the
    # scatter; every row against the oracle, and bit for bit the two calls
    q_lens, seq_lens, Hq, Hkv, D = PREFILL[case]
    nb = sum(-(-s // 16) for s in seq_lens) + 64
    lay = W.custom_layout(q_lens, seq_lens, Hq, Hkv, D, nb, seed=200 + case)
    b = W.make_batch(lay, device="cuda", q_gain=q_gain)
    _, _, out, plan = run_fused(b)
    tok, want = oracle_subset(b, range(lay.num_seqs))
    assert_parity(gpu_rows(out, tok), want, f"fused prefill case {case} q_gain={q_gain} plan={plan.info()}")
    check_against_two_calls(b)


def test_fused_side_by_side_fresh_prompts(cuda_lib):
    # decodes beside fresh prompts: the scatter, then the pair kernel by
    # programmatic launch (nothing to stage), then the decode kernel behind
    # it on the other SMs, each waiting for its predecessor only at its end
    q = [1] * 300 + [1024, 512]
    s = [2000] * 300 + [1024, 512]
    nb = sum(-(-x // 16) for x in s) + 64
    lay = W.custom_layout(q, s, 12, 2, 128, nb, seed=501)
    b = W.make_batch(lay, device="cuda", q_gain=8.0)
    _, _, out, plan = run_fused(b)
    info = plan.info()
    assert info["overlap_sms"] > 0 and info["prefill_pair"] == 1 and info["num_decode_units"] > 0
    check_against_two_calls(b)
    seqs = [0, 1, 150, 299, 300, 301]
    tok, want = oracle_subset(b, seqs)
    assert_parity(gpu_rows(out, tok), want, f"fused side by side, plan={info}")


@pytest.mark.parametrize("name", ["decode_tinyllama_b64", "prefix_llama3_70b_b128"])
def test_fused_consecutive_calls_and_side_stream(cuda_lib, name):
    # the same step three times on one plan and workspace (merge tickets
    # reset, each call's kernels ordered after the previous call's: with the
    # shared prefix, the scatter queued behind the side-by-side kernels and
    # the programmatic merge launch), on a stream of its own
    b = W.make_batch(W.layout(name), device="cuda")
    _, _, ref, _ = run_step(b)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        _, _, out, _ = run_fused(b, stream=s, repeats=3)
    assert same_bits(out, ref)


def test_fused_without_host_tables(cuda_lib):
    # no shared-prefix detection: the prefix workload runs as plain decode
    check_against_two_calls(W.make_batch(W.layout("prefix_llama3_70b_b128"), device="cuda"), with_tables=False)


@pytest.mark.parametrize("name", ["tiny_mixed", "decode_tinyllama_b64", "prefix_llama3_70b_b128",
                                  "mixed_qwen25_1p5b_t8192", "prefill_qwen25_1p5b_4x2048"])
def test_fused_step_captured_in_a_cuda_graph(cuda_lib, name):
    # the step (scatter + attention, one call) captured once and replayed:
    # decode only, shared prefix beside the suffix decode (merge kernel) and
    # the side-by-side mixed step (a second stream joins the capture)
    b = W.make_batch(W.layout(name), device="cuda")
    kc_ref, vc_ref, ref, _ = run_step(b)
    lay = b.layout
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    bt, cu, sl, slots = b.device_ints("cuda")
    plan = pa.Plan(lay.cu_seqlens_q, lay.seq_lens, dims_for(lay), block_tables=lay.block_tables)
    ws = pa.workspace_for(plan)
    out = torch.empty_like(b.q)

    def step():
        pa.reshape_and_attention(b.k, b.v, slots, b.q, kc, vc, bt, cu, sl, b.scale, out, plan, ws)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # warm-up outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    out.fill_(float("nan"))
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert pa.workspace_status(ws) == 0
    assert same_bits(kc, kc_ref) and same_bits(vc, vc_ref)
    assert same_bits(out, ref)
    del g
