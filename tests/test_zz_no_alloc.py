"""pa_attention_varlen_noalloc checked against pa_attention_varlen (GPU).

Some callers cannot allocate device memory: an engine that gave nearly all of
the GPU to its KV pool at start-up and keeps no allocator in its step loop, a
host or plugin interface that hands an op only its inputs, outputs and a
stream, or a loop that must not stall on a cudaMalloc/cudaFree pair.  For them
the library offers an attention entry point whose scratch is a fixed array in
the library's own device memory.  These tests call it through the C ABI and
compare its output with the workspace-taking entry point's, on consecutive
calls that share that array.

The file is named so that pytest collects it last: a run that stops at the
first failure has then already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_attention_token_b200 as pa
import workloads as W
from tests.parity import assert_parity

pytestmark = pytest.mark.gpu


def _dims(lay):
    return pa.Dims(lay.num_tokens, lay.num_seqs, lay.num_q_heads, lay.num_kv_heads,
                   lay.head_dim, lay.num_blocks, lay.max_blocks_per_seq, 16)


def _prepare(name, q_gain=1.0, host_tables=False):
    lay = W.layout(name)
    b = W.make_batch(lay, device="cuda", q_gain=q_gain)
    kc, vc = b.k_cache.clone(), b.v_cache.clone()
    bt, cu, sl, slots = b.device_ints("cuda")
    pa.reshape_and_cache(b.k, b.v, slots, kc, vc)
    plan = pa.Plan(lay.cu_seqlens_q, lay.seq_lens, _dims(lay),
                   block_tables=lay.block_tables if host_tables else None)
    ws = pa.workspace_for(plan)
    ref = torch.full_like(b.q, float("nan"))
    pa.attention_varlen(b.q, kc, vc, bt, cu, sl, b.scale, ref, plan, ws)
    return b, kc, vc, bt, cu, sl, plan, ref


def _call_noalloc(lib, b, kc, vc, bt, cu, sl, plan, out):
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return lib.pa_attention_varlen_noalloc(
        p(b.q), p(kc), p(vc), p(bt), p(cu), p(sl), ctypes.c_float(b.scale), p(out),
        ctypes.byref(plan.dims), plan.handle, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(cuda_lib):
    lib = pa.load_library()
    # the split-KV decode kernel; the two-head prefill kernel (head_dim 64);
    # the pair kernel on staged prompts; the pair kernel on a shared prefix
    # read from the paged cache, beside the decode kernel (partials, merges)
    cases = [_prepare("decode_tinyllama_b64"), _prepare("tiny_mixed", q_gain=8.0),
             _prepare("prefill_qwen25_1p5b_4x2048"), _prepare("prefix_llama3_70b_b128", host_tables=True)]
    assert cases[2][6].info()["prefill_pair"] == 1 and cases[3][6].info()["num_prefix_groups"] == 1
    # two calls in a row per case, alternating cases, so each call starts from
    # the array contents the previous (different) call left behind
    for rnd in range(2):
        for b, kc, vc, bt, cu, sl, plan, ref in cases:
            out = torch.full_like(b.q, float("nan"))
            st = _call_noalloc(lib, b, kc, vc, bt, cu, sl, plan, out)
            assert st == pa.PA_OK, pa.status_string(st)
            torch.cuda.synchronize()
            assert_parity(out.float().cpu().numpy(), ref.float().cpu().numpy().astype(np.float64),
                          f"no-alloc call {rnd} ({b.layout.name})")
    # the array's status word: no bounded wait ran out in any of the calls;
    # reading it with clear leaves it zero
    st = ctypes.c_uint32(7)
    assert lib.pa_noalloc_status(ctypes.byref(st), 1, None) == pa.PA_OK
    assert st.value == 0
    assert pa.noalloc_status() == 0


def test_noalloc_rejects_plans_beyond_its_array(cuda_lib):
    lib = pa.load_library()
    cap = int(lib.pa_noalloc_scratch_bytes())
    # one 8192-token prompt with 8 kv heads of 128 dims and an odd group (3
    # query heads per kv head: the two-head kernel, which reads staged K/V)
    # stages 64 key tiles of K and V per kv head in the scratch: 32 MiB
    S, n = 1, 8192
    cu = np.array([0, n], dtype=np.int32)
    sl = np.array([n], dtype=np.int32)
    d = pa.Dims(n, S, 24, 8, 128, 1024, n // 16, 16)
    plan = pa.Plan(cu, sl, d)
    assert plan.workspace_bytes > cap
    fake = ctypes.c_void_p(0x10000)         # never used: the call is rejected first
    st = lib.pa_attention_varlen_noalloc(fake, fake, fake, fake, fake, fake, ctypes.c_float(0.1),
                                         fake, ctypes.byref(d), plan.handle, None)
    assert st == pa.PA_ERR_TOO_LARGE
    assert "16 MiB" in pa.status_string(st)
