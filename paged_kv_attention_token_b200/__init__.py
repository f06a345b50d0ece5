"""Python binding of libpa.so, the paged-KV attention step for B200 (sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/pa.h.  There is no CPU or
PyTorch fallback; if the library is missing or cannot be loaded, every call
raises.  PyTorch supplies device memory and streams.

    import paged_kv_attention_token_b200 as pa
    pa.reshape_and_cache(k, v, slot_mapping, k_cache, v_cache)
    plan = pa.Plan(cu_seqlens_q_host, seq_lens_host, pa.dims_of(q, k_cache, block_tables, seq_lens))
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    pa.attention_varlen(q, k_cache, v_cache, block_tables, cu_seqlens_q, seq_lens,
                        scale, out, plan, ws)
"""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np
import torch

__all__ = ["load_library", "library_path", "PaError", "Dims", "dims_of", "Plan",
           "reshape_and_cache", "attention_varlen", "validate_inputs", "status_string", "Trace",
           "workspace_for",
           "PA_OK", "PA_ERR_NULL", "PA_ERR_SHAPE", "PA_ERR_DTYPE", "PA_ERR_ALIGN",
           "PA_ERR_UNSUPPORTED", "PA_ERR_WORKSPACE", "PA_ERR_BOUNDS", "PA_ERR_CUDA", "PA_ERR_PLAN",
           "PA_ERR_TOO_LARGE", "attention_varlen_noalloc", "noalloc_scratch_bytes", "noalloc_status",
           "workspace_status", "workspace_reset", "selftest_wait_timeout"]

PA_OK, PA_ERR_NULL, PA_ERR_SHAPE, PA_ERR_DTYPE, PA_ERR_ALIGN = 0, -1, -2, -3, -4
PA_ERR_UNSUPPORTED, PA_ERR_WORKSPACE, PA_ERR_BOUNDS, PA_ERR_CUDA, PA_ERR_PLAN = -5, -6, -7, -8, -9
PA_ERR_TOO_LARGE = -10

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libpa.so")
_lock = threading.Lock()
_lib = None


def library_path() -> str:
    return _LIB_PATH


class PaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = status_string(status) if _lib is not None else str(status)
        super().__init__(f"{what}: {msg} (status {status})" if what else f"{msg} (status {status})")


class Dims(ctypes.Structure):
    _fields_ = [("num_tokens", ctypes.c_int32), ("num_seqs", ctypes.c_int32),
                ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
                ("max_blocks_per_seq", ctypes.c_int32), ("block_size", ctypes.c_int32)]

    def __repr__(self):
        return "Dims(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


class PlanInfo(ctypes.Structure):
    _fields_ = [("num_sms", ctypes.c_int32), ("num_decode_rows", ctypes.c_int32),
                ("num_decode_units", ctypes.c_int32), ("num_partials", ctypes.c_int32),
                ("num_combine_rows", ctypes.c_int32), ("num_prefill_tiles", ctypes.c_int32),
                ("decode_kv_blocks", ctypes.c_int64), ("prefill_causal_pairs", ctypes.c_int64),
                ("table_bytes", ctypes.c_uint64), ("workspace_bytes", ctypes.c_uint64),
                ("num_staged_kv_tiles", ctypes.c_int32), ("num_prefill_ctas", ctypes.c_int32),
                ("num_prefix_groups", ctypes.c_int32), ("attention_launches", ctypes.c_int32),
                ("decode_kv_keys", ctypes.c_int64), ("prefill_pair", ctypes.c_int32),
                ("overlap_sms", ctypes.c_int32)]

    def as_dict(self):
        return {n: int(getattr(self, n)) for n, _ in self._fields_}


def load_library():
    """Load libpa.so (once).  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"CUDA library {_LIB_PATH} is missing: build it with "
                               "`python -m paged_kv_attention_token_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        P, I, SZ, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
        DP = ctypes.POINTER(Dims)
        sig = {
            "pa_reshape_and_cache": (I, [P, P, P, P, P, DP, P]),
            "pa_plan_build": (I, [P, P, P, DP, I, ctypes.POINTER(P)]),
            "pa_plan_get_info": (I, [P, ctypes.POINTER(PlanInfo)]),
            "pa_plan_workspace_bytes": (SZ, [P]),
            "pa_plan_destroy": (None, [P]),
            "pa_attention_varlen": (I, [P, P, P, P, P, P, F, P, DP, P, P, SZ, P]),
            "pa_attention_varlen_ex": (I, [P, P, P, P, P, P, F, P, DP, P, P, SZ, P, P]),
            "pa_attention_varlen_noalloc": (I, [P, P, P, P, P, P, F, P, DP, P, P]),
            "pa_reshape_and_attention": (I, [P, P, P, P, P, P, P, P, P, F, P, DP, P, P, SZ, P]),
            "pa_kv_export": (I, [P, P, P, P, P, P, DP, P]),
            "pa_kv_import": (I, [P, P, P, P, P, P, DP, P]),
            "pa_noalloc_scratch_bytes": (SZ, []),
            "pa_workspace_status": (I, [P, P, ctypes.POINTER(ctypes.c_uint32)]),
            "pa_workspace_reset": (I, [P, P, P]),
            "pa_noalloc_status": (I, [ctypes.POINTER(ctypes.c_uint32), I, P]),
            "pa_selftest_wait_timeout": (I, [P, ctypes.c_longlong, P]),
            "pa_validate_scratch_bytes": (SZ, [DP]),
            "pa_validate_inputs": (I, [P, P, P, P, DP, P, SZ, P]),
            "pa_status_string": (ctypes.c_char_p, [I]),
            "pa_version": (ctypes.c_char_p, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def status_string(status: int) -> str:
    return load_library().pa_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != PA_OK:
        raise PaError(status, what)


def _dev_ptr(t: torch.Tensor | None, name: str, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise PaError(PA_ERR_SHAPE, f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise PaError(PA_ERR_DTYPE, f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise PaError(PA_ERR_SHAPE, f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def dims_of(q: torch.Tensor, k_cache: torch.Tensor, block_tables: torch.Tensor,
            seq_lens) -> Dims:
    """Dims of a call from the tensors' shapes (q [T,Hq,D], cache [NB,16,Hkv,D],
    block_tables [S,MB])."""
    T, Hq, D = q.shape
    NB, B, Hkv, D2 = k_cache.shape
    if D2 != D:
        raise PaError(PA_ERR_SHAPE, "q and cache head_dim differ")
    S = len(seq_lens)
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    return Dims(T, S, Hq, Hkv, D, NB, MB, B)


def reshape_and_cache(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor,
                      k_cache: torch.Tensor, v_cache: torch.Tensor, stream=None) -> None:
    """Write k[t], v[t] into the caches at slot_mapping[t] (pa_reshape_and_cache)."""
    lib = load_library()
    T, Hkv, D = k.shape
    if v.shape != k.shape or k_cache.shape != v_cache.shape or tuple(k_cache.shape[2:]) != (Hkv, D):
        raise PaError(PA_ERR_SHAPE, "reshape_and_cache shapes")
    if slot_mapping.shape != (T,):
        raise PaError(PA_ERR_SHAPE, "slot_mapping must be [T]")
    d = Dims(T, 0, Hkv, Hkv, D, k_cache.shape[0], 0, k_cache.shape[1])
    bf = torch.bfloat16
    _check(lib.pa_reshape_and_cache(_dev_ptr(k, "k", bf), _dev_ptr(v, "v", bf),
                                    _dev_ptr(slot_mapping, "slot_mapping", torch.int64),
                                    _dev_ptr(k_cache, "k_cache", bf), _dev_ptr(v_cache, "v_cache", bf),
                                    ctypes.byref(d), _stream_ptr(stream)), "pa_reshape_and_cache")


def _host_i32(a, name):
    if isinstance(a, torch.Tensor):
        if a.is_cuda:
            raise PaError(PA_ERR_SHAPE, f"{name} must be a host array for planning")
        a = a.numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


class Plan:
    """Work partition for one step (pa_plan_build); reusable for every layer.

    The plan must stay alive until the GPU work queued with it has completed
    (like every other input).  ``rebuild`` re-partitions for the next step in
    place, reusing the plan's buffers.  With host ``block_tables`` ([S][MB]
    int32, the values of the device array), runs of decodes that share
    their leading blocks are attended to them once (cascade)."""

    def __init__(self, cu_seqlens_q, seq_lens, dims: Dims, device: int | None = None, block_tables=None):
        lib = load_library()
        self._lib = lib
        if device is None:
            device = torch.cuda.current_device() if torch.cuda.is_available() else -1
        self.device = int(device)
        self._h = ctypes.c_void_p()
        self.rebuild(cu_seqlens_q, seq_lens, dims, block_tables)

    def rebuild(self, cu_seqlens_q, seq_lens, dims: Dims, block_tables=None):
        self._cu = _host_i32(cu_seqlens_q, "cu_seqlens_q")
        self._sl = _host_i32(seq_lens, "seq_lens")
        self._bt = None if block_tables is None else _host_i32(block_tables, "block_tables")
        self.dims = Dims(*[getattr(dims, n) for n, _ in Dims._fields_])
        if self._bt is not None and (self._bt.ndim != 2 or self._bt.shape[0] != self.dims.num_seqs
                                     or self._bt.shape[1] != self.dims.max_blocks_per_seq):
            raise ValueError(f"block_tables must be [{self.dims.num_seqs}][{self.dims.max_blocks_per_seq}]")
        bt_ptr = None if self._bt is None else self._bt.ctypes.data
        _check(self._lib.pa_plan_build(self._cu.ctypes.data, self._sl.ctypes.data, bt_ptr,
                                       ctypes.byref(self.dims), self.device, ctypes.byref(self._h)),
               "pa_plan_build")
        return self

    @property
    def handle(self):
        return self._h

    @property
    def workspace_bytes(self) -> int:
        return int(self._lib.pa_plan_workspace_bytes(self._h))

    def info(self) -> dict:
        inf = PlanInfo()
        _check(self._lib.pa_plan_get_info(self._h, ctypes.byref(inf)), "pa_plan_get_info")
        return inf.as_dict()

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            self._lib.pa_plan_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def workspace_for(plan: Plan, device=None) -> torch.Tensor:
    """A zero-filled device workspace of the size a plan needs (256-byte
    aligned by torch)."""
    return torch.zeros(max(plan.workspace_bytes, 1), dtype=torch.uint8,
                       device=device if device is not None else "cuda")


class Trace(ctypes.Structure):
    """Events recorded around the kernels of one attention call (pa_trace)."""
    _fields_ = [("events", ctypes.c_void_p * 6)]

    # "staging" is the K/V staging kernel when the call runs its kernels one
    # after the other (no decode kernel beside the prefill kernel)
    MARKS = {"plan_wait": (0, 1), "decode": (1, 2), "combine": (2, 3), "staging": (3, 4), "prefill": (4, 5)}

    def __init__(self, stages=("plan_wait", "decode", "combine", "prefill")):
        """Record only the marks the named stages need (each record costs a
        couple of microseconds of GPU time)."""
        super().__init__()
        self.stages = tuple(stages)
        used = sorted({i for st in self.stages for i in self.MARKS[st]})
        self.torch_events = {i: torch.cuda.Event(enable_timing=True) for i in used}

    def arm(self, stream):
        # torch only reports elapsed times of events it has recorded itself;
        # record them once here, the library records them again at its marks
        # (the latest record on the stream sets an event's timestamp).
        # torch creates the CUDA event on its first record, so the handles
        # are taken only after that
        for i, e in self.torch_events.items():
            e.record(stream)
            self.events[i] = ctypes.c_void_p(e.cuda_event)

    def elapsed_ms(self) -> dict:
        """Per-stage times (ms) once the stream has reached the last event."""
        ev = self.torch_events
        return {st: ev[self.MARKS[st][0]].elapsed_time(ev[self.MARKS[st][1]]) for st in self.stages}


def attention_varlen(q, k_cache, v_cache, block_tables, cu_seqlens_q, seq_lens, scale,
                     out, plan: Plan, workspace: torch.Tensor, stream=None,
                     trace: "Trace | None" = None) -> torch.Tensor:
    """Varlen causal paged attention (pa_attention_varlen); writes and returns out.
    With ``trace``, CUDA events are recorded around each kernel."""
    lib = load_library()
    d = plan.dims
    bf = torch.bfloat16
    if tuple(q.shape) != (d.num_tokens, d.num_q_heads, d.head_dim) or out.shape != q.shape:
        raise PaError(PA_ERR_SHAPE, "q/out shape does not match the plan")
    if tuple(k_cache.shape) != (d.num_blocks, d.block_size, d.num_kv_heads, d.head_dim) or \
            v_cache.shape != k_cache.shape:
        raise PaError(PA_ERR_SHAPE, "cache shape does not match the plan")
    if tuple(block_tables.shape) != (d.num_seqs, d.max_blocks_per_seq):
        raise PaError(PA_ERR_SHAPE, "block_tables shape does not match the plan")
    if workspace.dtype != torch.uint8:
        raise PaError(PA_ERR_DTYPE, "workspace must be uint8")
    args = (_dev_ptr(q, "q", bf), _dev_ptr(k_cache, "k_cache", bf), _dev_ptr(v_cache, "v_cache", bf),
            _dev_ptr(block_tables, "block_tables", torch.int32),
            _dev_ptr(cu_seqlens_q, "cu_seqlens_q", torch.int32),
            _dev_ptr(seq_lens, "seq_lens", torch.int32),
            ctypes.c_float(scale), _dev_ptr(out, "out", bf), ctypes.byref(d), plan.handle,
            _dev_ptr(workspace, "workspace"), ctypes.c_size_t(workspace.numel()), _stream_ptr(stream))
    if trace is None:
        _check(lib.pa_attention_varlen(*args), "pa_attention_varlen")
    else:
        trace.arm(stream if stream is not None else torch.cuda.current_stream())
        _check(lib.pa_attention_varlen_ex(*args, ctypes.byref(trace)), "pa_attention_varlen_ex")
    return out


def reshape_and_attention(k, v, slot_mapping, q, k_cache, v_cache, block_tables, cu_seqlens_q, seq_lens,
                          scale, out, plan: Plan, workspace: torch.Tensor, stream=None) -> torch.Tensor:
    """A step's cache write and attention in one call (pa_reshape_and_attention):
    writes the caches like reshape_and_cache and out like attention_varlen."""
    lib = load_library()
    d = plan.dims
    bf = torch.bfloat16
    if tuple(q.shape) != (d.num_tokens, d.num_q_heads, d.head_dim) or out.shape != q.shape:
        raise PaError(PA_ERR_SHAPE, "q/out shape does not match the plan")
    if tuple(k.shape) != (d.num_tokens, d.num_kv_heads, d.head_dim) or v.shape != k.shape:
        raise PaError(PA_ERR_SHAPE, "k/v shape does not match the plan")
    if tuple(slot_mapping.shape) != (d.num_tokens,):
        raise PaError(PA_ERR_SHAPE, "slot_mapping must be [T]")
    if tuple(k_cache.shape) != (d.num_blocks, d.block_size, d.num_kv_heads, d.head_dim) or \
            v_cache.shape != k_cache.shape:
        raise PaError(PA_ERR_SHAPE, "cache shape does not match the plan")
    if tuple(block_tables.shape) != (d.num_seqs, d.max_blocks_per_seq):
        raise PaError(PA_ERR_SHAPE, "block_tables shape does not match the plan")
    if workspace.dtype != torch.uint8:
        raise PaError(PA_ERR_DTYPE, "workspace must be uint8")
    _check(lib.pa_reshape_and_attention(
        _dev_ptr(k, "k", bf), _dev_ptr(v, "v", bf), _dev_ptr(slot_mapping, "slot_mapping", torch.int64),
        _dev_ptr(q, "q", bf), _dev_ptr(k_cache, "k_cache", bf), _dev_ptr(v_cache, "v_cache", bf),
        _dev_ptr(block_tables, "block_tables", torch.int32), _dev_ptr(cu_seqlens_q, "cu_seqlens_q", torch.int32),
        _dev_ptr(seq_lens, "seq_lens", torch.int32), ctypes.c_float(scale), _dev_ptr(out, "out", bf),
        ctypes.byref(d), plan.handle, _dev_ptr(workspace, "workspace"), ctypes.c_size_t(workspace.numel()),
        _stream_ptr(stream)), "pa_reshape_and_attention")
    return out


def _kv_transfer(name, src_k, src_v, dst_k, dst_v, cache, buf, block_tables, cu_tokens, stream):
    lib = load_library()
    if buf.dim() != 3 or cache.dim() != 4 or tuple(cache.shape[2:]) != tuple(buf.shape[1:]):
        raise PaError(PA_ERR_SHAPE, f"{name}: cache [NB,16,Hkv,D] and buffers [N,Hkv,D] disagree")
    if block_tables.dim() != 2 or tuple(cu_tokens.shape) != (block_tables.shape[0] + 1,):
        raise PaError(PA_ERR_SHAPE, f"{name}: block_tables [S,MB] and cu_tokens [S+1]")
    N, Hkv, D = buf.shape
    d = Dims(N, block_tables.shape[0], Hkv, Hkv, D, cache.shape[0], block_tables.shape[1], cache.shape[1])
    bf = torch.bfloat16
    _check(getattr(lib, name)(_dev_ptr(src_k, "src_k", bf), _dev_ptr(src_v, "src_v", bf),
                              _dev_ptr(block_tables, "block_tables", torch.int32),
                              _dev_ptr(cu_tokens, "cu_tokens", torch.int32),
                              _dev_ptr(dst_k, "dst_k", bf), _dev_ptr(dst_v, "dst_v", bf),
                              ctypes.byref(d), _stream_ptr(stream)), name)


def kv_export(k_cache, v_cache, block_tables, cu_tokens, k_out, v_out, stream=None) -> None:
    """Gather requests' K/V from the paged caches into contiguous [N,Hkv,D]
    buffers (pa_kv_export)."""
    if k_out.shape != v_out.shape or k_cache.shape != v_cache.shape:
        raise PaError(PA_ERR_SHAPE, "pa_kv_export: k/v shapes differ")
    _kv_transfer("pa_kv_export", k_cache, v_cache, k_out, v_out, k_cache, k_out, block_tables, cu_tokens, stream)


def kv_import(k_in, v_in, block_tables, cu_tokens, k_cache, v_cache, stream=None) -> None:
    """Write contiguous [N,Hkv,D] K/V buffers into the paged caches through
    the block tables (pa_kv_import)."""
    if k_in.shape != v_in.shape or k_cache.shape != v_cache.shape:
        raise PaError(PA_ERR_SHAPE, "pa_kv_import: k/v shapes differ")
    _kv_transfer("pa_kv_import", k_in, v_in, k_cache, v_cache, k_cache, k_in, block_tables, cu_tokens, stream)


def workspace_status(workspace: torch.Tensor, stream=None) -> int:
    """Error bits the attention calls since the last reset left in a
    workspace (0 = none); waits for the stream."""
    st = ctypes.c_uint32(0)
    _check(load_library().pa_workspace_status(_dev_ptr(workspace, "workspace"), _stream_ptr(stream),
                                              ctypes.byref(st)), "pa_workspace_status")
    return int(st.value)


def workspace_reset(workspace: torch.Tensor, plan: "Plan", stream=None) -> None:
    """Zero a workspace's status word and merge tickets (after an error)."""
    _check(load_library().pa_workspace_reset(_dev_ptr(workspace, "workspace"), plan.handle, _stream_ptr(stream)),
           "pa_workspace_reset")


def noalloc_status(clear: bool = False, stream=None) -> int:
    """Error bits in the no-alloc array's status word on the current device
    (0 = none); with clear, zero the word afterwards.  Waits for the stream."""
    st = ctypes.c_uint32(0)
    _check(load_library().pa_noalloc_status(ctypes.byref(st), 1 if clear else 0, _stream_ptr(stream)),
           "pa_noalloc_status")
    return int(st.value)


def selftest_wait_timeout(workspace: torch.Tensor, limit_cycles: int, stream=None) -> None:
    """Queue the bounded-wait self-test: a kernel whose mbarrier wait runs out
    after limit_cycles sets bit 0 of the workspace's status word."""
    _check(load_library().pa_selftest_wait_timeout(_dev_ptr(workspace, "workspace"), int(limit_cycles),
                                                   _stream_ptr(stream)), "pa_selftest_wait_timeout")


def noalloc_scratch_bytes() -> int:
    """Size of the fixed device array pa_attention_varlen_noalloc uses."""
    return int(load_library().pa_noalloc_scratch_bytes())


def attention_varlen_noalloc(q, k_cache, v_cache, block_tables, cu_seqlens_q, seq_lens, scale,
                             out, plan: Plan, stream=None) -> torch.Tensor:
    """pa_attention_varlen_noalloc: the same attention with no caller workspace
    (the library's fixed device array serves as scratch; see include/pa.h for
    who needs this and the rules for concurrent calls)."""
    lib = load_library()
    d = plan.dims
    bf = torch.bfloat16
    if tuple(q.shape) != (d.num_tokens, d.num_q_heads, d.head_dim) or out.shape != q.shape:
        raise PaError(PA_ERR_SHAPE, "q/out shape does not match the plan")
    _check(lib.pa_attention_varlen_noalloc(
        _dev_ptr(q, "q", bf), _dev_ptr(k_cache, "k_cache", bf), _dev_ptr(v_cache, "v_cache", bf),
        _dev_ptr(block_tables, "block_tables", torch.int32),
        _dev_ptr(cu_seqlens_q, "cu_seqlens_q", torch.int32), _dev_ptr(seq_lens, "seq_lens", torch.int32),
        ctypes.c_float(scale), _dev_ptr(out, "out", bf), ctypes.byref(d), plan.handle,
        _stream_ptr(stream)), "pa_attention_varlen_noalloc")
    return out


def validate_inputs(slot_mapping, block_tables, cu_seqlens_q, seq_lens, dims: Dims,
                    stream=None) -> int:
    """Device check of the data-dependent preconditions; returns PA_OK or
    PA_ERR_BOUNDS (synchronizes the stream)."""
    lib = load_library()
    nbytes = int(lib.pa_validate_scratch_bytes(ctypes.byref(dims)))
    scratch = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=cu_seqlens_q.device)
    st = lib.pa_validate_inputs(_dev_ptr(slot_mapping, "slot_mapping", torch.int64),
                                _dev_ptr(block_tables, "block_tables", torch.int32),
                                _dev_ptr(cu_seqlens_q, "cu_seqlens_q", torch.int32),
                                _dev_ptr(seq_lens, "seq_lens", torch.int32), ctypes.byref(dims),
                                _dev_ptr(scratch, "scratch"), ctypes.c_size_t(nbytes),
                                _stream_ptr(stream))
    if st not in (PA_OK, PA_ERR_BOUNDS):
        _check(st, "pa_validate_inputs")
    return int(st)
