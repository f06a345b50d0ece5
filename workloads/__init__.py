"""Seeded synthetic inputs for the paged-KV attention step.

This module serves both sides (the CUDA path and the CPU oracle) and holds
none of the attention arithmetic: it only draws lengths, block tables and
random tensors, and lays them out in the input format the op consumes.

Input format (the op's contract, not computed by either side):
  q            [T, Hq, D]   bf16   queries of all scheduled tokens, flat
  k, v         [T, Hkv, D]  bf16   K/V of the scheduled tokens (to be cached)
  k/v_cache    [NB, 16, Hkv, D] bf16  the paged pool
  block_tables [S, MB] int32  physical block of each logical block
  cu_seqlens_q [S+1] int32    segment boundaries in the flat token stream
  seq_lens     [S] int32      tokens of each request after this step
  slot_mapping [T] int64      pool row of each scheduled token

The scheduler side assigns a scheduled token at logical position p of request
i to pool row ``block_tables[i][p // 16] * 16 + p % 16`` (the slot); this
module forms the slot mapping that way, as "vLLM 学习笔记 01" §1.6 describes
the model runner doing, so that both sides receive the same inputs.

Pool contents: every slot a request reads as history gets N(0,1); every
other slot (the tail of a request's last block, the slots the scheduled
tokens will be written to, and every unallocated block) holds NaN, so that
reading anything the method must not read shows up in the output.  Block
table padding points at an unallocated (NaN) block rather than at an
out-of-range id, so that a kernel that wrongly reads it produces NaN instead
of an invalid address.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

BLOCK_SIZE = 16


@dataclass
class Layout:
    """Integer structure of one batch (host numpy arrays)."""
    name: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    num_blocks: int
    q_lens: np.ndarray          # int32 [S]
    seq_lens: np.ndarray        # int32 [S]
    block_tables: np.ndarray    # int32 [S, MB]
    poison_block: int           # an unallocated block id (NaN-filled)
    shared_prefix_blocks: int = 0
    block_size: int = BLOCK_SIZE
    seed: int = 0
    description: str = ""

    @property
    def num_seqs(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def cu_seqlens_q(self) -> np.ndarray:
        cu = np.zeros(self.num_seqs + 1, dtype=np.int32)
        np.cumsum(self.q_lens, out=cu[1:])
        return cu

    @property
    def num_tokens(self) -> int:
        return int(self.q_lens.sum())

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def slot_mapping(self) -> np.ndarray:
        """Pool row of each scheduled token (int64 [T])."""
        out = np.empty(self.num_tokens, dtype=np.int64)
        cu = self.cu_seqlens_q
        for i in range(self.num_seqs):
            n, L = int(self.seq_lens[i]), int(self.q_lens[i])
            pos = np.arange(n - L, n, dtype=np.int64)
            out[cu[i]:cu[i + 1]] = (self.block_tables[i, pos // self.block_size].astype(np.int64)
                                    * self.block_size + pos % self.block_size)
        return out

    def used_blocks(self) -> np.ndarray:
        """Sorted distinct physical block ids that requests own."""
        ids = [self.block_tables[i, :_cdiv(int(n), self.block_size)]
               for i, n in enumerate(self.seq_lens)]
        return np.unique(np.concatenate(ids)) if ids else np.zeros(0, np.int32)

    def history_mask_rows(self):
        """Pool rows that must hold NaN among allocated blocks: tail slots past
        seq_len and the slots the scheduled tokens are written to."""
        rows = []
        for i in range(self.num_seqs):
            n, L = int(self.seq_lens[i]), int(self.q_lens[i])
            nb = _cdiv(n, self.block_size)
            blocks = self.block_tables[i, :nb].astype(np.int64)
            pos = np.arange(n - L, nb * self.block_size, dtype=np.int64)
            rows.append(blocks[pos // self.block_size] * self.block_size + pos % self.block_size)
        return np.concatenate(rows) if rows else np.zeros(0, np.int64)

    def kv_bytes_read(self) -> int:
        """Distinct K+V bytes the step must read: every cached position of
        every request once (shared blocks counted once)."""
        per_tok = 2 * self.num_kv_heads * self.head_dim * 2
        if self.shared_prefix_blocks:
            shared = self.shared_prefix_blocks * self.block_size
            return per_tok * (shared + int((self.seq_lens.astype(np.int64) - shared).sum()))
        return per_tok * int(self.seq_lens.astype(np.int64).sum())

    def kv_bytes_logical(self) -> int:
        """K+V bytes summed per request (shared blocks counted per reader)."""
        return 2 * self.num_kv_heads * self.head_dim * 2 * int(self.seq_lens.astype(np.int64).sum())


def _cdiv(a: int, b: int) -> int:
    return -(-a // b)


def _tables(rng, seq_lens, num_blocks, shared_prefix_blocks=0):
    """Allocate blocks as consecutive runs of a seeded permutation of the pool.
    With shared_prefix_blocks > 0, the first run is shared by every request."""
    perm = rng.permutation(num_blocks).astype(np.int32)
    nbs = [_cdiv(int(n), BLOCK_SIZE) for n in seq_lens]
    mb = max(nbs) if nbs else 0
    used = shared_prefix_blocks + sum(nb - shared_prefix_blocks for nb in nbs)
    if used >= num_blocks:
        raise ValueError(f"pool of {num_blocks} blocks cannot hold {used} blocks plus a poison block")
    poison = int(perm[-1])
    bt = np.full((len(nbs), max(mb, 1)), poison, dtype=np.int32)
    cur = shared_prefix_blocks
    for i, nb in enumerate(nbs):
        if shared_prefix_blocks:
            bt[i, :shared_prefix_blocks] = perm[:shared_prefix_blocks]
        own = nb - shared_prefix_blocks
        bt[i, shared_prefix_blocks:nb] = perm[cur:cur + own]
        cur += own
    return bt, poison


def custom_layout(q_lens, seq_lens, num_q_heads, num_kv_heads, head_dim, num_blocks,
                  seed=0, name="custom", shared_prefix_blocks=0) -> Layout:
    q_lens = np.asarray(q_lens, dtype=np.int32)
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    if np.any(q_lens > seq_lens) or np.any(q_lens < 0):
        raise ValueError("need 0 <= q_len <= seq_len")
    rng = np.random.default_rng(seed)
    bt, poison = _tables(rng, seq_lens, num_blocks, shared_prefix_blocks)
    return Layout(name, num_q_heads, num_kv_heads, head_dim, num_blocks, q_lens,
                  seq_lens, bt, poison, shared_prefix_blocks, seed=seed)


# ---------------------------------------------------------------------------
# The five workloads.  Model names only give attention shapes; no weights.
# ---------------------------------------------------------------------------

def _tiny_mixed(seed):
    # Two decodes and one 6-token fresh prefill in one unpadded batch, the mix
    # "vLLM 学习笔记 01" §1.6 gives as its example.  Context lengths 17/40/6
    # count the scheduled tokens (computed-vs-total view, §1.4).
    return custom_layout([1, 1, 6], [17, 40, 6], 4, 2, 64, 64, seed, "tiny_mixed")


def _decode_tinyllama(seed):
    rng = np.random.default_rng(seed)
    seq = rng.integers(128, 2048, size=64, endpoint=True).astype(np.int32)
    lay = custom_layout(np.ones(64, np.int32), seq, 32, 4, 64, 16384, seed + 1,
                        "decode_tinyllama_b64")
    return lay


def _decode_llama3_8b(seed):
    rng = np.random.default_rng(seed)
    seq = np.floor(np.exp(rng.uniform(math.log(512), math.log(8192), size=256)))
    seq = np.clip(seq, 512, 8192).astype(np.int32)
    return custom_layout(np.ones(256, np.int32), seq, 32, 8, 128, 160000, seed + 1,
                         "decode_llama3_8b_b256")


def _mixed_qwen25(seed):
    rng = np.random.default_rng(seed)
    dec = rng.integers(1024, 4096, size=1152, endpoint=True).astype(np.int32)
    # decodes first, then the prefill chunk (2048 new on 6144 cached), then
    # three fresh prompts: 8192 scheduled tokens in all.
    q_lens = np.concatenate([np.ones(1152, np.int32), [2048, 1024, 1536, 2432]]).astype(np.int32)
    seq = np.concatenate([dec, [8192, 1024, 1536, 2432]]).astype(np.int32)
    return custom_layout(q_lens, seq, 12, 2, 128, 300000, seed + 1, "mixed_qwen25_1p5b_t8192")


def _prefix_llama3_70b(seed):
    rng = np.random.default_rng(seed)
    suffix = rng.integers(256, 1024, size=128, endpoint=True).astype(np.int32)
    seq = (4096 + suffix).astype(np.int32)
    return custom_layout(np.ones(128, np.int32), seq, 64, 8, 128, 16384, seed + 1,
                         "prefix_llama3_70b_b128", shared_prefix_blocks=256)


def _prefill_qwen25(seed):
    # the mixed step's prefill side alone, at a size a profiler captures in
    # seconds: four fresh 2048-token prompts with the Qwen2.5-1.5B head shape
    return custom_layout(np.full(4, 2048, np.int32), np.full(4, 2048, np.int32), 12, 2, 128,
                         4 * 128 + 16, seed + 1, "prefill_qwen25_1p5b_4x2048")


WORKLOADS = {
    "tiny_mixed": (_tiny_mixed, 1001,
                   "3 requests, seq 17/40/6, q 1/1/6; Hq 4, Hkv 2, D 64; pool 64 blocks"),
    "decode_tinyllama_b64": (_decode_tinyllama, 1002,
                             "64 decodes, seq U[128,2048]; Hq 32, Hkv 4, D 64; pool 16384 blocks"),
    "decode_llama3_8b_b256": (_decode_llama3_8b, 1003,
                              "256 decodes, seq log-U[512,8192]; Hq 32, Hkv 8, D 128; pool 160000 blocks"),
    "mixed_qwen25_1p5b_t8192": (_mixed_qwen25, 1004,
                                "8192-token step: 1152 decodes seq U[1024,4096], chunk 2048 on 6144, "
                                "fresh 1024/1536/2432; Hq 12, Hkv 2, D 128; pool 300000 blocks"),
    "prefix_llama3_70b_b128": (_prefix_llama3_70b, 1005,
                               "128 decodes sharing a 4096-token prefix (256 blocks) + suffix "
                               "U[256,1024]; Hq 64, Hkv 8, D 128; pool 16384 blocks"),
    "prefill_qwen25_1p5b_4x2048": (_prefill_qwen25, 1006,
                                   "4 fresh 2048-token prompts; Hq 12, Hkv 2, D 128; pool 528 blocks"),
}


def layout(name: str, seed: int | None = None) -> Layout:
    fn, default_seed, desc = WORKLOADS[name]
    lay = fn(default_seed if seed is None else seed)
    lay.description = desc
    return lay


@dataclass
class Batch:
    layout: Layout
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    k_cache: torch.Tensor      # pool before the scheduled tokens are written
    v_cache: torch.Tensor
    scale: float
    extra: dict = field(default_factory=dict)

    def device_ints(self, device):
        """block_tables, cu_seqlens_q, seq_lens, slot_mapping as device tensors."""
        L = self.layout
        return (torch.from_numpy(L.block_tables).to(device),
                torch.from_numpy(L.cu_seqlens_q).to(device),
                torch.from_numpy(L.seq_lens).to(device),
                torch.from_numpy(L.slot_mapping).to(device))


def make_batch(lay: Layout, device="cpu", seed: int | None = None,
               q_gain: float = 1.0) -> Batch:
    """Draw q, k, v and the pool contents for a layout.

    q, k, v and history slots ~ N(0,1) (q multiplied by q_gain: >1 gives the
    peaked variant whose softmax concentrates on few keys).  Drawn with a
    seeded torch.Generator on ``device``.
    """
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(lay.seed * 7 + 11 if seed is None else seed)
    T, Hq, Hkv, D = lay.num_tokens, lay.num_q_heads, lay.num_kv_heads, lay.head_dim
    bf = torch.bfloat16

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=torch.float32).to(bf)

    q = randn(T, Hq, D)
    if q_gain != 1.0:
        q = (q.float() * q_gain).to(bf)
    k = randn(T, Hkv, D)
    v = randn(T, Hkv, D)
    caches = []
    used = torch.from_numpy(lay.used_blocks().astype(np.int64)).to(dev)
    nan_rows = torch.from_numpy(lay.history_mask_rows()).to(dev)
    for _ in range(2):
        c = torch.full((lay.num_blocks, lay.block_size, Hkv, D), float("nan"), dtype=bf, device=dev)
        # fill block by block group to bound the float32 temporary
        step = max(1, (1 << 27) // (lay.block_size * Hkv * D))
        for s in range(0, used.numel(), step):
            ids = used[s:s + step]
            c[ids] = randn(ids.numel(), lay.block_size, Hkv, D)
        if nan_rows.numel():
            c.view(-1, Hkv, D)[nan_rows] = float("nan")
        caches.append(c)
    return Batch(lay, q, k, v, caches[0], caches[1], 1.0 / math.sqrt(D))


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Host uint16 bit patterns of a bf16 tensor (copies to the host)."""
    if t.dtype != torch.bfloat16:
        raise TypeError("expected bf16")
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


@dataclass
class HostSubset:
    """A subset of a batch's requests, moved to the host with a compacted pool.

    Only the blocks the chosen requests own are copied; block tables and slots
    are renumbered into the compact pool.  Data movement only."""
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    k_cache: np.ndarray
    v_cache: np.ndarray
    block_tables: np.ndarray
    cu_seqlens_q: np.ndarray
    seq_lens: np.ndarray
    slot_mapping: np.ndarray
    token_index: np.ndarray     # flat token ids of the subset in the full batch
    seq_index: np.ndarray


def host_subset(batch: Batch, seq_ids) -> HostSubset:
    L = batch.layout
    seq_ids = np.asarray(sorted(set(int(s) for s in seq_ids)), dtype=np.int64)
    cu = L.cu_seqlens_q
    nbs = [_cdiv(int(L.seq_lens[i]), L.block_size) for i in seq_ids]
    owned = np.concatenate([L.block_tables[i, :nb] for i, nb in zip(seq_ids, nbs)]) \
        if len(seq_ids) else np.zeros(0, np.int32)
    uniq, inv = np.unique(owned, return_inverse=True)
    poison = len(uniq)          # one extra NaN block for table padding
    mb = max(nbs) if nbs else 1
    bt = np.full((len(seq_ids), max(mb, 1)), poison, dtype=np.int32)
    o = 0
    for r, nb in enumerate(nbs):
        bt[r, :nb] = inv[o:o + nb]
        o += nb
    dev = batch.k_cache.device
    ids = torch.from_numpy(np.append(uniq.astype(np.int64), L.poison_block)).to(dev)
    kc = bf16_bits(batch.k_cache[ids])
    vc = bf16_bits(batch.v_cache[ids])
    tok = np.concatenate([np.arange(cu[i], cu[i + 1]) for i in seq_ids]) \
        if len(seq_ids) else np.zeros(0, np.int64)
    tok = tok.astype(np.int64)
    remap = {int(b): j for j, b in enumerate(uniq)}
    slots_full = L.slot_mapping[tok]
    slots = np.array([remap[int(s) // L.block_size] * L.block_size + int(s) % L.block_size
                      for s in slots_full], dtype=np.int64)
    q_lens = L.q_lens[seq_ids]
    cu_s = np.zeros(len(seq_ids) + 1, dtype=np.int32)
    np.cumsum(q_lens, out=cu_s[1:])
    tok_t = torch.from_numpy(tok).to(batch.q.device)
    return HostSubset(bf16_bits(batch.q[tok_t]), bf16_bits(batch.k[tok_t]), bf16_bits(batch.v[tok_t]),
                      kc, vc, bt, cu_s, L.seq_lens[seq_ids].astype(np.int32), slots, tok, seq_ids)
