"""Seeded synthetic workloads for the paged decode path.

This module only draws inputs: context lengths, shuffled physical block ids,
query / key / value values and request traces.  It holds none of the method's
arithmetic (no attention, no slot addressing, no bookkeeping policy), so both
the CUDA path and the CPU oracle may use it without sharing any logic.

Storage convention: ``"f32"`` values are ``numpy.float32``; ``"f16"`` and
``"bf16"`` values are raw 16-bit patterns in ``numpy.uint16`` (rounded to
nearest-even from float32 by torch's CPU cast).

Workload shapes follow the pages' serving set-ups: Llama-2-7B-shaped heads
(32 query = 32 KV heads, head_dim 128), Llama-3-70B-shaped heads with grouped
KV (64 query / 8 KV heads), up to 256 concurrent sequences (max-num-seqs 256)
and long-tailed, power-law context lengths, 16-token blocks by default and
8-token blocks for the small-model trace.  No public dataset is read: these
draws stand in for the pages' serving traces.
"""

from dataclasses import dataclass, field
import math

import numpy as np

ELEMENT_BYTES = {"f32": 4, "f16": 2, "bf16": 2}


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    dtype: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    lengths: str                  # "fixed" | "uniform" | "zipf" | "const"
    fixed_lengths: tuple = ()
    len_lo: int = 0
    len_hi: int = 0
    zipf_a: float = 0.0
    num_blocks: int = 0           # 0: needed blocks + spare fraction
    spare: float = 0.25
    partition_size: int = 0       # 0: library default
    outlier_frac: float = 0.0     # fraction of K rows scaled by outlier_scale
    outlier_scale: float = 8.0

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.head_dim)


CONFIGS = {
    # 4 sequences, contexts {1,16,17,90}, MHA 4/4, D=64, 16-token blocks,
    # 32-block pool, fp32.
    "tiny": DecodeConfig("tiny", "f32", 4, 4, 4, 64, 16, "fixed",
                         fixed_lengths=(1, 16, 17, 90), num_blocks=32),
    # Llama-2-7B-shaped layer: 64 sequences, contexts uniform on [128, 2048].
    "7b": DecodeConfig("7b", "f16", 64, 32, 32, 128, 16, "uniform",
                       len_lo=128, len_hi=2048),
    # Llama-3-70B-shaped layer, GQA group 8: 256 sequences, contexts from a
    # truncated power law p(L) ~ L^-1.2 on [16, 8192].
    "70b": DecodeConfig("70b", "bf16", 256, 64, 8, 128, 16, "zipf",
                        len_lo=16, len_hi=8192, zipf_a=1.2),
    # Long-context split-K: 8 sequences of 32768 tokens, 512-token partitions,
    # 1% of K rows scaled by 8 to stress softmax stability.
    "long": DecodeConfig("long", "bf16", 8, 64, 8, 128, 16, "const",
                         len_lo=32768, len_hi=32768, partition_size=512,
                         outlier_frac=0.01),
}


def rng(seed):
    return np.random.default_rng(int(seed))


def context_lengths(cfg, r):
    """Draw the post-write context length of every sequence."""
    if cfg.lengths == "fixed":
        return np.array(cfg.fixed_lengths, dtype=np.int64)
    if cfg.lengths == "const":
        return np.full(cfg.num_seqs, cfg.len_lo, dtype=np.int64)
    if cfg.lengths == "uniform":
        return r.integers(cfg.len_lo, cfg.len_hi + 1, size=cfg.num_seqs).astype(np.int64)
    if cfg.lengths == "zipf":
        support = np.arange(cfg.len_lo, cfg.len_hi + 1, dtype=np.int64)
        p = support.astype(np.float64) ** (-cfg.zipf_a)
        p /= p.sum()
        return r.choice(support, size=cfg.num_seqs, p=p).astype(np.int64)
    raise ValueError(cfg.lengths)


def shuffled_tables(r, blocks_per_seq, num_blocks=0, spare=0.25):
    """Assign physical block ids from a seeded permutation of the pool.

    blocks_per_seq: how many blocks each sequence holds.  The pool is
    ``num_blocks`` (or needed * (1 + spare), rounded up) blocks; a random
    permutation of all ids is dealt out to the sequences in order.  Returns
    (num_blocks, tables int32 [S, max(blocks_per_seq)] padded with -1).
    """
    blocks_per_seq = np.asarray(blocks_per_seq, dtype=np.int64)
    need = int(blocks_per_seq.sum())
    nb = int(num_blocks) if num_blocks else int(math.ceil(need * (1.0 + spare)))
    if nb < need:
        raise ValueError("pool smaller than the blocks needed")
    perm = r.permutation(nb).astype(np.int32)
    width = max(1, int(blocks_per_seq.max()) if len(blocks_per_seq) else 1)
    tables = np.full((len(blocks_per_seq), width), -1, dtype=np.int32)
    at = 0
    for s, n in enumerate(blocks_per_seq.tolist()):
        tables[s, :n] = perm[at:at + n]
        at += n
    return nb, tables


def to_storage(x32, dtype):
    """Round float32 values to ``dtype`` storage (RNE via torch's CPU cast)."""
    x32 = np.ascontiguousarray(x32, dtype=np.float32)
    if dtype == "f32":
        return x32
    import torch
    t = torch.from_numpy(x32)
    tt = {"f16": torch.float16, "bf16": torch.bfloat16}[dtype]
    return t.to(tt).view(torch.int16).numpy().view(np.uint16)


def normal_storage(r, shape, dtype):
    """Standard-normal values of ``shape`` in ``dtype`` storage form."""
    return to_storage(r.standard_normal(shape, dtype=np.float32), dtype)


def outlier_rows(r, num_rows, frac):
    """Indices of exactly floor(frac * num_rows) rows, uniform without replacement."""
    k = int(math.floor(frac * num_rows))
    return np.sort(r.choice(num_rows, size=k, replace=False)) if k else np.zeros(0, dtype=np.int64)


@dataclass
class DecodeInputs:
    cfg: DecodeConfig
    context_lens: np.ndarray      # int64 [S], post-write lengths
    num_blocks: int
    block_tables: np.ndarray      # int32 [S, max_blocks], -1 padded
    q: np.ndarray                 # storage [S, Hq, D]
    k_hist: list = field(default_factory=list)   # per seq storage [ctx, Hkv, D]
    v_hist: list = field(default_factory=list)


def blocks_for(context_lens, block_size):
    return [-(-int(n) // block_size) for n in context_lens]


def make_decode_inputs(cfg, seed, context_lens=None, block_size=None, num_blocks=None):
    """Draw one decode step's inputs on the host (small and medium sizes).

    The K/V history of every sequence is drawn in logical order; the last row
    of each history is the step's new token.  Physical placement is only the
    block table (a permutation of the pool), never applied here.
    """
    r = rng(seed)
    bs = block_size or cfg.block_size
    lens = np.asarray(context_lens if context_lens is not None else context_lengths(cfg, r), dtype=np.int64)
    nb, tables = shuffled_tables(r, blocks_for(lens, bs),
                                 num_blocks if num_blocks is not None else cfg.num_blocks, cfg.spare)
    S, Hq, Hkv, D = len(lens), cfg.num_heads, cfg.num_kv_heads, cfg.head_dim
    q = normal_storage(r, (S, Hq, D), cfg.dtype)
    kh, vh = [], []
    for n in lens.tolist():
        k32 = r.standard_normal((n, Hkv, D), dtype=np.float32)
        if cfg.outlier_frac > 0:
            rows = outlier_rows(r, n * Hkv, cfg.outlier_frac)
            flat = k32.reshape(n * Hkv, D)
            flat[rows] *= np.float32(cfg.outlier_scale)
        kh.append(to_storage(k32, cfg.dtype))
        vh.append(normal_storage(r, (n, Hkv, D), cfg.dtype))
    return DecodeInputs(cfg, lens, nb, tables, q, kh, vh)


# ---------------------------------------------------------------------------
# Continuous-batching trace (fp16, 8-token blocks, 32/32 heads, D=128)
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class TraceConfig:
    dtype: str = "f16"
    num_heads: int = 32
    num_kv_heads: int = 32
    head_dim: int = 128
    block_size: int = 8
    max_running: int = 128
    num_requests: int = 256
    steps: int = 200
    prefix_len: int = 1024
    prompt_lo: int = 1
    prompt_hi: int = 512
    output_mean: float = 256.0
    fork_every: int = 8           # 1 in fork_every requests forks a child
    pool_frac: float = 0.75       # pool = this fraction of the unbounded peak

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.head_dim)


TRACE = TraceConfig()


@dataclass
class TraceRequest:
    seq_id: int
    prompt_len: int
    output_len: int
    shares_prefix: bool
    fork_child: int
    fork_output_len: int


PREFIX_SEQ = 1 << 40                # id of the sequence holding the shared prefix


def make_trace_requests(tc, seed):
    """All requests waiting at step 0, in arrival (FCFS) order.

    Unique prompt lengths uniform on [prompt_lo, prompt_hi]; output lengths
    geometric with the given mean (support >= 1); every other request shares
    the system prefix; one in ``fork_every`` forks a parallel-sampling child
    (child id = num_requests + request id).
    """
    r = rng(seed)
    n = tc.num_requests
    prompts = r.integers(tc.prompt_lo, tc.prompt_hi + 1, size=n)
    outs = r.geometric(1.0 / tc.output_mean, size=n)
    child_outs = r.geometric(1.0 / tc.output_mean, size=n)
    share = r.permutation(np.arange(n) % 2 == 0)
    fork = r.permutation(np.arange(n) % tc.fork_every == 0)
    reqs = []
    for i in range(n):
        reqs.append(TraceRequest(i, int(prompts[i]), int(outs[i]), bool(share[i]),
                                 n + i if fork[i] else -1, int(child_outs[i])))
    return reqs


def token_values(seed, stream, pos, shape, dtype, salt=0):
    """Values of one token row from a counter-keyed stream.

    ``stream`` names whose history the row belongs to (a sequence id, or the
    prefix holder), ``pos`` its logical position, ``salt`` separates K (0),
    V (1) and Q (2).  Keyed generation lets a preempted sequence's history be
    drawn again identically.
    """
    r = np.random.default_rng([int(seed), int(stream) & 0xFFFFFFFF, int(stream) >> 32, int(pos), int(salt)])
    return to_storage(r.standard_normal(shape, dtype=np.float32), dtype)


# ---------------------------------------------------------------------------
# Device-side draws for full-size workloads (torch RNG on the GPU)
# ---------------------------------------------------------------------------

@dataclass
class DeviceDraw:
    cfg: DecodeConfig
    context_lens: np.ndarray      # int64 [S]
    offsets: np.ndarray           # int64 [S + 1]: sequence s owns history rows [off[s], off[s+1])
    num_blocks: int
    free_order: np.ndarray        # int32 permutation of the pool (blocks are taken from its end)
    q: object                     # torch [S, Hq, D]
    k_hist: object                # torch [sum(ctx), Hkv, D]
    v_hist: object


def draw_device(cfg, seed, device="cuda", context_lens=None, block_size=None):
    """Draw one decode step's inputs directly on the GPU.

    Lengths, the pool size and its shuffled free order come from numpy's
    seeded generator; values are standard normal from a seeded torch CUDA
    generator, rounded to the dtype (1% of K rows scaled by 8 first when the
    config asks for outliers).
    """
    import torch
    r = rng(seed)
    bs = block_size or cfg.block_size
    lens = np.asarray(context_lens if context_lens is not None else context_lengths(cfg, r), dtype=np.int64)
    need = sum(blocks_for(lens, bs))
    nb = cfg.num_blocks if cfg.num_blocks else int(math.ceil(need * (1.0 + cfg.spare)))
    order = r.permutation(nb).astype(np.int32)
    offsets = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    total = int(offsets[-1])
    S, Hq, Hkv, D = len(lens), cfg.num_heads, cfg.num_kv_heads, cfg.head_dim
    tt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[cfg.dtype]
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000003 + 17)
    q = torch.randn((S, Hq, D), generator=g, device=device, dtype=torch.float32).to(tt)
    k32 = torch.randn((total, Hkv, D), generator=g, device=device, dtype=torch.float32)
    if cfg.outlier_frac > 0:
        rows = outlier_rows(r, total * Hkv, cfg.outlier_frac)
        idx = torch.from_numpy(rows).to(device)
        flat = k32.view(total * Hkv, D)
        flat[idx] *= cfg.outlier_scale
    k = k32.to(tt)
    del k32
    v = torch.randn((total, Hkv, D), generator=g, device=device, dtype=torch.float32).to(tt)
    return DeviceDraw(cfg, lens, offsets, nb, order, q, k, v)


# ---------------------------------------------------------------------------
# Counter-based rows for traces: any (stream, position) can be regenerated
# ---------------------------------------------------------------------------

_M64 = np.uint64(0xFFFFFFFFFFFFFFFF)


def _splitmix64(x):
    """SplitMix64 finaliser (Steele, Lea, Flood 2014) on uint64 arrays."""
    x = np.asarray(x, dtype=np.uint64)
    z = x + np.uint64(0x9E3779B97F4A7C15)
    z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def generated_token(seq, pos, vocab):
    """Token id a synthetic decode produced for position ``pos`` of sequence
    ``seq``: SplitMix64 of (seq x 0x100000001B3 + pos) mod 2^64, modulo vocab.
    Stands in for the sampled token when a scheduler names blocks by their
    token ids."""
    m = 0xFFFFFFFFFFFFFFFF
    z = ((int(seq) * 0x100000001B3 + int(pos)) + 0x9E3779B97F4A7C15) & m
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & m
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & m
    return (z ^ (z >> 31)) % int(vocab)


_ROW_TABLES = {}


def _row_tables(seed, width):
    key = (int(seed), int(width))
    if key not in _ROW_TABLES:
        r = np.random.default_rng([int(seed) & 0xFFFFFFFF, 0x5EED, width])
        _ROW_TABLES[key] = (r.standard_normal((4096, width), dtype=np.float32),
                            r.standard_normal((4096, width), dtype=np.float32))
    return _ROW_TABLES[key]


def token_rows(seed, stream, positions, heads, head_dim, dtype, salt=0):
    """Standard-normal rows [len(positions), heads, head_dim] in storage form,
    keyed by (seed, stream, position, salt) so any row can be drawn again.

    Two tables A, B of 4096 standard-normal rows are drawn once per seed; a
    row is (A[i] + B[j]) / sqrt(2) with (i, j) taken from a SplitMix64 hash of
    the key -- 16.7M distinct rows, each element N(0, 1).  salt separates K (0),
    V (1) and queries (2).
    """
    pos = np.asarray(positions, dtype=np.uint64).reshape(-1)
    with np.errstate(over="ignore"):
        h = _splitmix64(np.uint64(int(seed) & 0xFFFFFFFFFFFFFFFF) ^ _splitmix64(
            np.uint64(int(stream) & 0xFFFFFFFFFFFFFFFF) ^ _splitmix64(np.uint64(int(salt) + 1))))
        h = _splitmix64(h ^ _splitmix64(pos + np.uint64(0x632BE59BD9B4E019)))
    i = (h & np.uint64(4095)).astype(np.int64)
    j = ((h >> np.uint64(12)) & np.uint64(4095)).astype(np.int64)
    A, B = _row_tables(seed, heads * head_dim)
    z = A[i]
    z += B[j]
    z *= np.float32(0.7071067811865476)
    return to_storage(z.reshape(len(pos), heads, head_dim), dtype)


def prefix_keys(tokens):
    """uint64 key of every prefix tokens[:p+1], p = 0..n-1 (a SplitMix64 chain),
    so the K/V rows drawn from these keys depend on the whole prefix, as a
    model's K/V at a position does."""
    toks = np.asarray(tokens, dtype=np.int64).astype(np.uint64)
    with np.errstate(over="ignore"):
        mixed = _splitmix64(toks + np.uint64(0x13198A2E03707344)).tolist()
    m = 0xFFFFFFFFFFFFFFFF
    keys = []
    h = 0x243F6A8885A308D3
    for x in mixed:                      # the chain itself, in Python integers
        z = ((h ^ x) + 0x9E3779B97F4A7C15) & m
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & m
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & m
        h = z ^ (z >> 31)
        keys.append(h)
    return np.array(keys, dtype=np.uint64)


def prefix_rows(seed, tokens, start, heads, head_dim, dtype, salt=0):
    """Rows [n - start, heads, head_dim] for positions start..n-1 of the token
    sequence, each keyed by its whole prefix (prefix_keys) and salt (K 0, V 1)."""
    keys = prefix_keys(tokens)[start:]
    return token_rows(seed, 0x9F, keys, heads, head_dim, dtype, salt)
