"""Seeded synthetic inputs for paged decode attention.

This module only draws random numbers and lays them out as plain arrays.  It
holds none of the method's arithmetic (no slot formula, no attention math), so
both the CPU oracle (through the tests) and the CUDA path (through the tests and
the benchmark) can consume the same inputs without sharing any computation.

Floating-point tensors are returned as ``numpy.uint16`` arrays holding fp16 or
bf16 bit patterns; ``dtype`` says which.  Values are drawn in fp32 and rounded
to the storage type with round-to-nearest-even (numpy for fp16, torch for bf16).

Workloads follow the five decode batches used throughout the project:

* ``tiny``     4 seqs, 8/8 heads, D=64, B=16, fp16, 64-frame pool, L ~ U{1..100}
* ``mha13b``   32 seqs, 40/40 heads, D=128, B=16, fp16, 4096 frames, L ~ U{1..2048}
               (13B-shaped: 40 heads x 128 = the 5120 hidden size of the slides)
* ``gqa8b``    256 seqs, 32/8 heads, D=128, B=16, bf16, 65536 frames,
               L = clip(round(exp(N(ln 512, 1))), 16, 4096), K scaled by 0.5
* ``shared``   16 prompts x 4 samples, 32/8 heads, D=128, B=16, bf16, prompt
               1000 tokens, 0..200 private tokens per sample, 65536 frames
* ``long``     4 seqs, 32/8 heads, D=128, B=32, bf16, 8192 frames,
               L ~ U{16384..32768}
* ``prefill``  16 seqs, 32/8 heads, D=128, B=16, bf16, 8192 frames: each a chunk
               of T ~ U{256..2048} new tokens after p0 ~ U{0..4096} cached ones
               (p0 = 0 for the first 4: whole prompts)

Draw order inside one workload: context lengths, the physical frame order of
the pool, q, K, V (for ``shared``: generated lengths, frame order, q, prompt K,
prompt V, generated K, generated V).  The default seed of a workload is its
position in the list above (0 for ``tiny`` ... 4 for ``long``).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

F16 = 0
BF16 = 1
DTYPE_NAMES = {F16: "f16", BF16: "bf16"}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    dtype: int
    max_blocks_per_seq: int
    scale: float
    k_scale: float = 1.0
    # length law: ("uniform", lo, hi) | ("lognormal", median, sigma, lo, hi) | ("shared", prompt, gmax)
    # | ("beam", prompt, steps) | ("prefix", system prompt, max own tokens)
    lengths: tuple = ()
    # shared-prefix workloads only
    num_prompts: int = 0
    samples_per_prompt: int = 0

    @property
    def group(self) -> int:
        return self.num_heads // self.num_kv_heads

    @property
    def elt_bytes(self) -> int:
        return 2

    def with_block_size(self, block_size: int) -> "Workload":
        """Same batch on a pool of the same token capacity with another block size."""
        tokens = self.num_blocks * self.block_size
        max_tokens = self.max_blocks_per_seq * self.block_size
        return dataclasses.replace(
            self,
            name=f"{self.name}-B{block_size}",
            block_size=block_size,
            num_blocks=tokens // block_size,
            max_blocks_per_seq=max_tokens // block_size,
        )


WORKLOADS = {
    "tiny": Workload("tiny", 0, 4, 8, 8, 64, 16, 64, F16, 7, 1.0 / 8.0,
                     lengths=("uniform", 1, 100)),
    "mha13b": Workload("mha13b", 1, 32, 40, 40, 128, 16, 4096, F16, 128, 1.0 / math.sqrt(128),
                       lengths=("uniform", 1, 2048)),
    "gqa8b": Workload("gqa8b", 2, 256, 32, 8, 128, 16, 65536, BF16, 256, 1.0 / math.sqrt(128),
                      k_scale=0.5, lengths=("lognormal", 512, 1.0, 16, 4096)),
    "shared": Workload("shared", 3, 64, 32, 8, 128, 16, 65536, BF16, 75, 1.0 / math.sqrt(128),
                       lengths=("shared", 1000, 200), num_prompts=16, samples_per_prompt=4),
    "long": Workload("long", 4, 4, 32, 8, 128, 32, 8192, BF16, 1024, 1.0 / math.sqrt(128),
                     lengths=("uniform", 16384, 32768)),
    # prefix caching: 64 requests on 4 shared 1024-token system prompts + 16-256 own tokens
    "prefix": Workload("prefix", 6, 64, 32, 8, 128, 16, 8192, BF16, 81, 1.0 / math.sqrt(128),
                       lengths=("prefix", 1024, 256), num_prompts=4),
    # beam search over a block tree: one 1000-token prompt, 4 beams, 200 steps
    "beam": Workload("beam", 5, 4, 32, 8, 128, 16, 4096, BF16, 76, 1.0 / math.sqrt(128),
                     lengths=("beam", 1000, 200)),
    # chunked prefill, Llama-3-8B-shaped GQA: 16 sequences, each a chunk of
    # U{256..2048} new tokens after U{0..4096} cached ones (the first 4 whole
    # prompts, nothing cached)
    "prefill": Workload("prefill", 7, 16, 32, 8, 128, 16, 8192, BF16, 384, 1.0 / math.sqrt(128),
                        lengths=("prefill", 4096, 256, 2048, 4)),
}


def to_bits(x: np.ndarray, dtype: int) -> np.ndarray:
    """Round fp32 values to fp16/bf16 (RNE) and return the bit patterns as uint16."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == F16:
        return x.astype(np.float16).view(np.uint16)
    if dtype == BF16:
        import torch

        return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    raise ValueError(f"unknown dtype {dtype}")


def _normal_bits(rng: np.random.Generator, shape, dtype: int, scale: float = 1.0,
                 chunk: int = 1 << 24) -> np.ndarray:
    """N(0, scale^2) values drawn in fp32 in chunks, stored as dtype bit patterns."""
    n = int(np.prod(shape, dtype=np.int64))
    out = np.empty(n, dtype=np.uint16)
    for lo in range(0, n, chunk):
        hi = min(n, lo + chunk)
        x = rng.standard_normal(hi - lo, dtype=np.float32)
        if scale != 1.0:
            x *= np.float32(scale)
        out[lo:hi] = to_bits(x, dtype)
    return out.reshape(shape)


def draw_lengths(w: Workload, rng: np.random.Generator) -> np.ndarray:
    law = w.lengths
    if law[0] == "uniform":
        return rng.integers(law[1], law[2], size=w.num_seqs, endpoint=True).astype(np.int32)
    if law[0] == "lognormal":
        median, sigma, lo, hi = law[1:]
        x = np.exp(rng.normal(math.log(median), sigma, size=w.num_seqs))
        return np.clip(np.rint(x), lo, hi).astype(np.int32)
    raise ValueError(law)


@dataclasses.dataclass
class DecodeInputs:
    """One decode batch.

    ``k_stream``/``v_stream`` hold every token's K/V in logical order, sequence
    after sequence: sequence s owns rows ``offsets[s]:offsets[s+1]``, each row
    ``[num_kv_heads, head_dim]``.  The last row of each sequence is the token the
    decode step appends; the rows before it are the already-cached context.
    ``frame_order`` is the order in which the pool hands out physical frames.
    """
    w: Workload
    context_lens: np.ndarray  # int32 [S]
    frame_order: np.ndarray   # int32 [N], a permutation of 0..N-1
    q: np.ndarray             # uint16 [S, Hq, D]
    k_stream: np.ndarray      # uint16 [sum L, Hkv, D]
    v_stream: np.ndarray      # uint16 [sum L, Hkv, D]
    offsets: np.ndarray       # int64 [S+1]

    @property
    def total_tokens(self) -> int:
        return int(self.offsets[-1])


def make_decode_inputs(name_or_w, seed: int | None = None, num_seqs: int | None = None,
                       lengths: np.ndarray | None = None) -> DecodeInputs:
    """Seeded decode batch for one of the workloads (not ``shared`` or ``beam``).

    ``num_seqs`` truncates the batch (the first sequences of the same draw of
    lengths are kept, so a truncated batch is a prefix of the full one only in
    its lengths); ``lengths`` overrides the drawn lengths (edge-case tests).
    """
    w = WORKLOADS[name_or_w] if isinstance(name_or_w, str) else name_or_w
    if w.lengths and w.lengths[0] == "shared":
        raise ValueError("use make_shared_inputs for the shared-prefix workload")
    if w.lengths and w.lengths[0] in ("beam", "prefix"):
        raise ValueError("use make_beam_inputs / make_prefix_inputs for these workloads")
    rng = np.random.default_rng(w.seed if seed is None else seed)
    lens = draw_lengths(w, rng)
    if lengths is not None:
        lens = np.asarray(lengths, dtype=np.int32)
    elif num_seqs is not None:
        lens = lens[:num_seqs]
    if num_seqs is not None or lengths is not None:
        w = dataclasses.replace(w, num_seqs=int(lens.shape[0]))
    frame_order = rng.permutation(w.num_blocks).astype(np.int32)
    q = _normal_bits(rng, (w.num_seqs, w.num_heads, w.head_dim), w.dtype)
    total = int(lens.astype(np.int64).sum())
    k = _normal_bits(rng, (total, w.num_kv_heads, w.head_dim), w.dtype, w.k_scale)
    v = _normal_bits(rng, (total, w.num_kv_heads, w.head_dim), w.dtype)
    offsets = np.zeros(w.num_seqs + 1, dtype=np.int64)
    np.cumsum(lens, out=offsets[1:])
    return DecodeInputs(w, lens, frame_order, q, k, v, offsets)


@dataclasses.dataclass
class SharedInputs:
    """Shared-prefix parallel sampling batch.

    Prompt p is shared by samples ``p*n .. p*n+n-1`` (n = samples per prompt).
    ``prompt_k[p]`` holds the prompt's K rows in logical order; sample i then
    generates ``gen_lens[i]`` private tokens whose K rows are
    ``gen_k[gen_offsets[i]:gen_offsets[i+1]]``.
    """
    w: Workload
    prompt_len: int
    gen_lens: np.ndarray      # int32 [S]
    frame_order: np.ndarray   # int32 [N]
    q: np.ndarray             # uint16 [S, Hq, D]
    prompt_k: np.ndarray      # uint16 [P, prompt_len, Hkv, D]
    prompt_v: np.ndarray
    gen_k: np.ndarray         # uint16 [sum g, Hkv, D]
    gen_v: np.ndarray
    gen_offsets: np.ndarray   # int64 [S+1]


def make_shared_inputs(seed: int | None = None, num_prompts: int | None = None) -> SharedInputs:
    w = WORKLOADS["shared"]
    if num_prompts is not None:
        w = dataclasses.replace(w, num_prompts=num_prompts,
                                num_seqs=num_prompts * w.samples_per_prompt)
    rng = np.random.default_rng(w.seed if seed is None else seed)
    prompt_len, gmax = w.lengths[1], w.lengths[2]
    gen = rng.integers(0, gmax, size=w.num_seqs, endpoint=True).astype(np.int32)
    frame_order = rng.permutation(w.num_blocks).astype(np.int32)
    q = _normal_bits(rng, (w.num_seqs, w.num_heads, w.head_dim), w.dtype)
    pk = _normal_bits(rng, (w.num_prompts, prompt_len, w.num_kv_heads, w.head_dim), w.dtype)
    pv = _normal_bits(rng, (w.num_prompts, prompt_len, w.num_kv_heads, w.head_dim), w.dtype)
    total = int(gen.astype(np.int64).sum())
    gk = _normal_bits(rng, (total, w.num_kv_heads, w.head_dim), w.dtype)
    gv = _normal_bits(rng, (total, w.num_kv_heads, w.head_dim), w.dtype)
    offs = np.zeros(w.num_seqs + 1, dtype=np.int64)
    np.cumsum(gen, out=offs[1:])
    return SharedInputs(w, prompt_len, gen, frame_order, q, pk, pv, gk, gv, offs)


@dataclasses.dataclass
class BeamInputs:
    """Beam-search script over a block tree (slide 14).

    One prompt of ``prompt_len`` tokens; at each of ``steps`` steps the ``k``
    beams are replaced by ``k`` candidates, candidate j continuing beam
    ``parents[step, j]`` with one token whose K/V rows are ``step_k[step, j]``
    (step 0 starts from the prompt alone, so ``parents[0]`` is all 0).
    Parents are drawn skewed towards the first beams (geometric, p = 1/2), the
    way the best-scoring beams collect most continuations; the scores themselves
    are not modelled.  ``q`` holds the final beams' queries.
    """
    w: Workload
    prompt_len: int
    k: int
    steps: int
    parents: np.ndarray       # int32 [steps, k]
    frame_order: np.ndarray   # int32 [N]
    q: np.ndarray             # uint16 [k, Hq, D]
    prompt_k: np.ndarray      # uint16 [prompt_len, Hkv, D]
    prompt_v: np.ndarray
    step_k: np.ndarray        # uint16 [steps, k, Hkv, D]
    step_v: np.ndarray


@dataclasses.dataclass
class PrefixInputs:
    """Requests that share system prompts (automatic prefix caching).

    Request i is system prompt ``system[i]`` (``prompt_len`` tokens) followed by
    ``own_lens[i]`` tokens of its own; ``token_ids[i]`` holds its whole prompt.
    K/V rows depend on the token's prefix: system prompt p's rows are
    ``system_k[p]`` (equal in every request that uses p), request i's own rows
    are ``own_k[own_offsets[i]:own_offsets[i+1]]``.
    """
    w: Workload
    prompt_len: int
    system: np.ndarray        # int32 [S]
    own_lens: np.ndarray      # int32 [S]
    token_ids: list           # S int32 arrays
    frame_order: np.ndarray   # int32 [N]
    q: np.ndarray             # uint16 [S, Hq, D]
    system_k: np.ndarray      # uint16 [P, prompt_len, Hkv, D]
    system_v: np.ndarray
    own_k: np.ndarray         # uint16 [sum own, Hkv, D]
    own_v: np.ndarray
    own_offsets: np.ndarray   # int64 [S + 1]


def make_prefix_inputs(seed: int | None = None, num_seqs: int | None = None) -> PrefixInputs:
    w = WORKLOADS["prefix"]
    if num_seqs is not None:
        w = dataclasses.replace(w, num_seqs=num_seqs)
    rng = np.random.default_rng(w.seed if seed is None else seed)
    plen, omax = w.lengths[1], w.lengths[2]
    system = rng.integers(0, w.num_prompts, size=w.num_seqs).astype(np.int32)
    own = rng.integers(16, omax, size=w.num_seqs, endpoint=True).astype(np.int32)
    sys_tokens = rng.integers(0, 128000, size=(w.num_prompts, plen)).astype(np.int32)
    token_ids = [np.concatenate([sys_tokens[system[i]], rng.integers(0, 128000, size=own[i]).astype(np.int32)])
                 for i in range(w.num_seqs)]
    frame_order = rng.permutation(w.num_blocks).astype(np.int32)
    q = _normal_bits(rng, (w.num_seqs, w.num_heads, w.head_dim), w.dtype)
    sk = _normal_bits(rng, (w.num_prompts, plen, w.num_kv_heads, w.head_dim), w.dtype)
    sv = _normal_bits(rng, (w.num_prompts, plen, w.num_kv_heads, w.head_dim), w.dtype)
    total = int(own.astype(np.int64).sum())
    ok = _normal_bits(rng, (total, w.num_kv_heads, w.head_dim), w.dtype)
    ov = _normal_bits(rng, (total, w.num_kv_heads, w.head_dim), w.dtype)
    offs = np.zeros(w.num_seqs + 1, dtype=np.int64)
    np.cumsum(own, out=offs[1:])
    return PrefixInputs(w, plen, system, own, token_ids, frame_order, q, sk, sv, ok, ov, offs)


def make_beam_inputs(seed: int | None = None, steps: int | None = None) -> BeamInputs:
    w = WORKLOADS["beam"]
    rng = np.random.default_rng(w.seed if seed is None else seed)
    prompt_len, nsteps = w.lengths[1], w.lengths[2] if steps is None else steps
    k = w.num_seqs
    parents = np.minimum(rng.geometric(0.5, size=(nsteps, k)) - 1, k - 1).astype(np.int32)
    parents[0] = 0  # the first step continues the single prompt beam k times
    frame_order = rng.permutation(w.num_blocks).astype(np.int32)
    q = _normal_bits(rng, (k, w.num_heads, w.head_dim), w.dtype)
    pk = _normal_bits(rng, (prompt_len, w.num_kv_heads, w.head_dim), w.dtype)
    pv = _normal_bits(rng, (prompt_len, w.num_kv_heads, w.head_dim), w.dtype)
    sk = _normal_bits(rng, (nsteps, k, w.num_kv_heads, w.head_dim), w.dtype)
    sv = _normal_bits(rng, (nsteps, k, w.num_kv_heads, w.head_dim), w.dtype)
    return BeamInputs(w, prompt_len, k, nsteps, parents, frame_order, q, pk, pv, sk, sv)


def make_token_rows(rng_seed: int, num_tokens: int, num_kv_heads: int, head_dim: int,
                    dtype: int):
    """Random new-token K and V rows ``[T, Hkv, D]`` (cache-write tests)."""
    rng = np.random.default_rng(rng_seed)
    k = _normal_bits(rng, (num_tokens, num_kv_heads, head_dim), dtype)
    v = _normal_bits(rng, (num_tokens, num_kv_heads, head_dim), dtype)
    return k, v


def random_slots(rng_seed: int, num_tokens: int, num_slots: int, num_skipped: int = 0) -> np.ndarray:
    """``num_tokens`` distinct slot indices in ``[0, num_slots)``; ``num_skipped``
    of them (at random positions) replaced by -1, the padding sentinel."""
    rng = np.random.default_rng(rng_seed)
    slots = rng.choice(num_slots, size=num_tokens, replace=False).astype(np.int64)
    if num_skipped:
        slots[rng.choice(num_tokens, size=num_skipped, replace=False)] = -1
    return slots


def random_pool(rng_seed: int, num_blocks: int, num_kv_heads: int, block_size: int,
                head_dim: int, dtype: int):
    """A K pool and a V pool ``[N, Hkv, B, D]`` filled with N(0,1) values."""
    rng = np.random.default_rng(rng_seed)
    shape = (num_blocks, num_kv_heads, block_size, head_dim)
    return _normal_bits(rng, shape, dtype), _normal_bits(rng, shape, dtype)


@dataclasses.dataclass
class PrefillInputs:
    """One prefill batch.  Sequence s has ``cached[s]`` tokens already in the
    cache and ``chunk[s]`` new ones after them.  ``k_stream``/``v_stream`` hold
    all of its cached + new tokens in logical order (rows
    ``offsets[s]:offsets[s+1]``); ``q`` holds the new tokens' queries, sequence
    after sequence (rows ``query_start[s]:query_start[s+1]``)."""
    w: Workload
    cached: np.ndarray        # int32 [S]
    chunk: np.ndarray         # int32 [S]
    frame_order: np.ndarray   # int32 [N]
    q: np.ndarray             # uint16 [sum chunk, Hq, D]
    k_stream: np.ndarray      # uint16 [sum (cached + chunk), Hkv, D]
    v_stream: np.ndarray
    offsets: np.ndarray       # int64 [S + 1]
    query_start: np.ndarray   # int32 [S + 1]

    @property
    def context_lens(self) -> np.ndarray:
        return (self.cached + self.chunk).astype(np.int32)


def make_prefill_inputs(name_or_w="prefill", seed: int | None = None, cached=None,
                        chunk=None) -> PrefillInputs:
    """Seeded prefill batch.  Draw order: cached lengths, chunk lengths, frame
    order, q, K, V.  ``cached`` / ``chunk`` override the drawn lengths (tests)."""
    w = WORKLOADS[name_or_w] if isinstance(name_or_w, str) else name_or_w
    rng = np.random.default_rng(w.seed if seed is None else seed)
    _, max_cached, lo, hi, n_whole = w.lengths
    p0 = rng.integers(0, max_cached, size=w.num_seqs, endpoint=True).astype(np.int32)
    p0[:n_whole] = 0
    T = rng.integers(lo, hi, size=w.num_seqs, endpoint=True).astype(np.int32)
    if cached is not None or chunk is not None:
        p0 = np.asarray(cached if cached is not None else p0, np.int32)
        T = np.asarray(chunk if chunk is not None else T, np.int32)
        w = dataclasses.replace(w, num_seqs=int(T.shape[0]))
    frame_order = rng.permutation(w.num_blocks).astype(np.int32)
    total_q = int(T.astype(np.int64).sum())
    q = _normal_bits(rng, (total_q, w.num_heads, w.head_dim), w.dtype)
    lens = (p0 + T).astype(np.int64)
    k = _normal_bits(rng, (int(lens.sum()), w.num_kv_heads, w.head_dim), w.dtype, w.k_scale)
    v = _normal_bits(rng, (int(lens.sum()), w.num_kv_heads, w.head_dim), w.dtype)
    offsets = np.zeros(w.num_seqs + 1, dtype=np.int64)
    np.cumsum(lens, out=offsets[1:])
    qs = np.zeros(w.num_seqs + 1, dtype=np.int32)
    np.cumsum(T, out=qs[1:])
    return PrefillInputs(w, p0, T, frame_order, q, k, v, offsets, qs)
