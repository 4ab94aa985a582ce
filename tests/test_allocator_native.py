"""The C++ block allocator in libpkv agrees with the Python reference model:
same slots, tables, copy pairs, reference counts, statistics and errors, on the
pages' traces and on long random operation scripts.  Host code only."""
import numpy as np
import pytest

from oracle.allocator_model import AllocatorModel, AllocatorError
from paged_kv_cache_419_b200.binding import BlockAllocator, PkvError, PKV_ENOMEM, PKV_EINVAL
import workloads as wl


def same_state(native, model, seqs, max_blocks):
    if seqs:
        table, lens = native.block_table(seqs, max_blocks)
        mt, ml = model.block_table(seqs, max_blocks)
        assert table.tolist() == mt and lens.tolist() == ml
    for b in range(model.N):
        assert native.refcount(b) == model.ref[b]
    st = native.stats()
    for k, v in model.stats().items():
        assert st[k] == v, k


def test_pages_trace_new_frame_only_when_last_fills():
    n = BlockAllocator(8, 16)
    assert n.add_seq(0, 15).tolist() == list(range(15))
    assert n.append(0) == (15, -1, -1)
    assert n.append(0) == (16, -1, -1)


def test_cow_batch_step_emits_one_pair_per_writer_while_shared():
    order = np.random.default_rng(0).permutation(256).astype(np.int32)
    n, m = BlockAllocator(256, 16, order), AllocatorModel(256, 16, order)
    for a in (n, m):
        a.add_seq(0, 1000)
        for c in (1, 2, 3):
            a.fork(0, c)
    slots, pairs = n.append_batch([0, 1, 2, 3])
    exp_slots, exp_pairs = [], []
    for s in range(4):
        slot, src, dst = m.append(s)
        exp_slots.append(slot)
        if src >= 0:
            exp_pairs.append([src, dst])
    assert slots.tolist() == exp_slots and pairs.tolist() == exp_pairs and len(exp_pairs) == 3
    same_state(n, m, [0, 1, 2, 3], 80)


def test_enomem_changes_nothing():
    n = BlockAllocator(4, 16)
    n.add_seq(0, 40)
    before = n.stats()
    with pytest.raises(PkvError) as e:
        n.add_seq(1, 17)
    assert e.value.status == PKV_ENOMEM and n.stats() == before
    n.add_seq(1, 16)
    n.fork(1, 2)
    # the step needs 2 frames (seq 1 and seq 2 both start a new block), 0 free
    with pytest.raises(PkvError) as e:
        n.append_batch([1, 2])
    assert e.value.status == PKV_ENOMEM and n.stats()["tokens"] == 40 + 16 + 16


def test_bad_ids_are_rejected():
    n = BlockAllocator(8, 4)
    n.add_seq(0, 3)
    for call in (lambda: n.add_seq(0, 1), lambda: n.fork(5, 6), lambda: n.fork(0, 0),
                 lambda: n.append(9), lambda: n.free_seq(9), lambda: n.append_batch([0, 0])):
        with pytest.raises(PkvError) as e:
            call()
        assert e.value.status == PKV_EINVAL
    with pytest.raises(PkvError):
        BlockAllocator(4, 4, frame_order=[0, 1, 1, 2])


@pytest.mark.parametrize("seed", range(6))
def test_random_scripts_match_the_model(seed):
    rng = np.random.default_rng(100 + seed)
    N, Bsz = int(rng.integers(16, 200)), int(rng.choice([8, 16, 32]))
    order = rng.permutation(N).astype(np.int32)
    n, m = BlockAllocator(N, Bsz, order), AllocatorModel(N, Bsz, order)
    live, next_id = [], 0
    for step in range(400):
        op = rng.choice(["add", "fork", "append", "batch", "free"], p=[0.2, 0.15, 0.3, 0.2, 0.15])
        if op == "add" or not live:
            L = int(rng.integers(0, 3 * Bsz))
            try:
                exp = m.add_seq(next_id, L)
            except AllocatorError:
                with pytest.raises(PkvError):
                    n.add_seq(next_id, L)
            else:
                assert n.add_seq(next_id, L).tolist() == exp
                live.append(next_id)
            next_id += 1
        elif op == "fork":
            p = int(rng.choice(live))
            m.fork(p, next_id)
            n.fork(p, next_id)
            live.append(next_id)
            next_id += 1
        elif op == "append":
            s = int(rng.choice(live))
            try:
                exp = m.append(s)
            except AllocatorError:
                with pytest.raises(PkvError):
                    n.append(s)
            else:
                assert n.append(s) == exp
        elif op == "batch":
            k = int(rng.integers(1, len(live) + 1))
            ids = [int(x) for x in rng.choice(live, size=k, replace=False)]
            snapshot = (list(m.free), list(m.ref), {s: list(t) for s, t in m.tables.items()},
                        dict(m.lens))
            try:
                exp = [m.append(s) for s in ids]
            except AllocatorError:
                m.free, m.ref = type(m.free)(snapshot[0]), snapshot[1]
                m.tables, m.lens = snapshot[2], snapshot[3]
                with pytest.raises(PkvError):
                    n.append_batch(ids)
            else:
                slots, pairs = n.append_batch(ids)
                assert slots.tolist() == [e[0] for e in exp]
                assert pairs.tolist() == [[e[1], e[2]] for e in exp if e[1] >= 0]
        else:
            s = int(rng.choice(live))
            live.remove(s)
            m.free_seq(s)
            n.free_seq(s)
        if step % 25 == 0:
            same_state(n, m, live, 64)
    same_state(n, m, live, 64)


@pytest.mark.parametrize("seed", range(6))
def test_beam_search_scripts_match_the_model(seed):
    """Beam-search steps (slide 14's block tree) on the native allocator and the
    model: same ids, slots, copy pairs, tables, counts and free queue, including
    width changes, dropped beams and pool exhaustion (all-or-nothing)."""
    rng = np.random.default_rng(300 + seed)
    N, Bsz = int(rng.integers(12, 64)), int(rng.choice([8, 16, 32]))
    order = rng.permutation(N).astype(np.int32)
    n, m = BlockAllocator(N, Bsz, order), AllocatorModel(N, Bsz, order)
    P = int(rng.integers(1, 4 * Bsz))
    assert n.add_seq(0, P).tolist() == m.add_seq(0, P)
    beams, nid_n, nid_m, failures = [0], 1, 1, 0
    for step in range(120):
        k = len(beams)
        # mostly narrow steps; now and then a wide one that can exhaust the pool
        k_new = int(rng.integers(8, 33)) if rng.random() < 0.1 else int(rng.integers(1, 6))
        # skewed parents: most candidates continue the first (best) beams
        parents = [int(min(k - 1, rng.geometric(0.5) - 1)) for _ in range(k_new)]
        try:
            ids, slots, pairs, nid_m = m.beam_step(beams, parents, nid_m)
        except AllocatorError:
            failures += 1
            with pytest.raises(PkvError) as e:
                n.beam_step(beams, parents, nid_n)
            assert e.value.status == PKV_ENOMEM
            # free a beam to make room, as a scheduler would
            if len(beams) > 1:
                victim = beams.pop()
                m.free_seq(victim)
                n.free_seq(victim)
            continue
        ids_n, slots_n, pairs_n, nid_n = n.beam_step(beams, parents, nid_n)
        assert ids_n.tolist() == ids and slots_n.tolist() == slots
        assert pairs_n.tolist() == pairs and nid_n == nid_m
        beams = ids
        if step % 10 == 0:
            same_state(n, m, beams, 4 * N)
    same_state(n, m, beams, 4 * N)
    assert n.stats() == m.stats()
    assert failures > 0 or seed in (2, 4)  # the pool runs out in most scripts


def test_beam_step_rejects_bad_arguments():
    n = BlockAllocator(16, 4)
    n.add_seq(0, 5)
    n.add_seq(1, 5)
    for beams, parents, nid in (([0, 0], [0], 5), ([0, 7], [0], 5), ([0, 1], [2], 5), ([0, 1], [0, 0], 1)):
        with pytest.raises(PkvError) as e:
            n.beam_step(beams, parents, nid)
        assert e.value.status == PKV_EINVAL
    assert n.stats()["logical_blocks"] == 4  # nothing changed


def test_decode_workload_tables_follow_the_frame_order():
    w = wl.WORKLOADS["gqa8b"]
    inp = wl.make_decode_inputs(w, num_seqs=16)
    n = BlockAllocator(w.num_blocks, w.block_size, inp.frame_order)
    for s, L in enumerate(inp.context_lens):
        n.add_seq(s, int(L))
    table, lens = n.block_table(list(range(16)), w.max_blocks_per_seq)
    used = np.concatenate([table[s][table[s] >= 0] for s in range(16)])
    assert used.tolist() == inp.frame_order[: used.size].tolist()
    assert lens.tolist() == inp.context_lens.tolist()


def test_kv_memory_report_matches_the_model():
    """The bench's KV memory report (native allocator) against the Python model
    on the same batches: useful-KV share of the gqa8b batch (the pages report
    96.3 % useful KV memory, dataarena note section 2) and the frames saved by
    sharing prompts among 4 samples with copy-on-write (slides 13-14)."""
    import bench

    w = wl.WORKLOADS["gqa8b"]
    lens = wl.make_decode_inputs(w).context_lens
    rep = bench.kv_memory_report(w, lens)
    m = AllocatorModel(w.num_blocks, w.block_size)
    for s, L in enumerate(lens):
        m.add_seq(s, int(L))
    st = m.stats()
    assert rep["frames"] == st["used_blocks"] == int(sum(-(-int(L) // w.block_size) for L in lens))
    assert rep["tokens"] == int(lens.sum())
    assert rep["useful_kv_pct"] == round(100.0 * lens.sum() / (st["used_blocks"] * w.block_size), 2)
    assert rep["useful_kv_pct"] > 96.3  # only each sequence's last block is partial

    sh = wl.make_shared_inputs()
    ws = sh.w
    m = AllocatorModel(ws.num_blocks, ws.block_size, sh.frame_order)
    n = ws.samples_per_prompt
    for p in range(ws.num_prompts):
        m.add_seq(p * n, sh.prompt_len)
        for c in range(1, n):
            m.fork(p * n, p * n + c)
    copies = 0
    for step in range(int(sh.gen_lens.max())):
        for s in range(ws.num_seqs):
            if sh.gen_lens[s] > step:
                _, src, _ = m.append(s)
                copies += src >= 0
    ms = m.stats()
    assert rep["sharing_frames"] == ms["used_blocks"]
    assert rep["sharing_unshared_frames"] == ms["logical_blocks"]
    assert rep["sharing_cow_copies"] == copies

    bm = wl.make_beam_inputs()
    m = AllocatorModel(bm.w.num_blocks, bm.w.block_size, bm.frame_order)
    m.add_seq(0, bm.prompt_len)
    beams, nid, copies = [0], 1, 0
    for step in range(bm.steps):
        beams, _, pairs, nid = m.beam_step(beams, bm.parents[step], nid)
        copies += len(pairs)
    ms = m.stats()
    assert rep["beam_frames"] == ms["used_blocks"] and rep["beam_unshared_frames"] == ms["logical_blocks"]
    assert rep["beam_cow_copies"] == copies
    assert rep["beam_saving_pct"] == round(100.0 * (1 - ms["used_blocks"] / ms["logical_blocks"]), 2)

    px = wl.make_prefix_inputs()
    m = AllocatorModel(px.w.num_blocks, px.w.block_size, px.frame_order)
    cached = sum(m.add_seq_cached(i, px.token_ids[i])[1] for i in range(px.w.num_seqs))
    ms = m.stats()
    total = sum(len(t) for t in px.token_ids)
    assert rep["prefix_cache_frames"] == ms["used_blocks"]
    assert rep["prefix_cache_uncached_frames"] == ms["logical_blocks"]
    assert rep["prefix_cache_reused_tokens_pct"] == round(100.0 * cached / total, 2)
    # every request after the first on a system prompt reuses that prompt's 64 full blocks
    firsts = len(set(px.system.tolist()))
    assert cached == (px.w.num_seqs - firsts) * px.prompt_len


def test_block_hash_is_sha256():
    """pkv_block_hash is SHA-256 (FIPS 180-4) of the parent key and the token ids
    as little-endian int32, checked against hashlib on messages of 0 to 300
    tokens (1 to 20 SHA-256 blocks) with and without a parent key."""
    import hashlib
    from paged_kv_cache_419_b200.binding import block_hash

    rng = np.random.default_rng(11)
    for n in (0, 1, 7, 8, 15, 16, 31, 32, 100, 300):
        toks = rng.integers(-2**31, 2**31, size=n, dtype=np.int64).astype(np.int32)
        for parent in (None, bytes(rng.integers(0, 256, size=32, dtype=np.uint8))):
            msg = (parent if parent is not None else bytes(32)) + toks.astype("<i4").tobytes()
            assert block_hash(parent, toks) == hashlib.sha256(msg).digest()
    assert AllocatorModel.block_key(None, [1, 2, 3]) == block_hash(None, [1, 2, 3])


@pytest.mark.parametrize("seed", range(4))
def test_prefix_cache_scripts_match_the_model(seed):
    """Requests built from a few shared system prompts plus private suffixes,
    mixed with frees, appends and forks: the native allocator and the model agree
    on slots, cached-token counts, tables, counts and the cache size."""
    rng = np.random.default_rng(500 + seed)
    N, Bsz = int(rng.integers(24, 120)), int(rng.choice([4, 8, 16]))
    order = rng.permutation(N).astype(np.int32)
    n, m = BlockAllocator(N, Bsz, order), AllocatorModel(N, Bsz, order)
    systems = [[int(x) for x in rng.integers(0, 1000, size=int(rng.integers(0, 5 * Bsz)))] for _ in range(3)]
    live, next_id, hits = [], 0, 0
    for step in range(300):
        op = rng.choice(["req", "free", "append", "fork"], p=[0.4, 0.3, 0.2, 0.1])
        if op == "req" or not live:
            toks = systems[int(rng.integers(0, 3))] + [int(x) for x in rng.integers(0, 1000, size=int(rng.integers(0, 2 * Bsz)))]
            try:
                exp_slots, exp_cached = m.add_seq_cached(next_id, toks)
            except AllocatorError:
                with pytest.raises(PkvError) as e:
                    n.add_seq_cached(next_id, toks)
                assert e.value.status == PKV_ENOMEM
            else:
                slots, cached = n.add_seq_cached(next_id, toks)
                assert slots.tolist() == exp_slots and cached == exp_cached
                hits += cached > 0
                live.append(next_id)
            next_id += 1
        elif op == "free":
            s = int(rng.choice(live))
            live.remove(s)
            m.free_seq(s)
            n.free_seq(s)
        elif op == "append":
            s = int(rng.choice(live))
            try:
                exp = m.append(s)
            except AllocatorError:
                with pytest.raises(PkvError):
                    n.append(s)
            else:
                assert n.append(s) == exp
        else:
            p = int(rng.choice(live))
            m.fork(p, next_id)
            n.fork(p, next_id)
            live.append(next_id)
            next_id += 1
        if step % 20 == 0:
            same_state(n, m, live, 4 * N)
    same_state(n, m, live, 4 * N)
    assert hits > 0


@pytest.mark.parametrize("seed", range(4))
def test_mixed_scripts_match_the_model(seed):
    """Everything at once: cached and plain prompts, forks, appends and batches,
    beam steps over a live group of sequences, and frees (which also release
    cached frames for revival or eviction).  Native allocator and model agree on
    every result and on the whole state."""
    rng = np.random.default_rng(900 + seed)
    N, Bsz = int(rng.integers(20, 96)), int(rng.choice([4, 8, 16]))
    order = rng.permutation(N).astype(np.int32)
    n, m = BlockAllocator(N, Bsz, order), AllocatorModel(N, Bsz, order)
    systems = [[int(x) for x in rng.integers(0, 50, size=int(rng.integers(Bsz, 4 * Bsz)))] for _ in range(2)]
    live, next_id = [], 0
    for step in range(400):
        op = rng.choice(["cached", "plain", "fork", "append", "batch", "beam", "free"],
                        p=[0.2, 0.1, 0.1, 0.15, 0.1, 0.15, 0.2])
        if op in ("cached", "plain") or not live:
            toks = systems[int(rng.integers(0, 2))] + [int(x) for x in rng.integers(0, 50, size=int(rng.integers(0, Bsz)))]
            try:
                exp = m.add_seq_cached(next_id, toks) if op == "cached" else (m.add_seq(next_id, len(toks)), 0)
            except AllocatorError:
                with pytest.raises(PkvError):
                    n.add_seq_cached(next_id, toks) if op == "cached" else n.add_seq(next_id, len(toks))
            else:
                got = n.add_seq_cached(next_id, toks) if op == "cached" else (n.add_seq(next_id, len(toks)), 0)
                assert got[0].tolist() == exp[0] and got[1] == exp[1]
                live.append(next_id)
            next_id += 1
        elif op == "fork":
            p = int(rng.choice(live))
            m.fork(p, next_id)
            n.fork(p, next_id)
            live.append(next_id)
            next_id += 1
        elif op == "append":
            s = int(rng.choice(live))
            try:
                exp = m.append(s)
            except AllocatorError:
                with pytest.raises(PkvError):
                    n.append(s)
            else:
                assert n.append(s) == exp
        elif op == "batch":
            ids = [int(x) for x in rng.choice(live, size=int(rng.integers(1, len(live) + 1)), replace=False)]
            snap = (type(m.free)(m.free), list(m.ref), {k: list(v) for k, v in m.tables.items()}, dict(m.lens),
                    dict(m.cache), dict(m.frame_key))
            try:
                exp = [m.append(s) for s in ids]
            except AllocatorError:
                m.free, m.ref, m.tables, m.lens, m.cache, m.frame_key = snap
                with pytest.raises(PkvError):
                    n.append_batch(ids)
            else:
                slots, pairs = n.append_batch(ids)
                assert slots.tolist() == [e[0] for e in exp]
                assert pairs.tolist() == [[e[1], e[2]] for e in exp if e[1] >= 0]
        elif op == "beam":
            k = int(rng.integers(1, len(live) + 1))
            beams = [int(x) for x in rng.choice(live, size=k, replace=False)]
            parents = [int(rng.integers(0, k)) for _ in range(int(rng.integers(0, k + 3)))]
            try:
                ids, slots, pairs, nid = m.beam_step(beams, parents, next_id)
            except AllocatorError:
                with pytest.raises(PkvError):
                    n.beam_step(beams, parents, next_id)
            else:
                ids_n, slots_n, pairs_n, nid_n = n.beam_step(beams, parents, next_id)
                assert ids_n.tolist() == ids and slots_n.tolist() == slots and pairs_n.tolist() == pairs
                assert nid_n == nid
                live = [s for s in live if s not in beams] + ids
                next_id = nid
        else:
            s = int(rng.choice(live))
            live.remove(s)
            m.free_seq(s)
            n.free_seq(s)
        if step % 25 == 0:
            same_state(n, m, live, 8 * N)
    same_state(n, m, live, 8 * N)


def test_prefix_cache_and_beam_edge_cases():
    n, m = BlockAllocator(8, 4), AllocatorModel(8, 4)
    # an empty prompt and a prompt shorter than a block: nothing is cached
    for obj in (n, m):
        assert obj.add_seq_cached(0, [])[1] == 0
        assert obj.add_seq_cached(1, [7, 8, 9])[1] == 0
    assert n.stats()["cached_blocks"] == m.stats()["cached_blocks"] == 0
    # exactly one full block is cached and reused, the partial one is not
    for obj in (n, m):
        obj.add_seq_cached(2, [1, 2, 3, 4, 5])
        assert obj.add_seq_cached(3, [1, 2, 3, 4, 6])[1] == 4
    assert n.stats() == m.stats() and n.stats()["cached_blocks"] == 1
    # a beam step with no candidates frees every beam
    ids, slots, pairs, nid = n.beam_step([2, 3], [], 50)
    e_ids, e_slots, e_pairs, e_nid = m.beam_step([2, 3], [], 50)
    assert ids.tolist() == e_ids == [] and nid == e_nid == 50
    assert n.stats() == m.stats()
    # a fresh id that is already live is refused, nothing changes
    before = n.stats()
    with pytest.raises(PkvError) as e:
        n.beam_step([0], [0, 0], 1)
    assert e.value.status == PKV_EINVAL and n.stats() == before
