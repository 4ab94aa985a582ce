"""The allocator model's pins catch plausible mistakes.

Each case plants one mistake in a copy of oracle/allocator_model.py (a fork
that does not count, a beam that is never freed, a cache key that forgets its
prefix ...), loads the copy as a module and runs the model's pin tests against
it; at least one pin must fail.  The unchanged copy passes them all.
"""
import importlib.util
import os
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
MODEL = os.path.join(ROOT, "oracle", "allocator_model.py")


def _load_pins():
    spec = importlib.util.spec_from_file_location(
        "allocator_model_pins", os.path.join(os.path.dirname(os.path.abspath(__file__)), "test_allocator_model.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


PINS = _load_pins()
PIN_CALLS = [
    PINS.test_new_frame_only_when_last_block_fills,
    PINS.test_cow_four_samples_only_last_block_copied,
    PINS.test_full_shared_last_block_is_never_copied,
    PINS.test_free_returns_frames_in_fifo_order_and_refcounts,
    PINS.test_all_or_nothing_exhaustion,
    lambda: PINS.test_only_last_block_partial_and_waste_below_4_percent("gqa8b"),
    PINS.test_shared_workload_memory_saving,
    PINS.test_beam_step_candidates_share_the_prefix_like_forked_processes,
    PINS.test_beam_step_frees_dropped_beams_and_copies_only_on_divergence,
    PINS.test_beam_tree_frames_closed_form,
    PINS.test_beam_step_enomem_changes_nothing,
    PINS.test_prefix_cache_second_request_maps_to_the_same_frames,
    PINS.test_prefix_cache_keys_chain_the_whole_prefix,
    PINS.test_prefix_cache_survives_free_and_is_evicted_only_by_reuse,
    PINS.test_prefix_cache_enomem_changes_nothing,
    PINS.test_prefix_cache_block_after_a_different_prefix_is_not_reused,
]

MUTATIONS = {
    "fork_does_not_count": ("        for b in self.tables[child]:\n            self.ref[b] += 1",
                            "        for b in self.tables[child]:\n            pass"),
    "copy_on_write_when_unshared": ("            if self.ref[last] > 1:", "            if self.ref[last] >= 1:"),
    "dropped_beams_kept": ("                if i not in first:\n                    self.free_seq(b)",
                           "                if False:\n                    self.free_seq(b)"),
    "every_candidate_forks": ("            if p not in first:\n                first.add(p)",
                              "            if False:\n                first.add(p)"),
    "key_forgets_prefix": ("        data = (parent if parent is not None else bytes(32)) + b\"\".join(",
                           "        data = bytes(32) + b\"\".join("),
    "partial_block_cached": ("        nb, full = -(-L // self.B), L // self.B", "        nb, full = -(-L // self.B), -(-L // self.B)"),
    "revived_frame_stays_free": ("            if self.ref[f] == 0:\n                self.free.remove(f)",
                                 "            if False:\n                self.free.remove(f)"),
    "eviction_keeps_key": ("        key = self.frame_key.pop(b, None)", "        key = None"),
    "free_queue_lifo": ("                self.free.append(b)", "                self.free.appendleft(b)"),
}


def _mutant(old: str, new: str):
    src = open(MODEL).read()
    if old:
        assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
        src = src.replace(old, new)
    mod = types.ModuleType("allocator_model_mutant")
    exec(compile(src, MODEL + " (mutant)", "exec"), mod.__dict__)
    return mod


def _failing_pins(mod, monkeypatch):
    monkeypatch.setattr(PINS, "AllocatorModel", mod.AllocatorModel)
    monkeypatch.setattr(PINS, "AllocatorError", mod.AllocatorError)
    failed = []
    for call in PIN_CALLS:
        try:
            call()
        except (Exception, pytest.fail.Exception):  # assertion, pytest.raises miss or other error
            failed.append(getattr(call, "__name__", "lambda"))
    return failed


def test_unchanged_model_passes_every_pin(monkeypatch):
    assert _failing_pins(_mutant("", ""), monkeypatch) == []


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    failed = _failing_pins(_mutant(*MUTATIONS[name]), monkeypatch)
    assert failed, f"no pin caught the planted mistake {name}"
