"""Plant one plausible mistake at a time in a copy of the oracle's C source and
check that at least one pin catches it. This shows the pins constrain every
part of the oracle: decoders, slot arithmetic, pool layout, scores, softmax,
head grouping, the split-context merge, and the write / copy routines."""
import os
import subprocess

import pytest

import oracle
import pins

MUTANTS = {
    "scale_dropped": ("s[t] = scale * dot;", "s[t] = dot;"),
    "group_by_modulo": ("int g = h / group;", "int g = h % num_kv_heads;"),
    "slot_without_block_size": ("return (int64_t)table_row[logical_block] * block_size + offset;",
                                "return (int64_t)table_row[logical_block] + offset;"),
    "slot_offset_shifted": ("int64_t offset = pos % block_size;",
                            "int64_t offset = (pos + 1) % block_size;"),
    "pool_transposed": ("* block_size + offset) * head_dim + d;",
                        "* head_dim + d) * block_size + offset;"),
    "no_normalisation": ("out[d] /= denom;", "out[d] /= 1.0;"),
    "softmax_sign": ("double w = exp(s[t] - m);", "double w = exp(m - s[t]);"),
    "dot_drops_last": ("for (int d = 0; d < head_dim; ++d)\n            dot += q[d]",
                       "for (int d = 0; d < head_dim - 1; ++d)\n            dot += q[d]"),
    "v_is_k": ("out[d] += w * V[(size_t)t * head_dim + d];",
               "out[d] += w * K[(size_t)t * head_dim + d];"),
    "merge_unweighted": ("L += exp(m[p] - M) * l[p];", "L += l[p];"),
    "partition_drops_tail": ("int t1 = t0 + partition_tokens < n ? t0 + partition_tokens : n;",
                             "int t1 = t0 + partition_tokens < n ? t0 + partition_tokens : n - 1;"),
    "f16_bias": ("mag = ldexp((double)(1024 + f), e - 25);", "mag = ldexp((double)(1024 + f), e - 24);"),
    "bf16_bias": ("mag = ldexp((double)(128 + f), e - 134);", "mag = ldexp((double)(128 + f), e - 133);"),
    "write_skips_slot0": ("if (slot < 0)\n            continue;", "if (slot <= 0)\n            continue;"),
    "window_one_short": ("int lo = (window > 0 && n > window) ? n - window : 0;",
                         "int lo = (window > 0 && n > window) ? n - window + 1 : 0;"),
    "window_ignored": ("int lo = (window > 0 && n > window) ? n - window : 0;",
                       "int lo = 0;"),
    "window_rows_shifted": ("dst[(size_t)(t - lo) * head_dim + d] =\n                widen(pool[pool_index(block, kv_head, offset, d,",
                            "dst[(size_t)(t - lo) * head_dim + d] =\n                widen(pool[pool_index(block, kv_head, offset > 0 ? offset - 1 : 0, d,"),
    "swap_v_from_k": ("dst_v[(size_t)dst * block_elems + i] = src_v[(size_t)src * block_elems + i];",
                      "dst_v[(size_t)dst * block_elems + i] = src_k[(size_t)src * block_elems + i];"),
    "prefill_not_causal": ("int p = n - m + (tok - q_start[b]);", "int p = n - 1;"),
    "prefill_position_shifted": ("int p = n - m + (tok - q_start[b]);",
                                 "int p = n - m + (tok - q_start[b]) - (tok > q_start[b]);"),
    "prefill_window_one_short": ("int lo = (window > 0 && p + 1 > window) ? p + 1 - window : 0;",
                                 "int lo = (window > 0 && p + 1 > window) ? p + 2 - window : 0;"),
    "prefill_window_ignored": ("int lo = (window > 0 && p + 1 > window) ? p + 1 - window : 0;",
                               "int lo = 0;"),
    "copy_k_only": ("v_cache[(size_t)dst * block_elems + i] = v_cache[(size_t)src * block_elems + i];",
                    ";"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(oracle.SRC).read()
    assert old in src, f"anchor of mutant {name} not found in oracle.c"
    mutated = src.replace(old, new)
    c_path = os.path.join(tmp_path, "oracle_mutant.c")
    so_path = os.path.join(tmp_path, "liboracle_mutant.so")
    with open(c_path, "w") as f:
        f.write(mutated)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared", "-std=c11",
                    "-o", so_path, c_path, "-lm"], check=True)
    caught = []
    with oracle.using(so_path):
        for pin in pins.ALL_ORACLE_PINS:
            try:
                pin()
            except Exception as e:  # noqa: BLE001 -- any failure of a pin counts
                caught.append((pin.__name__, type(e).__name__))
                break
    assert caught, f"no pin caught the planted mistake {name}"


# Plausible mistakes in the block-manager model (oracle/allocator_model.py);
# the model pins must catch each.
MODEL_MUTANTS = {
    "cow_at_three_users": ("if self.ref[blk] > 1:", "if self.ref[blk] > 2:"),
    "window_releases_partial_block": ("for i in range(start // self.block_size):",
                                      "for i in range(-(-start // self.block_size)):"),
    "prefix_lookup_reaches_last_token": ("for i in range(max(n - 1, 0) // bs):",
                                         "for i in range(n // bs):"),
    "prefix_partial_block_cached": ("for i in range(len(shared), n // bs):",
                                    "for i in range(len(shared), -(-n // bs)):"),
    "prefix_evicts_newest": ("blk = next(iter(self.idle))", "blk = next(reversed(self.idle))"),
    "prefix_idle_not_free": ("return len(self.free) + len(self.idle)", "return len(self.free)"),
    "prefix_hit_left_idle": ("self.idle.pop(b, None)", "pass"),
    "prefix_hits_not_counted": ("unused = sum(1 for b in shared if self.ref[b] == 0)",
                                "unused = 0"),
    "prefix_not_kept_after_free": ("if blk in self.prefix_of:\n            self.idle[blk] = None",
                                   "if False:\n            self.idle[blk] = None"),
}


@pytest.mark.parametrize("name", sorted(MODEL_MUTANTS))
def test_model_pins_catch_mutant(name, tmp_path, monkeypatch):
    import importlib.util

    import oracle.allocator_model as am
    old, new = MODEL_MUTANTS[name]
    src = open(am.__file__).read()
    assert src.count(old) == 1, f"anchor of mutant {name} not found once in allocator_model.py"
    path = os.path.join(tmp_path, "allocator_model_mutant.py")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    spec = importlib.util.spec_from_file_location("allocator_model_mutant", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    monkeypatch.setattr(pins, "BlockManagerModel", mod.BlockManagerModel)
    monkeypatch.setattr(pins, "OutOfBlocks", mod.OutOfBlocks)
    caught = []
    for pin in pins.ALL_MODEL_PINS:
        try:
            pin()
        except Exception as e:  # noqa: BLE001 -- any failure of a pin counts
            caught.append((pin.__name__, type(e).__name__))
            break
    assert caught, f"no model pin caught the planted mistake {name}"


# Plausible mistakes in the oracle's Python placement helpers
# (oracle/__init__.py: place_history, new_token_slots), which build the pools
# every GPU parity test compares against; the oracle pins must catch each.
HELPER_MUTANTS = {
    "history_keeps_new_token": ("n = int(batch.context_lens[b]) - (0 if include_new else 1)",
                                "n = int(batch.context_lens[b])"),
    "history_drops_one_more": ("n = int(batch.context_lens[b]) - (0 if include_new else 1)",
                               "n = int(batch.context_lens[b]) - 1"),
    "new_token_at_len": ("slot(batch.block_tables[b], int(batch.context_lens[b]) - 1,",
                         "slot(batch.block_tables[b], int(batch.context_lens[b]),"),
    "new_token_first_position": ("slot(batch.block_tables[b], int(batch.context_lens[b]) - 1,",
                                 "slot(batch.block_tables[b], 0 * int(batch.context_lens[b]),"),
}


@pytest.mark.parametrize("name", sorted(HELPER_MUTANTS))
def test_pins_catch_helper_mutant(name, monkeypatch):
    old, new = HELPER_MUTANTS[name]
    src = open(oracle.__file__).read()
    assert src.count(old) == 1, f"anchor of mutant {name} not found once in oracle/__init__.py"
    # the module re-executed from the mutated text; it loads the same compiled oracle
    ns = {"__name__": "oracle_mutant", "__file__": oracle.__file__}
    exec(compile(src.replace(old, new), oracle.__file__, "exec"), ns)
    monkeypatch.setattr(oracle, "place_history", ns["place_history"])
    monkeypatch.setattr(oracle, "new_token_slots", ns["new_token_slots"])
    caught = []
    for pin in pins.ALL_ORACLE_PINS:
        try:
            pin()
        except Exception as e:  # noqa: BLE001 -- any failure of a pin counts
            caught.append((pin.__name__, type(e).__name__))
            break
    assert caught, f"no pin caught the planted mistake {name}"
