"""Pins against numbers the pages print (tests/golden/page_constants.json)."""

import json
import math
import os

from oracle import spark_oracle as so
from spark_gen import WORKLOADS

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")))


def test_reference_workload_matches_page_token_count():
    w = WORKLOADS["ref_72576"]
    assert w.N == GOLD["tokens_10s_768p"]["value"]
    assert w.nb == GOLD["blocks_10s_768p"]["value"]
    assert w.N % GOLD["block_tokens"]["value"] == 0
    W, H = GOLD["resolution"]["value"]
    assert w.grid[1:] == (H // 16, W // 16)


def test_ratio_sweep_matches_node_choices():
    w = WORKLOADS["ref_72576"]
    assert tuple(w.sweep()) == tuple(GOLD["topk_ratio_choices"]["value"])
    assert w.ratio == GOLD["topk_ratio_default"]["value"]
    # blocks kept at each ratio: ceil(r * 1134)
    assert [so.num_selected(w.nb, r) for r in w.sweep()] == [114, 227, 341]


def test_min_tokens_is_whole_blocks():
    mt = GOLD["min_tokens_default"]["value"]
    assert mt % 64 == 0 and mt // 64 == 192


def test_every_workload_is_whole_blocks_and_tiles():
    for w in WORKLOADS.values():
        assert w.N % 64 == 0
        F, Hl, Wl = w.grid
        assert F % 2 == 0 and Hl % 8 == 0 and Wl % 4 == 0     # 2x8x4 positional tiles fit
        assert w.nb >= 2 and math.ceil(math.log2(w.nb)) >= 1
