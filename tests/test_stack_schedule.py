"""The model's own layer stack (no GPU): workloads.production_stack against
the schedule and shapes the pages print ("Model Setup Numbers Without Jargon";
mengman.github.io 3.3, 3.4), and the cache sharing the three modes imply
("The Three Modes Full Reindex And Reuse": FULL builds its own main KV and
indexer keys, REINDEX and REUSE use the latest FULL's)."""
import json
import os

from fp4_kv_cache_step_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def _facts():
    with open(GOLDEN) as f:
        return json.load(f)


def test_schedule_matches_the_pages():
    f = _facts()
    ls = f["layer_schedule"]
    st = wl.production_stack(1 << 20, 4)
    assert st.swa_only + len(st.layers) == ls["layers"]
    assert st.swa_only == ls["swa_only_layers"]
    enc = st.segments[:ls["encoder_groups"]]
    dec = st.segments[ls["encoder_groups"]:]
    assert len(dec) == 1                                    # one decoder cache
    assert sum(len(w.modes) for w in enc) == ls["encoder_csa2_layers"]
    for w in enc:
        assert list(w.modes) == ls["encoder_group"]
        assert w.N * ls["encoder_tokens_per_entry"] == 1 << 20
        assert w.C == 0                                     # no pool in the encoder
    d = dec[0]
    assert len(d.modes) == ls["decoder_layers"]
    groups = [list(d.modes[i:i + 4]) for i in range(0, 20, 4)]
    assert len(groups) == ls["decoder_groups"]
    assert groups[0] == ls["decoder_first_group"]
    assert all(g == ls["decoder_other_groups"] for g in groups[1:])
    assert d.N * ls["decoder_tokens_per_entry"] == 1 << 20


def test_shapes_and_pool_match_the_pages():
    f = _facts()
    st = wl.production_stack(1 << 20, 4)
    hp = f["hierarchical_pool"]
    for w in st.segments:
        assert w.K == f["model_top_k"]["value"]
        assert (w.Hi, w.Di) == (f["indexer_shape"]["heads"], f["indexer_shape"]["dim"])
        assert (w.Hq, w.D) == (f["attention_shape"]["query_heads"], f["attention_shape"]["head_dim"])
    d = st.segments[-1]
    assert d.pool_block == hp["block_size"] and d.C == hp["positions"]
    assert d.C // d.pool_block == hp["blocks"]


def test_layers_run_in_model_order_and_segments_have_their_own_caches():
    st = wl.production_stack(4096, 2)
    seen = [seg for seg, _ in st.layers]
    assert seen == sorted(seen)                             # encoder groups, then the decoder
    assert len({w.seed for w in st.segments}) == len(st.segments)   # distinct caches
    assert [l for seg, l in st.layers if seg == 0] == list(range(6))
