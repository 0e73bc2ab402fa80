"""The CPU oracle against its pins (golden example, closed forms, library routines,
invariants).  CPU only."""
import pytest

import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_config_constants_match_pages():
    """The workload sizes use the configuration values the pages print."""
    from synth import configs as C
    g = pins.load_golden("glm52_config_constants.txt")
    assert C.INDEX_HEADS == int(g["index_n_heads"][0])
    assert C.INDEX_DIM == int(g["index_head_dim"][0])
    assert C.DV == int(g["kv_lora_rank"][0])
    big = [w for w in C.WORKLOADS.values() if w.name != "tiny"]
    assert all(w.k == int(g["index_topk"][0]) for w in big)
    assert all(w.H == int(g["num_attention_heads"][0]) for w in big)
    assert all(w.L == int(g["index_topk_freq"][0]) for w in big if w.name != "mtp")
    assert C.WORKLOADS["mtp"].steps == int(g["mtp_steps"][0])
