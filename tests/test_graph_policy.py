"""Host logic of HostPipeline's graph use (no GPU): which steady-state calls
capture a CUDA graph, replay one, or enqueue their work directly."""
from mixture_experts_layer_53_b200 import GraphPolicy


def run(policy, keys):
    out = []
    for k in keys:
        how = policy.decide(k)
        if how == "capture":
            policy.stored(k, object())
        out.append(how)
    return out


def test_fresh_buffers_never_capture():
    p = GraphPolicy()
    assert run(p, [(i & 1, 1000 + i) for i in range(40)]) == ["direct"] * 40
    assert not p.graphs


def test_reused_buffers_capture_on_second_use_then_replay():
    p = GraphPolicy()
    keys = [(i & 1, 7 + (i & 1)) for i in range(8)]
    assert run(p, keys) == ["direct", "direct", "capture", "capture"] + ["replay"] * 4
    assert len(p.graphs) == 2


def test_graph_count_is_capped():
    p = GraphPolicy(max_graphs=2)
    keys = ["a", "b", "c"] * 4
    got = run(p, keys)
    assert got[:6] == ["direct", "direct", "direct", "capture", "capture", "direct"]
    assert got[6:] == ["replay", "replay", "direct"] * 2
    assert set(p.graphs) == {"a", "b"}


def test_memory_of_single_uses_is_bounded():
    p = GraphPolicy(max_seen=4)
    run(p, ["a", "b", "c", "d"])
    assert len(p.seen) == 4
    assert run(p, ["e"]) == ["direct"]  # full: cleared, then "e" remembered
    assert p.seen == {"e"}
    assert run(p, ["a", "e"]) == ["direct", "capture"]
