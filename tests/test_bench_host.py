"""Host-side pieces of bench.py (no GPU): the source hash that keys the
committed ncu traffic record, and the accept byte count."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_code_hash_ignores_comments_and_layout_only():
    b = load_bench()
    src = "int f(int x) {\n  // the next line\n  return x + 1; /* done */\n}\n"
    same = "int f(int x) { return x + 1; }  // reflowed, comments changed\n"
    other = "int f(int x) {\n  return x + 2;\n}\n"
    assert b._code_only(src) == b._code_only(same)
    assert b._code_only(src) != b._code_only(other)


def test_recorded_traffic_matches_only_its_workload_and_sources():
    b = load_bench()
    h = b.kernel_source_hash()
    assert len(h) == 16
    import json
    with open(os.path.join(ROOT, "profiles", "attention_traffic.json")) as f:
        rec = json.load(f)
    # another workload never borrows the record
    assert b.recorded_traffic(rec["workload"] + "_other") is None
    got = b.recorded_traffic(rec["workload"])
    if rec["kernel_hash"] == h:
        assert got == rec["dram_bytes_per_call"]
    else:
        assert got is None


def test_accept_bytes_chain_counts_the_pass_of_each_outcome():
    # 4VBN (every logit) + 4B(N-1) (draft probabilities at the drafts)
    # + 8V per sequence that stopped at a rejection (logit row + the rejected
    # child's draft row) + 4V per sequence that accepted every draft (p row)
    b = load_bench()

    class Acc:
        num_seqs, num_rows, vocab, temperature, tree_parents = 3, 5, 1000, 1.0, None

    lens = [0, 2, 4]
    paths = [[-1] * 4, [1, 2, -1, -1], [1, 2, 3, 4]]
    B, N, V, R = 3, 5, 1000, 2
    want = 4 * V * B * N + 4 * B * (N - 1) + 8 * V * R + 4 * V * (B - R)
    assert b.accept_bytes(Acc, lens, paths) == want
    Acc.temperature = 0.0
    assert b.accept_bytes(Acc, lens, paths) == 4 * V * B * N


def test_accept_bytes_tree_charges_every_rejected_child_row():
    b = load_bench()

    class Acc:
        num_seqs, num_rows, vocab, temperature = 2, 4, 100, 1.0
        tree_parents = [-1, 0, 0, 1]  # root with children 1, 2; node 1 with child 3

    # seq 0 stops at the root (two children rejected); seq 1 at node 3 (a leaf)
    lens = [0, 2]
    paths = [[-1, -1, -1], [1, 3, -1]]
    want = 4 * 100 * 2 * 4 + 4 * 2 * 3 + 4 * 100 * (1 + 2) + 4 * 100
    assert b.accept_bytes(Acc, lens, paths) == want
