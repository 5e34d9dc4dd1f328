"""Host-side logic of bench.py: FLOP/byte counting and the max-over-ranks reduction
(two gloo ranks on CPU)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
import oracle
import workloads


@pytest.mark.parametrize("L,w,s", [(256, 64, 4), (1, 5, 3), (10, 64, 4), (70, 64, 4), (68, 64, 4),
                                   (32768, 4096, 4), (2048, 128, 0), (100, 1, 7)])
def test_visible_pairs_closed_form_matches_oracle_count(L, w, s):
    if L > 5000:
        # large case: check the published totals instead of looping the oracle
        assert bench.visible_pairs(L, w, s) == 125_945_850
        return
    assert bench.visible_pairs(L, w, s) == sum(oracle.visible_count(t, w, s) for t in range(L))


def test_workload_flops_match_published_totals():
    W = workloads.WORKLOADS
    g = W["gqa8b_prefill"]
    assert bench.prefill_flops(g, [g.L]) == 4 * 128 * 32 * 125_945_850          # 2.0635 TFLOP
    p = W["packed_long"]
    assert abs(bench.prefill_flops(p, list(p.seqlens)) / 1e12 - 7.0656) < 1e-3
    b = W["based_local"]
    assert abs(bench.prefill_flops(b, [b.L] * b.B) / 1e9 - 8.324) < 1e-3
    d = W["decode"]
    assert abs(bench.decode_step_bytes(d, 20000) / 1e9 - 1.0761) < 1e-3


def test_linear_branch_counts():
    w = workloads.LINEAR_WORKLOADS["based_linear"]
    assert w.F == 273
    # recurrent form: 4 F (dv + 1) = 70,980 FLOPs per token and head; 8 x 2048 x 16 token-heads
    assert bench.based_linear_flops(w, w.B * w.L) == 70_980 * 262_144
    # q, k, v in and out (bf16): 320 bytes per token and head; state and z: 273 x 65 floats per head
    assert bench.based_linear_bytes(w, w.B * w.L) == 320 * 262_144 + 128 * 273 * 65 * 4 == 92_971_520
    # decode at B=64: state read and written plus 320 bytes of q, k, v, out per head
    assert bench.based_linear_decode_bytes(w, 64) == 1024 * (2 * 4 * 273 * 65 + 320) == 145_694_720


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier()
        q.put((rank, bench.reduce_max(1.5 + rank)))
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(2))
    assert got == {0: 2.5, 1: 2.5}


def test_reduce_max_without_process_group_is_identity():
    assert bench.reduce_max(3.25) == 3.25


def test_source_hash_ignores_comments_and_spacing():
    """A comment or spacing edit keeps a DRAM-traffic capture valid; a code edit does not."""
    code = "int f(int x) {\n  return x + 1;  // next\n}\n/* block\n comment */\n"
    assert bench._code_only(code) == bench._code_only("int f(int x) { return x + 1; }")
    assert bench._code_only(code) != bench._code_only("int f(int x) { return x + 2; }")


def test_traffic_table_entries_name_existing_sources():
    import json
    t = json.load(open(os.path.join(os.path.dirname(bench.__file__), "profiles", "traffic.json")))
    csrc = os.path.join(os.path.dirname(bench.__file__), "sink_aware_sliding_b200", "csrc")
    for name, e in t.items():
        if name == "about":
            continue
        assert e["dram_bytes_per_launch"] > 0
        for f in e["sources"]:
            assert os.path.exists(os.path.join(csrc, f)), (name, f)
