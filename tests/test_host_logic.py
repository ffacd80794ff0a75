"""Host-side logic without a GPU: byte accounting (whole sequences and sink +
window subsets, against a token-by-token count), the demotion workload's plan,
and the benchmark's replica plumbing (barrier + max over ranks) on two CPU
processes over gloo."""
import os
import subprocess
import sys
import textwrap

import pytest

from paged_long_context_b200 import accounting, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _brute_tokens(n, P, sink, window):
    pages = {}
    for j in range(n):
        if window <= 0 or j < sink or j >= n - window:
            pages[j // P] = pages.get(j // P, 0) + 1
    return pages


@pytest.mark.parametrize("n,P", [(1, 16), (100, 16), (513, 512), (4096, 256), (37, 8)])
@pytest.mark.parametrize("sink,window", [(0, 0), (0, 1), (4, 20), (50, 60), (3, 1000), (17, 5)])
def test_tokens_per_page_match_a_token_count(n, P, sink, window):
    want = _brute_tokens(n, P, sink, window)
    for p in range(-(-n // P)):
        assert accounting._tokens_in_page(n, p, P, sink, window) == want.get(p, 0)


def test_step_bytes_of_a_subset():
    spec = synth.CaseSpec("acct", 2, 4, 2, 64, 16, seq_lens=[100, 7], fmt="tiered",
                          tiers=[(0.5, "i8"), (0.5, "bf16")])
    case = synth.make_case(spec, 1, "cpu")
    full = accounting.step_bytes(case)
    sub = accounting.step_bytes(case, sink=4, window=20)
    # K+V bytes of exactly the tokens taking part, page by page in their formats
    kv = 0
    for b, n in enumerate([100, 7]):
        for p, cnt in _brute_tokens(n, 16, 4, 20).items():
            kv += cnt * 2 * case.num_kv_heads * synth.row_bytes(case.fmt_of_page(b, p), 64)
    assert sub["kv"] == kv and sub["kv"] < full["kv"]
    assert sub["tokens"] == 4 + 20 + 7
    assert full["tokens"] == 107


def test_cfr_byte_accounting_is_the_pages_figure():
    case = synth.workload("cfr")
    assert accounting.step_bytes(case)["kv"] == 32 * 33554432


def test_demotion_plan_covers_the_cold_pages_once():
    from paged_long_context_b200 import demote_workload
    spec = demote_workload.spec()
    # the plan without building pools: int4 for logical pages 0-31, int8 for 32-95
    assert demote_workload.TIERS == [(32, synth.I4), (96, synth.I8)]
    assert spec.batch * 96 == 768 and spec.page_tokens == 256


def test_replica_max_over_two_gloo_ranks(tmp_path):
    script = tmp_path / "ranks.py"
    script.write_text(textwrap.dedent(f"""
        import os, sys
        sys.path.insert(0, {ROOT!r})
        import bench
        d = bench.Dist(2, backend="gloo")
        d.barrier()
        m = d.max(10.0 + d.rank)          # each rank's own time
        d.barrier()
        print("rank", d.rank, "world", d.world, "max", m, flush=True)
        d.close()
    """))
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT="29617", WORLD_SIZE="2")
    procs = []
    for r in range(2):
        e = dict(env, RANK=str(r), LOCAL_RANK=str(r))
        procs.append(subprocess.Popen([sys.executable, str(script)], env=e, stdout=subprocess.PIPE,
                                      stderr=subprocess.STDOUT, text=True))
    outs = [p.communicate(timeout=120)[0] for p in procs]
    assert all(p.returncode == 0 for p in procs), outs
    for r, out in enumerate(outs):
        assert f"rank {r} world 2 max 11.0" in out, out
