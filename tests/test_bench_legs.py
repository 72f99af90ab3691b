"""The bench's CPU legs and bookkeeping (CPU only): the algorithmic bytes of
the memory-bound stages against hand-worked figures, the choice of the tensor
peak, the parity statistics of the CPU leg (zero against the oracle's own
results, and a planted mistake in the compared rows caught), the input
hashes, and one short run of the reference arm as the driver launches it."""
import hashlib
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import bench
import oracle
from moba_inputs import WORKLOADS, Workload, make_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_stage_bytes_hand_worked():
    # scaling_8k: 4 x 8192 tokens, 16 heads, d = 128, bf16, B = 512, k = 3
    w = WORKLOADS["scaling_8k"]
    sb = bench.stage_bytes(w)
    T = 4 * 8192
    assert sb["meanpool"] == T * 16 * 128 * 2 + 4 * 16 * 16 * 128 * 4
    idx = T * 16 * 3 * 4
    assert sb["gate_topk"] == T * 16 * 128 * 2 + idx
    # history pairs: min(2, c) per query of block c, 16 blocks of 512 queries
    pairs = 4 * 16 * 512 * sum(min(2, c) for c in range(16))
    assert bench.history_pairs(w) == pairs
    assert sb["regroup"] == 2 * idx + 4 * pairs


def test_history_pairs_million_token_shape():
    w = WORKLOADS["llama_1m"]
    # 256 blocks of 4096 queries, min(11, c) earlier blocks each, 32 heads
    assert bench.history_pairs(w) == 32 * 4096 * sum(min(11, c) for c in range(256))


def test_tensor_peak_choice():
    pk = {"bf16_tflops": 1671.7, "bf16_tflops_sustained": 1420.2}
    assert bench.tensor_peak(pk, 20.0) == (1420.2, "sustained")
    assert bench.tensor_peak(pk, 0.3) == (1671.7, "burst")
    assert bench.tensor_peak({"bf16_tflops": 1500.0}, 5.0) == (1500.0, "sustained")


def _leg():
    w = Workload("legs", (700, 300), 4, 2, 64, 64, 3, torch.float32, 4242, 1.0, 0.5)
    q, k, v, cu = make_inputs(w, "cpu")
    leg = bench.time_oracle(w, k, v, cu, bench.q_rows_from(q), budget_s=0.2, n_rows=500)
    return w, q, k, v, cu, leg


def test_parity_stats_zero_against_the_oracle_itself():
    w, q, k, v, cu, leg = _leg()
    out, lse, idx, gap = leg["result"]
    st = bench.parity_stats(w, leg, k, v, cu, out.astype(np.float32), lse.astype(np.float32), idx)
    assert st["pass"] and st["rows"] == 500
    assert st["index_mismatch_rows"] == 0 and st["index_mismatch_beyond_tie"] == 0
    assert st["max_abs_err"] < 1e-6
    assert sum(st["topk_margin_hist"].values()) == 500
    # rows with fewer than k - 1 earlier blocks reject nothing: margin "none"
    t = leg["rows"] // w.num_q_heads
    starts = np.array([0, 700])
    b = np.searchsorted(starts, t, side="right") - 1
    c = (t - starts[b]) // w.block_size
    assert st["topk_margin_hist"]["none"] == int((c <= w.topk - 1).sum())


def test_parity_stats_catch_a_planted_mistake():
    w, q, k, v, cu, leg = _leg()
    out, lse, idx, gap = leg["result"]
    bad_out = out.astype(np.float32).copy()
    bad_out[17, 5] += 1e-3  # beyond the fp32 tolerance
    st = bench.parity_stats(w, leg, k, v, cu, bad_out, lse.astype(np.float32), idx)
    assert not st["pass"] and st["max_abs_err"] >= 9e-4
    # a wrong block choice on a row with a clear margin
    bad_idx = idx.copy()
    r = int(np.nonzero((gap > 1e-2) & np.isfinite(gap))[0][0])
    row = bad_idx[r]
    row[0] = row[0] + 1 if row[1] != row[0] + 1 else row[0] - 1
    st = bench.parity_stats(w, leg, k, v, cu, out.astype(np.float32), lse.astype(np.float32),
                            bad_idx)
    assert st["index_mismatch_beyond_tie"] == 1 and not st["pass"]


def test_input_hashes_are_sha256_of_the_stored_bits():
    x = torch.arange(10, dtype=torch.float32).to(torch.bfloat16)
    h = bench.input_hashes({"x": x})["x"]
    assert h == hashlib.sha256(x.view(torch.int16).numpy().tobytes()).hexdigest()


@pytest.mark.skipif(torch.cuda.is_available(), reason="CPU run of the reference arm")
def test_reference_arm_prints_one_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_fp32", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["config"]["workload"] == "tiny_fp32"


def test_run_cli_workload_overrides():
    """The profiling CLI keeps the named workload's heads, dtype and seed and only replaces
    the shape fields it is given (one sequence of --tokens)."""
    from long_context_prefill_block_b200.run import workload
    from moba_inputs import WORKLOADS
    base = WORKLOADS["llama_1m"]
    assert workload("llama_1m", None, None, None) is base
    w = workload("llama_1m", 131072, 512, None)
    assert w.lengths == (131072,) and w.block_size == 512 and w.topk == base.topk
    assert (w.num_q_heads, w.num_kv_heads, w.head_dim, w.dtype, w.seed) == \
        (base.num_q_heads, base.num_kv_heads, base.head_dim, base.dtype, base.seed)
    assert -(-w.max_seqlen // w.block_size) == 256  # the million-token gate's block count
