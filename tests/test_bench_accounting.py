"""The bench's FLOP accounting (CPU): useful FLOPs are 4*d per (query, head,
attended key), counted over the chosen keys only. Pinned three ways: against
the per-workload figures worked out by hand from eq. (9)'s key count (the
own block contributes p - cB + 1 keys, each earlier chosen block B keys),
against the keys the oracle's own index rows select on small random inputs,
and the row-sampled and index-derived counters against the closed form."""
import numpy as np
import pytest
import torch

import bench
import oracle
from moba_inputs import WORKLOADS, Workload, small_case


# (workload, useful FLOPs, dense causal FLOPs) as the hand-worked table prints
# them; each figure must agree to half a unit of its last printed digit.
@pytest.mark.parametrize("name,useful,dense", [
    ("tiny_fp32", "7.1e7", "1.3e8"),
    ("scaling_8k", "3.18e11", "1.10e12"),
    ("long_32k", "6.75e11", "8.80e12"),
    ("micro_32k", "7.95e10", "2.75e11"),
    ("llama_1m", "7.91e14", "9.01e15"),
])
def test_workload_flops_match_the_hand_worked_table(name, useful, dense):
    def half_ulp(s):
        mant, exp = s.split("e")
        return 0.5 * 10.0 ** (int(exp) - (len(mant) - 2))

    u, h, c, dn = bench.flop_counts(WORKLOADS[name])
    assert u == h + c
    assert abs(u - float(useful)) <= half_ulp(useful)
    assert abs(dn - float(dense)) <= half_ulp(dense)


def test_scaling_shape_closed_form():
    # 4 x 8192 tokens, 16 heads, d = 128, B = 512, k = 3: per sequence the
    # own block gives 16 blocks x (512 * 513 / 2) keys, the history blocks
    # 512 keys for each earlier chosen block: min(2, c) per query of block c.
    w = WORKLOADS["scaling_8k"]
    own = 16 * 512 * 513 // 2
    hist = 512 * 512 * sum(min(2, c) for c in range(16))
    expect = 4 * 128 * (own + hist) * 16 * 4
    assert bench.flop_counts(w)[0] == expect


@pytest.mark.parametrize("lengths,B,topk", [((300, 0, 517), 64, 3), ((1000,), 100, 4), ((64, 64), 16, 1)])
def test_flops_equal_the_keys_the_oracle_selects(lengths, B, topk):
    Hq, Hkv, d = 2, 1, 64
    q, k, v, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=torch.float32, seed=77)
    idx, _ = oracle.gate_topk(q, k, cu, B, topk)
    # attended keys per (row, head) from the oracle's index rows
    keys = 0
    cu_np = cu.numpy()
    for b in range(len(lengths)):
        for p in range(int(cu_np[b + 1] - cu_np[b])):
            t = int(cu_np[b]) + p
            c = p // B
            for h in range(Hq):
                for e in idx[t, h]:
                    if e < 0:
                        continue
                    keys += B if e < c else p - c * B + 1
    w = Workload("t", tuple(lengths), Hq, Hkv, d, B, topk, torch.float32, 0, 1.0, 0.3)
    useful, hist, cur, _ = bench.flop_counts(w)
    assert useful == 4 * d * keys
    fh, fc = bench.flops_from_indices(torch.from_numpy(idx), cu, B, d)
    assert (fh, fc) == (hist, cur)
    rows = np.arange(sum(lengths) * Hq)
    assert bench.row_flops(w, rows) == useful


def test_gate_flops_count_the_complete_earlier_blocks():
    # 2 * d per scored block: query p of block c scores blocks 0 .. c-1
    w = Workload("g", (1000, 1), 3, 1, 64, 128, 3, torch.float32, 0, 1.0, 0.3)
    scored = sum(p // 128 for p in range(1000))
    assert bench.gate_flops(w) == 2 * 64 * 3 * scored
    assert bench.gate_flops(WORKLOADS["llama_1m"]) == 2 * 128 * 32 * 4096 * (256 * 255 // 2)
