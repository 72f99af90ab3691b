"""The bounds-checked build (libmoba_checked.so, the sources compiled with
MOBA_CHECKED): its device index and bounds checks -- query rows, list
entries, partial rows, output and index rows, regroup positions -- record
MOBA_ERR_CHECK in the status word and skip the access instead of trapping.
On valid inputs no check may fire, and the results must equal the oracle's
as the ordinary build's do: the tensor-core and SIMT paths, varlen with an
empty sequence, GQA, shared routing, the prefix-mean gate, the sorting-
network gate, decode and backward. Each case runs in a child process (the
binding loads one library per process)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import torch
import long_context_prefill_block_b200 as moba
from long_context_prefill_block_b200 import build
from moba_inputs import small_case
from parity import check_forward
moba.use_library(build.LIB_CHECKED)
DEV = "cuda"
cases = [
    ((1000, 333, 0, 2048), 4, 2, 128, 128, 3, torch.bfloat16, False, False),
    ((2048, 700), 8, 2, 128, 128, 12, torch.bfloat16, False, False),
    ((900, 517), 4, 4, 64, 64, 4, torch.float32, False, False),
    ((2048, 1500), 8, 2, 128, 128, 4, torch.bfloat16, True, False),
    ((1500, 900), 4, 2, 128, 128, 3, torch.bfloat16, False, True),
]
for lengths, Hq, Hkv, d, B, topk, dtype, shared, prefix in cases:
    q, k, v, cu = small_case(lengths, Hq, Hkv, d, B, topk, dtype=dtype, seed=901)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    out, lse = moba.moba_forward(qd, kd, vd, cu, B, topk, return_lse=True,
                                 shared_routing=shared, prefix_mean=prefix)
    idx = moba.moba_gate_topk(qd, kd, cu, B, topk, shared_routing=shared, prefix_mean=prefix)
    torch.cuda.synchronize()
    st = moba.moba_device_status()
    assert st == 0, ("status", st, lengths)
    check_forward(q, k, v, cu, B, topk, out, lse, idx, shared_routing=shared, prefix_mean=prefix)
    dense = moba.dense_causal_forward(qd, kd, vd, cu)
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(5)).to(dtype).to(DEV)
    moba.moba_backward(qd, kd, vd, cu, out, lse, dout, B, topk, idx=idx, shared_routing=shared,
                       prefix_mean=prefix)
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0
# decode: the last position of every request
q, k, v, cu = small_case((700, 1100), 4, 2, 128, 128, 3, dtype=torch.bfloat16, seed=902)
kd, vd = k.to(DEV), v.to(DEV)
lens = (cu[1:] - cu[:-1]).tolist()
rows = torch.tensor([int(cu[r + 1]) - 1 for r in range(len(lens))])
qd = q[rows].contiguous().to(DEV)
kbar = moba.moba_meanpool(kd, cu, 128)
cu_q = torch.arange(0, len(lens) + 1, dtype=torch.int32)
out_d = moba.moba_decode(qd, kd, vd, cu, cu_q, kbar, 128, 3)
full = moba.moba_forward(q.to(DEV), kd, vd, cu, 128, 3)
torch.cuda.synchronize()
assert moba.moba_device_status() == 0
err = (out_d.float() - full[rows.to(DEV)].float()).abs().max().item()
assert err <= 2e-2, err
print("checked ok")
"""


def test_checked_build_fires_no_check_and_matches_the_oracle():
    from long_context_prefill_block_b200 import build

    if not os.path.exists(build.LIB_CHECKED):
        pytest.skip("checked build absent (python -m long_context_prefill_block_b200.build --checked)")
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "checked ok" in r.stdout
