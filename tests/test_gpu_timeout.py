"""The bounded waits of the tensor-core kernel, run out on purpose.

Every on-chip wait of the kernel (for a copy, an MMA, or other warps) gives
up after a limit; ``mla_dims.wait_limit_kcycles`` sets that limit.  With a
limit of a thousand cycles the first waits for copies from memory run out,
so each CTA records MLA_DEV_TIMEOUT in the workspace error word, lets the
copies and MMAs it has in flight finish, frees its tensor memory and exits.
Nothing traps and nothing hangs: the host reads the error word, and the next
call on the same stream computes the right answer with a clear error word.
"""
import pytest
import torch

import mla_latent_attention_b200 as mla
import mla_workloads as W
import oracle
from gpu_common import assert_matches_oracle, require_gpu

pytestmark = pytest.mark.gpu

MLA_DEV_TIMEOUT = 4


@pytest.mark.parametrize("kv", [W.KV_FP8, W.KV_BF16])
def test_wait_that_runs_out_stops_the_call_cleanly(kv):
    require_gpu()
    w = W.make_workload("long_ctx_142k", kv=kv, ctx_override=("fixed", 9001))
    wd = w.to("cuda")
    ws = torch.zeros(1 << 26, dtype=torch.uint8, device="cuda")
    mla.decode_workload(wd, kernel="tcgen05", workspace=ws, wait_limit_kcycles=1)
    code, info = mla.read_device_error(ws)
    assert code == MLA_DEV_TIMEOUT and info >= 0, (code, info)
    # the same stream goes on: a call with the default limit is clean and right
    mla.reset_device_error(ws)
    out, lse = mla.decode_workload(wd, kernel="tcgen05", workspace=ws)
    assert mla.read_device_error(ws) == (0, 0)
    ref_o, ref_l = oracle.decode_workload(w)
    assert_matches_oracle(out, lse, ref_o, ref_l, w.kv_dtype, f"after a stop ({kv})")
