"""The bounded-wait timeout path, made to run out without a fault or a hang.

sq_wait_selftest has one GPU thread wait on an mbarrier that nothing arrives
on, through the helper every tensor-core kernel of the library waits with,
with a limit of a few milliseconds: the wait gives up, SQ_FLAG_TIMEOUT is set
in the flag word, the kernel returns, and the context stays usable (a normal
compress afterwards still matches the oracle).
"""

import time

import numpy as np
import pytest
import torch

from gpu_helpers import calibrate_oracle, compare_compressed, records_to_device
from synthetic import make_workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

from compressed_attention_head_b200 import sq  # noqa: E402


def test_wait_runs_out_sets_the_flag_and_the_context_stays_usable():
    flags = torch.zeros(4, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    sq.sq_wait_selftest(3000, flags)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert flags[0].item() & sq.SQ_FLAG_TIMEOUT
    assert elapsed < 1.0, elapsed            # a 3 ms limit, not the kernels' 2 s
    # the context still works: a compress call matches the oracle
    w = make_workload("llama8b", batch=1, tokens=200)
    d = w.cfg["d"]
    cals = calibrate_oracle(w.k_cal[:2], 3.0, True)
    recs = records_to_device(cals)
    k = w.k[:, :2].contiguous().cuda()
    cache = sq.alloc_cache(1, 2, 224, cals[0].words, True)
    f2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    sq.sq_compress_kv(recs, None, k, None, 1, 2, d, 200, None, cache, None, f2)
    torch.cuda.synchronize()
    assert f2.item() == 0
    words = cache.words_u32()
    for h in range(2):
        compare_compressed(words[0, h, :200], cache.norm[0, h, :200].cpu().numpy(),
                           cache.rnorm[0, h, :200].cpu().numpy(), k[0, h].double().cpu().numpy(), cals[h])


def test_selftest_rejects_bad_arguments():
    flags = torch.zeros(4, dtype=torch.int32, device="cuda")
    for bad in (0, 2000001):
        with pytest.raises(sq.SqError) as e:
            sq.sq_wait_selftest(bad, flags)
        assert e.value.status == sq.SQ_ERR_ARG
