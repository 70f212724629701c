"""The CUDA-core decode kernel (built with -DPA_DECODE_TENSOR_MIN_GROUP=16)
against the oracle. The default library runs the tensor-core kernel for every
head group; this builds the alternative into a temporary library and checks it
on the same parity cases in a separate process."""
import os
import subprocess
import sys

import pytest

from paged_kv_cache_372_b200 import build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHECK = r'''
import sys
sys.path.insert(0, sys.argv[1])
import torch
import paged_kv_cache_372_b200 as pa
from paged_kv_cache_372_b200 import workloads
from tests import gpu_harness as H
for wl in (workloads.tiny(0), workloads.llama7b(1, num_seqs=6), workloads.llama3_8b(2, num_seqs=12)):
    for P in (None, 64):
        kp, vp = H.to_gpu(wl)
        okp, ovp = H.oracle_state(wl)
        out = H.gpu_step(wl, 0, kp, vp, P)
        ref = H.oracle_step(wl, 0, okp, ovp)
        torch.cuda.synchronize()
        assert pa.pa_device_errors() == 0
        assert H.pools_equal(kp, vp, okp, ovp)
        err = H.max_err(out, ref)
        assert err <= H.TOL[wl.dtype], (wl.name, P, err)
print("ok")
'''


def test_cuda_core_kernel_matches_oracle(tmp_path):
    lib = build.build(force=True, extra=["-DPA_DECODE_TENSOR_MIN_GROUP=16"], out=str(tmp_path / "libpa_cc.so"))
    env = dict(os.environ, PA_B200_LIB=lib)
    res = subprocess.run([sys.executable, "-c", CHECK, ROOT], cwd=ROOT, env=env, capture_output=True,
                         text=True, timeout=900)
    assert res.returncode == 0 and res.stdout.strip().endswith("ok"), res.stderr[-3000:]
