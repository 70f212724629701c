"""pa_decode_noalloc against pa_decode, through the C ABI.

pa_decode_noalloc serves callers that cannot allocate device memory while they
decode (a plugin whose host pre-partitions device memory, a real-time loop
that must not take cudaMalloc's implicit synchronisation). It keeps its scratch
in a fixed 16 MiB array inside the library instead of a caller workspace.
These checks call it twice in a row on the same inputs (the second call runs
on the array the first one left behind) and compare each output with
pa_decode's, within the attention tolerance of the parity tests. This file is
collected last so a failure here never hides the other tests' results.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_372_b200 as pa
from paged_kv_cache_372_b200 import build, workloads

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "bf16": 1e-2}


def _inputs(wl):
    st = wl.steps[0]
    dev = torch.device("cuda", 0)
    return dict(q=st.q.to(dev), kp=wl.k_pool.to(dev), vp=wl.v_pool.to(dev),
                tab=torch.from_numpy(st.block_tables).to(dev), ctx=torch.from_numpy(st.context_lens).to(dev),
                max_ctx=int(st.context_lens.max()))


def _call_noalloc(lib, wl, x, out, partition):
    B, H, D = x["q"].shape
    return lib.pa_decode_noalloc(
        out.data_ptr(), x["q"].data_ptr(), x["kp"].data_ptr(), x["vp"].data_ptr(), x["tab"].data_ptr(),
        x["ctx"].data_ptr(), B, H, wl.num_kv_heads, D, wl.block_size, x["tab"].shape[1], wl.num_blocks,
        x["max_ctx"], ctypes.c_float(wl.scale), pa.PA_F16 if wl.dtype == "f16" else pa.PA_BF16, partition,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("name,kw,partition", [
    ("llama7b", {"num_seqs": 16}, 0),      # split into 512-token partitions, merged in-kernel
    ("llama3_8b", {"num_seqs": 12}, 256),  # grouped heads, many partitions
    ("tiny", {}, 0),                       # one partition per sequence
])
def test_noalloc_matches_pa_decode_on_two_calls(name, kw, partition):
    build.build()
    lib = pa.lib()
    wl = workloads.build(name, 11, **kw)
    x = _inputs(wl)
    ref = torch.empty_like(x["q"])
    pa.pa_decode(ref, x["q"], x["kp"], x["vp"], x["tab"], x["ctx"], wl.scale, x["max_ctx"], partition)
    torch.cuda.synchronize()
    for call in range(2):
        out = torch.full_like(x["q"], float("nan"))
        status = _call_noalloc(lib, wl, x, out, partition)
        assert status == pa.PA_OK, (call, lib.pa_last_error())
        torch.cuda.synchronize()
        assert pa.pa_device_errors() == 0
        err = (out.float() - ref.float()).abs().max().item()
        assert np.isfinite(err) and err <= TOL[wl.dtype], (call, err)


def test_noalloc_rejects_sizes_beyond_its_array():
    lib = pa.lib()
    # 256 sequences x 32 heads x 64 partitions of fp32 partials is far above 16 MiB.
    need = pa.pa_decode_workspace_size(256, 32, 8, 128, 16, 32768, 512)
    assert need > pa.NOALLOC_SCRATCH_BYTES
    dummy = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    p = dummy.data_ptr()
    status = lib.pa_decode_noalloc(p, p, p, p, p, p, 256, 32, 8, 128, 16, 2048, 16, 32768,
                                   ctypes.c_float(0.1), pa.PA_BF16, 512, None)
    assert status == pa.PA_ERR_UNSUPPORTED
    assert b"16777216" in lib.pa_last_error()
    torch.cuda.synchronize()
    assert pa.pa_device_errors() == 0
