"""pa_decode_noalloc against pa_decode and the oracle, through the C ABI.

pa_decode_noalloc serves callers that cannot allocate device memory while they
decode (a plugin whose host pre-partitions device memory, a real-time loop
that must not take cudaMalloc's implicit synchronisation). It keeps its scratch
in a fixed 16 MiB array inside the library instead of a caller workspace.

Each case makes two calls in a row on different inputs: the second batch has
fewer sequences and shorter contexts than the first, so it has fewer work-list
entries and partitions than the first call left in the shared array, and a
missing reset of the cursor, the entry count or the merge counters would show.
Both calls run the same kernels with the same partitioning as pa_decode, so
each output must equal pa_decode's on the same inputs bit for bit; each is
also compared with the fp64 oracle within the attention tolerance. This file
is collected last so a failure here never hides the other tests' results.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_372_b200 as pa
from paged_kv_cache_372_b200 import build, workloads
from tests.bruteforce import bits_of

pytestmark = pytest.mark.gpu

TOL = {"f16": 2e-3, "bf16": 1e-2}


def _inputs(wl, num_seqs=None, ctx_div=1):
    """The first step of `wl` on cuda:0, optionally cut to its first num_seqs
    sequences with every context shortened to ceil(ctx / ctx_div)."""
    st = wl.steps[0]
    B = st.q.shape[0] if num_seqs is None else num_seqs
    ctx = -(-st.context_lens[:B].astype(np.int64) // ctx_div)
    dev = torch.device("cuda", 0)
    return dict(q_host=st.q[:B].contiguous(), tab_host=np.ascontiguousarray(st.block_tables[:B]),
                ctx_host=ctx.astype(np.int32),
                q=st.q[:B].contiguous().to(dev), kp=wl.k_pool.to(dev), vp=wl.v_pool.to(dev),
                tab=torch.from_numpy(np.ascontiguousarray(st.block_tables[:B])).to(dev),
                ctx=torch.from_numpy(ctx.astype(np.int32)).to(dev), max_ctx=int(ctx.max()))


def _call_noalloc(lib, wl, x, out, partition):
    B, H, D = x["q"].shape
    return lib.pa_decode_noalloc(
        out.data_ptr(), x["q"].data_ptr(), x["kp"].data_ptr(), x["vp"].data_ptr(), x["tab"].data_ptr(),
        x["ctx"].data_ptr(), B, H, wl.num_kv_heads, D, wl.block_size, x["tab"].shape[1], wl.num_blocks,
        x["max_ctx"], ctypes.c_float(wl.scale), pa.PA_F16 if wl.dtype == "f16" else pa.PA_BF16, partition,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("name,kw,partition", [
    ("llama7b", {"num_seqs": 16}, 0),      # split into 256-token partitions, merged in-kernel
    ("llama3_8b", {"num_seqs": 12}, 256),  # grouped heads, many partitions
    ("tiny", {}, 0),                       # one partition per sequence
])
def test_noalloc_equals_pa_decode_on_two_calls(name, kw, partition):
    build.build()
    lib = pa.lib()
    wl = workloads.build(name, 11, **kw)
    B = wl.num_seqs
    # Second call: fewer sequences, contexts a third as long (fewer entries and partitions).
    cases = [_inputs(wl), _inputs(wl, num_seqs=max(1, B // 2), ctx_div=3)]
    for call, x in enumerate(cases):
        ref = torch.empty_like(x["q"])
        pa.pa_decode(ref, x["q"], x["kp"], x["vp"], x["tab"], x["ctx"], wl.scale, x["max_ctx"], partition)
        out = torch.full_like(x["q"], float("nan"))
        status = _call_noalloc(lib, wl, x, out, partition)
        assert status == pa.PA_OK, (call, lib.pa_last_error())
        torch.cuda.synchronize()
        assert pa.pa_device_errors() == 0
        assert torch.equal(out, ref), (call, (out.float() - ref.float()).abs().max().item())
        want = oracle.paged_attention(bits_of(x["q_host"]), bits_of(wl.k_pool), bits_of(wl.v_pool),
                                      x["tab_host"], x["ctx_host"], wl.scale, wl.dtype)
        err = float(np.abs(out.float().cpu().double().numpy() - want).max())
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
