"""The allocation-free decode entry point (kvq_decode_attention_noalloc).

It exists for callers that cannot call cudaMalloc or hand the library a workspace
(for example a plugin inside a host program that owns the device allocator, or a C
caller whose device footprint must stay fixed after start-up). It runs the same
decode with its partials in a fixed device array inside the library. This file
checks, through the C ABI, that two calls in a row give the same output as the
workspace entry point within the parity tolerance (and as the CPU oracle), and that a
cache too large for the array is refused before anything runs. It is collected last on
purpose.
"""
import ctypes

import numpy as np
import pytest

from harness import check_close

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_workspace_decode():
    import torch
    from quantized_mixed_precision_qx_b200 import kvq
    from quantized_mixed_precision_qx_b200.synth import KVRecipe, Workload

    import oracle as orc
    wl = Workload(1, 1, 4, 24, 256, 3000, KVRecipe("outlier"), seed=21)
    g = kvq.KVCache(1, 1, 4, 24, 256, 3000, kvq.Q6_0, kvq.Q5_0, kvq.Q8_0, 1024)
    o = orc.Cache(1, 1, 4, 24, 256, 3000, orc.Q6_0, orc.Q5_0, orc.Q8_0, 1024)
    k, v = wl.kv_chunk(0, 0, 3000, "k"), wl.kv_chunk(0, 0, 3000, "v")
    g.append(0, torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda())
    o.append(0, k, v)
    assert kvq.kvq_decode_workspace_bytes(g.handle, 1) <= kvq.NOALLOC_WORKSPACE_BYTES
    q = torch.from_numpy(wl.q_decode(0, 0)).cuda()
    ref = g.decode(0, q, 0.8).cpu().numpy()
    vmax = float(np.abs(v).max())
    ref_oracle = o.decode(0, wl.q_decode(0, 0), 0.8)
    L = kvq.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        st = L.kvq_decode_attention_noalloc(g.handle, 0, ctypes.c_void_p(q.data_ptr()), ctypes.c_float(0.8),
                                            ctypes.c_void_p(out.data_ptr()), stream)
        assert st == kvq.OK, kvq.status_string(st)
        torch.cuda.synchronize()
        check_close(out.cpu().numpy(), ref, vmax, "noalloc decode")
        check_close(out.cpu().numpy(), ref_oracle, vmax, "noalloc decode vs oracle")


def test_noalloc_rejects_oversized_cache():
    import torch
    from quantized_mixed_precision_qx_b200 import kvq

    # 64 x 8 (batch x kv heads) units of 8 heads x 256 dims need more partials than the array holds
    g = kvq.KVCache(1, 64, 8, 64, 256, 64, kvq.Q4_0, kvq.Q4_0)
    assert kvq.kvq_decode_workspace_bytes(g.handle, 1) > kvq.NOALLOC_WORKSPACE_BYTES
    q = torch.zeros(64, 64, 256, device="cuda")
    out = torch.zeros_like(q)
    st = kvq.lib().kvq_decode_attention_noalloc(g.handle, 0, ctypes.c_void_p(q.data_ptr()), ctypes.c_float(1.0),
                                                ctypes.c_void_p(out.data_ptr()),
                                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == kvq.ERR_CAPACITY
    torch.cuda.synchronize()
    assert (out == 0).all()
