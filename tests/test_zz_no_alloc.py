"""kv2d_decode_attn_noalloc -- decode for callers that cannot allocate
device memory (a plugin inside a host that owns all memory, a runtime with a
fixed memory plan, or a loop that must not risk a device-synchronising
cudaMalloc).  It takes no workspace; its scratch is a fixed array inside the
library.  Its output must match the workspace entry point's, within the
decode tolerance, on two calls in a row (the second call must not be
disturbed by what the first left in the shared array).  Self-contained, so it
passes alone in a fresh process and after the rest of the suite."""
import pytest
import torch

from kv_cache_compression_kv2d_b200 import binding as B
from kv_cache_compression_kv2d_b200 import synth
from kv_cache_compression_kv2d_b200.synth import Workload

from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_workspace_decode():
    from kv_cache_compression_kv2d_b200 import build
    build.build()
    assert torch.cuda.is_available()
    wl = Workload("noalloc", 3, 2, 4, 128, 1537, 64, 24, 0.3, ragged_min=700)
    host = synth.generate(wl, seed=11, extra_capacity=8)
    run = H.make_run(wl, H.to_device(host), H.params_for(wl))
    H.compress(run)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        _, _, q = synth.decode_tokens(wl, call, seed=11, device="cuda", mu=run.batch.mu)
        ref = H.gpu_decode(run, q)
        out = torch.full_like(ref, float("nan"))
        B.kv2d_decode_attn_noalloc(run.p, wl.batch, run.cc.struct, run.dv, run.seq_len,
                                   run.batch.capacity, q, out, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert not torch.isnan(out).any()
        err = float((out.float() - ref.float()).abs().max())
        assert err <= H.TOL_OUT, f"call {call}: max abs difference {err}"
