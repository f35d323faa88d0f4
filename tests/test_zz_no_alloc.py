"""kv2d_decode_attn_noalloc -- decode for callers that cannot allocate
device memory (a plugin inside a host that owns all memory, a runtime with a
fixed memory plan, or a loop that must not risk a device-synchronising
cudaMalloc).  It takes no workspace; its scratch is a fixed array inside the
library.  It runs the same deterministic kernel with the same split as the
workspace entry point, so its output must equal that entry point's bit for
bit, on two calls in a row (the second call must not be disturbed by what
the first left in the shared array).  Two batch shapes: few units (every
unit cut into the same number of CTA pieces) and more units than half the
SMs (the batch's bytes shared out evenly, units straddling CTAs, so the
per-unit tickets in the shared array decide which CTA merges).
Self-contained, so it passes alone in a fresh process and after the rest of
the suite."""
import pytest
import torch

from kv_cache_compression_kv2d_b200 import binding as B
from kv_cache_compression_kv2d_b200 import synth
from kv_cache_compression_kv2d_b200.synth import Workload

from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [
    # 6 units of up to 1537 tokens: each unit gets its own CTAs
    Workload("noalloc_few", 3, 2, 4, 128, 1537, 64, 24, 0.3, ragged_min=700),
    # 160 units of 300..900 tokens (more units than half the SMs): shares
    # of the batch-wide byte range, several units per CTA
    Workload("noalloc_many", 20, 8, 4, 128, 900, 64, 32, 0.3, ragged_min=300),
], ids=lambda w: w.name)
def test_noalloc_decode_equals_workspace_decode(shape):
    from kv_cache_compression_kv2d_b200 import build
    build.build()
    assert torch.cuda.is_available()
    wl = shape
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
        assert torch.equal(out, ref), (
            f"call {call}: max abs difference {float((out.float() - ref.float()).abs().max())}")
