"""pa_decode_noalloc: decode without a caller-allocated workspace.

For callers that cannot allocate device memory (an engine whose memory is all
reserved at start-up, a C program that only receives ready-made buffers), the
library offers a decode entry point whose split-K scratch is its own fixed
16 MiB device array.  Checked here through the C ABI against pa_decode with a
caller workspace, on two calls in a row (the second reuses the array with the
first call's contents still in it), within the attention tolerance the other
tests use, with a checked-mode error flag that must stay 0.  A case short
enough to need no scratch at all (one partition) goes through the same entry
point.  This file is collected last so a stop at the first failure has
already run everything else; it also passes alone in a fresh process.
"""

from __future__ import annotations

import pytest
import torch

from paged_kv_attention_35_b200 import synth
from paged_kv_attention_35_b200.workloads import DecodeWorkload
from tests.gpu_cases import TOL_MAX, TOL_MEAN

pytestmark = pytest.mark.gpu


def _close(a: torch.Tensor, b: torch.Tensor):
    err = (a.double() - b.double()).abs()
    assert torch.isfinite(a.float()).all()
    assert float(err.max()) <= TOL_MAX and float(err.mean()) <= TOL_MEAN


def _twice_against_pa_decode(w, expect_scratch: bool):
    from paged_kv_attention_35_b200 import ops
    need = ops.decode_workspace_size(w.B, w.hq, w.hkv, w.d, w.max_context_len)
    assert (0 < need <= ops.NOALLOC_SCRATCH_BYTES) if expect_scratch else need == 0
    ref = w.step().clone()                                 # pa_decode, caller workspace
    torch.cuda.synchronize()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = []
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        ops.decode_noalloc(w.d_q, w.kc, w.vc, w.d_bt, w.d_cl, w.max_context_len, out=out,
                           err_flag=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        _close(out, ref)
        outs.append(out)
    _close(outs[1], outs[0])


def test_noalloc_decode_matches_pa_decode(cuda_device):
    w = DecodeWorkload.from_spec(synth.WORKLOADS["qwen3_0p6b_decode"]).upload("cuda")
    _twice_against_pa_decode(w, expect_scratch=True)       # the split-K path


def test_noalloc_decode_other_shape_after_first(cuda_device):
    """A second workload (7B-GQA shape, block 16) through the same shared scratch."""
    lens = synth.uniform_lengths(64, 512, 4096, 77).tolist()
    w = DecodeWorkload(lens, 28, 4, 128, 16, seed=77).upload("cuda")
    _twice_against_pa_decode(w, expect_scratch=True)


def test_noalloc_decode_without_scratch(cuda_device):
    """The tiny decode step (4 seqs, contexts <= 255) fits one partition: no scratch used."""
    w = DecodeWorkload.from_spec(synth.WORKLOADS["tiny_decode"]).upload("cuda")
    _twice_against_pa_decode(w, expect_scratch=False)


def test_noalloc_rejects_sizes_beyond_the_scratch(cuda_device):
    from paged_kv_attention_35_b200 import ops
    # 256 seqs x 28 heads x 64 partitions of 64 tokens: ~238 MB of partials > 16 MiB
    need = ops.decode_workspace_size(256, 28, 4, 128, 4096, 64)
    assert need > ops.NOALLOC_SCRATCH_BYTES
    q = torch.zeros(256, 28, 128, dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros(64, 256, 4, 128, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(256, 16, dtype=torch.int32, device="cuda")
    cl = torch.full((256,), 4096, dtype=torch.int32, device="cuda")
    with pytest.raises(RuntimeError, match="PA_ERR_WORKSPACE"):
        ops.decode_noalloc(q, pool, pool, bt, cl, 4096, partition_size=64)
