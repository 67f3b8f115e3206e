"""The allocation-free forward (svdq_linear_forward_noalloc) against the workspace forward.

Some callers cannot allocate device memory while they run (a host framework that owns all device
memory and gives plugins no allocator, or a latency-critical path that cannot afford cudaMalloc's
possible device synchronisation).  For them the library keeps a fixed 20 MiB scratch array in its
own device module.  This file is collected last on purpose: it must pass both on its own in a
fresh process and after every other test.
"""
import numpy as np
import pytest

import synth
from oracle import svdq_oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import w4a4_rank_corrected_smooth_b200 as S  # noqa: E402

REL_FRO_TOL = 5e-3
MAX_ABS_TOL = 1e-2


def _bf16_dev(x_bits):
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).view(torch.bfloat16).cuda()


def _f64(Y):
    return O.bf16_to_f32(Y.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)


def test_noalloc_forward_matches_workspace_forward_on_two_calls():
    spec = synth.custom("noalloc", M=1000, K=1024, N=768, rank=32, seed=21)
    X = synth.activations_bf16(spec)
    lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(X), "nvfp4", spec.rank)
    Xd = _bf16_dev(X)
    Y_ws = lin.forward(Xd)  # existing entry point, caller-provided workspace
    torch.cuda.synchronize()
    ref = _f64(Y_ws)
    for _ in range(2):  # the second call reuses the scratch the first one left behind
        Y = torch.full((spec.M, spec.N), float("nan"), dtype=torch.bfloat16, device="cuda")
        lin.svdq_linear_forward_noalloc(Xd, spec.M, spec.K, Y, spec.N)
        torch.cuda.synchronize()
        S.svdq_get_device_error()
        got = _f64(Y)
        assert np.all(np.isfinite(got))
        assert O.rel_fro(got, ref) <= REL_FRO_TOL
        assert np.max(np.abs(got - ref)) <= MAX_ABS_TOL * np.max(np.abs(ref))
        # the same deterministic kernels on the same operands: identical bits, not just close
        assert torch.equal(Y.view(torch.int16), Y_ws.view(torch.int16))
    lin.close()


def test_noalloc_forward_rejects_shapes_beyond_the_fixed_scratch():
    spec = synth.custom("noalloc_big", M=16, K=3072, N=256, rank=32, seed=22)
    X = synth.activations_bf16(spec)
    lin = S.SVDQLinear(synth.weight_bf16(spec), None, synth.act_absmax(X), "nvfp4", spec.rank)
    # the row limit is the largest M whose workspace fits the 20 MiB scratch, found from the
    # library's own svdq_workspace_size (it moves with the workspace layout)
    lo, hi = 1, 1 << 20
    assert lin.workspace_size(lo) <= 20 << 20 < lin.workspace_size(hi)
    while hi - lo > 1:
        mid = (lo + hi) // 2
        lo, hi = (mid, hi) if lin.workspace_size(mid) <= 20 << 20 else (lo, mid)
    M = hi  # the first M that no longer fits
    assert all(lin.workspace_size(m) <= 20 << 20 for m in (1, lo // 2, lo))
    Yok = torch.zeros((lo, spec.N), dtype=torch.bfloat16, device="cuda")
    lin.svdq_linear_forward_noalloc(torch.zeros((lo, spec.K), dtype=torch.bfloat16, device="cuda"), lo, spec.K,
                                    Yok, spec.N)
    torch.cuda.synchronize()
    S.svdq_get_device_error()
    Xd = torch.zeros((M, spec.K), dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros((M, spec.N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(S.SVDQError) as ei:
        lin.svdq_linear_forward_noalloc(Xd, M, spec.K, Y, spec.N)
    assert ei.value.status == 1 and "fixed scratch" in str(ei.value)
    lin.close()


def test_noalloc_w4a16_needs_no_scratch_and_has_no_row_limit():
    """The W4A16 layer's one kernel uses no scratch: the allocation-free forward takes any M (here
    beyond the W4A4 layer's 20 MiB limit) and equals the ordinary forward bit for bit."""
    spec = synth.custom("noalloc_w4a16", M=64, K=3072, N=256, rank=0, seed=23)
    Xs = synth.activations_bf16(spec)
    lin = S.SVDQLinear(synth.weight_bf16(spec), synth.bias_bf16(spec), synth.act_absmax(Xs), "w4a16", 0)
    M = 12000
    X = np.tile(Xs, (M // 64 + 1, 1))[:M]
    Xd = _bf16_dev(X)
    Y_ref = lin.forward(Xd)
    Y = torch.full((M, spec.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    lin.svdq_linear_forward_noalloc(Xd, M, spec.K, Y, spec.N)
    torch.cuda.synchronize()
    S.svdq_get_device_error()
    assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16))
    lin.close()
