"""dsv4v_linear_residual_noalloc: the residual GEMM for callers that cannot allocate device
memory (no workspace; the library's static scratch holds the split-tile partials and counters).
Called through the C ABI twice in a row on shapes whose GEMM plan splits tiles, so the static
scratch is really used and reused; each result must match dsv4v_linear_residual with a
caller-allocated workspace."""
import numpy as np
import pytest
import torch

from vision_transformer_encoder_dsv4v_b200 import dsv4v as A

pytestmark = pytest.mark.gpu


def _bf16(shape, scale, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16).cuda()


def test_noalloc_matches_workspace_entry_point_twice():
    cfg = A.make_config(1024, 16, 2816, 2, 4096, 1)
    for call, (rows, k) in enumerate([(784, 2816), (784, 2816), (3562, 1024)]):
        a = _bf16((rows, k), 1.0, 10 + call)
        w = _bf16((1024, k), 0.02, 20 + call)
        x = _bf16((rows, 1024), 1.0, 30 + call)
        ws = torch.zeros(A.dsv4v_workspace_size(cfg, A.BatchRef([(rows, 1)])), dtype=torch.uint8, device="cuda")
        x_ref = x.clone()
        A.dsv4v_linear_residual(cfg, rows, k, a, w, x_ref, ws)
        x_new = x.clone()
        A.dsv4v_linear_residual_noalloc(cfg, rows, k, a, w, x_new)
        torch.cuda.synchronize()
        assert A.dsv4v_device_error() == 0
        g = x_new.float().cpu().numpy().astype(np.float64)
        r = x_ref.float().cpu().numpy().astype(np.float64)
        # the element-wise bf16 tolerance of the GEMM parity tests
        assert np.all(np.abs(g - r) <= 2.0 ** -8 * np.abs(r) + 2e-5), f"call {call}: max err {np.abs(g - r).max()}"


def test_noalloc_rejects_sizes_beyond_its_limit():
    cfg = A.make_config(1024, 16, 2816, 2, 4096, 1)
    a = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(A.Dsv4vError) as e:
        A.dsv4v_linear_residual_noalloc(cfg, A.DSV4V_NOALLOC_MAX_ROWS + 1, 1024, a, a, a)
    assert e.value.status == 2   # DSV4V_ERR_UNSUPPORTED, nothing launched


def test_noalloc_rejected_calls_enqueue_nothing():
    """A call the entry point refuses (an fp32 config, a K that is neither D nor F, too many rows)
    returns its error before putting any work on the stream: captured into a graph, it leaves
    the graph empty (so it cannot clear counters that a call on another stream is using)."""
    from cuda.bindings import runtime as rt

    cfg_bf16 = A.make_config(1024, 16, 2816, 2, 4096, 1)
    cfg_f32 = A.make_config(1024, 16, 2816, 2, 4096, 1, dtype=A.DSV4V_F32)
    a = _bf16((784, 1024), 1.0, 1)
    w = _bf16((1024, 1024), 0.02, 2)
    x = _bf16((784, 1024), 1.0, 3)
    A.dsv4v_linear_residual_noalloc(cfg_bf16, 784, 1024, a, w, x)  # first call on the device: outside capture
    torch.cuda.synchronize()
    err, s = rt.cudaStreamCreateWithFlags(rt.cudaStreamNonBlocking)
    assert err == rt.cudaError_t.cudaSuccess
    try:
        for cfg, rows, k, status in [(cfg_f32, 784, 1024, 2), (cfg_bf16, 784, 1000, 1),
                                     (cfg_bf16, A.DSV4V_NOALLOC_MAX_ROWS + 1, 1024, 2)]:
            (err,) = rt.cudaStreamBeginCapture(s, rt.cudaStreamCaptureMode.cudaStreamCaptureModeRelaxed)
            assert err == rt.cudaError_t.cudaSuccess
            with pytest.raises(A.Dsv4vError) as e:
                A.dsv4v_linear_residual_noalloc(cfg, rows, k, a, w, x, stream=int(s))
            err, graph = rt.cudaStreamEndCapture(s)
            assert err == rt.cudaError_t.cudaSuccess
            err, _, n_nodes = rt.cudaGraphGetNodes(graph, 0)
            assert err == rt.cudaError_t.cudaSuccess
            rt.cudaGraphDestroy(graph)
            assert e.value.status == status and n_nodes == 0
    finally:
        rt.cudaStreamDestroy(s)
