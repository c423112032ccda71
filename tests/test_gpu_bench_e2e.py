"""The benchmark's end-to-end leg (host buffers, copies pipelined across
layers on two copy streams) returns exactly what direct device calls of
fqt_linear_fwd / fqt_linear_bwd compute: a missing stream or event
dependency would let a layer read inputs before they land or copy out
outputs before they are written."""
import pytest
import torch

import bench
import fqt_synth as S

pytestmark = pytest.mark.gpu


def test_pipelined_e2e_outputs_match_direct_calls(gpu_lib):
    F = gpu_lib
    dev = torch.device("cuda", 0)
    N = K = 4096
    cfg = F.linear_cfg(F.NVFP4, out_dtype=F.OUT_BF16, seed=0)
    src = S.llama_linear(N, K, M=bench.M_TOKENS, seed=0)
    cache = {(N, K): src}
    layers = [bench.Layer(F, f"l{i}", N, K, cfg, src, dev) for i in range(3)]
    for L in layers:                      # stale device contents must not leak through
        L.x.zero_(); L.w.zero_(); L.dy.zero_(); L.y.fill_(7); L.dx.fill_(7); L.dw.fill_(7)
    ws = F.Workspace(device=dev)
    _ms, h2d, d2h, host = bench.e2e_run(F, layers, cache, cfg, ws, 2, dev)
    assert ws.status() == 0
    assert h2d == 3 * (2 * bench.M_TOKENS * K + 2 * N * K + 2 * bench.M_TOKENS * N)
    assert d2h == 3 * (2 * bench.M_TOKENS * N + 2 * bench.M_TOKENS * K + 4 * N * K)

    # the same layer computed directly on the device
    sv = F.Saved.empty(bench.M_TOKENS, N, K, cfg, device=dev, logical_scales=False)
    y = torch.empty((bench.M_TOKENS, N), dtype=torch.bfloat16, device=dev)
    dx = torch.empty((bench.M_TOKENS, K), dtype=torch.bfloat16, device=dev)
    dw = torch.empty((N, K), dtype=torch.float32, device=dev)
    F.fqt_linear_fwd(cfg, src["X"].to(dev), src["W"].to(dev), y, sv, ws)
    F.fqt_linear_bwd(cfg, src["dY"].to(dev), sv, dx, dw, ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    h = host[(N, K)]
    assert torch.equal(h["Y"], y.cpu())
    assert torch.equal(h["dX"], dx.cpu())
    assert torch.equal(h["dW"], dw.cpu())
