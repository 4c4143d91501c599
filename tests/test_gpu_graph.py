"""The hot path captured in a CUDA graph (one graph per refinement step, as a
serving loop would run it) replays to the same bits as the eager calls.

Every entry point launches on the caller's stream, allocates nothing and
takes its scratch from the caller, so a whole step -- merge, re-noise, a
merged-LoRA layer, an Euler step, the last projection with the Euler update
and the MXFP8 layer -- can be captured; the eager run that comes first also
fills the host-side caches (kernel attributes, occupancy queries) that must
not be filled during a capture.
"""

import pytest
import torch

import lora_gemm_b200 as lg
import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_step_in_a_cuda_graph_matches_eager():
    w = synth.WORKLOADS["tiny"]
    K, N = w.shapes[0]
    T = w.height * w.width
    C = w.channels
    x = synth.activations(w, K, 0, DEV)
    W = synth.weight(w, 0, DEV)
    As, Bs = synth.adapters(w, 0, DEV)
    Wo = synth.weight(w, synth.PROJ_OUT_LAYER, DEV, shape=(K, C))
    up = synth.upscaled_latent(w, DEV)
    v = synth.velocity(w, 0, DEV)
    R = sum(synth.ADAPTER_RANKS)
    A_cat = torch.empty((R, K), dtype=torch.float32, device=DEV)
    B_cat = torch.empty((N, R), dtype=torch.float32, device=DEV)
    y = torch.empty((w.tokens, N), dtype=torch.bfloat16, device=DEV)
    y8 = torch.empty_like(y)
    z = torch.empty_like(up)
    zb = torch.empty(up.shape, dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(lg.lora_linear_workspace_size(w.tokens, K, N, R), dtype=torch.uint8, device=DEV)
    ws_e = torch.empty(lg.lora_linear_euler_workspace_size(w.tokens, K, C, R), dtype=torch.uint8, device=DEV)
    xq = lg.mx_quantize(x)
    wq = lg.mx_quantize(W)
    s = [float(torch.tensor(t, dtype=torch.float32)) for t in synth.SIGMA_SCHEDULE]

    def step():
        lg.lora_merge(As, Bs, synth.ADAPTER_SCALES, A_cat, B_cat)
        lg.renoise(up, s[0], w.seed, out=z)
        lg.lora_linear(x, W, A_cat, B_cat, y=y, workspace=ws)
        lg.euler_step(z, v, s[0], s[1])
        lg.mx_quantize(x, codes=xq[0], scales=xq[1])
        lg.lora_linear_mxfp8(x, xq, wq, A_cat, B_cat, y=y8, workspace=ws)
        lg.lora_linear_euler(x, Wo, A_cat, B_cat[:C], z, s[1], s[2], T, z_bf16=zb, workspace=ws_e)

    step()
    torch.cuda.synchronize()
    eager = [t.clone() for t in (A_cat, B_cat, y, y8, z, zb)]
    for t in (A_cat, B_cat, y, y8, z, zb):
        t.zero_()

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            step()
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert lg.get_last_device_error() == lg.LG_OK
    for got, ref in zip((A_cat, B_cat, y, y8, z, zb), eager):
        assert torch.equal(got.view(torch.uint8) if got.dtype == torch.bfloat16 else got,
                           ref.view(torch.uint8) if ref.dtype == torch.bfloat16 else ref)
    del g
