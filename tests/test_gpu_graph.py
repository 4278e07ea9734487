"""The step captured in a CUDA graph and replayed (as bench.py times it).

select -> plan -> attention through the C ABI on a side stream inside
torch.cuda.graph: every call of the step only enqueues work on the stream it
is given (no host synchronisation, allocation or host read-back), so the
captured graph replays the same kernels.  The replayed output must equal
the eagerly launched output bit for bit (the kernels are deterministic for
fixed inputs and lists), replays must repeat it, and the replayed lists must
be the eager lists.  Covered: the SDXL config with content selection, and a
head-masked layer of the stack (skipped heads zeroed by the graph too).
"""
import numpy as np
import pytest
import torch

from tests.gpu_util import dev_bf16
from workloads import WORKLOADS, head_mask_for_layer, make_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import prompt_aware_head_b200 as sa
    return sa


@pytest.mark.parametrize("name,rho,layer", [("sdxl", 0.3, None), ("stack", 0.5, 3)])
def test_step_replayed_as_graph_matches_eager(sa, name, rho, layer):
    w = WORKLOADS[name]
    B, H, N, d = w.B, w.H, w.N, w.d
    mask = head_mask_for_layer(w, layer) if layer is not None else None
    Qh, Kh, Vh = make_qkv(w, seed=5, layer=layer or 0)
    Q, K, V = dev_bf16(Qh), dev_bf16(Kh), dev_bf16(Vh)
    L = sa.Layout(list(w.segments), N)
    ws_bytes = sa.sa_workspace_size(B, H, N, d)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    sa.sa_workspace_init(ws, ws_bytes)
    idx = torch.zeros((B, H, w.nB, L.cap), dtype=torch.int32, device="cuda")
    counts = torch.zeros((B, H, w.nB), dtype=torch.int32, device="cuda")
    O = torch.full((B, H, N, d), float("nan"), dtype=torch.bfloat16, device="cuda")

    def step(st):
        sa.sa_select_blocks(L, Q, K, B, H, d, rho, mask, w.min_active, idx, counts, None, ws, ws_bytes, st)
        sa.sa_attention_plan(idx, counts, B, H, N, d, L.cap, mask, w.min_active, ws, ws_bytes, st)
        sa.sa_attention_run(Q, K, V, B, H, N, d, mask, w.min_active, 0.0, O, ws, ws_bytes, st)

    main = torch.cuda.current_stream()
    for _ in range(2):
        step(main)
    torch.cuda.synchronize()
    assert sa.sa_check(ws) == sa.SA_OK
    O_eager, idx_eager, cnt_eager = O.clone(), idx.clone(), counts.clone()

    side = torch.cuda.Stream()
    side.wait_stream(main)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        step(side)
    main.wait_stream(side)
    # capture enqueues nothing: poison the outputs, then only replays may fill them
    O.fill_(float("nan"))
    counts.zero_()
    for rep in range(3):
        graph.replay()
        torch.cuda.synchronize()
        assert sa.sa_check(ws) == sa.SA_OK
        assert torch.equal(counts, cnt_eager), "replay %d: counts differ from the eager step" % rep
        c = cnt_eager.cpu().numpy()
        i_r, i_e = idx.cpu().numpy(), idx_eager.cpu().numpy()
        for r in zip(*np.nonzero(c >= 0)):
            n = int(c[r])
            assert np.array_equal(i_r[r][:n], i_e[r][:n]), "replay %d: lists differ at %s" % (rep, r)
        assert torch.equal(O.view(torch.int16), O_eager.view(torch.int16)), "replay %d: O differs from eager" % rep
    if mask is not None:  # skipped heads are zero in the replayed output too
        off = [h for h in range(H) if not mask[h]]
        assert off and bool((O[:, off].float() == 0).all())
    del graph
    L.release()
