"""The allocation-free one-token forward (moe_layer_forward_noalloc) against
the workspace entry point moe_layer_forward, on a GPU.

The file name sorts last so that the suite also runs it after every other
test has used the library on the same device."""
import numpy as np
import pytest

import synth
from synth.layers import DeviceLayer

torch = pytest.importorskip("torch")
import int4_routed_expert_noaux_b200 as moe  # noqa: E402

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 512 * 1024


def needs_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("shape", [synth.TINY, synth.GLM], ids=["tiny", "glm"])
def test_noalloc_matches_workspace_forward(shape):
    needs_gpu()
    cfg = moe.Config.from_shape(shape)
    assert moe.workspace_bytes(cfg, 1) <= SCRATCH_BYTES
    dl = DeviceLayer(shape, 0, 0)
    layer = moe.Layer(cfg, dl.w_router, dl.bias, dl.routed, dl.shared)
    ws = moe.alloc_workspace(cfg, 1)
    x = torch.from_numpy(synth.tokens(shape, 0, 70, 2).view(np.int16)).cuda()
    k, H = shape.top_k, shape.hidden

    def outputs():
        return (torch.full((1, H), float("nan"), device="cuda"),
                torch.full((1, k), -1, dtype=torch.int32, device="cuda"),
                torch.full((1, k), float("nan"), device="cuda"))

    ref = [outputs() for _ in range(2)]
    got = [outputs() for _ in range(2)]
    status = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    for t in range(2):
        y, idx, w = ref[t]
        layer.forward(x[t:t + 1], y, ws, idx=idx, w=w)
    moe.ws_check(ws)
    # the first call on a device resolves the scratch array (module load)
    warm = outputs()
    moe.forward_noalloc(layer, x[1:2], warm[0], idx=warm[1], w=warm[2])
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    # two calls in a row on one stream: the second starts from the scratch
    # state the first one left behind
    for t in range(2):
        y, idx, w = got[t]
        moe.forward_noalloc(layer, x[t:t + 1], y, idx=idx, w=w, status=status[t:t + 1])
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
    assert status.tolist() == [0, 0]
    for t in range(2):
        for a, b in zip(ref[t], got[t]):
            assert torch.equal(a, b), t
    assert not torch.equal(ref[0][0], ref[1][0])


def test_noalloc_refuses_shapes_beyond_the_scratch():
    needs_gpu()
    # one token of a 8192 x 8192 layer needs more than the fixed array holds
    shape = synth.Shape(hidden=8192, inter=8192, n_experts=16, n_shared=1, top_k=8,
                        n_group=1, topk_group=1)
    cfg = moe.Config.from_shape(shape)
    assert moe.workspace_bytes(cfg, 1) > SCRATCH_BYTES
    H, I = shape.hidden, shape.inter
    # real, zero-filled buffers of the full size, shared by every expert
    ex = {"q_gate": torch.zeros(I * H // 2, dtype=torch.uint8, device="cuda"),
          "q_up": torch.zeros(I * H // 2, dtype=torch.uint8, device="cuda"),
          "s_gate": torch.zeros(I * H // 32, dtype=torch.int16, device="cuda"),
          "s_up": torch.zeros(I * H // 32, dtype=torch.int16, device="cuda"),
          "q_down": torch.zeros(H * I // 2, dtype=torch.uint8, device="cuda"),
          "s_down": torch.zeros(H * I // 32, dtype=torch.int16, device="cuda")}
    w_router = torch.zeros((shape.n_experts, H), dtype=torch.float32, device="cuda")
    bias = torch.zeros(shape.n_experts, dtype=torch.float32, device="cuda")
    layer = moe.Layer(cfg, w_router, bias, [ex] * shape.n_experts, ex)
    x = torch.zeros((1, H), dtype=torch.int16, device="cuda")
    y = torch.zeros((1, H), dtype=torch.float32, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.forward_noalloc(layer, x, y)
    assert moe.STATUS_NAMES[e.value.status] == "MOE_ERR_UNSUPPORTED"
    torch.cuda.synchronize()
    assert torch.count_nonzero(y).item() == 0
