"""The experts' SwiGLU FFN (moe_expert_gate_up, moe_expert_down) against the
oracle, on rows laid out by moe_dispatch_limited with 128-row expert blocks
(tolerances: gpu_check.check_expert_h / check_expert_y)."""
import numpy as np
import pytest
import torch

import token_dispatch_moe_b200 as moe
from gpu_check import check_expert_h, check_expert_y

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gen(seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    return g


def _layout(T, k, E, seed, hot=False, empty_expert=None):
    g = _gen(seed)
    ids = torch.randint(0, E, (T, k), generator=g, device=DEV, dtype=torch.int32)
    if hot:
        ids[:, 0] = 0
    if empty_expert is not None:
        ids[ids == empty_expert] = -1
    rows = moe.moe_dispatch_limited_rows(T, k, E, 0, 128)
    counts = torch.empty((E,), dtype=torch.int32, device=DEV)
    offsets = torch.empty((E + 1,), dtype=torch.int32, device=DEV)
    sorted_token = torch.empty((rows,), dtype=torch.int32, device=DEV)
    dest = torch.empty((T, k), dtype=torch.int32, device=DEV)
    ws = torch.empty((max(moe.moe_dispatch_workspace_size(T, k, E), 256),), dtype=torch.uint8,
                     device=DEV)
    moe.moe_dispatch_limited(ids, E, 0, 128, counts, offsets, sorted_token, dest, ws)
    return rows, offsets, sorted_token, dest


def _weights(E, d, F, seed, bias):
    g = _gen(seed)
    w1 = (torch.randn((E, F, d), generator=g, device=DEV) / d ** 0.5).to(torch.bfloat16)
    w3 = (torch.randn((E, F, d), generator=g, device=DEV) / d ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn((E, d, F), generator=g, device=DEV) / F ** 0.5).to(torch.bfloat16)
    b = [None, None, None]
    if bias:
        b = [torch.randn((E, F), generator=g, device=DEV) * 0.5,
             torch.randn((E, F), generator=g, device=DEV) * 0.5,
             torch.randn((E, d), generator=g, device=DEV) * 0.5]
    return w1, w3, w2, b


def _token_rows(sorted_token, offsets, n, seed):
    """Sampled rows that hold a token (padding rows excluded), first and last included."""
    total = int(offsets[-1].item())
    st = sorted_token[:total].cpu().numpy()
    real = np.nonzero(st >= 0)[0]
    rng = np.random.default_rng(seed)
    pick = rng.choice(real, size=min(n, real.size), replace=False)
    return np.unique(np.concatenate([pick, real[:1], real[-1:]]))


FFN_CASES = [
    # T, k, E, d, F, act, bias, hot
    (500, 2, 8, 256, 128, moe.MOE_ACT_SWIGLU, False, False),
    (700, 4, 16, 384, 192, moe.MOE_ACT_SWIGLU_OAI, True, True),    # N tiles 96 (up) and 192 (down)
    (300, 8, 4, 2048, 768, moe.MOE_ACT_SWIGLU, False, False),      # the qwen3 expert shape
    (200, 4, 4, 2880, 2880, moe.MOE_ACT_SWIGLU_OAI, True, False),  # the gpt-oss expert shape
    (129, 1, 3, 64, 32, moe.MOE_ACT_SWIGLU, True, True),
    (4000, 8, 8, 512, 256, moe.MOE_ACT_SWIGLU, False, True),      # several tiles per CTA
]


@pytest.mark.parametrize("case", FFN_CASES, ids=lambda c: "-".join(map(str, c)))
def test_expert_ffn_parity(case):
    T, k, E, d, F, act, bias, hot = case
    rows, offsets, sorted_token, dest = _layout(T, k, E, T + E, hot=hot,
                                                empty_expert=E - 1 if E > 3 else None)
    x = torch.randn((T, d), generator=_gen(3), device=DEV).to(torch.bfloat16)
    xs = torch.zeros((rows, d), dtype=torch.bfloat16, device=DEV)
    moe.moe_permute(x, dest, xs)
    w1, w3, w2, (b1, b3, b2) = _weights(E, d, F, 11 + E, bias)
    h = torch.full((rows, F), 9.0, dtype=torch.bfloat16, device=DEV)
    y = torch.full((rows, d), 9.0, dtype=torch.bfloat16, device=DEV)
    st = torch.zeros((1,), dtype=torch.int32, device=DEV)
    moe.moe_expert_gate_up(xs, offsets, w1, w3, h, b1, b3, act, st)
    moe.moe_expert_down(h, offsets, w2, y, b2, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    sample = _token_rows(sorted_token, offsets, 96, T)
    check_expert_h(h, xs, offsets, w1, w3, b1, b3, act, sample)
    check_expert_y(y, h, offsets, w2, b2, sample)
    # Rows past the last expert block are not touched.
    total = int(offsets[-1].item())
    assert torch.all(h[total:] == 9.0) and torch.all(y[total:] == 9.0)


def test_expert_ffn_misaligned_offsets_are_reported():
    """Blocks that do not start on 128-row boundaries: nothing written, status set."""
    E, d, F, rows = 2, 64, 32, 256
    offsets = torch.tensor([0, 100, 256], dtype=torch.int32, device=DEV)
    xs = torch.zeros((rows, d), dtype=torch.bfloat16, device=DEV)
    w1, w3, w2, _ = _weights(E, d, F, 1, False)
    h = torch.full((rows, F), 9.0, dtype=torch.bfloat16, device=DEV)
    st = torch.zeros((1,), dtype=torch.int32, device=DEV)
    moe.moe_expert_gate_up(xs, offsets, w1, w3, h, d_status=st)
    torch.cuda.synchronize()
    assert st.item() == moe.MOE_ERR_DEVICE_INDEX
    assert torch.all(h[:128] == 9.0)  # the straddling tile is skipped


def test_expert_ffn_validation():
    E, d, F, rows = 2, 64, 32, 128
    offsets = torch.tensor([0, 128, 128], dtype=torch.int32, device=DEV)
    xs = torch.zeros((rows, d), dtype=torch.bfloat16, device=DEV)
    w1, w3, w2, _ = _weights(E, d, F, 1, False)
    h = torch.empty((rows, F), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(moe.MoeError):
        moe.moe_expert_gate_up(xs, offsets, w1, w3, h, act=7)
    with pytest.raises(ValueError):
        moe.moe_expert_down(h, offsets, w2, torch.empty((rows, d + 16), dtype=torch.bfloat16,
                                                        device=DEV))
