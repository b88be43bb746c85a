"""Device memory of one layer, training and inference, from the buffer sizes the
C ABI reports (host only: the layer's buffers are allocated on the CPU here, no
kernel runs).  The byte counts are written out from the tensor shapes the
header documents, not from the layer's own bookkeeping."""
import pytest
import torch

from dynamic_block_sparse_macro_b200 import _abi
from dynamic_block_sparse_macro_b200.layer import PrismSparseAttention


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from dynamic_block_sparse_macro_b200 import build
    build.build()


def _layer(with_backward, T=16, H=48, W=80, heads=2, d=128, dtype="bf16"):
    return PrismSparseAttention(T, H, W, heads, d, 64, dtype, 8, 0.9, device="cpu", with_backward=with_backward)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_training_layer_bytes_by_stage(dtype):
    T, H, W, heads, d = 16, 48, 80, 2, 128
    m = _layer(True, T, H, W, heads, d, dtype)
    s = _abi.query_sizes(_abi.problem(T, H, W, heads, d, 64, dtype))
    N, Z, MB, SW = T * H * W, T * H * W // 512, T * H * W // 64, (T * H * W // 64 + 31) // 32
    el = 2 if dtype == "bf16" else 4
    rep = m.memory_report()
    assert rep["blocked_qkv"] == 3 * heads * N * d * el
    assert rep["scores"] == 2 * heads * MB * d * 4 + heads * MB * MB * 4
    # sel, gsel, gselT words + count + margin + the status word
    assert rep["selection"] == 3 * heads * MB * SW * 4 + 2 * heads * MB * 4 + 4
    of32 = heads * N * d * 4 if dtype == "bf16" else 0
    assert rep["forward"] == heads * N * d * el + of32 + heads * N * 4 + max(16, s.ws_attn_fwd)
    assert rep["backward"] == 4 * heads * N * d * el + max(16, s.ws_attn_bwd)
    assert rep["total"] == sum(v for k, v in rep.items() if k != "total")
    assert rep["plan"] >= N * 4 + (MB + 1) * 4 + Z * (3 + 1 + 1 + 8 + 2) * 4


def test_inference_layer_keeps_no_backward_state():
    heads, d = 2, 128
    m = _layer(False, heads=heads, d=d)
    t = _layer(True, heads=heads, d=d)
    N, MB, SW = m.sizes.n_tokens, m.sizes.max_blocks, m.sizes.sel_words
    a, b = m.memory_report(), t.memory_report()
    assert m.lse is None and m.Of32 is None and m.gselT is None
    assert a["backward"] == 0
    assert b["selection"] - a["selection"] == heads * MB * SW * 4           # no key-major selection
    assert b["forward"] - a["forward"] == heads * N * d * 4 + heads * N * 4  # no fp32 O, no LSE
    assert a["plan"] == b["plan"] and a["blocked_qkv"] == b["blocked_qkv"] and a["scores"] == b["scores"]
    with pytest.raises(RuntimeError):
        m.backward(torch.empty(1))


def test_long_clip_layer_fits_one_gpu():
    # 112x72x128 grid (1,032,192 tokens), 24 heads of 128, bf16: the training layer's buffers
    # (P at its worst case, n_blk = N/64) plus raster Q, K, V, dO, O, dQ, dK, dV and hhat stay
    # inside the 180 GB of one GPU; inference needs about half
    T, H, W, heads, d = 112, 72, 128, 24, 128
    N = T * H * W
    io_train = 8 * N * heads * d * 2 + N * 64 * 2
    io_infer = 4 * N * heads * d * 2 + N * 64 * 2
    for wb, io in ((True, io_train), (False, io_infer)):
        m = PrismSparseAttention(T, H, W, heads, d, 64, "bf16", 8, 0.95, device="meta", with_backward=wb)
        tot = m.memory_report()["total"] + io
        assert tot < 180e9, (wb, tot)
    assert m.memory_report()["scores"] == 2 * heads * (N // 64) * d * 4 + heads * (N // 64) ** 2 * 4
