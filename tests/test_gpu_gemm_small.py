"""GPU parity: the small-M (1..32 tokens) tensor-core path vs the oracle.

The whole method runs on the GPU (per-token or per-group quantization of bf16
X, then the swap-AB tcgen05 product with K split across the SMs and the
split tiles summed by their last contributor); the oracle runs the same
definition.  The quantized tokens, their scales and (int8) the int32
accumulators come back through the debug hook and must be bit-exact; bf16
outputs are bit-exact for int8 and within 2^-7 |y| + 1e-3 for E4M3.

Without the debug hook, five to eight tokens within K <= 8192 on at most 8 MiB
of weights run on the GEMV kernel, each product as two products of four tokens
or fewer over the same weights in one launch: those calls are checked on their
outputs (and, int8, bit-equal to the split-K kernel's).
"""
import numpy as np
import pytest
import torch

import fp8_linear_layers_b200 as ql
import oracle
from fp8_linear_layers_b200 import synthetic
from tests._util import assert_y_close, bf16_dev, bits, f32_dev, u8_dev

pytestmark = pytest.mark.gpu


def _run(scheme, M, N, K, seed=0, outliers=None, tag="small", sample=None, ws=None, check_q=True):
    if outliers is None:
        outliers = synthetic.outlier_count(K) if scheme != ql.FP8_E4M3_BLOCK128 else 0
    x = synthetic.make_x(M, K, seed=seed, tag=f"{tag}-x", outliers=outliers)
    w = synthetic.make_w(N, K, seed=seed, tag=f"{tag}-w")
    wq, sw = oracle.quantize_weight(scheme, w)
    dbg = ql.Debug(qx=torch.empty((M, K), dtype=torch.uint8, device="cuda"),
                   sx=torch.empty(ql.act_scale_shape(scheme, M, K), dtype=torch.float32, device="cuda"),
                   acc_i32=torch.empty((M, N), dtype=torch.int32, device="cuda")
                   if scheme == ql.W8A8_INT8_ROW else None,
                   acc_f32=torch.empty((M, N), dtype=torch.float32, device="cuda")
                   if scheme == ql.FP8_E4M3_ROW else None)
    if ws is None:
        ws = ql.new_workspace(ql.workspace_bytes(scheme, M, N, K))
    ypad = torch.full((M * N + 64,), -3.0, dtype=torch.bfloat16, device="cuda")
    y = ypad[:M * N].view(M, N)
    ql.gemm_small(scheme, bf16_dev(x), u8_dev(wq), f32_dev(sw), ws, y=y, debug=dbg)
    st, detail = ql.device_status()
    assert st == 0, f"device status {st} detail {detail:#x}"
    assert np.all(bits(ypad[M * N:]) == bits(torch.tensor([-3.0], dtype=torch.bfloat16))[0])
    rqx, rsx = oracle.quantize_act(scheme, x)
    if check_q:
        assert np.array_equal(dbg.qx.cpu().numpy(), rqx)
        assert np.array_equal(dbg.sx.cpu().numpy().view(np.uint32), rsx.view(np.uint32))
    gy = bits(y)
    if sample is None:
        ry, racc_i, racc_d = oracle.linear(scheme, rqx, rsx, wq, sw, want_acc=True)
        if scheme == ql.W8A8_INT8_ROW:
            assert np.array_equal(dbg.acc_i32.cpu().numpy(), racc_i), "int32 accumulators differ"
            assert np.array_equal(gy, ry), "int8 outputs must be bit-exact"
        else:
            assert_y_close(gy, ry, f"small {scheme} {M}x{N}x{K}")
            if scheme == ql.FP8_E4M3_ROW:
                acc = dbg.acc_f32.cpu().numpy().astype(np.float64)
                assert np.all(np.abs(acc - racc_d) <= 1e-5 * np.abs(racc_d).max() + 1e-6)
    else:
        rng = np.random.default_rng(seed + 7)
        pm = np.concatenate([rng.integers(0, M, sample), np.full(N, M - 1)])
        pn = np.concatenate([rng.integers(0, N, sample), np.arange(N)])
        ry, racc_i, _ = oracle.linear_sampled(scheme, rqx, rsx, wq, sw, pm, pn, want_acc=True)
        if scheme == ql.W8A8_INT8_ROW:
            assert np.array_equal(dbg.acc_i32.cpu().numpy()[pm, pn], racc_i)
            assert np.array_equal(gy[pm, pn], ry)
        else:
            assert_y_close(gy[pm, pn], ry, f"small {scheme} {M}x{N}x{K} sampled")
    return ws


def test_config_w8a8_k_proj_m8_seed0(cuda):
    """W8A8, X [8, 4096] with 8 outlier channels x20, W [1024, 4096], seed 0: every output."""
    _run(ql.W8A8_INT8_ROW, 8, 1024, 4096, seed=0, outliers=8, tag="cfg0")


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW])
@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (2, 300, 1040), (5, 128, 48), (16, 1000, 4096),
                                   (17, 640, 2048), (32, 256, 8192), (3, 129, 272), (32, 4096, 128),
                                   # up to four tokens ride on the GEMV kernel's B columns; past
                                   # its K limits they take the split-K kernel
                                   (2, 1000, 4096), (2, 129, 16384), (2, 64, 16400), (3, 1001, 4096),
                                   (4, 777, 2064), (4, 300, 8192), (3, 64, 8208), (4, 130, 16),
                                   # five to eight tokens (with the debug hook: the split-K kernel)
                                   (5, 1000, 4096), (7, 129, 8192), (8, 4096, 4096), (6, 64, 8208),
                                   (8, 4100, 4096)])
def test_small_shapes_full_compare(cuda, scheme, M, N, K):
    _run(scheme, M, N, K)


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (2, 256, 384), (16, 384, 4096), (32, 1280, 1024),
                                   (7, 128, 12288), (2, 384, 4096), (3, 256, 1024), (4, 512, 8192),
                                   (4, 128, 8320), (6, 1024, 4096), (8, 4096, 4096)])
def test_small_block_shapes(cuda, M, N, K):
    _run(ql.FP8_E4M3_BLOCK128, M, N, K, outliers=2)


@pytest.mark.parametrize("M", [2, 3, 4, 8, 16, 32])
@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW])
@pytest.mark.parametrize("name,N,K", synthetic.LLAMA31_8B)
def test_small_llama_shapes_full_size(cuda, M, scheme, name, N, K):
    full = M <= 4 or (scheme == ql.W8A8_INT8_ROW and M <= 8)
    _run(scheme, M, N, K, tag=f"llama.{name}", sample=None if full else 1500)


@pytest.mark.parametrize("M", [2, 4, 32])
@pytest.mark.parametrize("name,N,K", synthetic.QWEN3_8B)
def test_small_qwen_block_full_size(cuda, M, name, N, K):
    _run(ql.FP8_E4M3_BLOCK128, M, N, K, tag=f"qwen.{name}", sample=None if M <= 4 else 1000)


def test_workspace_reused_across_calls(cuda):
    """The split-tile sums and counters are left at zero, so one workspace
    serves call after call of one shape; re-zeroed, it serves another shape
    that fits in it."""
    for scheme in (ql.FP8_E4M3_ROW, ql.W8A8_INT8_ROW):
        ws = _run(scheme, 8, 1024, 4096, tag="reuse")
        nbytes = ws.numel()
        for _ in range(3):
            _run(scheme, 8, 1024, 4096, tag="reuse", ws=ws)
        need = ql.workspace_bytes(ql.W8A8_INT8_ROW, 4, 512, 2048)
        assert need <= nbytes
        ws.zero_()
        _run(ql.W8A8_INT8_ROW, 4, 512, 2048, tag="reuse2", ws=ws)
        _run(ql.W8A8_INT8_ROW, 4, 512, 2048, tag="reuse2", ws=ws)


def test_workspace_too_small_is_rejected(cuda):
    M, N, K = 8, 1024, 4096
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    sw = torch.ones(N, dtype=torch.float32, device="cuda")
    with pytest.raises(ql.QLinearError) as e:
        ql.gemm_small(ql.W8A8_INT8_ROW, x, wq, sw, ws)
    assert e.value.status == 7


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW, ql.FP8_E4M3_BLOCK128])
def test_forward_dispatch_small_m(cuda, scheme):
    M, N, K = 12, 384, 1024
    x = synthetic.make_x(M, K, seed=5, tag="fwd-small-x", outliers=3)
    w = synthetic.make_w(N, K, seed=5, tag="fwd-small-w")
    wq, sw = oracle.quantize_weight(scheme, w)
    ws = ql.new_workspace(ql.forward_workspace_bytes(scheme, M, N, K))
    y = ql.forward(scheme, bf16_dev(x), u8_dev(wq), f32_dev(sw), workspace=ws)
    torch.cuda.synchronize()
    ry = oracle.forward(scheme, x, wq, sw)
    if scheme == ql.W8A8_INT8_ROW:
        assert np.array_equal(bits(y), ry)
    else:
        assert_y_close(bits(y), ry, "forward small M")


def _run_plain(scheme, M, N, K, seed=0, outliers=None, tag="plain", sample=None):
    """The call without the debug hook; y (and a canary past it) against the
    oracle.  Returns the output bits."""
    if outliers is None:
        outliers = synthetic.outlier_count(K) if scheme != ql.FP8_E4M3_BLOCK128 else 0
    x = synthetic.make_x(M, K, seed=seed, tag=f"{tag}-x", outliers=outliers)
    w = synthetic.make_w(N, K, seed=seed, tag=f"{tag}-w")
    wq, sw = oracle.quantize_weight(scheme, w)
    ws = ql.new_workspace(ql.workspace_bytes(scheme, M, N, K))
    ypad = torch.full((M * N + 64,), -3.0, dtype=torch.bfloat16, device="cuda")
    y = ypad[:M * N].view(M, N)
    ql.gemm_small(scheme, bf16_dev(x), u8_dev(wq), f32_dev(sw), ws, y=y)
    st, detail = ql.device_status()
    assert st == 0, f"device status {st} detail {detail:#x}"
    assert np.all(bits(ypad[M * N:]) == bits(torch.tensor([-3.0], dtype=torch.bfloat16))[0]), "wrote past y"
    gy = bits(y)
    what = f"small {scheme} {M}x{N}x{K} (no debug hook)"
    if sample is None:
        ry = oracle.forward(scheme, x, wq, sw)
        if scheme == ql.W8A8_INT8_ROW:
            assert np.array_equal(gy, ry), what + ": int8 outputs must be bit-exact"
        else:
            assert_y_close(gy, ry, what)
    else:
        rqx, rsx = oracle.quantize_act(scheme, x)
        rng = np.random.default_rng(seed + 11)
        pm = np.concatenate([rng.integers(0, M, sample), np.full(N, M - 1), np.full(N, 4 % M)])
        pn = np.concatenate([rng.integers(0, N, sample), np.arange(N), np.arange(N)])
        ry = oracle.linear_sampled(scheme, rqx, rsx, wq, sw, pm, pn)
        if scheme == ql.W8A8_INT8_ROW:
            assert np.array_equal(gy[pm, pn], ry), what
        else:
            assert_y_close(gy[pm, pn], ry, what + " sampled")
    return gy


def test_config_w8a8_k_proj_m8_seed0_plain(cuda):
    """The same product without the debug hook (the GEMV kernel, two 4-token
    halves): every output bit-exact."""
    _run_plain(ql.W8A8_INT8_ROW, 8, 1024, 4096, seed=0, outliers=8, tag="cfg0")


@pytest.mark.parametrize("M", [5, 6, 7, 8])
@pytest.mark.parametrize("scheme,N,K", [(ql.W8A8_INT8_ROW, 1000, 4096), (ql.W8A8_INT8_ROW, 8, 8192),
                                        (ql.W8A8_INT8_ROW, 4100, 48), (ql.W8A8_INT8_ROW, 64, 8208),
                                        (ql.W8A8_INT8_ROW, 2048, 4096), (ql.W8A8_INT8_ROW, 2056, 4096),
                                        (ql.FP8_E4M3_ROW, 129, 4096), (ql.FP8_E4M3_ROW, 520, 8192),
                                        (ql.FP8_E4M3_ROW, 16, 272),
                                        (ql.FP8_E4M3_BLOCK128, 1024, 4096), (ql.FP8_E4M3_BLOCK128, 128, 8192),
                                        (ql.FP8_E4M3_BLOCK128, 384, 8320)])
def test_five_to_eight_tokens_full_compare(cuda, M, scheme, N, K):
    """Ragged N (partial stages, a product smaller than one stage per CTA), K at
    and past the GEMV's four-token limit (8208, 8320: the split-K kernel),
    weights of exactly 8 MiB (2048 x 4096: the GEMV) and just past it (2056 x
    4096: the split-K kernel); int8 outputs also bit-equal to the split-K
    kernel's (the debug-hook call)."""
    gy = _run_plain(scheme, M, N, K, seed=M, tag=f"t58.{N}.{K}", outliers=3)
    if scheme == ql.W8A8_INT8_ROW:
        x = synthetic.make_x(M, K, seed=M, tag=f"t58.{N}.{K}-x", outliers=3)
        w = synthetic.make_w(N, K, seed=M, tag=f"t58.{N}.{K}-w")
        wq, sw = oracle.quantize_weight(scheme, w)
        dbg = ql.Debug(acc_i32=torch.empty((M, N), dtype=torch.int32, device="cuda"))
        ws = ql.new_workspace(ql.workspace_bytes(scheme, M, N, K))
        y = ql.gemm_small(scheme, bf16_dev(x), u8_dev(wq), f32_dev(sw), ws, debug=dbg)
        torch.cuda.synchronize()
        assert np.array_equal(bits(y), gy), "GEMV route and split-K kernel differ"


@pytest.mark.parametrize("M", [5, 8])
@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW])
@pytest.mark.parametrize("name,N,K", synthetic.LLAMA31_8B)
def test_five_to_eight_tokens_llama_full_size(cuda, M, scheme, name, N, K):
    """The Llama-3.1-8B layer at M = 5 and 8 without the debug hook (down_proj,
    K = 14336, takes the split-K kernel): int8 every output up to 4096 rows,
    else sampled outputs plus the last token's and the fifth token's rows."""
    full = scheme == ql.W8A8_INT8_ROW and N <= 4096
    _run_plain(scheme, M, N, K, seed=M, tag=f"llama58.{name}", sample=None if full else 1500)


@pytest.mark.parametrize("name,N,K", synthetic.QWEN3_8B)
def test_five_to_eight_tokens_qwen_block(cuda, name, N, K):
    _run_plain(ql.FP8_E4M3_BLOCK128, 8, N, K, seed=8, tag=f"qwen58.{name}", sample=1000)
