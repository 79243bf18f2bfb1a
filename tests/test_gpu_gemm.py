"""GPU: the tcgen05/TMEM/TMA GEMM and the mma.sync GEMM against a float64
reference of the same bf16 operands (relative error bound of fp32
accumulation over K terms: 1e-5 x sqrt(K) is generous; we use 2e-4 abs on
O(1) outputs), on the engine's shapes, ragged M and every tile width."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)
from streaming_speaker_diarization_b200 import binding as b  # noqa: E402
from _helpers import make_engine, tiny_weights  # noqa: E402


@pytest.fixture(scope="module")
def eng():
    e = make_engine(tiny_weights(), 1, 2, 2)
    yield e
    b.sf_destroy(e)


# engine shapes at the 90 s workload (M = 1125), streaming batches, ragged M,
# every tile width and split-K counts 1..8 (e.g. (300, 64, 4096): 3 tiles -> 8 splits)
SHAPES = [(1125, 2048, 512), (1125, 512, 2048), (1125, 1536, 512), (1125, 192, 192), (1125, 576, 192),
          (1125, 192, 768), (1125, 512, 4096), (1, 64, 64), (333, 768, 192), (128, 128, 128), (129, 256, 4096),
          (24896, 1024, 512), (70, 16, 64), (300, 64, 4096), (2000, 256, 1024),
          # more tiles than SMs: persistent kernel, BN 256 / 128, ragged M and N tails
          (20000, 192, 256), (19001, 256, 512), (50000, 576, 192), (72000, 256, 256),
          # K >= 1024, N >= 256, multi-wave: CTA pairs on the default path
          (20608, 512, 2048)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("path", [1, 0])
def test_gemm_vs_float64(eng, M, N, K, path):
    g = torch.Generator().manual_seed(M * 7 + N * 3 + K)
    A = (torch.randn(M, K, generator=g) / np.sqrt(K)).to(torch.bfloat16)
    W = torch.randn(N, K, generator=g).to(torch.bfloat16)
    bias = torch.randn(N, generator=g)
    ref = A.double().numpy() @ W.double().numpy().T + bias.double().numpy()
    C = torch.full((M, N), float("nan"), device="cuda")
    b.sf_gemm_bf16(eng, A.cuda(), W.cuda(), C, bias=bias.cuda(), path=path)
    b.sf_check(eng)
    err = np.max(np.abs(C.cpu().numpy() - ref))
    assert err <= 2e-4 * max(1.0, np.sqrt(K / 512)), err


def test_gemm_tc_strided_a(eng):
    """A with a row stride larger than K (a column slice of a wider matrix)."""
    M, N, K = 300, 128, 256
    g = torch.Generator().manual_seed(3)
    big = torch.randn(M, 3 * K, generator=g).to(torch.bfloat16)
    W = torch.randn(N, K, generator=g).to(torch.bfloat16)
    A = big.cuda()
    C = torch.zeros((M, N), device="cuda")
    sub = A[:, K:2 * K]
    rc = b.lib.sf_gemm_bf16(eng, sub.data_ptr(), A.stride(0), W.cuda().data_ptr(), M, N, K, None, C.data_ptr(), 1,
                            torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    b.sf_check(eng)
    ref = big[:, K:2 * K].double().numpy() @ W.double().numpy().T
    assert np.max(np.abs(C.cpu().numpy() - ref)) < 2e-3


def test_gemm_tc_split_k_is_deterministic(eng):
    """Split-K partials are summed in split order by whichever CTA arrives
    last: repeated launches must agree bit for bit."""
    M, N, K = 1125, 512, 2048
    g = torch.Generator().manual_seed(11)
    A = (torch.randn(M, K, generator=g) / 40).to(torch.bfloat16).cuda()
    W = torch.randn(N, K, generator=g).to(torch.bfloat16).cuda()
    outs = []
    for _ in range(4):
        C = torch.zeros((M, N), device="cuda")
        b.sf_gemm_bf16(eng, A, W, C, path=1)
        outs.append(C.cpu())
    b.sf_check(eng)
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


@pytest.mark.parametrize("M,N,K", [(1125, 2048, 512), (20000, 192, 256), (19001, 256, 512), (333, 768, 192)])
def test_gemm_tc_bf16_output(eng, M, N, K):
    """Path 2: the engine's bf16 projection epilogue; each output is the
    float64 result rounded to bf16 (within one bf16 ulp of it)."""
    g = torch.Generator().manual_seed(M + N + K)
    A = (torch.randn(M, K, generator=g) / np.sqrt(K)).to(torch.bfloat16)
    W = torch.randn(N, K, generator=g).to(torch.bfloat16)
    bias = torch.randn(N, generator=g)
    ref = A.double().numpy() @ W.double().numpy().T + bias.double().numpy()
    C = torch.full((M, N), float("nan"), device="cuda", dtype=torch.bfloat16)
    b.sf_gemm_bf16(eng, A.cuda(), W.cuda(), C, bias=bias.cuda(), path=2)
    b.sf_check(eng)
    got = C.float().cpu().numpy()
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 2e-4)


@pytest.mark.parametrize("M,N,K", [(1125, 1024, 512), (20000, 192, 256), (19001, 512, 512)])
@pytest.mark.parametrize("path", [3, 4, 5])
def test_gemm_tc_fused_epilogues(eng, M, N, K, path):
    """Paths 3-5: residual update (f32), swish (bf16) and gated linear unit
    (bf16, interleaved value/gate columns) against float64."""
    _check_fused(eng, M, N, K, path)


@pytest.mark.parametrize("M,N,K", [(20608, 512, 512), (20608, 512, 2048), (20001, 512, 2048), (19030, 1536, 512)])
def test_gemm_tc_resid_streaming_shapes(eng, M, N, K):
    """Path 3 at the streaming step's residual projections (the persistent
    and CTA-pair kernels, residual boxes loaded by TMA), and with ragged M
    whose last tile leaves whole 32-row warps past M."""
    _check_fused(eng, M, N, K, 3)


@pytest.fixture(scope="module", params=[0, 128, 192, 256])
def eng_pairs(request):
    """Engine on the CTA-pair GEMM path: planned tile width (0) or forced."""
    e = make_engine(tiny_weights(), 1, 2, 2)
    b.sf_set_option(e, b.SF_OPT_GEMM_PATH, 2)
    b.sf_set_option(e, b.SF_OPT_GEMM_PAIR_BN, request.param)
    yield e
    b.sf_destroy(e)


# multi-wave shapes with N >= 256 (the CTA-pair kernel): ragged last pair tile
# whose second CTA is entirely past M (19001 = 74 x 256 + 57), N not a
# multiple of 256 (the second CTA's weight rows of the last tile all past N),
# long K, many tiles per pair
PAIR_SHAPES = [(19001, 256, 512), (20000, 320, 256), (24896, 1024, 512), (20608, 512, 2048), (72000, 256, 256),
               (20608, 2048, 512), (20608, 192, 768), (20608, 576, 192), (33000, 192, 192)]


@pytest.mark.parametrize("M,N,K", PAIR_SHAPES)
def test_gemm_tc_pairs_vs_float64(eng_pairs, M, N, K):
    g = torch.Generator().manual_seed(M * 5 + N * 3 + K)
    A = (torch.randn(M, K, generator=g) / np.sqrt(K)).to(torch.bfloat16)
    W = torch.randn(N, K, generator=g).to(torch.bfloat16)
    bias = torch.randn(N, generator=g)
    ref = A.double().numpy() @ W.double().numpy().T + bias.double().numpy()
    C = torch.full((M, N), float("nan"), device="cuda")
    b.sf_gemm_bf16(eng_pairs, A.cuda(), W.cuda(), C, bias=bias.cuda(), path=1)
    b.sf_check(eng_pairs)
    err = np.max(np.abs(C.cpu().numpy() - ref))
    assert err <= 2e-4 * max(1.0, np.sqrt(K / 512)), err


@pytest.mark.parametrize("path", [2, 3, 4, 5])
def test_gemm_tc_pairs_fused_epilogues(eng_pairs, path):
    _check_fused(eng_pairs, 20608, 1024, 512, path)


def _check_fused(eng, M, N, K, path):
    g = torch.Generator().manual_seed(M + 3 * N + K + path)
    A = (torch.randn(M, K, generator=g) / np.sqrt(K)).to(torch.bfloat16)
    W = torch.randn(N, K, generator=g).to(torch.bfloat16)
    bias = torch.randn(N, generator=g)
    r = A.double().numpy() @ W.double().numpy().T + bias.double().numpy()
    if path == 2:
        C = torch.full((M, N), float("nan"), device="cuda", dtype=torch.bfloat16)
        ref, tol_rel, tol_abs = r, 2.0 ** -8, 2e-4
    elif path == 3:
        x0 = torch.randn(M, N, generator=g)
        C = x0.cuda()
        ref, tol_rel, tol_abs = x0.double().numpy() + r, 0.0, 4e-4
    elif path == 4:
        C = torch.full((M, N), float("nan"), device="cuda", dtype=torch.bfloat16)
        ref, tol_rel, tol_abs = r / (1 + np.exp(-r)), 2.0 ** -8, 2e-4
    else:
        C = torch.full((M, N // 2), float("nan"), device="cuda", dtype=torch.bfloat16)
        ref, tol_rel, tol_abs = r[:, 0::2] / (1 + np.exp(-r[:, 1::2])), 2.0 ** -8, 2e-4
    b.sf_gemm_bf16(eng, A.cuda(), W.cuda(), C, bias=bias.cuda(), path=path)
    b.sf_check(eng)
    got = C.float().cpu().numpy()
    assert np.all(np.abs(got - ref) <= np.abs(ref) * tol_rel + tol_abs)


# --------------------------------------------------------------------------
# Residual projection with the LayerNorm fused into the epilogue (the
# conformer's "x += f(x); h = LN(x)" steps and the Transformer's post-LN),
# against float64 of the same bf16 operands: x to fp32 accumulation
# accuracy, h (bf16) to one bf16 rounding (2^-8 relative) plus that.

def _ln64(v, g, b):
    mu = v.mean(1, keepdims=True)
    var = ((v - mu) ** 2).mean(1, keepdims=True)
    return (v - mu) / np.sqrt(var + 1e-5) * g + b


LN_SHAPES = [(1125, 512, 512, 0.5, 0, False), (1125, 512, 2048, 0.5, 1, True), (1125, 512, 512, 1.0, 0, False),
             (1125, 192, 192, 1.0, 1, False), (1125, 192, 768, 1.0, 1, False), (1, 512, 64, 1.0, 0, False),
             (130, 192, 128, 0.5, 1, True), (1000, 64, 256, 1.0, 0, False), (513, 320, 192, 1.0, 1, False)]


@pytest.mark.parametrize("M,N,K,alpha,xnorm,two", LN_SHAPES)
def test_gemm_resid_layernorm_fused(eng, M, N, K, alpha, xnorm, two):
    g = torch.Generator().manual_seed(M + 3 * N + 5 * K)
    A = (torch.randn(M, K, generator=g) / np.sqrt(K)).to(torch.bfloat16)
    W = torch.randn(N, K, generator=g).to(torch.bfloat16)
    bias = torch.randn(N, generator=g)
    x0 = torch.randn(M, N, generator=g) * 2 + 0.3
    lg, lb = 1 + 0.3 * torch.randn(N, generator=g), 0.2 * torch.randn(N, generator=g)
    lg2, lb2 = 1 + 0.3 * torch.randn(N, generator=g), 0.2 * torch.randn(N, generator=g)
    x = x0.cuda().contiguous()
    h = torch.full((M, N), float("nan"), device="cuda", dtype=torch.bfloat16)
    b.sf_gemm_bf16_ln(eng, A.cuda(), W.cuda(), x, lg.cuda(), lb.cuda(), h, bias=bias.cuda(), alpha=alpha, xnorm=xnorm,
                      g2=lg2.cuda() if two else None, b2=lb2.cuda() if two else None)
    b.sf_check(eng)
    d = lambda t: t.double().numpy()  # noqa: E731
    xn = d(x0) + alpha * (d(A) @ d(W).T + d(bias))
    y = _ln64(xn, d(lg), d(lb))
    x_ref = y if xnorm else xn
    h_ref = _ln64(y, d(lg2), d(lb2)) if two else y
    gx, gh = x.cpu().numpy(), h.float().cpu().numpy()
    assert np.max(np.abs(gx - x_ref)) <= 2e-4 * max(1.0, np.sqrt(K / 512)) * (2 if xnorm else 4)
    assert np.max(np.abs(gh - h_ref) / (np.abs(h_ref) + 1e-2)) <= 1e-2
    assert np.max(np.abs(gh - h_ref)) <= 3e-2


def test_gemm_resid_layernorm_rejects_unfusable(eng):
    A = torch.zeros((10, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((576, 64), dtype=torch.bfloat16, device="cuda")     # 9 tiles of 64: more than a cluster
    x = torch.zeros((10, 576), device="cuda")
    h = torch.zeros((10, 576), dtype=torch.bfloat16, device="cuda")
    one = torch.ones(576, device="cuda")
    with pytest.raises(b.SFError, match="SF_ESHAPE"):
        b.sf_gemm_bf16_ln(eng, A, W, x, one, one, h)


def test_offline_forward_with_and_without_layernorm_fusion():
    """The bf16 offline forward with the fused residual LayerNorms equals the
    unfused engine to bf16 accuracy and the oracle within 2e-2 (xavier
    weights, so the probabilities spread over ~[0.45, 0.8])."""
    import oracle as O
    from synth import synth_batch
    from _helpers import to_dev
    w = tiny_weights(xavier=True)
    e = make_engine(w, 1, 2, 2, max_batch=4)
    try:
        audio, lens, _ = synth_batch(85, [9.0, 4.1])
        Tp = int(O.encoder_frames(audio.shape[1] // 160))
        outs = []
        for fuse in (1, 0):
            b.sf_set_option(e, b.SF_OPT_LN_FUSE, fuse)
            p = torch.zeros((2, Tp, 4), device="cuda")
            b.sf_forward_offline(e, to_dev(audio), lens, p)
            b.sf_check(e)
            outs.append(p.cpu().numpy())
    finally:
        b.sf_destroy(e)
    ref, tp = O.forward_offline(audio, lens, w)
    for i in range(2):
        assert np.max(np.abs(outs[0][i, :tp[i]] - ref[i, :tp[i]])) <= 2e-2
    assert np.max(np.abs(outs[0] - outs[1])) <= 1e-2
