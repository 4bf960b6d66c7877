"""Parity of the CUDA path with the CPU oracle at sizes the oracle finishes in
seconds: several tiles plus ragged tails in M, N and K-chunks, every format,
several N:M ratios, LayerNorm with and without affine parameters, and the
degenerate inputs. Prep outputs must be bit-exact; the GEMM within
1e-3 * sum|a||w| per element."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_common import (assert_bits_equal, assert_linear_close, assert_prep_matches, assert_weight_matches,
                        cuda16, gpu_prepare)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import sparsity_gemm_b200 as sq
    assert torch.cuda.is_available()
    sq.lib()
    yield


def test_single_linear_16x256x256_nvfp4_2of4():
    """The single-linear workload: X ~ N(0,1) with 4 of 256 channels x50,
    W ~ N(0, 0.02^2), LayerNorm gamma=1 beta=0, NVFP4, 2:4."""
    import sparsity_gemm_b200 as sq
    x = synth.activations_gaussian(0, 16, 256, 4, 50.0)
    w = synth.weights(1, 256, 256)
    ones, zeros = np.ones(256, np.float16), np.zeros(256, np.float16)
    op = oracle.prepare(x, ones, zeros, 1e-5, 2, 4, oracle.NVFP4)
    p, ex = gpu_prepare(x, ones, zeros, 1e-5, 2, 4, sq.NVFP4)
    assert_prep_matches(ex, op)
    ow = oracle.quantize_weight(w, oracle.NVFP4)
    qw = sq.quantize_weight(cuda16(w), sq.NVFP4)
    assert_weight_matches(sq.weight_export(qw), ow)
    out = sq.linear(p, qw).cpu().numpy()
    want, bound = oracle.linear_prepared(op, ow)
    assert_linear_close(out, want, bound)
    assert sq.get_last_error() == sq.OK


PREP_CASES = [
    # (m_tok, k, fmt, n, m, affine)
    (37, 256, 0, 2, 4, False),
    (300, 512, 0, 2, 4, True),
    (300, 512, 1, 2, 4, False),
    (129, 768, 1, 4, 8, True),
    (64, 512, 0, 4, 8, False),
    (33, 256, 0, 1, 2, False),
    (33, 256, 1, 3, 8, True),   # m = 8 with odd n: metadata chunks share bytes
    (17, 512, 0, 5, 8, False),
    (40, 512, 0, 8, 16, True),
    (40, 512, 1, 4, 4, False),  # n = m: plain quantization
    (24, 256, 0, 1, 4, False),
    (9, 1024, 1, 16, 16, True),
]


@pytest.mark.parametrize("m_tok,k,fmt,n,m,affine", PREP_CASES)
def test_prepare_bit_exact(m_tok, k, fmt, n, m, affine):
    x = synth.activations_student(100 + m_tok + k + n * 7 + m, m_tok, k)
    g, b = synth.ln_params(5, k) if affine else (None, None)
    op = oracle.prepare(x, g, b, 1e-5, n, m, fmt)
    _, ex = gpu_prepare(x, g, b, 1e-5, n, m, fmt)
    assert_prep_matches(ex, op)


@pytest.mark.parametrize("m_tok,k,fmt,norm", [(5000, 256, 0, "layer"), (10007, 512, 1, "layer"),
                                               (9500, 768, 0, "rms")])
def test_prepare_many_short_rows_bit_exact(m_tok, k, fmt, norm):
    """Rows enough for several rows per statistics warp (their sums finished
    together after all warps are done), with a ragged last CTA: every row's
    statistics and every code and scale bit-exact."""
    import sparsity_gemm_b200 as sq
    x = synth.activations_student(700 + m_tok, m_tok, k)
    op = oracle.prepare(x, None, None, 1e-5, 2, 4, fmt, norm=norm)
    p = sq.prepare(cuda16(x), None, None, 1e-5, 2, 4, fmt, norm=norm)
    assert_prep_matches(sq.prep_export(p), op)


@pytest.mark.parametrize("norm", ["layer", "rms"])
@pytest.mark.parametrize("affine", [False, True])
def test_certified_short_rows_and_exact_fallback(norm, affine):
    """Rows of at most 2048 elements, enough of them (>= 8 per SM) that the
    warp kernel takes its certified form (several rows per warp without the
    affine parameters); rows the error bound cannot decide (constant rows, fp16
    extremes, a large mean over a small spread, subnormals) spread over
    different warps and CTAs are summed again exactly. Every row bit-exact."""
    import sparsity_gemm_b200 as sq
    m_tok, k = 3001, 768
    x = synth.activations_student(940 + affine, m_tok, k)
    for r in (0, 37, 1500, 2999):
        x[r] = np.float16(3.5)
    for r in (5, 1201):
        x[r, ::2] = np.float16(65504.0)
        x[r, 1::2] = np.float16(-65504.0)
    for r in (9, 640, 3000):
        x[r] = np.float16(1000.0)
        x[r, ::7] = np.float16(1000.5)
    x[11] = 0
    x[13].view(np.uint16)[:] = np.arange(k, dtype=np.uint16) % 64 + 1  # fp16 subnormals
    x[17, : k // 2] = np.float16(65504.0)
    g, b = synth.ln_params(941, k) if affine else (None, None)
    if norm == "rms":
        b = None
    op = oracle.prepare(x, g, b, 1e-5, 2, 4, 1, norm=norm)
    p = sq.prepare(cuda16(x), None if g is None else cuda16(g), None if b is None else cuda16(b), 1e-5, 2, 4, 1,
                   norm=norm)
    assert_prep_matches(sq.prep_export(p), op)
    assert sq.get_last_error() == sq.OK


def test_maximum_k_statistics_at_the_lane_sum_bound():
    """K = SHARQ_K_MAX with rows enough for one warp per row: each lane adds
    2048 values, the bound of its 32-bit sums; rows of fp16 extremes (all
    +65504, alternating +-65504, all -65504) and Student-t rows. Statistics
    bit-exact for every row, LayerNorm and RMSNorm."""
    import sparsity_gemm_b200 as sq
    m_tok, k = 1200, sq.K_MAX
    x = synth.activations_student(910, m_tok, k)
    x[0] = np.float16(65504.0)
    x[1, ::2] = np.float16(65504.0)
    x[1, 1::2] = np.float16(-65504.0)
    x[2] = np.float16(-65504.0)
    x[3, : k // 2] = np.float16(65504.0)
    xd = cuda16(x)
    for norm, stats in (("layer", oracle.ln_stats), ("rms", oracle.rms_stats)):
        mu, rstd = stats(x, 1e-5)
        ex = sq.prep_export(sq.prepare(xd, None, None, 1e-5, 2, 4, sq.NVFP4, norm=norm))
        assert_bits_equal("mu", ex["mu"], mu)
        assert_bits_equal("rstd", ex["rstd"], rstd)


@pytest.mark.parametrize("norm", ["layer", "rms"])
@pytest.mark.parametrize("affine", [False, True])
def test_certified_statistics_and_exact_fallback(norm, affine):
    """Rows longer than 2048 elements (one warp per row) take binary64 sums
    whose error bound must decide the binary32 rstd; rows where it does not
    (a constant row, fp16 extremes of both signs, a large mean over a small
    spread) are summed again by the exact method. Every row bit-exact, with
    and without the affine parameters."""
    import sparsity_gemm_b200 as sq
    m_tok, k = 48, 4096
    x = synth.activations_student(920 + affine, m_tok, k)
    x[0] = np.float16(3.5)
    x[1, ::2] = np.float16(65504.0)
    x[1, 1::2] = np.float16(-65504.0)
    x[2] = np.float16(1000.0)
    x[2, ::7] = np.float16(1000.5)
    x[3] = 0
    x[4].view(np.uint16)[:] = np.arange(k, dtype=np.uint16) % 64 + 1  # fp16 subnormals
    x[5, : k // 2] = np.float16(65504.0)
    g, b = synth.ln_params(921, k) if affine else (None, None)
    if norm == "rms":
        b = None
    op = oracle.prepare(x, g, b, 1e-5, 2, 4, 0, norm=norm)
    p = sq.prepare(cuda16(x), None if g is None else cuda16(g), None if b is None else cuda16(b), 1e-5, 2, 4, 0,
                   norm=norm)
    assert_prep_matches(sq.prep_export(p), op)
    assert sq.get_last_error() == sq.OK


def test_maximum_k_linear():
    """A linear at K = SHARQ_K_MAX (256 K steps, split over a cluster at 9
    rows): prep bit-exact, output within tolerance."""
    import sparsity_gemm_b200 as sq
    m_tok, n_out, k = 9, 256, sq.K_MAX
    x = synth.activations_student(911, m_tok, k)
    w = synth.weights(912, n_out, k)
    op = oracle.prepare(x, None, None, 1e-5, 2, 4, 0)
    p, ex = gpu_prepare(x, None, None, 1e-5, 2, 4, 0)
    assert_prep_matches(ex, op)
    out = sq.linear(p, sq.quantize_weight(cuda16(w), 0)).cpu().numpy()
    want, bound = oracle.linear_prepared(op, oracle.quantize_weight(w, 0))
    assert_linear_close(out, want, bound)
    assert sq.get_last_error() == sq.OK


@pytest.mark.parametrize("n_out,k,fmt", [(32, 256, 0), (544, 512, 0), (544, 512, 1), (256, 1024, 1)])
def test_weight_quantization_bit_exact(n_out, k, fmt):
    import sparsity_gemm_b200 as sq
    w = synth.weights(7 + n_out, n_out, k)
    ow = oracle.quantize_weight(w, fmt)
    qw = sq.quantize_weight(cuda16(w), fmt)
    assert_weight_matches(sq.weight_export(qw), ow)


LINEAR_CASES = [
    # (m_tok, n_out, k, fmt, n, m)
    (16, 256, 256, 0, 2, 4),
    (300, 544, 512, 0, 2, 4),   # ragged M (3 tiles) and N (2 tiles + 32)
    (300, 544, 512, 1, 2, 4),
    (1, 256, 256, 0, 2, 4),
    (129, 512, 1024, 0, 4, 8),
    (129, 512, 1024, 1, 4, 8),
    (256, 288, 768, 0, 1, 2),
    (45, 1024, 2048, 0, 2, 4),  # 8 K tiles, more than the pipeline depth
    # Few tiles: K is split across a cluster (300 x 544: 2 CTAs per tile,
    # 129 x 512: 4, 45 x 1024: 8) and reduced through distributed shared
    # memory; the rows below end the MXFP4 and 16-tile variants.
    (3, 512, 2048, 1, 2, 4),
    (130, 2048, 2048, 0, 2, 4),
]


@pytest.mark.parametrize("m_tok,n_out,k,fmt,n,m", LINEAR_CASES)
def test_linear_within_tolerance(m_tok, n_out, k, fmt, n, m):
    import sparsity_gemm_b200 as sq
    x = synth.activations_student(200 + m_tok, m_tok, k)
    w = synth.weights(300 + n_out, n_out, k)
    op = oracle.prepare(x, None, None, 1e-5, n, m, fmt)
    ow = oracle.quantize_weight(w, fmt)
    p, ex = gpu_prepare(x, None, None, 1e-5, n, m, fmt)
    assert_prep_matches(ex, op)
    qw = sq.quantize_weight(cuda16(w), fmt)
    out = sq.linear(p, qw).cpu().numpy()
    want, bound = oracle.linear_prepared(op, ow)
    assert_linear_close(out, want, bound)
    assert sq.get_last_error() == sq.OK


def test_empty_activation():
    import sparsity_gemm_b200 as sq
    x = np.zeros((0, 256), np.float16)
    p = sq.prepare(torch.zeros((0, 256), dtype=torch.float16, device="cuda"), None, None, 1e-5, 2, 4, sq.NVFP4)
    assert sq.prep_export(p)["s_t"] == 1.0
    qw = sq.quantize_weight(cuda16(synth.weights(1, 256, 256)), sq.NVFP4)
    out = sq.linear(p, qw)
    assert out.shape == (0, 256)
    assert sq.get_last_error() == sq.OK


@pytest.mark.parametrize("fmt", [0, 1])
def test_degenerate_rows(fmt):
    """All-zero tensor (tensor scale 1), constant rows (variance 0), -0
    entries, fp16 extremes (65504 and subnormals)."""
    import sparsity_gemm_b200 as sq
    zero = np.zeros((5, 256), np.float16)
    op = oracle.prepare(zero, None, None, 1e-5, 2, 4, fmt)
    _, ex = gpu_prepare(zero, None, None, 1e-5, 2, 4, fmt)
    assert_prep_matches(ex, op)
    assert ex["s_t"] == 1.0

    x = synth.activations_student(9, 6, 512)
    x[0] = np.float16(3.5)                       # constant row
    x[1, ::2] = np.float16(65504.0)              # extremes
    x[1, 1::2] = np.float16(-65504.0)
    x[2] = 0
    x[2].view(np.uint16)[::3] = 0x8000            # -0 entries
    x[3].view(np.uint16)[:] = np.arange(512, dtype=np.uint16) % 64 + 1  # fp16 subnormals
    x[4].view(np.uint16)[::2] |= 0x8000
    op = oracle.prepare(x, None, None, 1e-5, 2, 4, fmt)
    _, ex = gpu_prepare(x, None, None, 1e-5, 2, 4, fmt)
    assert_prep_matches(ex, op)


def test_all_zero_weight():
    import sparsity_gemm_b200 as sq
    w = np.zeros((64, 256), np.float16)
    ow = oracle.quantize_weight(w, 0)
    qw = sq.quantize_weight(cuda16(w), 0)
    assert_weight_matches(sq.weight_export(qw), ow)
    assert ow.s_tw == 1.0


def test_launch_counts_and_no_host_sync():
    import sparsity_gemm_b200 as sq
    x = cuda16(synth.activations_student(1, 64, 512))
    p = sq.prepare(x, None, None, 1e-5, 2, 4, sq.NVFP4)
    assert sq.last_launch_count() == 2
    qw = sq.quantize_weight(cuda16(synth.weights(2, 256, 512)), sq.NVFP4)
    assert sq.last_launch_count() == 2
    sq.linear(p, qw)
    assert sq.last_launch_count() == 1
    assert sq.get_last_error() == sq.OK


def test_bounded_wait_reports_timeout_and_context_survives():
    """A wait on a barrier nothing arrives at runs out after its limit; the
    status comes back as SHARQ_ERR_TIMEOUT and the context stays usable."""
    import sparsity_gemm_b200 as sq
    assert sq.get_last_error() == sq.OK
    sq.selftest_wait(50_000_000)  # 50 ms
    assert sq.get_last_error() == sq.ERR_TIMEOUT
    assert sq.last_timeout_site() == 0x1FF
    assert sq.get_last_error() == sq.OK  # cleared
    test_single_linear_16x256x256_nvfp4_2of4()


def test_results_do_not_depend_on_stream_or_buffer_reuse():
    import sparsity_gemm_b200 as sq
    x = synth.activations_student(77, 200, 512)
    p1, ex1 = gpu_prepare(x, None, None, 1e-5, 2, 4, 0)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        p2 = sq.prepare(cuda16(x), None, None, 1e-5, 2, 4, 0, out=p1, stream=s)
        ex2 = sq.prep_export(p2, stream=s)
    for key in ex1:
        np.testing.assert_array_equal(np.asarray(ex1[key]), np.asarray(ex2[key]))


def test_quantizer_division_is_correctly_rounded():
    """The encode kernels' reciprocal-and-correction division equals the
    correctly rounded quotient on 2^26 operand pairs."""
    import sparsity_gemm_b200 as sq
    assert sq.selftest_division(1 << 26, seed=12345) == 0


def test_tiny_and_huge_scales_bit_exact():
    """Activation tensors far from unit scale (large eps shrinks X_ln) and
    weights with tiny magnitudes still match the oracle bit for bit."""
    import sparsity_gemm_b200 as sq
    x = synth.activations_student(31, 40, 512)
    for eps in [1e-5, 1e20, 3e38]:
        op = oracle.prepare(x, None, None, eps, 2, 4, 0)
        _, ex = gpu_prepare(x, None, None, eps, 2, 4, 0)
        assert_prep_matches(ex, op)
    w = (synth.weights(32, 64, 256).astype(np.float32) * 1e-3).astype(np.float16)
    ow = oracle.quantize_weight(w, 0)
    qw = sq.quantize_weight(cuda16(w), 0)
    assert_weight_matches(sq.weight_export(qw), ow)


RMS_CASES = [
    # (m_tok, k, fmt, n, m, weight): warp-per-row statistics (k <= 8192) and
    # CTA-per-row statistics (few rows of k = 14336)
    (37, 256, 0, 2, 4, False),
    (300, 1024, 1, 2, 4, True),
    (129, 768, 0, 4, 8, True),
    (5, 14336, 0, 2, 4, False),
    (3, 14336, 1, 2, 4, True),
]


@pytest.mark.parametrize("m_tok,k,fmt,n,m,weight", RMS_CASES)
def test_prepare_rms_bit_exact(m_tok, k, fmt, n, m, weight):
    import sparsity_gemm_b200 as sq
    x = synth.activations_student(500 + m_tok + k, m_tok, k)
    g = synth.ln_params(501, k)[0] if weight else None
    op = oracle.prepare(x, g, None, 1e-5, n, m, fmt, norm="rms")
    p = sq.prepare(cuda16(x), None if g is None else cuda16(g), None, 1e-5, n, m, fmt, norm="rms")
    assert_prep_matches(sq.prep_export(p), op)
    assert sq.get_last_error() == sq.OK


def test_linear_on_rms_prepared_input():
    import sparsity_gemm_b200 as sq
    m_tok, k, n_out = 200, 1024, 544
    x = synth.activations_student(510, m_tok, k)
    g = synth.ln_params(511, k)[0]
    w = synth.weights(512, n_out, k)
    op = oracle.prepare(x, g, None, 1e-5, 2, 4, 0, norm="rms")
    ow = oracle.quantize_weight(w, 0)
    p = sq.prepare(cuda16(x), cuda16(g), None, 1e-5, 2, 4, 0, norm="rms")
    out = sq.linear(p, sq.quantize_weight(cuda16(w), 0)).cpu().numpy()
    want, bound = oracle.linear_prepared(op, ow)
    assert_linear_close(out, want, bound)
    assert sq.get_last_error() == sq.OK
