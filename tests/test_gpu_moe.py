"""Parity of the mixture-of-experts grouped path with the oracle: grouped
weight quantization and the row gather bit for bit, the grouped dual-path
linear within 1e-3 * sum|a||w| per element, the edge cases of a routing
(experts with no rows, with exactly one tile, with one row past a tile, no
rows at all, one expert), device-side rejection of invalid routing arrays,
and the Qwen3-30B-A3B-shaped FFN (hidden 2048, 128 experts of intermediate
768, top-8 of 4096 tokens) on sampled outputs."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_common import assert_bits_equal, assert_linear_close, cuda16

pytestmark = pytest.mark.gpu

EPS = 1e-5


@pytest.fixture(scope="module")
def sq():
    import sparsity_gemm_b200 as sq
    assert torch.cuda.is_available()
    sq.lib()
    return sq


def _i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).cuda()


def padded_rows(offsets):
    """Row of the grouped prep that holds grouped row i, for every i (the
    layout the header documents: group g starts at row 128 * T_g, T_g the
    128-row tiles of the groups before it)."""
    offsets = np.asarray(offsets, np.int64)
    counts = np.diff(offsets)
    tiles = np.concatenate([[0], np.cumsum((counts + 127) // 128)])
    dst = np.empty(int(offsets[-1]), np.int64)
    for g in range(len(counts)):
        dst[offsets[g]:offsets[g + 1]] = 128 * tiles[g] + np.arange(counts[g])
    return dst, int(128 * tiles[-1])


def custom_routing(seed, tokens, counts):
    """Grouped rows with the given per-group counts, each a random token."""
    rng = np.random.default_rng(seed)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    row_idx = rng.integers(0, tokens, size=int(offsets[-1])).astype(np.int32)
    return row_idx, offsets


COUNTS = [0, 128, 129, 5, 0, 300, 1]


def check_gather(sq, gp, ex_src_rows, op, row_idx, offsets, local=None):
    """Exported grouped prep vs the oracle's prepared rows: every grouped row
    at its padded position, the rest of the groups' tiles zero."""
    ex = sq.prep_export(gp)
    dst, used = padded_rows(offsets)
    src = row_idx if local is None else local
    sel = np.arange(len(dst)) if ex_src_rows is None else ex_src_rows
    for name, key, want in [("mask idx", "idx", op.idx), ("S codes", "s_codes", op.s_codes),
                            ("S scales", "s_scales", op.s_scales), ("R codes", "r_codes", op.r_codes),
                            ("R scales", "r_scales", op.r_scales), ("mu", "mu", op.mu), ("rstd", "rstd", op.rstd)]:
        assert_bits_equal(name, ex[key][dst[sel]], want[src[sel]])
    pad = np.ones(used, bool)
    pad[dst] = False
    for key in ["idx", "s_codes", "s_scales", "r_codes", "r_scales", "mu", "rstd"]:
        assert not np.any(np.asarray(ex[key])[:used][pad]), key
    assert_bits_equal("s_t", np.float32([ex["s_t"]]), np.float32([op.s_t]))


@pytest.mark.parametrize("fmt", [0, 1])
def test_grouped_weight_quantization(sq, fmt):
    groups, n_out, k = 5, 96, 512
    w = np.stack([synth.weights(200 + g, n_out, k, std=0.02 * (g + 1)) for g in range(groups)])
    w[3] = 0  # an all-zero expert: tensor scale 1, zero codes
    qw = sq.quantize_weight_grouped(cuda16(w), fmt)
    assert qw.desc.groups == groups
    for g, ow in enumerate(oracle.quantize_weight_grouped(w, fmt)):
        wx = sq.weight_export(sq.group_view(qw, g))
        assert_bits_equal(f"group {g} codes", wx["codes"], ow.codes)
        assert_bits_equal(f"group {g} scales", wx["scales"], ow.scales)
        assert_bits_equal(f"group {g} s_tW", np.float32([wx["s_tw"]]), np.float32([ow.s_tw]))
    assert sq.get_last_error() == sq.OK


@pytest.mark.parametrize("fmt,n,m", [(0, 2, 4), (1, 2, 4), (0, 5, 8)])
def test_gather_rows_bit_exact(sq, fmt, n, m):
    tokens, k = 300, 512
    x = synth.activations_student(210, tokens, k)
    op = oracle.prepare(x, None, None, EPS, n, m, fmt)
    p = sq.prepare(cuda16(x), None, None, EPS, n, m, fmt)
    row_idx, offsets = custom_routing(211, tokens, COUNTS)
    gp = sq.gather_rows(p, _i32(row_idx), _i32(offsets), len(row_idx))
    assert gp.desc.groups == len(COUNTS) and gp.m_tok == sq.grouped_rows(len(row_idx), len(COUNTS))
    check_gather(sq, gp, None, op, row_idx, offsets)
    assert sq.get_last_error() == sq.OK


@pytest.mark.parametrize("fmt,n,m,norm", [(0, 2, 4, "layer"), (1, 2, 4, "layer"), (0, 3, 8, "layer"),
                                          (0, 2, 4, "rms")])
def test_prepare_grouped_equals_prepare_then_gather(sq, fmt, n, m, norm):
    """Rows in grouped order prepared straight into the grouped layout: the
    codes, scales, mask metadata and tensor scale equal a preparation
    followed by the identity gather bit for bit (over the groups' tiles),
    the statistics equal the plain preparation's (indexed by source row),
    and a grouped linear on either gives the same output bit for bit."""
    k = 512
    rows = int(sum(COUNTS))
    offsets = np.concatenate([[0], np.cumsum(COUNTS)]).astype(np.int32)
    x = cuda16(synth.activations_student(270, rows, k))
    off = _i32(offsets)
    gp = sq.prepare_grouped(x, off, None, None, EPS, n, m, fmt, norm=norm)
    p = sq.prepare(x, None, None, EPS, n, m, fmt, norm=norm)
    gg = sq.gather_rows(p, None, off, rows)
    assert gp.m_tok == gg.m_tok and gp.desc.groups == gg.desc.groups
    eg, ed, ep = sq.prep_export(gp), sq.prep_export(gg), sq.prep_export(p)
    used = padded_rows(offsets)[1]
    for key in ("idx", "s_codes", "s_scales", "r_codes", "r_scales"):
        assert_bits_equal(key, eg[key][:used], ed[key][:used])
    assert_bits_equal("s_t", np.float32([eg["s_t"]]), np.float32([ed["s_t"]]))
    assert_bits_equal("mu", eg["mu"][:rows], ep["mu"])
    assert_bits_equal("rstd", eg["rstd"][:rows], ep["rstd"])
    qw = sq.quantize_weight_grouped(cuda16(np.stack([synth.weights(271 + g, 96, k) for g in range(len(COUNTS))])), fmt)
    a = sq.linear_grouped(gp, off, qw, rows).cpu().numpy()
    b = sq.linear_grouped(gg, off, qw, rows).cpu().numpy()
    assert_bits_equal("grouped linear", a.view(np.uint16), b.view(np.uint16))
    assert sq.get_last_error() == sq.OK


def test_prepare_grouped_edge_cases(sq):
    """No rows (every tile row zero, tensor scale 1), and invalid offsets
    (recorded on the device, output untouched)."""
    k = 256
    empty = sq.prepare_grouped(torch.zeros((0, k), dtype=torch.float16, device="cuda"), _i32([0, 0, 0]))
    assert sq.prep_export(empty)["s_t"] == 1.0
    assert sq.get_last_error() == sq.OK
    x = cuda16(synth.activations_student(280, 40, k))
    good = sq.prepare_grouped(x, _i32([0, 20, 40]))
    sentinel = torch.full_like(good.buf, 0xA5)
    sq.prepare_grouped(x, _i32([0, 30, 20]), out=sq.Prepared(sentinel, None))
    assert sq.get_last_error() == sq.ERR_INVALID_ARG
    assert sq.last_timeout_site() == 0x201
    # the encode pass wrote nothing; only the statistics area and words may change
    n_codes = good.desc.m_tok * (k // 2)
    assert bool((sentinel[:n_codes] == 0xA5).all())


@pytest.mark.parametrize("fmt,n_out", [(0, 544), (1, 256), (0, 96)])
def test_linear_grouped_matches_oracle(sq, fmt, n_out):
    tokens, k = 300, 512
    groups = len(COUNTS)
    x = synth.activations_student(220 + fmt, tokens, k)
    w = np.stack([synth.weights(230 + g, n_out, k) for g in range(groups)])
    op = oracle.prepare(x, None, None, EPS, 2, 4, fmt)
    qws = oracle.quantize_weight_grouped(w, fmt)
    row_idx, offsets = custom_routing(221, tokens, COUNTS)
    p = sq.prepare(cuda16(x), None, None, EPS, 2, 4, fmt)
    qw = sq.quantize_weight_grouped(cuda16(w), fmt)
    off = _i32(offsets)
    gp = sq.gather_rows(p, _i32(row_idx), off, len(row_idx))
    out = sq.linear_grouped(gp, off, qw, len(row_idx)).cpu().numpy()
    want, bound = oracle.linear_grouped(op, row_idx, offsets, qws)
    assert_linear_close(out, want, bound)
    assert sq.get_last_error() == sq.OK


def test_one_group_identity_equals_dense_linear(sq):
    """One expert over all rows in order: the grouped path runs the dense
    path's arithmetic, so the outputs are identical (a shape with enough
    tiles that the dense launch does not split K)."""
    tokens, k, n_out = 1217, 768, 2048
    x = synth.activations_student(240, tokens, k)
    w = synth.weights(241, n_out, k)
    p = sq.prepare(cuda16(x), None, None, EPS, 2, 4, 0)
    qw1 = sq.quantize_weight(cuda16(w), 0)
    qwg = sq.quantize_weight_grouped(cuda16(w[None]), 0)
    off = _i32([0, tokens])
    gp = sq.gather_rows(p, None, off, tokens)
    dense = sq.linear(p, qw1).cpu().numpy()
    grouped = sq.linear_grouped(gp, off, qwg, tokens).cpu().numpy()
    assert np.array_equal(dense.view(np.uint16), grouped.view(np.uint16))
    assert sq.get_last_error() == sq.OK


def test_no_rows(sq):
    k = 256
    x = synth.activations_student(250, 4, k)
    p = sq.prepare(cuda16(x), None, None, EPS, 2, 4, 0)
    qw = sq.quantize_weight_grouped(cuda16(np.stack([synth.weights(251, 64, k)] * 3)), 0)
    off = _i32([0, 0, 0, 0])
    gp = sq.gather_rows(p, _i32(np.zeros(1, np.int32)), off, 0)
    out = sq.linear_grouped(gp, off, qw, 0)
    assert out.shape == (0, 64)
    assert sq.get_last_error() == sq.OK


def test_invalid_routing_is_rejected_on_the_device(sq):
    """Offsets that decrease, that do not end at rows, or a row index past
    the source: the kernels write nothing for them and the status word
    reports SHARQ_ERR_INVALID_ARG; the context stays usable."""
    tokens, k, n_out = 64, 256, 64
    x = synth.activations_student(260, tokens, k)
    p = sq.prepare(cuda16(x), None, None, EPS, 2, 4, 0)
    qw = sq.quantize_weight_grouped(cuda16(np.stack([synth.weights(261, n_out, k)] * 2)), 0)
    good_off = _i32([0, 20, 40])
    gp = sq.gather_rows(p, _i32(np.arange(40) % tokens), good_off, 40)
    assert sq.get_last_error() == sq.OK
    for bad in ([0, 30, 20], [0, 10, 39], [1, 20, 40]):
        off = _i32(bad)
        out = torch.full((40, n_out), 7.0, dtype=torch.float16, device="cuda")
        sq.linear_grouped(gp, off, qw, 40, out=out)
        assert sq.get_last_error() == sq.ERR_INVALID_ARG, bad
        assert sq.last_timeout_site() == 0x201
        assert bool((out == 7.0).all())
        sentinel = torch.full_like(gp.buf, 0xA5)
        gp2 = sq.gather_rows(p, _i32(np.arange(40) % tokens), off, 40, out=sq.Prepared(sentinel, None))
        assert sq.get_last_error() == sq.ERR_INVALID_ARG, bad
        assert bool((sentinel == 0xA5).all())
    bad_idx = np.arange(40) % tokens
    bad_idx[17] = tokens  # one past the source
    gp3 = sq.gather_rows(p, _i32(bad_idx), good_off, 40)
    assert sq.get_last_error() == sq.ERR_INVALID_ARG
    assert sq.last_timeout_site() == 0x202
    # the rejected row is zero; the context still runs the valid path
    ex = sq.prep_export(gp3)
    dst, _ = padded_rows([0, 20, 40])
    assert not ex["s_codes"][dst[17]].any()
    out = sq.linear_grouped(gp, good_off, qw, 40)
    assert sq.get_last_error() == sq.OK and bool(torch.isfinite(out).all())


def _sample(n, count, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.r_[0, n - 1, rng.choice(n, size=min(count, n), replace=False)])


def _check_moe_linear(sq, gp, op, local, row_idx, offsets, qw, w, fmt, sel, seed):
    """Sampled rows and columns of a grouped linear vs the oracle (the
    oracle quantizes only the experts the sampled rows use)."""
    groups, n_out, _ = w.shape
    cols = _sample(n_out, 96, seed)
    off = _i32(offsets)
    out = sq.linear_grouped(gp, off, qw, len(row_idx)).cpu().numpy()
    used = sorted({oracle.expert_of(offsets, int(i)) for i in sel})
    qws = [None] * groups
    for g in used:
        qws[g] = oracle.quantize_weight(w[g], fmt)
        wx = sq.weight_export(sq.group_view(qw, g))
        assert_bits_equal(f"expert {g} codes", wx["codes"], qws[g].codes)
        assert_bits_equal(f"expert {g} scales", wx["scales"], qws[g].scales)
    qws = [q if q is not None else qws[used[0]] for q in qws]  # unused experts are never read
    want, bound = oracle.linear_grouped(op, local, offsets, qws, sel=sel, cols=cols)
    assert_linear_close(out[np.ix_(sel, cols)], want, bound)
    assert sq.get_last_error() == sq.OK


def test_qwen3_30b_a3b_moe_ffn_full_size(sq):
    """Gate and up projections (2048 -> 768) read one gathered prep of the
    4096-token activation; the down projection (768 -> 2048) reads a
    grouped-order activation of all 32768 (token, expert) rows."""
    cfg = synth.QWEN3_MOE
    tokens, hidden, inter, groups, top_k = 4096, cfg["hidden"], cfg["inter"], cfg["n_experts"], cfg["top_k"]
    fmt, n, m = 0, 2, 4
    row_idx, offsets = synth.moe_routing(300, tokens, groups, top_k)
    rows = len(row_idx)
    assert rows == tokens * top_k
    off = _i32(offsets)
    sel = _sample(rows, 20, 301)

    # gate / up: token-order prep, then the gather
    x = synth.activations_student(302, tokens, hidden)
    p = sq.prepare(cuda16(x), None, None, EPS, n, m, fmt)
    gp = sq.gather_rows(p, _i32(row_idx), off, rows)
    s_t = oracle.tensor_scale_of(x, None, None, EPS, fmt)
    toks = np.unique(row_idx[sel])
    op = oracle.prepare(x[toks], None, None, EPS, n, m, fmt, s_t=s_t)
    local = np.zeros(rows, np.int64)
    local[sel] = np.searchsorted(toks, row_idx[sel])
    check_gather(sq, gp, sel, op, row_idx, offsets, local=local)
    for j, name in enumerate(["gate", "up"]):
        w = np.stack([synth.weights(310 + 1000 * j + g, inter, hidden) for g in range(groups)])
        qw = sq.quantize_weight_grouped(cuda16(w), fmt)
        _check_moe_linear(sq, gp, op, local, row_idx, offsets, qw, w, fmt, sel, 320 + j)
        del qw, w

    # down: a fresh activation already in grouped order
    xd = synth.activations_student(330, rows, inter)
    pd = sq.prepare(cuda16(xd), None, None, EPS, n, m, fmt)
    gpd = sq.gather_rows(pd, None, off, rows)
    s_td = oracle.tensor_scale_of(xd, None, None, EPS, fmt)
    opd = oracle.prepare(xd[sel], None, None, EPS, n, m, fmt, s_t=s_td)
    local_d = np.zeros(rows, np.int64)
    local_d[sel] = np.arange(len(sel))
    check_gather(sq, gpd, sel, opd, np.arange(rows), offsets, local=local_d)
    wd = np.stack([synth.weights(340 + g, hidden, inter) for g in range(groups)])
    qwd = sq.quantize_weight_grouped(cuda16(wd), fmt)
    _check_moe_linear(sq, gpd, opd, local_d, np.arange(rows), offsets, qwd, wd, fmt, sel, 350)
