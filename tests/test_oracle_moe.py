"""Pins for the oracle's mixture-of-experts grouped linear (each expert's
dual-path linear over the rows routed to it, the activation prepared once):

- one group with the identity routing is the dense layer;
- experts with one-hot weight rows that differ per expert reveal, through
  an independent codec library, which prepared row and which expert every
  output row used, and that each expert's own tensor scale applies;
- relabelling the experts permutes nothing but the grouping;
- each expert's weight is quantized on its own;
- the routing generator gives every token top_k distinct experts.
"""
import ml_dtypes
import numpy as np

import synth


def _deq(codes, scales, fmt):
    blk = 16 if fmt == 0 else 32
    v = (codes & 0xF).astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    t = ml_dtypes.float8_e4m3fn if fmt == 0 else ml_dtypes.float8_e8m0fnu
    return v * np.repeat(scales.view(t).astype(np.float64), blk, axis=1)


def test_one_group_identity_routing_is_the_dense_layer(orc):
    x = synth.activations_student(80, 9, 256)
    w = synth.weights(81, 64, 256)
    p = orc.prepare(x, None, None, 1e-5, 2, 4, 0)
    qw = orc.quantize_weight(w, 0)
    dense, db = orc.linear_prepared(p, qw)
    got, gb = orc.linear_grouped(p, np.arange(9), [0, 9], [qw])
    assert np.array_equal(got, dense) and np.array_equal(gb, db)


def test_one_hot_experts_reveal_row_and_expert(orc):
    """Expert g's weight row j is one-hot at column (7 g + j) % k with value
    (g + 1) * 0.5 * 2^-g in fp16; with NVFP4 its tensor scale and block
    scale differ per expert, and the output is the dequantized activation at
    that column times the expert's dequantized one-hot value (equal up to
    the binary64 rounding of the product's order)."""
    k, n_out, groups, tokens = 256, 32, 4, 6
    fmt = 0
    x = synth.activations_student(82, tokens, k)
    p = orc.prepare(x, None, None, 1e-5, 2, 4, fmt)
    w = np.zeros((groups, n_out, k), np.float16)
    for g in range(groups):
        for j in range(n_out):
            w[g, j, (7 * g + j) % k] = np.float16((g + 1) * 0.5 * 2.0 ** -g)
    qws = orc.quantize_weight_grouped(w, fmt)
    row_idx, offsets = synth.moe_routing(83, tokens, groups, 2)
    out, _ = orc.linear_grouped(p, row_idx, offsets, qws)
    a = (_deq(p.s_codes, p.s_scales, fmt) + _deq(p.r_codes, p.r_scales, fmt)) * float(p.s_t)
    for i in range(len(row_idx)):
        g = int(np.searchsorted(offsets, i, side="right")) - 1
        wv = _deq(qws[g].codes, qws[g].scales, fmt) * float(qws[g].s_tw)
        for j in range(n_out):
            c = (7 * g + j) % k
            assert abs(wv[j, c] - float(w[g, j, c])) <= 0.07 * float(w[g, j, c])  # FP4 keeps the one-hot value
            assert np.isclose(out[i, j], a[row_idx[i], c] * wv[j, c], rtol=1e-14, atol=0)


def test_relabelling_experts_only_regroups(orc):
    k, n_out, groups, tokens = 256, 32, 5, 7
    x = synth.activations_student(84, tokens, k)
    p = orc.prepare(x, None, None, 1e-5, 2, 4, 1)
    w = np.stack([synth.weights(85 + g, n_out, k) for g in range(groups)])
    qws = orc.quantize_weight_grouped(w, 1)
    row_idx, offsets = synth.moe_routing(86, tokens, groups, 2)
    out, _ = orc.linear_grouped(p, row_idx, offsets, qws)
    perm = np.array([3, 0, 4, 1, 2])  # new label of old expert g is perm[g]
    inv = np.argsort(perm)
    new_rows, new_off = [], [0]
    for h in range(groups):
        g = inv[h]
        new_rows.append(row_idx[offsets[g]:offsets[g + 1]])
        new_off.append(new_off[-1] + offsets[g + 1] - offsets[g])
    out2, _ = orc.linear_grouped(p, np.concatenate(new_rows), new_off, [qws[inv[h]] for h in range(groups)])
    for h in range(groups):
        g = inv[h]
        assert np.array_equal(out2[new_off[h]:new_off[h + 1]], out[offsets[g]:offsets[g + 1]])


def test_experts_are_quantized_independently(orc):
    w = np.stack([synth.weights(87, 32, 256), synth.weights(88, 32, 256)])
    a = orc.quantize_weight_grouped(w, 0)
    w2 = w.copy()
    w2[1] = (w2[1].astype(np.float32) * 8).astype(np.float16)
    b = orc.quantize_weight_grouped(w2, 0)
    assert np.array_equal(a[0].codes, b[0].codes) and a[0].s_tw == b[0].s_tw
    assert np.array_equal(a[1].codes, b[1].codes) and b[1].s_tw == np.float32(a[1].s_tw * 8)


def test_routing_gives_each_token_top_k_distinct_experts():
    tokens, groups, top_k = 50, 16, 4
    row_idx, offsets = synth.moe_routing(89, tokens, groups, top_k)
    assert offsets[0] == 0 and offsets[-1] == tokens * top_k and np.all(np.diff(offsets) >= 0)
    per_token = [[] for _ in range(tokens)]
    for g in range(groups):
        seg = row_idx[offsets[g]:offsets[g + 1]]
        assert np.all(np.diff(seg) > 0)  # ascending, no token twice in an expert
        for t in seg:
            per_token[t].append(g)
    assert all(len(set(e)) == top_k for e in per_token)
