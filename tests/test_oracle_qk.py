"""Pins for per-head QK RMSNorm + 3D RoPE."""
import numpy as np
import torch

from conftest import closed_form, load_golden


def test_golden(orc):
    g = load_golden("qk_rope.json")
    hd, pairs, theta = g["hd"], tuple(g["pairs"]), g["theta"]
    for case in g["cases"]:
        H = case.get("heads", 1)
        x = orc.f64_to_bf16(np.array(case["x"], dtype=np.float64)).reshape(1, H * hd)
        pos = np.array([case["pos"]], dtype=np.int32)
        out = orc.qk_rmsnorm_rope3d(x, np.array(case["w"], dtype=np.float64), H, hd, pos, pairs,
                                    theta, case["eps"])
        want = np.array([closed_form(e) for e in case["out"]])
        assert np.allclose(out.reshape(-1), want, rtol=0, atol=1e-14), case["name"]


def _setup(orc, R=6, H=3, hd=16, pairs=(3, 3, 2), seed=0):
    rng = np.random.default_rng(seed)
    x = orc.f64_to_bf16(rng.standard_normal((R, H * hd)) * 1.5)
    w = 1.0 + 0.02 * rng.standard_normal(hd)
    return x, w, H, hd, pairs


def test_position_zero_is_library_rms_norm(orc):
    x, w, H, hd, pairs = _setup(orc)
    eps = 1e-6
    out = orc.qk_rmsnorm_rope3d(x, w, H, hd, np.zeros((x.shape[0], 3), np.int32), pairs, 1e4, eps)
    v = torch.from_numpy(orc.bf16_to_f64(x)).reshape(-1, H, hd)
    ref = torch.nn.functional.rms_norm(v, (hd,), weight=torch.from_numpy(w), eps=eps)
    assert np.allclose(out, ref.reshape(x.shape[0], -1).numpy(), rtol=0, atol=1e-13)


def test_rotation_preserves_pair_norms(orc):
    x, w, H, hd, pairs = _setup(orc, seed=1)
    R = x.shape[0]
    rng = np.random.default_rng(2)
    pos = rng.integers(0, 90, (R, 3)).astype(np.int32)
    base = orc.qk_rmsnorm_rope3d(x, w, H, hd, np.zeros((R, 3), np.int32), pairs, 1e4, 1e-6)
    rot = orc.qk_rmsnorm_rope3d(x, w, H, hd, pos, pairs, 1e4, 1e-6)
    nb = np.hypot(base[:, 0::2], base[:, 1::2])
    nr = np.hypot(rot[:, 0::2], rot[:, 1::2])
    assert np.allclose(nb, nr, rtol=1e-13, atol=1e-15)
    assert not np.allclose(base, rot)


def test_relative_position_invariance_per_axis(orc):
    """q(p + d) . k(p' + d) == q(p) . k(p') per head, shifting one axis at a time."""
    x, w, H, hd, pairs = _setup(orc, R=2, seed=3)
    q, k = x[0:1], x[1:2]
    p, pp = np.array([[3, 5, 7]], np.int32), np.array([[11, 2, 9]], np.int32)

    def dots(a, b):
        qa = orc.qk_rmsnorm_rope3d(q, w, H, hd, a, pairs, 1e4, 1e-6).reshape(H, hd)
        kb = orc.qk_rmsnorm_rope3d(k, w, H, hd, b, pairs, 1e4, 1e-6).reshape(H, hd)
        return (qa * kb).sum(axis=1)

    ref = dots(p, pp)
    for axis in range(3):
        d = np.zeros((1, 3), np.int32)
        d[0, axis] = 17
        assert np.allclose(dots(p + d, pp + d), ref, rtol=1e-12, atol=1e-12)
        # a shift of one side alone does change the dot product
        assert not np.allclose(dots(p + d, pp), ref, rtol=1e-6, atol=1e-6)


def test_only_the_axis_segment_of_a_nonzero_axis_turns(orc):
    x, w, H, hd, pairs = _setup(orc, R=1, seed=4)
    pt, ph, pw = pairs
    base = orc.qk_rmsnorm_rope3d(x, w, H, hd, np.zeros((1, 3), np.int32), pairs, 1e4, 1e-6)
    bounds = [(0, pt), (pt, pt + ph), (pt + ph, pt + ph + pw)]
    for axis in range(3):
        pos = np.zeros((1, 3), np.int32)
        pos[0, axis] = 9
        out = orc.qk_rmsnorm_rope3d(x, w, H, hd, pos, pairs, 1e4, 1e-6).reshape(H, hd // 2, 2)
        b = base.reshape(H, hd // 2, 2)
        lo, hi = bounds[axis]
        changed = ~np.all(np.isclose(out, b, rtol=0, atol=0), axis=(0, 2))
        assert np.all(changed[lo:hi]) and not np.any(changed[:lo]) and not np.any(changed[hi:])


def test_normalised_head_rms_closed_form(orc):
    x, w, H, hd, pairs = _setup(orc, seed=5)
    eps = 0.05
    out = orc.qk_rmsnorm_rope3d(x, np.ones(hd), H, hd, np.zeros((x.shape[0], 3), np.int32), pairs,
                                1e4, eps).reshape(-1, H, hd)
    v = orc.bf16_to_f64(x).reshape(-1, H, hd)
    ms = (v ** 2).mean(axis=2)
    assert np.allclose(np.sqrt((out ** 2).mean(axis=2)), np.sqrt(ms / (ms + eps)), rtol=1e-13)


def test_grid_positions_match_row_major_indices(orc):
    T, Hg, Wg = 3, 4, 5
    ref = np.stack(np.indices((T, Hg, Wg)), axis=-1).reshape(-1, 3)
    assert np.array_equal(orc.grid_positions(T, Hg, Wg, 0, T * Hg * Wg), ref)
    assert np.array_equal(orc.grid_positions(T, Hg, Wg, 17, 20), ref[17:37])


def test_row_stride_reads_a_fused_buffer(orc):
    """Rows of k inside a [R, 3*H*hd] qkv buffer, read with row stride 3*H*hd,
    give the same as the dense rows."""
    x, w, H, hd, pairs = _setup(orc, seed=6)
    R, D = x.shape
    rng = np.random.default_rng(7)
    qkv = orc.f64_to_bf16(rng.standard_normal((R, 3 * D)))
    qkv[:, D:2 * D] = x
    pos = rng.integers(0, 50, (R, 3)).astype(np.int32)
    dense = orc.qk_rmsnorm_rope3d(x, w, H, hd, pos, pairs, 1e4, 1e-6)
    flat = np.concatenate([qkv.reshape(-1)[D:], np.zeros(D, np.uint16)])
    via_stride = orc.qk_rmsnorm_rope3d(flat, w, H, hd, pos, pairs, 1e4, 1e-6, row_stride=3 * D)
    assert np.array_equal(dense, via_stride)


# ------------------------------------------------ layout and norm options


def test_options_golden(orc):
    g = load_golden("qk_rope.json")
    hd, pairs, theta = g["hd"], tuple(g["pairs"]), g["theta"]
    for case in g["rotate_half_cases"]:
        x = orc.f64_to_bf16(np.array(case["x"], dtype=np.float64)).reshape(1, hd)
        out = orc.qk_rmsnorm_rope3d_ex(x, np.array(case["w"], dtype=np.float64), 1, hd,
                                       np.array([case["pos"]], np.int32), pairs, theta,
                                       case["eps"], layout=1)
        want = np.array([closed_form(e) for e in case["out"]])
        assert np.allclose(out.reshape(-1), want, rtol=0, atol=1e-14), case["name"]
    for case in g["row_norm_cases"]:
        H = case["heads"]
        x = orc.f64_to_bf16(np.array(case["x"], dtype=np.float64)).reshape(1, H * hd)
        out = orc.qk_rmsnorm_rope3d_ex(x, np.array(case["w"], dtype=np.float64), H, hd,
                                       np.array([case["pos"]], np.int32), pairs, theta,
                                       case["eps"], norm=1)
        want = np.array([closed_form(e) for e in case["out"]])
        assert np.allclose(out.reshape(-1), want, rtol=0, atol=1e-14), case["name"]


def test_default_options_are_the_pinned_operator(orc):
    x, w, H, hd, pairs = _setup(orc, seed=8)
    pos = np.random.default_rng(9).integers(0, 60, (x.shape[0], 3)).astype(np.int32)
    assert np.array_equal(orc.qk_rmsnorm_rope3d_ex(x, w, H, hd, pos, pairs, 1e4, 1e-6),
                          orc.qk_rmsnorm_rope3d(x, w, H, hd, pos, pairs, 1e4, 1e-6))


def test_rotate_half_is_interleaved_after_a_fixed_permutation(orc):
    """Moving element p to slot 2p and element p + hd/2 to slot 2p + 1 turns
    rotate-half pairs into interleaved pairs of the same index, so the
    rotate-half operator equals the (pinned) interleaved one conjugated by
    that permutation."""
    x, w, H, hd, pairs = _setup(orc, seed=10)
    R = x.shape[0]
    pos = np.random.default_rng(11).integers(0, 60, (R, 3)).astype(np.int32)
    perm = np.empty(hd, dtype=np.int64)           # interleaved slot -> rotate-half element
    perm[0::2] = np.arange(hd // 2)
    perm[1::2] = np.arange(hd // 2) + hd // 2
    xi = x.reshape(R, H, hd)[:, :, perm].reshape(R, H * hd)
    out_i = orc.qk_rmsnorm_rope3d(xi, w[perm], H, hd, pos, pairs, 1e4, 1e-6).reshape(R, H, hd)
    out_h = orc.qk_rmsnorm_rope3d_ex(x, w, H, hd, pos, pairs, 1e4, 1e-6, layout=1).reshape(R, H, hd)
    back = np.empty_like(out_i)
    back[:, :, perm] = out_i
    assert np.allclose(out_h, back, rtol=0, atol=1e-14)


def test_row_norm_at_position_zero_is_library_rms_norm(orc):
    x, _, H, hd, pairs = _setup(orc, seed=12)
    w = 1.0 + 0.02 * np.random.default_rng(13).standard_normal(H * hd)
    out = orc.qk_rmsnorm_rope3d_ex(x, w, H, hd, np.zeros((x.shape[0], 3), np.int32), pairs, 1e4,
                                   1e-6, norm=1)
    v = torch.from_numpy(orc.bf16_to_f64(x))
    ref = torch.nn.functional.rms_norm(v, (H * hd,), weight=torch.from_numpy(w), eps=1e-6)
    assert np.allclose(out, ref.numpy(), rtol=0, atol=1e-13)


def test_row_norm_with_one_head_is_the_head_norm(orc):
    x, w, _, hd, pairs = _setup(orc, H=1, seed=14)
    pos = np.random.default_rng(15).integers(0, 60, (x.shape[0], 3)).astype(np.int32)
    for layout in (0, 1):
        a = orc.qk_rmsnorm_rope3d_ex(x, w, 1, hd, pos, pairs, 1e4, 1e-6, layout=layout, norm=0)
        b = orc.qk_rmsnorm_rope3d_ex(x, w, 1, hd, pos, pairs, 1e4, 1e-6, layout=layout, norm=1)
        assert np.array_equal(a, b)


def test_options_keep_norms_and_relative_positions(orc):
    x, w, H, hd, pairs = _setup(orc, R=2, seed=16)
    wrow = np.tile(w, H)
    q, k = x[0:1], x[1:2]
    p, pp = np.array([[3, 5, 7]], np.int32), np.array([[11, 2, 9]], np.int32)
    for layout, norm in ((1, 0), (0, 1), (1, 1)):
        ww = wrow if norm else w
        f = lambda t, ps: orc.qk_rmsnorm_rope3d_ex(t, ww, H, hd, ps, pairs, 1e4, 1e-6,
                                                   layout=layout, norm=norm).reshape(H, hd)
        base = f(q, np.zeros((1, 3), np.int32))
        rot = f(q, p)
        half = hd // 2
        if layout == 0:
            nb, nr = np.hypot(base[:, 0::2], base[:, 1::2]), np.hypot(rot[:, 0::2], rot[:, 1::2])
        else:
            nb, nr = np.hypot(base[:, :half], base[:, half:]), np.hypot(rot[:, :half], rot[:, half:])
        assert np.allclose(nb, nr, rtol=1e-13)
        ref = (f(q, p) * f(k, pp)).sum(axis=1)
        for axis in range(3):
            d = np.zeros((1, 3), np.int32)
            d[0, axis] = 13
            assert np.allclose((f(q, p + d) * f(k, pp + d)).sum(axis=1), ref, rtol=1e-12, atol=1e-12)
