"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

None of these re-types the oracle's own formula.  Each pin is one of
  * a value or shape the pages print (tests/golden/, each entry cited),
  * a library routine for a special case (torch.nn.functional.conv3d in fp64,
    torch's bf16 conversion, numpy integer matmul),
  * an identity of the mathematics (Conv3d == flatten-and-dot, one-hot,
    linearity, exact integer arithmetic, the duplicated-frame identity).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _bits(a):
    return np.asarray(a, dtype=np.float32).view(np.uint32)


def _torch_norm_volume(frames, grid, tp, mean, std):
    """Normalised, time-padded volume built with torch ops (an independent
    construction): repeat the last frame, (x-mean)/std in fp32, torch bf16 RNE."""
    f = frames.float()
    T = f.shape[0]
    tpad = grid[0] * tp
    if tpad > T:
        f = torch.cat([f, f[-1:].expand(tpad - T, *f.shape[1:])], 0)
    f = f[:tpad]
    m = torch.tensor(mean, dtype=torch.float32).view(1, -1, 1, 1)
    s = torch.tensor(std, dtype=torch.float32).view(1, -1, 1, 1)
    return ((f - m) / s).to(torch.bfloat16).double()


def _torch_conv_rows(vol, w, bias, tp, p, grid, merge):
    """torch conv3d (kernel == stride) in fp64, rows put in merge order by a
    view/permute of the output grid."""
    wb = w.float().to(torch.bfloat16).double()
    x = vol.permute(1, 0, 2, 3).unsqueeze(0)                   # [1, C, Tpad, H, W]
    y = torch.nn.functional.conv3d(x, wb, None if bias is None else bias.double(),
                                   stride=(tp, p, p))[0]     # [E, gt, gh, gw]
    E, gt, gh, gw = y.shape
    if merge == 1:
        return y.permute(1, 2, 3, 0).reshape(-1, E)
    m = merge
    y = y.view(E, gt, gh // m, m, gw // m, m).permute(1, 2, 4, 3, 5, 0)
    return y.reshape(-1, E)


# --------------------------------------------------------------------------- bf16

def test_bf16_round_matches_torch_rne():
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-40, 38, 20000),
        # exact ties at bf16 precision: low 16 bits 0x8000 with even and odd kept lsb
        (np.arange(2000, dtype=np.uint32) * 0x10000 + 0x3f808000).view(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.4e38, np.inf, -np.inf, 1e-40, -1e-45,
                  1.00390625, 1.01171875], dtype=np.float32),
    ]).astype(np.float32)
    ours = oracle.bf16_round(vals)
    ref = torch.from_numpy(vals).to(torch.bfloat16).float().numpy()
    assert np.array_equal(_bits(ours), _bits(ref))
    nan = oracle.bf16_round(np.array([np.nan], dtype=np.float32))
    assert np.isnan(nan).all()


@pytest.mark.parametrize("mean,std", [(workloads.CLIP_MEAN, workloads.CLIP_STD),
                                      ((0.5, 0.25, -1.5), (0.5, 3.0, 0.1))])
def test_normalization_exhaustive_over_bf16_inputs(mean, std):
    """Every finite bf16 pixel value, every channel: oracle == torch fp32 (x-m)/s -> bf16."""
    bits = np.arange(65536, dtype=np.uint32) << 16
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    C = len(mean)
    frames = torch.from_numpy(np.tile(x, C).reshape(1, C, 1, -1).copy())
    ref = _torch_norm_volume(frames, (1, 1, 1), 1, mean, std).float().numpy()
    for c in range(C):
        ours = np.array([oracle.normalize_pixel(float(v), mean[c], std[c]) for v in x[::97]],
                        dtype=np.float32)
        assert np.array_equal(_bits(ours), _bits(ref[0, c, 0, ::97]))
    # the whole volume through the oracle's patchify (p=1 makes rows = pixels)
    rows = oracle.patchify(frames, (1, 1, x.size), 1, mean, std, C, 1, 1)
    assert np.array_equal(_bits(rows.T.reshape(C, -1)), _bits(ref[0, :, 0, :]))


# ------------------------------------------------------------- library special case

TINY = [
    # C, tp, p, E, T, gh, gw, merge, bias
    (1, 1, 1, 3, 1, 2, 2, 2, False),
    (1, 2, 2, 5, 3, 2, 4, 2, True),
    (3, 2, 3, 4, 4, 4, 2, 2, True),
    (3, 1, 4, 2, 2, 3, 5, 1, False),
    (3, 2, 2, 8, 1, 2, 2, 2, True),
    (1, 2, 3, 7, 5, 1, 3, 1, True),
]


@pytest.mark.parametrize("C,tp,p,E,T,gh,gw,merge,with_bias", TINY)
def test_frames_form_matches_torch_conv3d(C, tp, p, E, T, gh, gw, merge, with_bias):
    gt = -(-T // tp)
    frames = workloads.uniform01((T, C, gh * p, gw * p), 100 + C * 10 + p)
    w = workloads.normal((E, C, tp, p, p), 200 + E)
    bias = workloads.normal((E,), 300 + E) if with_bias else None
    mean = tuple(0.1 * (c + 1) for c in range(C))
    std = tuple(0.2 + 0.05 * c for c in range(C))
    out, mag = oracle.conv3d_frames(frames, (gt, gh, gw), merge, mean, std, w, bias, C, tp, p)
    vol = _torch_norm_volume(frames, (gt, gh, gw), tp, mean, std)
    ref = _torch_conv_rows(vol, w, bias, tp, p, (gt, gh, gw), merge).numpy()
    assert out.shape == ref.shape == (gt * gh * gw, E)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    assert np.all(mag >= np.abs(out - (0 if bias is None else bias.double().numpy())) - 1e-12)


@pytest.mark.parametrize("C,tp,p,E", [(3, 2, 2, 6), (1, 1, 3, 4), (3, 2, 14, 9), (2, 2, 4, 16)])
def test_patches_form_matches_torch_conv3d(C, tp, p, E):
    """view(-1, C, tp, p, p) -> Conv3d(kernel=stride) -> view(-1, E), as printed on
    Optimize VLM PatchEmbed (Qwen3VLVisionPatchEmbed.forward) and patch详解 §4.3."""
    N = 37
    K = C * tp * p * p
    x = workloads.normal((N, K), 400 + p)
    w = workloads.normal((E, C, tp, p, p), 500 + p)
    b = workloads.normal((E,), 600 + p)
    out, _ = oracle.conv3d_patches(x, w, b, C, tp, p)
    xb = x.to(torch.bfloat16).double().view(-1, C, tp, p, p)
    wb = w.to(torch.bfloat16).double()
    ref = torch.nn.functional.conv3d(xb, wb, b.double(), stride=(tp, p, p)).view(-1, E)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------- identities of the maths

def test_conv_equals_flatten_and_matmul():
    """Qwen2.5VL-Vision Encode-PatchEmbed, python验证: the Conv3d equals the
    flattened input times the flattened weight transposed."""
    C, tp, p, E = 3, 2, 14, 24
    frames = workloads.uniform01((3, C, 4 * p, 6 * p), 7)
    grid = (2, 4, 6)
    w = workloads.normal((E, C, tp, p, p), 8, std=0.02, dtype=torch.bfloat16)
    out, _ = oracle.conv3d_frames(frames, grid, 2, workloads.CLIP_MEAN, workloads.CLIP_STD,
                                  w, None, C, tp, p)
    rows = oracle.patchify(frames, grid, 2, workloads.CLIP_MEAN, workloads.CLIP_STD, C, tp, p)
    flat = rows.astype(np.float64) @ w.double().reshape(E, -1).numpy().T
    np.testing.assert_allclose(out, flat, rtol=1e-12, atol=1e-13)
    # and the patches form on those rows is the same thing again
    out2, _ = oracle.conv3d_patches(rows, w, None, C, tp, p)
    np.testing.assert_allclose(out2, flat, rtol=1e-12, atol=1e-13)


def test_one_hot_recovers_weight_columns():
    C, tp, p, E = 3, 2, 4, 11
    K = C * tp * p * p
    w = workloads.normal((E, C, tp, p, p), 9)
    b = workloads.normal((E,), 10)
    x = np.eye(K, dtype=np.float32)
    out, _ = oracle.conv3d_patches(x, w, b, C, tp, p)
    wb = w.to(torch.bfloat16).double().reshape(E, K).numpy()
    assert np.array_equal(out, wb.T + b.double().numpy()[None, :])
    zero, _ = oracle.conv3d_patches(np.zeros((3, K), np.float32), w, b, C, tp, p)
    assert np.array_equal(zero, np.broadcast_to(b.double().numpy(), (3, E)))


def test_linearity():
    C, tp, p, E = 3, 2, 3, 6
    K = C * tp * p * p
    w = workloads.normal((E, C, tp, p, p), 11)
    b = workloads.normal((E,), 12)
    # bf16-exact inputs keep the check exact up to fp64 rounding
    x = workloads.small_ints((5, K), 13, -8, 8)
    y = workloads.small_ints((5, K), 14, -8, 8)
    a, c = 2.0, -3.0
    fx, _ = oracle.conv3d_patches(x, w, b, C, tp, p)
    fy, _ = oracle.conv3d_patches(y, w, b, C, tp, p)
    fz, _ = oracle.conv3d_patches(a * x + c * y, w, b, C, tp, p)
    bb = b.double().numpy()
    np.testing.assert_allclose(fz - bb, a * (fx - bb) + c * (fy - bb), rtol=1e-12, atol=1e-10)


def test_integer_inputs_are_exact():
    """Idea from Optimize VLM PatchEmbed (randint inputs, R1 == R2): small
    integers make every product and partial sum exact."""
    C, tp, p, E, N = 3, 2, 16, 33, 21
    K = C * tp * p * p
    x = workloads.small_ints((N, K), 15, 0, 2)
    w = workloads.small_ints((E, C, tp, p, p), 16, -4, 4)
    b = workloads.small_ints((E,), 17, -100, 100)
    out, _ = oracle.conv3d_patches(x, w, b, C, tp, p)
    ref = x.numpy().astype(np.int64) @ w.numpy().reshape(E, K).astype(np.int64).T \
        + b.numpy().astype(np.int64)[None, :]
    assert np.array_equal(out, ref.astype(np.float64))


def test_single_frame_is_duplicated_to_tp():
    """patch详解 §4.5: an image (T=1) with temporal patch 2 still yields one
    temporal patch; both temporal slices see the same frame, so the output is
    the frame against the sum of the two weight slices."""
    C, tp, p, E = 3, 2, 14, 10
    frames = workloads.uniform01((1, C, 2 * p, 4 * p), 18)
    w = workloads.normal((E, C, tp, p, p), 19, std=0.02, dtype=torch.bfloat16)
    out, _ = oracle.conv3d_frames(frames, (1, 2, 4), 2, workloads.CLIP_MEAN, workloads.CLIP_STD,
                                  w, None, C, tp, p)
    vol = _torch_norm_volume(frames, (1, 2, 4), 1, workloads.CLIP_MEAN, workloads.CLIP_STD)
    wsum = (w.double()[:, :, 0] + w.double()[:, :, 1]).unsqueeze(2)   # [E, C, 1, p, p]
    ref = torch.nn.functional.conv3d(vol.permute(1, 0, 2, 3).unsqueeze(0), wsum,
                                     stride=(1, p, p))[0]
    ref = ref.view(E, 1, 1, 2, 2, 2).permute(1, 2, 4, 3, 5, 0).reshape(-1, E)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-13)


def test_odd_frame_count_repeats_last_frame():
    """T=3, tp=2 -> ceil(3/2)=2 temporal patches (patch详解 §4.5 ceil); the
    second one pairs frame 2 with a copy of itself."""
    C, tp, p, E = 1, 2, 2, 3
    frames = workloads.uniform01((3, C, 2 * p, 2 * p), 20)
    w = workloads.normal((E, C, tp, p, p), 21)
    out, _ = oracle.conv3d_frames(frames, (2, 2, 2), 2, (0.0,), (1.0,), w, None, C, tp, p)
    last, _ = oracle.conv3d_frames(frames[2:3], (1, 2, 2), 2, (0.0,), (1.0,), w, None, C, tp, p)
    assert np.array_equal(out[4:], last)
    with pytest.raises(ValueError):
        oracle.conv3d_frames(frames, (1, 2, 2), 2, (0.0,), (1.0,), w, None, C, tp, p)


# ------------------------------------------------------------- indexing and ordering

def test_patchify_is_a_permutation_of_pixels():
    """Index-encoding frames (value = flat pixel index, exact in bf16 below 256),
    identity normalisation: every pixel appears exactly once across the rows."""
    C, tp, p, T, gh, gw = 2, 2, 2, 2, 4, 4
    frames = workloads.index_frames(T, C, gh * p, gw * p)
    assert frames.numel() <= 256
    rows = oracle.patchify(frames, (1, gh, gw), 2, (0.0,) * C, (1.0,) * C, C, tp, p)
    assert sorted(rows.ravel().astype(np.int64).tolist()) == list(range(frames.numel()))


def test_patchify_matches_torch_unfold():
    """Rows equal an independent patch extraction with torch view/permute in
    view(-1, C, tp, p, p) order, then put in merge order."""
    C, tp, p, T, gh, gw = 3, 2, 14, 4, 6, 4
    frames = workloads.uniform01((T, C, gh * p, gw * p), 22)
    mean, std = workloads.CLIP_MEAN, workloads.CLIP_STD
    rows = oracle.patchify(frames, (2, gh, gw), 2, mean, std, C, tp, p)
    vol = _torch_norm_volume(frames, (2, gh, gw), tp, mean, std).float()   # [4, C, H, W]
    v = vol.view(2, tp, C, gh, p, gw, p).permute(0, 3, 5, 2, 1, 4, 6)     # gt,gh,gw,C,tp,i,j
    v = v.reshape(2, gh // 2, 2, gw // 2, 2, -1).permute(0, 1, 3, 2, 4, 5).reshape(-1, C * tp * p * p)
    assert np.array_equal(_bits(rows), _bits(v.numpy()))


def test_merge_order_matches_printed_mrope_positions():
    g = json.load(open(os.path.join(GOLD, "mrope_vision_positions_1_16_64.json")))
    t, h, w = g["grid_thw"]
    m = g["merge"]
    p = 2
    # frames encode (g_h, g_w) of each patch in channel 0 / channel 1 (exact small ints)
    C = 2
    f = torch.zeros(1, C, h * p, w * p)
    f[0, 0] = torch.arange(h).repeat_interleave(p).view(-1, 1).float()
    f[0, 1] = torch.arange(w).repeat_interleave(p).view(1, -1).float()
    rows = oracle.patchify(f, (t, h, w), m, (0.0, 0.0), (1.0, 1.0), C, 1, p)
    K = C * p * p
    gh_of_row = rows[:, 0].astype(int)
    gw_of_row = rows[:, K // 2].astype(int)
    n_tok = rows.shape[0] // (m * m)
    assert [3, n_tok] == g["shape"]
    off = g["text_prefix"]
    pos_h = np.array([off + gh_of_row[4 * v] // m for v in range(n_tok)])
    pos_w = np.array([off + gw_of_row[4 * v] // m for v in range(n_tok)])
    pr = g["printed"]
    assert pos_h[:3].tolist() == pr["h_head"] and pos_h[-3:].tolist() == pr["h_tail"]
    assert pr["h_contains"][:3] == pos_h[32:35].tolist()
    assert pos_w[:2].tolist() == pr["w_head"] and pos_w[-2:].tolist() == pr["w_tail"]
    assert pos_w[30:32].tolist() == pr["w_first_run_tail"]
    assert pos_w[32:34].tolist() == pr["w_second_run_head"]
    # every merged token's 4 rows form one 2x2 window
    for v in range(n_tok):
        win = {(int(gh_of_row[4 * v + d]), int(gw_of_row[4 * v + d])) for d in range(4)}
        hh, ww = pos_h[v] - off, pos_w[v] - off
        assert win == {(2 * hh + a, 2 * ww + b) for a in range(2) for b in range(2)}
    assert g["text_after"]["first"] == off + max(h // m, w // m)


def test_page_counts():
    g = json.load(open(os.path.join(GOLD, "page_counts.json")))
    for ent in g["entries"]:
        C, tp, p, m = ent["C"], ent["tp"], ent["p"], ent["merge"]
        gt, gh, gw = ent["grid_thw"]
        assert C * tp * p * p == ent["patch_dim"], ent["source"]
        T = ent["T"]
        H = ent.get("H", gh * p)
        W = ent.get("W", gw * p)
        frames = torch.zeros(T, C, H, W)
        w = torch.zeros(2, C, tp, p, p)
        out, _ = oracle.conv3d_frames(frames, (gt, gh, gw), m, (0.0,) * C, (1.0,) * C, w, None,
                                      C, tp, p)
        assert out.shape[0] == ent["patches"], ent["source"]
        if "merged_tokens" in ent:
            assert out.shape[0] // (m * m) == ent["merged_tokens"], ent["source"]
            assert [gt, gh // m, gw // m] == ent.get("merged_grid", [gt, gh // m, gw // m])


def test_kaiming_bound_of_config_weight():
    """PyTorch Conv default init bound 1/sqrt(fan_in), fan_in = 3*2*14*14 = 1176."""
    w = workloads.kaiming_uniform_conv((64, 3, 2, 14, 14), 2)
    b = 1.0 / np.sqrt(1176.0)
    assert abs(b - 0.02916) < 1e-5
    assert float(w.abs().max()) <= b and float(w.abs().max()) > 0.99 * b


# ------------------------------------------------ fp32-exact patches form

@pytest.mark.parametrize("C,tp,p,E", [(3, 2, 2, 5), (1, 1, 3, 4), (2, 2, 4, 3)])
def test_patches_fp32_matches_torch_conv3d(C, tp, p, E):
    """The unrounded patches form equals torch's fp64 Conv3d on the fp32 values
    (a library routine), with values that bf16 cannot represent."""
    K = C * tp * p * p
    g = torch.Generator().manual_seed(300 + K)
    x = torch.randn(7, K, generator=g) * 1.2345
    w = torch.randn(E, C, tp, p, p, generator=g) * 0.4321
    b = torch.randn(E, generator=g)
    out, mag = oracle.conv3d_patches_fp32(x, w, b, C, tp, p)
    ref = torch.nn.functional.conv3d(x.double().view(-1, C, tp, p, p), w.double(), b.double()).view(7, E)
    assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)
    absref = torch.nn.functional.conv3d(x.double().abs().view(-1, C, tp, p, p), w.double().abs()).view(7, E)
    assert np.allclose(mag, absref.numpy(), rtol=1e-12, atol=1e-12)
    # and it really does not round: bf16-rounded inputs give a different result
    out_b, _ = oracle.conv3d_patches(x, w, b, C, tp, p)
    assert not np.allclose(out, out_b, rtol=1e-6, atol=0)


def test_patches_fp32_equals_rounded_form_on_bf16_values():
    """On bf16-representable inputs both patches forms are the same definition."""
    C, tp, p, E = 3, 2, 3, 6
    K = C * tp * p * p
    x = workloads.normal((9, K), 310).to(torch.bfloat16).float()
    w = workloads.normal((E, C, tp, p, p), 311, std=0.1).to(torch.bfloat16).float()
    a, ma = oracle.conv3d_patches_fp32(x, w, None, C, tp, p)
    b, mb = oracle.conv3d_patches(x, w, None, C, tp, p)
    assert np.array_equal(a, b) and np.array_equal(ma, mb)


# ------------------------------------------------------------- PatchMerger

def _bf16(t):
    return t.to(torch.bfloat16).double()


@pytest.mark.parametrize("E,m2,H,with_bias,eps", [(8, 4, 5, True, 1e-6), (12, 4, 3, False, 1e-6),
                                                  (6, 1, 4, True, 1e-6), (8, 4, 5, True, 0.5)])
def test_patch_merger_matches_torch(E, m2, H, with_bias, eps):
    """LayerNorm -> concat of m2 rows -> fc1 -> exact GELU -> fc2, against torch's
    fp64 layer_norm / linear / gelu library routines with the same bf16 roundings
    of the LayerNorm output, the GELU output and the weights (mytransformer
    README §3.2 and §4.1).  The large eps makes the place of eps visible: it is
    added to the variance under the square root."""
    g = torch.Generator().manual_seed(400 + E + m2)
    V = 5
    D = E * m2
    x = torch.randn(V * m2, E, generator=g) * 2.0 + 0.5
    gamma = torch.randn(E, generator=g) * 0.5 + 1.0
    beta = torch.randn(E, generator=g) * 0.1
    w1 = torch.randn(D, D, generator=g) * 0.2
    w2 = torch.randn(H, D, generator=g) * 0.2
    b1 = torch.randn(D, generator=g) * 0.1 if with_bias else None
    b2 = torch.randn(H, generator=g) * 0.1 if with_bias else None
    out, mag = oracle.patch_merger(x, m2, gamma, beta, eps, w1, b1, w2, b2)
    ln = torch.nn.functional.layer_norm(x.double(), (E,), gamma.double(), beta.double(), eps)
    h = _bf16(ln.float()).view(V, D)
    y = torch.nn.functional.linear(h, _bf16(w1), None if b1 is None else b1.double())
    gl = _bf16(torch.nn.functional.gelu(y).float())
    ref = torch.nn.functional.linear(gl, _bf16(w2), None if b2 is None else b2.double())
    assert np.allclose(out, ref.numpy(), rtol=1e-9, atol=1e-9)
    refmag = torch.nn.functional.linear(gl.abs(), _bf16(w2).abs())
    assert np.allclose(mag, refmag.numpy(), rtol=1e-9, atol=1e-9)


def test_patch_merger_concatenates_the_window_rows_in_order():
    """With fc1 = identity and fc2 selecting one input column, the output is that
    column of the (bf16) LayerNorm of the right row: row q of a window lands at
    columns q*E .. q*E+E-1 of the merged row."""
    E, m2, V = 4, 4, 3
    D = E * m2
    x = workloads.normal((V * m2, E), 410)
    gamma, beta = torch.ones(E), torch.zeros(E)
    w1 = torch.eye(D) * 64.0      # fc1 passes each merged column through, scaled
    ln = torch.nn.functional.layer_norm(x.double(), (E,), None, None, 1e-6)
    for col in (0, E + 1, 2 * E + 3, 3 * E + 2):
        w2 = torch.zeros(1, D)
        w2[0, col] = 1.0
        out, _ = oracle.patch_merger(x, m2, gamma, beta, 1e-6, w1, None, w2, None)
        q, e = divmod(col, E)
        for v in range(V):
            y = 64.0 * float(_bf16(ln[v * m2 + q, e].float()))
            gl = 0.5 * y * (1.0 + math.erf(y / math.sqrt(2.0)))
            assert out[v, 0] == float(torch.tensor(gl, dtype=torch.float32).to(torch.bfloat16).double())


def test_frames_form_is_translation_invariant():
    """Patches that an image and its crop share (the crop drops the first patch
    column and the first patch row) must embed identically: the frames form
    locates every patch at (g_h * p, g_w * p) of its own image.  Raster order
    (merge 1) so that the shared rows are easy to pair up."""
    C, tp, p, E = 3, 2, 4, 6
    T, gh, gw = 3, 4, 5
    img = workloads.normal((T, C, gh * p, gw * p), 420)
    crop = img[:, :, p:, p:].contiguous()
    w = workloads.normal((E, C, tp, p, p), 421, std=0.3)
    gt = -(-T // tp)
    full, _ = oracle.conv3d_frames(img, (gt, gh, gw), 1, (0.1, 0.2, 0.3), (0.5, 0.7, 0.9), w, None, C, tp, p)
    part, _ = oracle.conv3d_frames(crop, (gt, gh - 1, gw - 1), 1, (0.1, 0.2, 0.3), (0.5, 0.7, 0.9), w, None,
                                   C, tp, p)
    for t in range(gt):
        for y in range(gh - 1):
            for x in range(gw - 1):
                a = full[(t * gh + (y + 1)) * gw + (x + 1)]
                b = part[(t * (gh - 1) + y) * (gw - 1) + x]
                assert np.array_equal(a, b), (t, y, x)
