"""Pins for the fp64 oracle, against things other than itself.

Each routine of oracle/ is checked against mathematics, a library routine or a
hand-worked fixture, chosen so that a dropped term, a wrong sign or index, or a
transposed operand fails at least one check:

- hand-worked fixtures (tests/golden/*.txt, each citing its passage), grouped
  pointwise included;
- the adjoint identity <conv_fwd(x), dY> = <x, dgrad(dY)> for every geometry
  the workloads use (reduced sizes), grouped and strided ones included;
- pointwise dgrad equals numpy's matmul of dY[M,K] and W[K,C];
- stride-1 depthwise dgrad equals the rotated-filter correlation;
- the row-streaming schedule equals the definition (strides 1..3, KH < S too);
- brute-force central differences of L(x) = <conv_fwd(x), dY>;
- torch.nn.grad.conv2d_input and torch.conv2d on CPU in fp64;
- closed forms: a delta dY gives the filter placed at (ho*S - ph, wo*S - pw);
  a centre-delta filter gives dX = dY; a constant dY gives sum(W) inside;
- planted mistakes (a wrong dY stride, an unrotated filter, a transposed filter)
  must each fail one of the pins.
"""
import os

import numpy as np
import pytest

import oracle
from convolution_backward_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rng(seed=0):
    return np.random.default_rng(seed)


def _read_golden(path):
    fields = {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, val = line.partition(":")
            fields[key.strip()] = val.strip()
    prob = dict(kv.split("=") for kv in fields["problem"].split())
    kind = prob.pop("kind")
    prob = {k: int(v) for k, v in prob.items()}
    arr = {k: np.array([float(t) for t in fields[k].split()]) for k in ("dY", "W", "dX")}
    return kind, prob, arr


@pytest.mark.parametrize("name", sorted(os.listdir(GOLDEN)))
def test_golden_fixture(name):
    if not name.endswith(".txt"):
        pytest.skip("not a fixture")
    kind, p, a = _read_golden(os.path.join(GOLDEN, name))
    Ho, Wo = oracle.out_dims(p["H"], p["W"], p["KH"], p["KW"], p["S"], p["ph"], p["pw"])
    K = p["C"] if kind == "depthwise" else p["K"]
    dy = a["dY"].reshape(p["N"], Ho, Wo, K)
    extra = {}
    if kind == "pointwise":
        w = a["W"].reshape(K, p["C"])
    elif kind == "depthwise":
        w = a["W"].reshape(p["KH"], p["KW"], p["C"])
    else:
        w = a["W"].reshape(K, p["KH"], p["KW"], p["C"] // p["groups"])
        extra = dict(groups=p["groups"], C=p["C"])
    dx = oracle.dgrad(dy, w, kind=kind, H=p["H"], W=p["W"], KH=p["KH"], KW=p["KW"], S=p["S"],
                      ph=p["ph"], pw=p["pw"], **extra)
    np.testing.assert_array_equal(dx.reshape(-1), a["dX"])
    pts = [(n, h, x, c) for n in range(p["N"]) for h in range(p["H"])
           for x in range(p["W"]) for c in range(p["C"])]
    got = oracle.dgrad_points(dy, w, pts, kind=kind, H=p["H"], W=p["W"], KH=p["KH"], KW=p["KW"],
                              S=p["S"], ph=p["ph"], pw=p["pw"], **extra)
    np.testing.assert_array_equal(got, a["dX"])


# Geometries: (N, H, W, C, K, KH, KW, S, ph, pw, kind, groups).  The workloads'
# filters at reduced batch, image and channel counts, plus grouped, strided and
# per-axis cases.
GEOMS = [
    (2, 5, 7, 6, 4, 1, 1, 1, 0, 0, "pointwise", 1),
    (1, 6, 6, 4, 4, 3, 3, 1, 1, 1, "depthwise", 4),
    (1, 9, 8, 3, 3, 31, 31, 1, 15, 15, "depthwise", 3),
    (1, 8, 9, 2, 2, 51, 5, 1, 25, 2, "depthwise", 2),
    (1, 9, 8, 2, 2, 5, 51, 1, 2, 25, "depthwise", 2),
    (2, 12, 11, 3, 3, 7, 7, 2, 3, 3, "depthwise", 3),
    (1, 7, 7, 2, 2, 7, 7, 1, 3, 3, "depthwise", 2),
    (1, 7, 6, 2, 2, 7, 7, 1, 1, 5, "depthwise", 2),
    (1, 5, 5, 2, 2, 5, 5, 1, 2, 0, "depthwise", 2),
    (1, 10, 9, 2, 2, 3, 3, 3, 1, 0, "depthwise", 2),
    (1, 9, 9, 2, 2, 2, 2, 3, 0, 1, "depthwise", 2),
    (1, 6, 7, 6, 4, 3, 2, 2, 1, 1, "grouped", 2),
    (1, 5, 6, 4, 6, 3, 3, 1, 1, 1, "grouped", 1),
]


def _rand_problem(g, seed):
    N, H, W, C, K, KH, KW, S, ph, pw, kind, groups = g
    r = rng(seed)
    Ho, Wo = oracle.out_dims(H, W, KH, KW, S, ph, pw)
    dy = r.standard_normal((N, Ho, Wo, K))
    if kind == "pointwise":
        w = r.standard_normal((K, C))
    elif kind == "depthwise":
        w = r.standard_normal((KH, KW, C))
    else:
        w = r.standard_normal((K, KH, KW, C // groups))
    x = r.standard_normal((N, H, W, C))
    return dy, w, x


def _kw(g):
    N, H, W, C, K, KH, KW, S, ph, pw, kind, groups = g
    return dict(kind=kind, H=H, W=W, KH=KH, KW=KW, S=S, ph=ph, pw=pw, groups=groups, C=C)


@pytest.mark.parametrize("g", GEOMS, ids=[f"{g[10]}{g[5]}x{g[6]}s{g[7]}p{g[8]}x{g[9]}" for g in GEOMS])
def test_adjoint_identity(g):
    dy, w, x = _rand_problem(g, 1)
    kw = _kw(g)
    dx = oracle.dgrad(dy, w, **kw)
    y = oracle.conv_fwd(x, w, kind=kw["kind"], K=g[4], KH=g[5], KW=g[6], S=g[7], ph=g[8],
                        pw=g[9], groups=g[11])
    lhs = float(np.sum(y * dy))
    rhs = float(np.sum(x * dx))
    scale = float(np.sum(np.abs(y * dy))) + 1e-300
    assert abs(lhs - rhs) <= 1e-12 * scale


@pytest.mark.parametrize("g", GEOMS, ids=[f"{g[10]}{g[5]}x{g[6]}s{g[7]}" for g in GEOMS])
def test_torch_conv2d_input_crosscheck(g):
    torch = pytest.importorskip("torch")
    N, H, W, C, K, KH, KW, S, ph, pw, kind, groups = g
    dy, w, _ = _rand_problem(g, 2)
    dx = oracle.dgrad(dy, w, **_kw(g))
    if kind == "pointwise":
        wt = torch.from_numpy(w).reshape(K, C, 1, 1)
    elif kind == "depthwise":
        wt = torch.from_numpy(np.ascontiguousarray(np.transpose(w, (2, 0, 1)))).reshape(C, 1, KH, KW)
    else:
        wt = torch.from_numpy(np.ascontiguousarray(np.transpose(w, (0, 3, 1, 2))))
    dyt = torch.from_numpy(np.ascontiguousarray(np.transpose(dy, (0, 3, 1, 2))))
    ref = torch.nn.grad.conv2d_input((N, C, H, W), wt, dyt, stride=S, padding=(ph, pw),
                                     groups=groups)
    ref = ref.permute(0, 2, 3, 1).numpy()
    np.testing.assert_allclose(dx, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("g", GEOMS, ids=[f"{g[10]}{g[5]}x{g[6]}s{g[7]}" for g in GEOMS])
def test_conv_fwd_matches_torch(g):
    torch = pytest.importorskip("torch")
    N, H, W, C, K, KH, KW, S, ph, pw, kind, groups = g
    _, w, x = _rand_problem(g, 3)
    y = oracle.conv_fwd(x, w, kind=kind, K=K, KH=KH, KW=KW, S=S, ph=ph, pw=pw, groups=groups)
    if kind == "pointwise":
        wt = torch.from_numpy(w).reshape(K, C, 1, 1)
    elif kind == "depthwise":
        wt = torch.from_numpy(np.ascontiguousarray(np.transpose(w, (2, 0, 1)))).reshape(C, 1, KH, KW)
    else:
        wt = torch.from_numpy(np.ascontiguousarray(np.transpose(w, (0, 3, 1, 2))))
    xt = torch.from_numpy(np.ascontiguousarray(np.transpose(x, (0, 3, 1, 2))))
    ref = torch.nn.functional.conv2d(xt, wt, stride=S, padding=(ph, pw), groups=groups)
    np.testing.assert_allclose(y, ref.permute(0, 2, 3, 1).numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("shape", [(1, 1, 1, 1, 1), (2, 3, 5, 8, 16), (1, 4, 7, 64, 40),
                                   (3, 2, 2, 5, 3)])
def test_pointwise_equals_matmul(shape):
    N, H, W, K, C = shape
    r = rng(4)
    dy = r.standard_normal((N, H, W, K))
    w = r.standard_normal((K, C))
    dx = oracle.dgrad(dy, w, kind="pointwise", H=H, W=W)
    ref = np.matmul(dy.reshape(-1, K), w).reshape(N, H, W, C)
    np.testing.assert_allclose(dx, ref, rtol=1e-13, atol=1e-13)


DW_S1 = [(3, 3, 1, 1), (31, 31, 15, 15), (51, 5, 25, 2), (5, 51, 2, 25), (7, 7, 3, 3),
         (7, 7, 1, 5), (5, 5, 2, 0), (1, 1, 0, 0), (4, 6, 3, 0), (64, 2, 40, 1)]


@pytest.mark.parametrize("f", DW_S1, ids=[f"{a}x{b}p{c}x{d}" for a, b, c, d in DW_S1])
def test_stride1_depthwise_equals_rotated_correlation(f):
    KH, KW, ph, pw = f
    r = rng(5)
    N, H, W, C = 2, 9, 10, 3
    Ho, Wo = oracle.out_dims(H, W, KH, KW, 1, ph, pw)
    dy = r.standard_normal((N, Ho, Wo, C))
    w = r.standard_normal((KH, KW, C))
    a = oracle.dgrad(dy, w, kind="depthwise", H=H, W=W, KH=KH, KW=KW, S=1, ph=ph, pw=pw)
    b = oracle.dw_rotated(dy, w, H=H, W=W, ph=ph, pw=pw)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


RS = [(7, 7, 2, 3, 3, 14, 13), (3, 3, 2, 1, 1, 8, 9), (3, 3, 1, 1, 1, 6, 6), (5, 3, 3, 2, 1, 10, 11),
      (2, 2, 3, 0, 0, 9, 10), (1, 1, 2, 0, 0, 5, 6), (7, 7, 2, 0, 0, 12, 12), (4, 5, 2, 3, 2, 9, 7),
      (7, 7, 1, 3, 3, 8, 8), (3, 3, 4, 1, 1, 13, 9)]


@pytest.mark.parametrize("f", RS, ids=[f"{a}x{b}s{c}p{d}x{e}" for a, b, c, d, e, _, _ in RS])
def test_rowstream_schedule_equals_definition(f):
    KH, KW, S, ph, pw, H, W = f
    r = rng(6)
    N, C = 2, 3
    Ho, Wo = oracle.out_dims(H, W, KH, KW, S, ph, pw)
    dy = r.standard_normal((N, Ho, Wo, C))
    w = r.standard_normal((KH, KW, C))
    a = oracle.dgrad(dy, w, kind="depthwise", H=H, W=W, KH=KH, KW=KW, S=S, ph=ph, pw=pw)
    b = oracle.dw_rowstream(dy, w, H=H, W=W, S=S, ph=ph, pw=pw)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)


def test_zero_contribution_rows_are_zero():
    # H = 12, 3x3 filter, stride 4, pad 0: Ho = 3 (rows 0..2, 4..6, 8..10 reached), row 3, 7, 11 not.
    r = rng(7)
    H = W = 12
    Ho, Wo = oracle.out_dims(H, W, 3, 3, 4, 0, 0)
    dy = r.standard_normal((1, Ho, Wo, 2))
    w = r.standard_normal((3, 3, 2))
    dx = oracle.dgrad(dy, w, kind="depthwise", H=H, W=W, KH=3, KW=3, S=4)
    for h in (3, 7, 11):
        assert np.all(dx[:, h] == 0)
        assert np.all(dx[:, :, h] == 0)
    assert np.any(dx[:, 10] != 0)


@pytest.mark.parametrize("g", [GEOMS[1], GEOMS[5], GEOMS[9], GEOMS[11], GEOMS[0]])
def test_points_equal_scatter(g):
    dy, w, _ = _rand_problem(g, 8)
    kw = _kw(g)
    dx = oracle.dgrad(dy, w, **kw)
    N, H, W, C = dx.shape
    pts = [(n, h, x, c) for n in range(N) for h in range(H) for x in range(W) for c in range(C)]
    got = oracle.dgrad_points(dy, w, pts, **kw)
    np.testing.assert_allclose(got, dx.reshape(-1), rtol=1e-13, atol=1e-13)


FD = [(1, 4, 5, 2, 3, 1, 1, 1, 0, 0, "pointwise", 1),
      (1, 5, 6, 3, 3, 3, 3, 1, 1, 1, "depthwise", 3),
      (1, 6, 5, 2, 2, 5, 2, 1, 2, 1, "depthwise", 2),
      (1, 6, 6, 3, 3, 3, 3, 2, 1, 1, "depthwise", 3),
      (1, 5, 5, 2, 4, 3, 3, 2, 1, 0, "grouped", 2)]


@pytest.mark.parametrize("g", FD, ids=[f"{g[10]}{g[5]}x{g[6]}s{g[7]}" for g in FD])
def test_finite_differences(g):
    dy, w, x = _rand_problem(g, 9)
    kw = _kw(g)
    dx = oracle.dgrad(dy, w, **kw)
    eps = 1e-3

    def L(xx):
        y = oracle.conv_fwd(xx, w, kind=g[10], K=g[4], KH=g[5], KW=g[6], S=g[7], ph=g[8],
                            pw=g[9], groups=g[11])
        return float(np.sum(y * dy))

    flat = x.reshape(-1)
    fd = np.empty_like(flat)
    for i in range(flat.size):
        xp = flat.copy()
        xm = flat.copy()
        xp[i] += eps
        xm[i] -= eps
        fd[i] = (L(xp.reshape(x.shape)) - L(xm.reshape(x.shape))) / (2 * eps)
    np.testing.assert_allclose(fd, dx.reshape(-1), rtol=1e-7, atol=1e-8)


@pytest.mark.parametrize("f", [(3, 3, 1, 1, 1), (7, 7, 2, 3, 3), (51, 5, 1, 25, 2),
                               (4, 6, 3, 2, 5)])
def test_delta_dy_places_filter(f):
    KH, KW, S, ph, pw = f
    H, W, C = 20, 21, 2
    Ho, Wo = oracle.out_dims(H, W, KH, KW, S, ph, pw)
    r = rng(10)
    w = r.standard_normal((KH, KW, C))
    for ho, wo in [(0, 0), (Ho - 1, Wo - 1), (Ho // 2, Wo // 3)]:
        dy = np.zeros((1, Ho, Wo, C))
        dy[0, ho, wo, 1] = 1.0
        dx = oracle.dgrad(dy, w, kind="depthwise", H=H, W=W, KH=KH, KW=KW, S=S, ph=ph, pw=pw)
        exp = np.zeros((1, H, W, C))
        for rr in range(KH):
            for ss in range(KW):
                h, x = ho * S - ph + rr, wo * S - pw + ss
                if 0 <= h < H and 0 <= x < W:
                    exp[0, h, x, 1] = w[rr, ss, 1]
        np.testing.assert_array_equal(dx, exp)


def test_centre_delta_filter_gives_dy():
    r = rng(11)
    for K in (3, 7, 31):
        P = K // 2
        w = np.zeros((K, K, 4))
        w[P, P, :] = 1.0
        dy = r.standard_normal((2, 9, 8, 4))
        dx = oracle.dgrad(dy, w, kind="depthwise", H=9, W=8, KH=K, KW=K, S=1, ph=P, pw=P)
        np.testing.assert_array_equal(dx, dy)


def test_constant_dy_gives_filter_sum_inside():
    r = rng(12)
    KH, KW, P = 5, 3, (2, 1)
    w = r.standard_normal((KH, KW, 3))
    H = W = 12
    Ho, Wo = oracle.out_dims(H, W, KH, KW, 1, *P)
    dy = np.full((1, Ho, Wo, 3), 2.5)
    dx = oracle.dgrad(dy, w, kind="depthwise", H=H, W=W, KH=KH, KW=KW, S=1, ph=P[0], pw=P[1])
    inner = dx[0, KH:H - KH, KW:W - KW, :]
    np.testing.assert_allclose(inner, np.broadcast_to(2.5 * w.sum(axis=(0, 1)), inner.shape),
                               rtol=1e-13)


# ------------------------------------------------------------ planted mistakes

def test_planted_wrong_dy_stride_is_caught():
    """dY pixel stride K+1 instead of K (the pointwise page's mutation) fails the matmul pin."""
    r = rng(13)
    N, H, W, K, C = 1, 3, 4, 8, 5
    buf = r.standard_normal(N * H * W * (K + 1))
    w = r.standard_normal((K, C))
    dy = buf[: N * H * W * K].reshape(N, H, W, K)
    ref = np.matmul(dy.reshape(-1, K), w).reshape(N, H, W, C)
    good = oracle.dgrad(buf, w, kind="pointwise", H=H, W=W, dy_shape=(N, H, W, K),
                        dy_strides=(H * W * K, W * K, K, 1))
    np.testing.assert_allclose(good, ref, rtol=1e-13, atol=1e-13)
    mutated = oracle.dgrad(buf, w, kind="pointwise", H=H, W=W, dy_shape=(N, H, W, K),
                           dy_strides=(H * W * (K + 1), W * (K + 1), K + 1, 1))
    assert not np.allclose(mutated, ref, rtol=1e-6, atol=1e-6)


def test_planted_unrotated_filter_is_caught():
    """Correlating with the unrotated filter (a dropped 180-degree turn) fails the adjoint pin."""
    r = rng(14)
    KH, KW, ph, pw = 3, 5, 1, 2
    N, H, W, C = 1, 7, 8, 2
    dy = r.standard_normal((N, H, W, C))
    w = r.standard_normal((KH, KW, C))
    x = r.standard_normal((N, H, W, C))
    wrong = oracle.dw_rotated(dy, w[::-1, ::-1, :], H=H, W=W, ph=ph, pw=pw)
    y = oracle.conv_fwd(x, w, kind="depthwise", KH=KH, KW=KW, S=1, ph=ph, pw=pw)
    lhs, rhs = float(np.sum(y * dy)), float(np.sum(x * wrong))
    assert abs(lhs - rhs) > 1e-6 * abs(lhs)


def test_planted_transposed_filter_is_caught():
    """Reading the depthwise filter as W[s][r][c] instead of W[r][s][c] fails the adjoint pin."""
    r = rng(15)
    KH = KW = 3
    N, H, W, C = 1, 7, 8, 2
    Ho, Wo = oracle.out_dims(H, W, KH, KW, 1, 1, 1)
    dy = r.standard_normal((N, Ho, Wo, C))
    w = r.standard_normal((KH, KW, C))
    x = r.standard_normal((N, H, W, C))
    y = oracle.conv_fwd(x, w, kind="depthwise", KH=KH, KW=KW, S=1, ph=1, pw=1)
    lhs = float(np.sum(y * dy))
    good = oracle.dgrad(dy, w, kind="depthwise", H=H, W=W, KH=KH, KW=KW, ph=1, pw=1,
                        w_strides=(1, KW * C, C, 0))
    assert abs(lhs - float(np.sum(x * good))) <= 1e-12 * abs(lhs)
    bad = oracle.dgrad(dy, w, kind="depthwise", H=H, W=W, KH=KH, KW=KW, ph=1, pw=1,
                       w_strides=(1, C, KW * C, 0))
    assert abs(lhs - float(np.sum(x * bad))) > 1e-6 * abs(lhs)


# --------------------------------------------------------------- input recipe

def test_synthetic_bf16_rounding_is_rne():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1e-40, np.inf, 3.0e38],
                 dtype=np.float32)
    b = synthetic.f32_to_bf16_bits(x)
    back = synthetic.bf16_bits_to_f32(b)
    torch = pytest.importorskip("torch")
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(back, ref)


def test_synthetic_f16_inputs_are_rne_and_bit_consistent():
    # binary16 has 11 significant bits: 1 + 2^-11 is halfway between 1 and
    # 1 + 2^-10 and rounds to the even neighbour 1; 1 + 3*2^-11 rounds up to
    # 1 + 2^-9; 2^-24 is the smallest subnormal and 2^-26 rounds to zero
    p = synthetic.Problem("f16_pin", "pointwise", "f16", 1, 1, 2, 8, 8, seed=5)
    inp = synthetic.make_inputs(p)
    np.testing.assert_array_equal(inp.dy_bits.view(np.float16).astype(np.float32), inp.dy)
    np.testing.assert_array_equal(inp.w_bits.view(np.float16).astype(np.float32), inp.w)
    x = np.array([1.0 + 2 ** -11, 1.0 + 3 * 2 ** -11, 2 ** -24, 2 ** -26, -65504.0], dtype=np.float32)
    np.testing.assert_array_equal(x.astype(np.float16).astype(np.float32),
                                  np.array([1.0, 1.0 + 2 ** -9, 2 ** -24, 0.0, -65504.0], dtype=np.float32))


def test_synthetic_workloads_shapes():
    p = synthetic.problem("dw7x7s2_bf16")
    assert (p.Ho, p.Wo) == (56, 56)
    assert synthetic.problem("pw_bf16").dy_shape == (32, 28, 28, 512)
    assert synthetic.problem("dw31x31_bf16").Ho == 64
    inp = synthetic.make_inputs(synthetic.problem("dw3x3_bf16"))
    assert inp.dy.shape == (8, 56, 56, 128) and inp.w.shape == (3, 3, 128)
    assert abs(float(np.std(inp.w)) - 1.0 / 3) < 0.02
    # the same seed gives the same draws
    again = synthetic.make_inputs(synthetic.problem("dw3x3_bf16"))
    np.testing.assert_array_equal(inp.dy_bits, again.dy_bits)


# --- the whole-array fp64 forms used for full-size comparisons -----------------

WHOLE_ARRAY_GEOMS = [
    # N, H, W, C, KH, KW, S, ph, pw
    (2, 7, 9, 3, 3, 3, 1, 1, 1),      # 3x3 'same'
    (1, 11, 10, 2, 7, 7, 2, 3, 3),    # 7x7 stride 2
    (2, 9, 8, 4, 5, 2, 3, 2, 1),      # stride 3, per-axis padding
    (1, 12, 5, 3, 4, 4, 2, 0, 3),     # even filter, unequal pads
    (1, 9, 9, 2, 2, 2, 3, 0, 0),      # filter smaller than the stride (gaps)
    (2, 13, 9, 3, 13, 5, 1, 6, 2),    # non-square stride-1 ('same')
    (1, 6, 6, 2, 1, 1, 1, 0, 0),      # 1x1
]


@pytest.mark.parametrize("geom", WHOLE_ARRAY_GEOMS)
def test_depthwise_taps_equals_scatter_loop(geom):
    """The per-tap slice form is the same sum as the scatter loop (up to fp64 rounding order)."""
    N, H, W, C, KH, KW, S, ph, pw = geom
    Ho = (H + 2 * ph - KH) // S + 1
    Wo = (W + 2 * pw - KW) // S + 1
    rng = np.random.default_rng(hash(geom) % 2**32)
    dy = rng.standard_normal((N, Ho, Wo, C))
    w = rng.standard_normal((KH, KW, C))
    got = oracle.depthwise_taps(dy, w, H=H, W=W, S=S, ph=ph, pw=pw)
    ref = oracle.dgrad(dy, w, kind="depthwise", H=H, W=W, KH=KH, KW=KW, S=S, ph=ph, pw=pw)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12 * (1 + np.abs(ref).max()))


def test_depthwise_taps_catches_a_dropped_tap():
    """A slice form that skips one tap must not pass the comparison above."""
    N, H, W, C, KH, KW, S, ph, pw = WHOLE_ARRAY_GEOMS[1]
    Ho = (H + 2 * ph - KH) // S + 1
    rng = np.random.default_rng(7)
    dy = rng.standard_normal((N, Ho, Ho, C))
    w = rng.standard_normal((KH, KW, C))
    w_dropped = w.copy()
    w_dropped[3, 4, :] = 0.0
    got = oracle.depthwise_taps(dy, w_dropped, H=H, W=W, S=S, ph=ph, pw=pw)
    ref = oracle.dgrad(dy, w, kind="depthwise", H=H, W=W, KH=KH, KW=KW, S=S, ph=ph, pw=pw)
    assert np.abs(got - ref).max() > 1e-3


def test_pointwise_matmul_equals_scatter_loop():
    rng = np.random.default_rng(11)
    dy = rng.standard_normal((2, 5, 7, 24))
    w = rng.standard_normal((24, 40))
    got = oracle.pointwise_matmul(dy, w)
    ref = oracle.dgrad(dy, w, kind="pointwise", H=5, W=7)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12 * (1 + np.abs(ref).max()))
