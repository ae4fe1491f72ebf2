"""CUDA path vs. the CPU oracle, element by element, on seeded inputs.

Bar: packed bytes, gamma, x~, eta, xsum and y_int are bit-exact; y (fp32 or
bf16) is bit-exact as well, which is stricter than the 1-ulp bound the
method's arithmetic allows, because both sides apply the same single fp32
rounding to each step (the pinned reading of the rescale).  Every call goes
through the C ABI (``ternary_weight_linear_04_b200.bitlinear``).
"""
import numpy as np
import pytest
import torch

from oracle import native as orc
from oracle import reference as ref
from ternary_weight_linear_04_b200 import _lib
from ternary_weight_linear_04_b200 import bitlinear as bl
from ternary_weight_linear_04_b200 import build as libbuild
from ternary_weight_linear_04_b200 import inputs

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "bf16": torch.bfloat16}


@pytest.fixture(scope="module", autouse=True)
def _built():
    libbuild.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    assert bl.device_error() == 0


def gpu_pack(W):
    packed, gamma = bl.pack_weights(torch.from_numpy(W).cuda())
    return packed.cpu().numpy(), np.float32(gamma.cpu().numpy()[0]), packed, gamma


def gpu_quant(x, act):
    xq, eta, xsum = bl.quant_act(torch.from_numpy(x).cuda().to(DT[act]))
    return xq, eta, xsum


def y_bits(y):
    """Bit patterns of a CPU fp32 / bf16 tensor, for exact comparison."""
    if y.dtype == torch.bfloat16:
        return y.view(torch.int16).numpy().view(np.uint16)
    return y.numpy().view(np.uint32)


def oracle_y_bits(y32, out):
    return orc.f32_to_bf16_bits(y32) if out == "bf16" else y32.view(np.uint32)


def check_layer(W, x, act="f32", out="f32", path="auto"):
    N, K = W.shape
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    packed_h, gamma_h, packed, gamma = gpu_pack(W)
    assert gamma_h.view(np.uint32) == ref_gamma.view(np.uint32), (gamma_h, ref_gamma)
    np.testing.assert_array_equal(packed_h, ref_packed)
    ref_xq, ref_eta, ref_xsum = orc.quant_act(x)
    xq, eta, xsum = gpu_quant(x, act)
    np.testing.assert_array_equal(xq.cpu().numpy(), ref_xq)
    np.testing.assert_array_equal(eta.cpu().numpy().view(np.uint32), ref_eta.view(np.uint32))
    np.testing.assert_array_equal(xsum.cpu().numpy(), ref_xsum)
    y, y_int = bl.forward(xq, eta, xsum, packed, gamma, N, out_dtype=DT[out], want_int=True, path=path)
    ref_yint, ref_y = orc.forward(ref_xq, ref_eta, ref_packed, ref_gamma, K, N)
    np.testing.assert_array_equal(y_int.cpu().numpy(), ref_yint)
    np.testing.assert_array_equal(y_bits(y.cpu()), oracle_y_bits(ref_y, out))


# ----------------------------------------------------------------- small cases

def test_worked_example_through_the_abi():
    import json, os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_example_2x4.json")))
    W = np.array(g["W"], np.float32)
    x = np.array(g["x"], np.float32)
    packed_h, gamma_h, packed, gamma = gpu_pack(W)
    assert float(gamma_h) == g["gamma"]
    np.testing.assert_array_equal(packed_h, g["packed"])
    xq, eta, xsum = gpu_quant(x, "f32")
    np.testing.assert_array_equal(xq.cpu().numpy(), g["xq"])
    for path in ("generic", "auto"):
        y, y_int = bl.forward(xq, eta, xsum, packed, gamma, 2, out_dtype=torch.bfloat16,
                              want_int=True, path=path)
        np.testing.assert_array_equal(y_int.cpu().numpy(), g["y_int"])
        np.testing.assert_array_equal(y_bits(y.cpu()), g["y_bf16_bits"])


@pytest.mark.parametrize("K", [1, 2, 3, 5, 63, 65, 130, 255])
def test_ragged_k_generic(K):
    W, x = inputs.make_case(10 + K, 3, K, 37)
    check_layer(W, x, "f32", "f32", path="auto")


@pytest.mark.parametrize("path", ["gemv", "tcgen05", "generic"])
@pytest.mark.parametrize("M,K,N", [(1, 64, 8), (1, 256, 256), (2, 192, 300), (3, 640, 129),
                                   (4, 3200, 1000), (8, 1024, 257)])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_paths_agree_with_oracle(path, M, K, N, out):
    if path == "gemv" and M > 4 and bl.decode_regm_shape(M, K, N) is None:
        pytest.skip("the CUDA-core decode kernels do not take this shape")
    W, x = inputs.make_case(1000 + M * 7 + K + N, M, K, N, act_dtype="bf16")
    check_layer(W, x, "bf16", out, path=path)


@pytest.fixture
def forced_split():
    yield bl.set_tc_split
    bl.set_tc_split(0)


@pytest.mark.parametrize("M", [1, 5, 16, 17, 32, 33, 64, 65, 128])
@pytest.mark.parametrize("ks", [2, 3, 5, 8])
def test_tcgen05_split_k_clusters(forced_split, M, ks):
    """K split across a cluster of ks CTAs, partial tiles added in CTA 0's
    shared memory: every token tile width, uneven K shares (K = 1600 = 12.5
    tiles of 128, so the last tile is ragged and the shares differ), N with a
    partial feature tile."""
    forced_split(ks)
    W, x = inputs.make_case(3100 + 7 * M + ks, M, 1600, 389, act_dtype="bf16")
    check_layer(W, x, "bf16", "bf16", path="tcgen05")


@pytest.mark.parametrize("M,K,N", [(16, 3200, 8640), (16, 8640, 3200), (8, 8192, 1000), (32, 28672, 512)])
def test_tcgen05_auto_split_decode_shapes(M, K, N):
    """The library's own split choice on decode-sized batches."""
    W, x = inputs.make_case(3300 + M + K, M, K, N, act_dtype="bf16")
    check_layer(W, x, "bf16", "bf16", path="tcgen05")


@pytest.mark.parametrize("M", [9, 16, 17, 31, 32, 33, 64, 65, 127, 128, 129, 200, 256, 257, 300])
def test_tcgen05_token_tiles_and_tails(M):
    """Every token-tile width (16..256) plus ragged tails in M, N and K
    (K = 704 = 5.5 stages of 128; N = 389 = 3 tiles + 5 rows)."""
    W, x = inputs.make_case(2000 + M, M, 704, 389, w_dist="laplace", act_dtype="bf16")
    check_layer(W, x, "bf16", "bf16", path="tcgen05")


def test_long_k_pipeline_wraps():
    """More K stages than pipeline slots (K = 4096: 32 stages)."""
    W, x = inputs.make_case(77, 40, 4096, 300, act_dtype="bf16")
    check_layer(W, x, "bf16", "bf16", path="tcgen05")
    check_layer(W, x[:3], "bf16", "bf16", path="gemv")


def test_all_zero_and_identity_weights():
    K = 256
    x = np.random.default_rng(0).normal(0, 1, (5, K)).astype(np.float32)
    for W in (np.zeros((130, K), np.float32), (K * np.eye(K)).astype(np.float32),
              (-K * np.eye(K)).astype(np.float32)):
        for path in ("gemv", "tcgen05", "generic"):
            check_layer(W, x if path != "gemv" else x[:4], "f32", "f32", path=path)


def test_quant_unaligned_and_scalar_paths():
    """bf16/fp32 rows whose K breaks the 16-byte vector width, and a
    misaligned base pointer (a column slice), take the scalar loop."""
    rng = np.random.default_rng(3)
    for act in ("f32", "bf16"):
        for K in (7, 13, 100, 1001):
            x = inputs.draw_activations(rng, 6, K, "student_t_outliers", act)
            ref = orc.quant_act(x)
            got = gpu_quant(x, act)
            for a, b in zip(got, ref):
                np.testing.assert_array_equal(a.cpu().numpy(), b)
        big = torch.from_numpy(inputs.draw_activations(rng, 4, 129, "normal", act)).cuda().to(DT[act])
        xs = big[:, 1:].contiguous()[:, :]  # contiguous copy: aligned
        off = big.reshape(-1)[1:1 + 4 * 128].reshape(4, 128)  # base offset by one element
        for t in (xs, off):
            ref = orc.quant_act(t.float().cpu().numpy())
            got = bl.quant_act(t)
            for a, b in zip(got, ref):
                np.testing.assert_array_equal(a.cpu().numpy(), b)


def test_empty_batch_is_a_no_op():
    W, _ = inputs.make_case(5, 1, 128, 64)
    _, _, packed, gamma = gpu_pack(W)
    xq = torch.empty((0, 128), dtype=torch.int8, device="cuda")
    eta = torch.empty(0, dtype=torch.float32, device="cuda")
    xsum = torch.empty(0, dtype=torch.int32, device="cuda")
    y = bl.forward(xq, eta, xsum, packed, gamma, 64)
    assert y.shape == (0, 64)
    q = bl.quant_act(torch.empty((0, 128), dtype=torch.bfloat16, device="cuda"))
    assert q[0].shape == (0, 128)


def test_gamma_exact_on_hard_sums():
    """The exact-sum reduction on inputs where a float reduction in any
    order would differ: huge dynamic range, ties, subnormals."""
    rng = np.random.default_rng(8)
    cases = [
        (rng.standard_normal((333, 77)) * np.exp2(rng.integers(-126, 100, (333, 77)))).astype(np.float32),
        np.concatenate([np.full((1, 5), 2.0 ** 53), np.ones((1, 3))], axis=1).astype(np.float32),
        np.full((64, 64), 2.0 ** -149, np.float32),
        rng.normal(0, 0.02, (1, 1)).astype(np.float32),
    ]
    for W in cases:
        ref_packed, ref_gamma, _ = orc.pack_weights(W)
        packed_h, gamma_h, _, _ = gpu_pack(W)
        assert gamma_h.view(np.uint32) == ref_gamma.view(np.uint32)
        np.testing.assert_array_equal(packed_h, ref_packed)


def _midpoint_matrix(N, K, k, extra, rng):
    """N*K/8 weights 2^k, N*K/8 weights -2^(k-24), optionally N*K/8 weights
    2^(k-50), the rest 0, shuffled: mean |W| = 2^k (1 + 2^-24) / 8, the
    midpoint between two fp32 values (or 2^-50 relative above it)."""
    n = N * K // 8
    W = np.zeros(N * K, np.float32)
    W[:n] = 2.0 ** k
    W[n:2 * n] = -(2.0 ** (k - 24))
    if extra:
        W[2 * n:3 * n] = 2.0 ** (k - 50)
    return rng.permutation(W).reshape(N, K)


@pytest.mark.parametrize("N,K", [(8, 64), (333, 80), (8640, 32)])
def test_pack_gamma_on_rounding_midpoints(N, K):
    """Matrices whose mean |W| sits exactly on the midpoint of two fp32
    values, or 2^-50 (relative) above it: the pack's fp64 sum of |W| cannot
    decide gamma, so its exact exponent buckets must (the tie to even, or
    rounded up).  gamma, packed bytes and base-3 bytes bit-exact."""
    rng = np.random.default_rng(N + K)
    for k in (-7, 0, 3):
        for extra in (False, True):
            W = _midpoint_matrix(N, K, k, extra, rng)
            ref_packed, ref_gamma, _ = orc.pack_weights(W)
            t = ref.ternarise(W, ref_gamma)
            want = np.float32(2.0 ** (k - 3))
            assert ref_gamma == (np.nextafter(want, np.float32(np.inf)) if extra else want)
            packed_h, gamma_h, _, _ = gpu_pack(W)
            assert gamma_h.view(np.uint32) == ref_gamma.view(np.uint32)
            np.testing.assert_array_equal(packed_h, ref_packed)
            p3, g3 = bl.pack_weights3(torch.from_numpy(W).cuda())
            assert np.float32(g3.cpu().numpy()[0]).view(np.uint32) == ref_gamma.view(np.uint32)
            np.testing.assert_array_equal(p3.cpu().numpy(), ref.pack3(t))


def test_pack_rejects_a_short_workspace():
    """The binding checks a caller's pack workspace against
    bitlinear_pack_workspace_bytes() (the C ABI takes a plain pointer and
    cannot); a workspace of exactly that size works."""
    W = torch.zeros((4, 64), device="cuda")
    with pytest.raises(ValueError):
        bl.pack_weights(W, workspace=torch.empty(2048, dtype=torch.uint8, device="cuda"))
    need = int(_lib.lib().bitlinear_pack_workspace_bytes())
    packed, gamma = bl.pack_weights(W, workspace=torch.empty(need, dtype=torch.uint8, device="cuda"))
    assert np.float32(gamma.cpu().numpy()[0]) == np.float32(1e-5)  # all-zero W: the floor
    assert np.all(packed.cpu().numpy() == 0x55)  # every code 01 (t = 0)


def _rd32(x):
    """The largest fp32 <= the fp64 value x."""
    f = np.float32(x)
    return np.nextafter(f, np.float32(-np.inf)) if float(f) > x else f


def _around(v, n=64):
    steps = [v]
    a = b = v
    for _ in range(n):
        a = np.nextafter(a, np.float32(-np.inf))
        b = np.nextafter(b, np.float32(np.inf))
        steps += [a, b]
    return np.array(steps, np.float32)


def test_pack_weights_at_the_ternary_threshold():
    """Weights at every fp32 within 64 ulps of gamma (0.5 + 2^-25) -- above
    it RN32(w / gamma) exceeds 0.5 -- and of gamma / 2, both signs, in a
    random matrix; re-placed until gamma (which they move) settles.  The
    kernels compare w with that threshold instead of dividing: packed bytes
    and gamma bit-exact, 2-bit and base-3."""
    rng = np.random.default_rng(12)
    W = rng.normal(0, 0.02, (96, 1000)).astype(np.float32)
    g = None
    for _ in range(30):
        g0, _ = ref.absmean_gamma(W)
        vals = np.concatenate([_around(_rd32(float(g0) * (0.5 + 2.0 ** -25))), _around(g0 * np.float32(0.5))])
        W[0, :vals.size] = vals
        W[1, :vals.size] = -vals
        g, _ = ref.absmean_gamma(W)
        if g == g0:
            break
    assert g == g0, "gamma did not settle"
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    t = ref.ternarise(W, ref_gamma)
    assert np.count_nonzero(t[0, :vals.size]) not in (0, vals.size)  # both sides of the threshold
    packed_h, gamma_h, _, _ = gpu_pack(W)
    assert gamma_h.view(np.uint32) == ref_gamma.view(np.uint32)
    np.testing.assert_array_equal(packed_h, ref_packed)
    p3, _ = bl.pack_weights3(torch.from_numpy(W).cuda())
    np.testing.assert_array_equal(p3.cpu().numpy(), ref.pack3(t))


# ----------------------------------------------------------------- full-size workloads

def sample_positions(M, N, rng, extra_rows=(), extra_cols=()):
    ms = list(rng.integers(0, M, 3000))
    ns = list(rng.integers(0, N, 3000))
    for m in extra_rows:
        ms += [m] * N
        ns += list(range(N))
    for n in extra_cols:
        ms += list(range(M))
        ns += [n] * M
    return np.array(ms, np.int64), np.array(ns, np.int64)


def check_full(W, x, batches, out="bf16", rows_full=True):
    N, K = W.shape
    rng = np.random.default_rng(N + K)
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    packed_h, gamma_h, packed, gamma = gpu_pack(W)
    assert gamma_h.view(np.uint32) == ref_gamma.view(np.uint32)
    np.testing.assert_array_equal(packed_h, ref_packed)
    del packed_h
    for M in batches:
        xm = x[:M]
        ref_xq, ref_eta, ref_xsum = orc.quant_act(xm)
        xq, eta, xsum = gpu_quant(xm, "bf16")
        np.testing.assert_array_equal(xq.cpu().numpy(), ref_xq)
        np.testing.assert_array_equal(eta.cpu().numpy(), ref_eta)
        np.testing.assert_array_equal(xsum.cpu().numpy(), ref_xsum)
        y, y_int = bl.forward(xq, eta, xsum, packed, gamma, N, out_dtype=DT[out], want_int=True)
        y_int = y_int.cpu().numpy()
        yb = y_bits(y.cpu())
        rows = (0, M - 1) if rows_full else ()
        cols = (0, N - 1, min(127, N - 1), min(128, N - 1))
        ms, ns = sample_positions(M, N, rng, rows, cols)
        ref_i, ref_y = orc.forward_at(ref_xq, ref_eta, ref_packed, ref_gamma, K, N, ms, ns)
        np.testing.assert_array_equal(y_int[ms, ns], ref_i)
        np.testing.assert_array_equal(yb[ms, ns], oracle_y_bits(ref_y, out))
        # a property that holds everywhere: y_int row sums against the packed codes
        # (sum_n y_int[m, n] = sum_k x~[m,k] * sum_n t[n,k]) on one random token
        m = int(rng.integers(0, M))
        col_t = np.zeros(K, np.int64)
        for n0 in range(0, N, 1024):
            from oracle import reference
            col_t += reference.unpack2(ref_packed[n0:n0 + 1024], K).astype(np.int64).sum(axis=0)
        assert int(y_int[m].astype(np.int64).sum()) == int(ref_xq[m].astype(np.int64) @ col_t)


def test_full_single_256():
    w = inputs.WORKLOADS["single_256"]
    W, x = inputs.make_matrix_inputs(w, 0)
    check_layer(W, x, "f32", "f32")


@pytest.mark.parametrize("idx", [0, 1])
def test_full_decode_3b(idx):
    w = inputs.WORKLOADS["decode_3b"]
    W, x = inputs.make_matrix_inputs(w, idx)
    check_full(W, x, w.batches)


def test_full_prefill_7b():
    w = inputs.WORKLOADS["prefill_7b"]
    W, x = inputs.make_matrix_inputs(w, 0)
    check_full(W, x, w.batches)


@pytest.mark.parametrize("idx", range(7))
def test_full_layer_70b(idx):
    w = inputs.WORKLOADS["layer_70b"]
    W, x = inputs.make_matrix_inputs(w, idx)
    check_full(W, x, w.batches)


def test_full_outlier_sweep():
    w = inputs.WORKLOADS["outlier_sweep"]
    W, x = inputs.make_matrix_inputs(w, 0)
    check_full(W, x, w.batches)


# ----------------------------------------------------------------- fused per-token layer

@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("K,N", [(64, 5), (3200, 1000), (4096, 700), (8640, 333), (16384, 77),
                                 (28672, 130)])
@pytest.mark.parametrize("static", [False, True])
def test_linear_fused_matches_oracle(M, K, N, static):
    W, x = inputs.make_case(5000 + M + K + N, M, K, N, x_dist="student_t_outliers", act_dtype="bf16")
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    _, _, packed, gamma = gpu_pack(W)
    torch.cuda.synchronize()
    xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
    y, (xq, eta, xsum), y_int = bl.linear(xd, packed, gamma, N, out_dtype=torch.bfloat16,
                                          want_quant=True, want_int=True, weights_static=static)
    ref_xq, ref_eta, ref_xsum = orc.quant_act(x)
    ref_yint, ref_y = orc.forward(ref_xq, ref_eta, ref_packed, ref_gamma, K, N)
    np.testing.assert_array_equal(xq.cpu().numpy(), ref_xq)
    np.testing.assert_array_equal(eta.cpu().numpy(), ref_eta)
    np.testing.assert_array_equal(xsum.cpu().numpy(), ref_xsum)
    np.testing.assert_array_equal(y_int.cpu().numpy(), ref_yint)
    np.testing.assert_array_equal(y_bits(y.cpu()), orc.f32_to_bf16_bits(ref_y))
    y2 = bl.linear(xd, packed, gamma, N, out_dtype=torch.float32)  # no optional outputs
    np.testing.assert_array_equal(y2.cpu().numpy().view(np.uint32), ref_y.view(np.uint32))


@pytest.mark.parametrize("act", ["f32", "bf16"])
def test_linear_two_kernel_path(act):
    """M above the decode range: quantise into caller scratch, then tcgen05."""
    W, x = inputs.make_case(6000, 37, 1024, 300, act_dtype=act)
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    _, _, packed, gamma = gpu_pack(W)
    y, (xq, eta, xsum) = bl.linear(torch.from_numpy(x).cuda().to(DT[act]), packed, gamma, 300,
                                   out_dtype=torch.float32, want_quant=True)
    ref_xq, ref_eta, _ = orc.quant_act(x)
    _, ref_y = orc.forward(ref_xq, ref_eta, ref_packed, ref_gamma, 1024, 300)
    np.testing.assert_array_equal(xq.cpu().numpy(), ref_xq)
    np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), ref_y.view(np.uint32))


def test_chained_layers_under_dependent_launch():
    """Layer 2 reads layer 1's output.  Launched back to back on one stream
    with static weights, the second kernel may start streaming its weights
    early but must read its activations only after the first has finished;
    a 20-deep chain checks that on every link."""
    rng = np.random.default_rng(99)
    K = 1024
    Ws = [inputs.draw_weights(rng, K, K) for _ in range(4)]
    packs = [gpu_pack(W)[2:] for W in Ws]
    ref = [orc.pack_weights(W)[:2] for W in Ws]
    torch.cuda.synchronize()
    x = inputs.draw_activations(rng, 1, K, "normal", "bf16")
    h = torch.from_numpy(x).cuda().to(torch.bfloat16)
    h_ref = x
    for i in range(20):
        pk, g = packs[i % 4]
        h = bl.linear(h, pk, g, K, out_dtype=torch.bfloat16, weights_static=True)
        rp, rg = ref[i % 4]
        xq, eta, _ = orc.quant_act(h_ref)
        _, y = orc.forward(xq, eta, rp, rg, K, K)
        h_ref = orc.f32_to_bf16_bits(y).astype(np.uint32) << 16
        h_ref = h_ref.view(np.float32)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(h.cpu().float().numpy().view(np.uint32), h_ref.view(np.uint32))


def test_bitlinear_module():
    W, x = inputs.make_case(7, 2, 512, 96, act_dtype="bf16")
    layer = bl.BitLinear.from_latent(torch.from_numpy(W).cuda())
    torch.cuda.synchronize()
    y = layer(torch.from_numpy(x).cuda().to(torch.bfloat16))
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    ref_xq, ref_eta, _ = orc.quant_act(x)
    _, ref_y = orc.forward(ref_xq, ref_eta, ref_packed, ref_gamma, 512, 96)
    np.testing.assert_array_equal(y_bits(y.cpu()), orc.f32_to_bf16_bits(ref_y))


@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("K", [64, 4096, 4160, 8192, 12288, 16384, 32768, 65536, 131072])
def test_decode_word_widths(M, K):
    """The decode kernel's own shape choice across K (padding words, ring
    stages, activations staged in shared memory or read from global), with
    N not a multiple of the rows per CTA."""
    if K * (1 if M == 1 else (2 if M == 2 else 4)) > 131072:
        pytest.skip("outside the decode kernel's shared-memory budget")
    W, x = inputs.make_case(9000 + M + K, M, K, 1237, act_dtype="bf16")
    check_layer(W, x, "bf16", "bf16", path="gemv")


@pytest.fixture
def forced_shape():
    yield bl.set_decode_shape
    bl.set_decode_shape(0, 0)


def _shape_or_skip(M, K, N, fused):
    try:
        return bl.decode_shape(M, K, N, fused=fused)
    except Exception as e:  # the forced shape cannot take this size
        if getattr(e, "status", None) == 2:
            pytest.skip("forced shape does not fit (M, K, N)")
        raise


@pytest.mark.parametrize("M", [1, 2, 3])
@pytest.mark.parametrize("RB", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("G", [1, 2, 7, 16])
@pytest.mark.parametrize("K,N", [(3200, 2000), (3200, 12400), (1024, 140)])
def test_decode_forced_shapes(forced_shape, M, RB, G, K, N):
    """Every (team width G, row block RB) instantiation of the decode kernel,
    fused and not: padding words (K/16 = 200 words against 32*G*nwj slots),
    partial row blocks, one row per CTA (N = 140), and a ring that wraps
    (N = 12400: 84 rows of 800 bytes per CTA)."""
    mt = 1 if M == 1 else (2 if M == 2 else 4)
    if RB * mt > 16:
        pytest.skip("RB * M' > 16")
    forced_shape(G, RB)
    shp = _shape_or_skip(M, K, N, True)
    assert (shp["team_warps"], shp["rows_per_block"]) == (G, RB)
    W, x = inputs.make_case(7000 + 17 * M + RB + 3 * G + N, M, K, N, act_dtype="bf16")
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    _, _, packed, gamma = gpu_pack(W)
    ref_xq, ref_eta, ref_xsum = orc.quant_act(x)
    ref_yint, ref_y = orc.forward(ref_xq, ref_eta, ref_packed, ref_gamma, K, N)
    xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
    # the fused kernel at every M (a one-matrix group always fuses)
    (yg,) = bl.linear_group(xd, [packed], [gamma], out_dtype=torch.bfloat16, weights_static=True)
    np.testing.assert_array_equal(y_bits(yg.cpu()), orc.f32_to_bf16_bits(ref_y))
    # bitlinear_linear (fused for M <= 2) with its optional outputs
    y, (xq, eta, xsum), y_int = bl.linear(xd, packed, gamma, N, out_dtype=torch.bfloat16,
                                          want_quant=True, want_int=True, weights_static=True)
    np.testing.assert_array_equal(xq.cpu().numpy(), ref_xq)
    np.testing.assert_array_equal(xsum.cpu().numpy(), ref_xsum)
    np.testing.assert_array_equal(y_int.cpu().numpy(), ref_yint)
    np.testing.assert_array_equal(y_bits(y.cpu()), orc.f32_to_bf16_bits(ref_y))
    _shape_or_skip(M, K, N, False)
    xq_d = torch.from_numpy(ref_xq).cuda()
    y2, y2_int = bl.forward(xq_d, torch.from_numpy(ref_eta).cuda(), torch.from_numpy(ref_xsum).cuda(),
                            packed, gamma, N, out_dtype=torch.float32, want_int=True, path="gemv")
    np.testing.assert_array_equal(y2_int.cpu().numpy(), ref_yint)
    np.testing.assert_array_equal(y2.cpu().numpy().view(np.uint32), ref_y.view(np.uint32))


def test_decode_shape_query_and_override(forced_shape):
    shp = bl.decode_shape(1, 3200, 8640)
    assert shp["team_warps"] * shp["teams"] <= 16 and shp["rows_per_block"] in (1, 2, 4, 8, 16)
    assert shp["words_per_lane"] * 32 * shp["team_warps"] >= 3200 // 16
    assert shp["rows_per_cta"] * shp["ctas"] >= 8640
    forced_shape(3, 4)
    shp = bl.decode_shape(1, 3200, 8640)
    assert (shp["team_warps"], shp["rows_per_block"], shp["teams"]) == (3, 4, 5)
    with pytest.raises(Exception):
        forced_shape(17, 0)
    with pytest.raises(Exception):
        forced_shape(0, 3)


# ----------------------------------------------------------------- exact ties of bf16 activations

def _all_bf16_below(eta):
    """Every bf16 value x with 0 < |x| < eta, both signs, then eta itself
    first (so eta is the row's absmax)."""
    bits = np.arange(1, 0x7F80, dtype=np.uint32)  # positive finite bf16 patterns
    vals = (bits << 16).view(np.float32)
    vals = vals[vals < eta]
    return np.concatenate([[eta], vals, -vals]).astype(np.float32)


def _tie_rows(mantissas, K):
    rows = []
    for m in mantissas:
        eta = np.float32(m / 128.0)  # a bf16 value in [1, 2)
        r = _all_bf16_below(eta)
        assert r.size <= K
        rows.append(np.concatenate([r, np.zeros(K - r.size, np.float32)]))
    return np.stack(rows)


def test_quantiser_exact_on_every_bf16_tie():
    """For each of the 128 bf16 mantissas of eta in [1, 2), a row holding
    every bf16 value below eta: 127x/eta hits every exact .5 tie and every
    near tie the lattice of bf16 ratios can produce.  Standalone quantiser
    (bf16 input) against the oracle's division."""
    K = 34816
    x = _tie_rows(range(128, 256), K)
    ref_xq, ref_eta, ref_xsum = orc.quant_act(x)
    xq, eta, xsum = gpu_quant(x, "bf16")
    np.testing.assert_array_equal(eta.cpu().numpy(), ref_eta)
    np.testing.assert_array_equal(xq.cpu().numpy(), ref_xq)
    np.testing.assert_array_equal(xsum.cpu().numpy(), ref_xsum)


# (M, K) reaching every launch shape of the vectorised bf16 quantiser: up to
# 64 rows one vector of 8 values per thread and 128 / 256 / 512 / 1024
# threads (K up to 1024 / 2048 / 4096 / 8192), then 1024 threads with four
# vectors each (K up to 32768, longer rows read again); from 65 rows four
# vectors per thread and 128 / 256 / 512 / 1024 threads (K up to 4096 /
# 8192 / 16384 / 32768, longer rows read again; 10000 rows of 64 make CTAs
# loop over rows).  Ragged K (not a multiple of the threads x 8) in most
# shapes.
_QUANT_SHAPES = [(3, 1000), (3, 1024), (5, 2040), (64, 4096), (2, 8192), (7, 8200), (1, 34816),
                 (65, 4096), (65, 4000), (70, 8192), (66, 16384), (65, 17072), (65, 34816),
                 (65, 51200), (65, 51208), (4000, 1024), (10000, 64)]


@pytest.mark.parametrize("M,K", _QUANT_SHAPES)
def test_quantiser_every_launch_shape(M, K):
    """Standalone bf16 quantiser on every launch shape: rows drawn from the
    bf16 values below a bf16 eta (eta itself, then every value whose 127x/eta
    is exactly a half-integer, up to half the row, then others at random,
    all at random positions: exact ties in many 8-value vectors, none in
    others) and heavy-tailed rows, against the oracle."""
    rng = np.random.default_rng(9000 + M + K)
    mant = rng.integers(128, 256, size=min(M, 128))  # many rows repeat these
    rows = []
    for m in mant:
        eta = np.float32(m / 128.0)
        r = _all_bf16_below(eta)
        h = 254.0 * r[1:].astype(np.float64) / np.float64(eta)  # exact: 16-bit products
        tie = 1 + np.flatnonzero((h == np.round(h)) & (np.round(h) % 2 == 1))
        tie = rng.permutation(tie)[:K // 2]
        rest = np.setdiff1d(np.arange(1, r.size), tie)
        fill = rng.choice(rest, size=min(K - 1 - tie.size, rest.size), replace=False)
        pick = np.concatenate([[0], tie, fill])
        row = np.zeros(K, np.float32)
        row[rng.permutation(K)[:pick.size]] = r[pick]
        rows.append(row)
    if M > 1:  # a row below the 1e-5 floor of eta: the IEEE-quotient branch
        bits = rng.integers(0x3000, 0x3727, size=K).astype(np.uint32)
        rows[-1] = (bits << 16).view(np.float32) * np.where(rng.random(K) < 0.5, -1, 1).astype(np.float32)
    ties = np.stack(rows)[np.arange(M) % len(rows)]
    for x in (ties, inputs.draw_activations(rng, M, K, "student_t_outliers", "bf16")):
        ref_xq, ref_eta, ref_xsum = orc.quant_act(x)
        xq, eta, xsum = gpu_quant(x, "bf16")
        np.testing.assert_array_equal(eta.cpu().numpy(), ref_eta)
        np.testing.assert_array_equal(xq.cpu().numpy(), ref_xq)
        np.testing.assert_array_equal(xsum.cpu().numpy(), ref_xsum)


@pytest.mark.parametrize("group", range(4))
def test_fused_decode_exact_on_every_bf16_tie(group):
    """The same rows through the fused decode kernel's own quantiser, two
    tokens per call (K = 34816, so K * 2 fits the decode kernel)."""
    K, N = 34816, 64
    W, _ = inputs.make_case(4242, 1, K, N)
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    _, _, packed, gamma = gpu_pack(W)
    mant = list(range(128 + 32 * group, 160 + 32 * group))
    x = _tie_rows(mant, K)
    ref_xq, ref_eta, ref_xsum = orc.quant_act(x)
    for i in range(0, len(mant), 2):
        xd = torch.from_numpy(x[i:i + 2]).cuda().to(torch.bfloat16)
        y, (xq, eta, xsum) = bl.linear(xd, packed, gamma, N, out_dtype=torch.float32, want_quant=True,
                                       weights_static=True)
        np.testing.assert_array_equal(xq.cpu().numpy(), ref_xq[i:i + 2])
        np.testing.assert_array_equal(eta.cpu().numpy(), ref_eta[i:i + 2])
        np.testing.assert_array_equal(xsum.cpu().numpy(), ref_xsum[i:i + 2])
        _, ref_y = orc.forward(ref_xq[i:i + 2], ref_eta[i:i + 2], ref_packed, ref_gamma, K, N)
        np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), ref_y.view(np.uint32))


def test_quantiser_tiny_rows_use_the_eta_floor():
    """Rows with max |x| < 1e-5: eta is the 1e-5 floor (not a bf16 value), so
    ties go through the IEEE quotient.  Both quantisers."""
    K = 4096
    rng = np.random.default_rng(11)
    bits = rng.integers(0x3000, 0x3727, size=(2, K)).astype(np.uint32)  # bf16 in ~[4.7e-10, 9.9e-6]
    x = ((bits << 16).view(np.float32) * np.where(rng.random((2, K)) < 0.5, -1, 1)).astype(np.float32)
    assert np.abs(x).max() < 1e-5
    ref_xq, ref_eta, ref_xsum = orc.quant_act(x)
    xq, eta, xsum = gpu_quant(x, "bf16")
    np.testing.assert_array_equal(xq.cpu().numpy(), ref_xq)
    np.testing.assert_array_equal(eta.cpu().numpy(), ref_eta)
    W, _ = inputs.make_case(4243, 1, K, 32)
    _, _, packed, gamma = gpu_pack(W)
    y, (xq2, eta2, xsum2) = bl.linear(torch.from_numpy(x).cuda().to(torch.bfloat16), packed, gamma, 32,
                                      out_dtype=torch.float32, want_quant=True)
    np.testing.assert_array_equal(xq2.cpu().numpy(), ref_xq)
    np.testing.assert_array_equal(xsum2.cpu().numpy(), ref_xsum)


# ----------------------------------------------------------------- shared-input groups

@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("Ns", [(1000, 256, 256), (3000, 3000), (777,), (130, 2, 517, 64)])
def test_linear_group_matches_each_matrix(M, Ns):
    """Up to 4 matrices sharing x in one launch: each output equals the
    oracle's layer on its own matrix (and bitlinear_linear on it)."""
    K = 4096
    packs, gams, refs = [], [], []
    x = None
    for i, N in enumerate(Ns):
        W, xi = inputs.make_case(8100 + 13 * i + N + M, M, K, N, act_dtype="bf16")
        if x is None:
            x = xi
        ref_packed, ref_gamma, _ = orc.pack_weights(W)
        _, _, packed, gamma = gpu_pack(W)
        packs.append(packed); gams.append(gamma)
        ref_xq, ref_eta, _ = orc.quant_act(x)
        refs.append(orc.forward(ref_xq, ref_eta, ref_packed, ref_gamma, K, N)[1])
    xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
    for static in (False, True):
        ys = bl.linear_group(xd, packs, gams, out_dtype=torch.bfloat16, weights_static=static)
        for y, ref_y, p, g in zip(ys, refs, packs, gams):
            np.testing.assert_array_equal(y_bits(y.cpu()), orc.f32_to_bf16_bits(ref_y))
            y1 = bl.linear(xd, p, g, p.shape[0], out_dtype=torch.bfloat16, weights_static=static)
            np.testing.assert_array_equal(y_bits(y1.cpu()), y_bits(y.cpu()))
    ys = bl.linear_group(xd, packs, gams, out_dtype=torch.float32)
    for y, ref_y in zip(ys, refs):
        np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), ref_y.view(np.uint32))


# ----------------------------------------------------------------- base-3 packing

@pytest.mark.parametrize("N,K", [(1, 1), (7, 5), (33, 81), (130, 640), (1000, 3200), (257, 8640)])
def test_pack3_bytes_match_the_oracle(N, K):
    W, _ = inputs.make_case(9100 + N + K, 1, K, N)
    t = orc.pack_weights(W, want_ternary=True)[2]
    packed3, gamma = bl.pack_weights3(torch.from_numpy(W).cuda())
    np.testing.assert_array_equal(packed3.cpu().numpy(), ref.pack3(t))
    assert np.float32(gamma.cpu().numpy()[0]).view(np.uint32) == orc.pack_weights(W)[1].view(np.uint32)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 9])
@pytest.mark.parametrize("K,N", [(64, 8), (645, 129), (3200, 1000), (8640, 333)])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_forward3_matches_the_oracle(M, K, N, out):
    """Base-3 accumulate: y_int and y bit-exact against the oracle (the same
    values as the 2-bit path on the same trits); ragged K (a partial last
    group and padding bytes), M above 4 (several launches)."""
    W, x = inputs.make_case(9200 + M + K + N, M, K, N, act_dtype="bf16")
    ref_packed, ref_gamma, t = orc.pack_weights(W, want_ternary=True)
    ref_xq, ref_eta, ref_xsum = orc.quant_act(x)
    ref_yint, ref_y = orc.forward(ref_xq, ref_eta, ref_packed, ref_gamma, K, N)
    packed3, gamma = bl.pack_weights3(torch.from_numpy(W).cuda())
    xq, eta, xsum = (torch.from_numpy(a).cuda() for a in (ref_xq, ref_eta, ref_xsum))
    y, y_int = bl.forward3(xq, eta, xsum, packed3, gamma, N, out_dtype=DT[out], want_int=True)
    np.testing.assert_array_equal(y_int.cpu().numpy(), ref_yint)
    np.testing.assert_array_equal(y_bits(y.cpu()), oracle_y_bits(ref_y, out))


# ----------------------------------------------------------------- the headline decode call

@pytest.mark.parametrize("M", [1, 2, 4, 16])
def test_headline_decode_call_every_output(M):
    """The call the decode benchmark times: bitlinear_linear on both decode_3b
    matrices (K=3200 -> N=8640 and K=8640 -> N=3200) with static weights,
    the benchmark's own seeded inputs, issued back to back on one stream with
    no synchronisation between them (as the timed step does).  Every output
    element, x~, eta, xsum and y_int are compared with the oracle bit for
    bit ([Production] "The MatMul-Free Breakthrough" and pipeline step 5)."""
    w = inputs.WORKLOADS["decode_3b"]
    mats = []
    for idx in range(2):
        W, x = inputs.make_matrix_inputs(w, idx, m_max=max(M, 64))
        ref_packed, ref_gamma, _ = orc.pack_weights(W)
        _, _, packed, gamma = gpu_pack(W)
        mats.append((W.shape, x[:M], ref_packed, ref_gamma, packed, gamma))
    torch.cuda.synchronize()
    outs = []
    for (N, K), x, _, _, packed, gamma in mats:
        xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
        outs.append(bl.linear(xd, packed, gamma, N, out_dtype=torch.bfloat16, want_quant=True,
                              want_int=True, weights_static=True))
    torch.cuda.synchronize()
    for ((N, K), x, ref_packed, ref_gamma, _, _), (y, (xq, eta, xsum), y_int) in zip(mats, outs):
        ref_xq, ref_eta, ref_xsum = orc.quant_act(x)
        ref_yint, ref_y = orc.forward(ref_xq, ref_eta, ref_packed, ref_gamma, K, N)
        np.testing.assert_array_equal(xq.cpu().numpy(), ref_xq)
        np.testing.assert_array_equal(eta.cpu().numpy().view(np.uint32), ref_eta.view(np.uint32))
        np.testing.assert_array_equal(xsum.cpu().numpy(), ref_xsum)
        np.testing.assert_array_equal(y_int.cpu().numpy(), ref_yint)
        np.testing.assert_array_equal(y_bits(y.cpu()), orc.f32_to_bf16_bits(ref_y))


@pytest.mark.parametrize("M,K", [(4, 8192), (4, 28672), (3, 16384), (9, 8192)])
def test_forward3_many_tokens_with_large_shared_memory(M, K):
    """Base-3 launches whose activation slots need more than 48 KB of shared
    memory (4 tokens at K = 8192 take 55 KB; at K = 28672 187 KB): each
    kernel instantiation raises its own shared-memory limit, so these run as
    four-token launches.  y_int and y bit-exact against the oracle."""
    N = 515
    W, x = inputs.make_case(9300 + M + K, M, K, N, act_dtype="bf16")
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    ref_xq, ref_eta, ref_xsum = orc.quant_act(x)
    ref_yint, ref_y = orc.forward(ref_xq, ref_eta, ref_packed, ref_gamma, K, N)
    packed3, gamma = bl.pack_weights3(torch.from_numpy(W).cuda())
    xq, eta, xsum = (torch.from_numpy(a).cuda() for a in (ref_xq, ref_eta, ref_xsum))
    for out in ("f32", "bf16"):
        y, y_int = bl.forward3(xq, eta, xsum, packed3, gamma, N, out_dtype=DT[out], want_int=True)
        np.testing.assert_array_equal(y_int.cpu().numpy(), ref_yint)
        np.testing.assert_array_equal(y_bits(y.cpu()), oracle_y_bits(ref_y, out))


# ----------------------------------------------------------------- one token, weights in registers

_REG_CASES = ([(K, 1000) for K in (1024, 2048, 3200, 4096, 6144, 8192, 8640, 12288)]
              + [(K, 3200) for K in (1024, 2048, 3200, 4096, 6144, 8192, 8640)]
              + [(K, 8640) for K in (1024, 2048, 3200, 4096)]
              + [(64, 5), (3200, 8641), (8640, 2369), (1024, 148), (1024, 149)])


@pytest.mark.parametrize("K,N", _REG_CASES)
def test_register_decode_kernel_every_shape(K, N):
    """bitlinear_linear for one token on the kernel that holds each CTA's
    weights in registers: every (rows per warp, words per lane)
    instantiation, ragged last CTAs (N = 8641, 149), padding words (K = 3200
    fills 200 of 224 word slots), static and non-static weights, fp32 and
    bf16 y, y_int and the optional x~ / eta / xsum outputs, all bit-exact
    against the oracle."""
    shp = bl.decode_reg_shape(K, N)
    assert shp is not None, "the register kernel takes (K, N)"
    W, x = inputs.make_case(12000 + K + N, 1, K, N, act_dtype="bf16")
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    _, _, packed, gamma = gpu_pack(W)
    ref_xq, ref_eta, ref_xsum = orc.quant_act(x)
    ref_yint, ref_y = orc.forward(ref_xq, ref_eta, ref_packed, ref_gamma, K, N)
    xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
    torch.cuda.synchronize()
    for static in (True, False):
        y, (xq, eta, xsum), y_int = bl.linear(xd, packed, gamma, N, out_dtype=torch.bfloat16,
                                              want_quant=True, want_int=True, weights_static=static)
        np.testing.assert_array_equal(xq.cpu().numpy(), ref_xq)
        np.testing.assert_array_equal(eta.cpu().numpy().view(np.uint32), ref_eta.view(np.uint32))
        np.testing.assert_array_equal(xsum.cpu().numpy(), ref_xsum)
        np.testing.assert_array_equal(y_int.cpu().numpy(), ref_yint)
        np.testing.assert_array_equal(y_bits(y.cpu()), orc.f32_to_bf16_bits(ref_y))
    y32 = bl.linear(xd, packed, gamma, N, out_dtype=torch.float32, weights_static=True)
    np.testing.assert_array_equal(y32.cpu().numpy().view(np.uint32), ref_y.view(np.uint32))


def test_register_decode_kernel_eta_floor_and_forced_ring(forced_shape):
    """A row with every |x| below 1e-5 (eta is the 1e-5 floor, not a bf16
    value: the kernel takes IEEE quotients), and the same call with a decode
    shape forced, which runs the shared-memory kernel instead: identical
    outputs."""
    K, N = 3200, 1000
    rng = np.random.default_rng(12)
    bits = rng.integers(0x3000, 0x3727, size=(1, K)).astype(np.uint32)
    x = ((bits << 16).view(np.float32) * np.where(rng.random((1, K)) < 0.5, -1, 1)).astype(np.float32)
    W, _ = inputs.make_case(12001, 1, K, N)
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    _, _, packed, gamma = gpu_pack(W)
    ref_xq, ref_eta, ref_xsum = orc.quant_act(x)
    _, ref_y = orc.forward(ref_xq, ref_eta, ref_packed, ref_gamma, K, N)
    xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
    outs = []
    for force in (False, True):
        if force:
            forced_shape(1, 4)
        y, (xq, eta, xsum) = bl.linear(xd, packed, gamma, N, out_dtype=torch.float32, want_quant=True,
                                       weights_static=True)
        np.testing.assert_array_equal(xq.cpu().numpy(), ref_xq)
        np.testing.assert_array_equal(xsum.cpu().numpy(), ref_xsum)
        np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), ref_y.view(np.uint32))
        outs.append(y.cpu())
    assert torch.equal(outs[0], outs[1])


# ----------------------------------------------------------------- 2..4 tokens, weights in registers

_REGM_CASES = ([(K, 1000) for K in (1024, 2048, 3200, 4096, 6144, 8640, 12288)]
               + [(K, 3200) for K in (1024, 2048, 3200, 4096, 6144, 8640)]
               + [(K, 8640) for K in (1024, 2048, 3200, 4096)]
               + [(64, 5), (3200, 8641), (8640, 2369), (1024, 149)])


@pytest.fixture
def register_kernels():
    yield bl.set_decode_reg
    bl.set_decode_reg(True)


@pytest.mark.parametrize("M", [2, 3, 4, 5, 8])
@pytest.mark.parametrize("K,N", _REGM_CASES)
def test_multi_token_register_kernel_every_shape(register_kernels, M, K, N):
    """bitlinear_forward (x~ given) for 2..8 tokens on the kernel that holds
    each CTA's weights in registers: every (token slots, rows per warp, words
    per lane) instantiation, ragged last CTAs, padding words and tokens (M =
    3 in 4 slots, 5 in 8), static and non-static weights, fp32 and bf16 y;
    y_int and y bit-exact against the oracle, and, up to 4 tokens, identical
    to the shared-memory decode kernel (register kernels off)."""
    shp = bl.decode_regm_shape(M, K, N)
    assert shp is not None, "the register kernel takes (M, K, N)"
    W, x = inputs.make_case(13000 + 7 * M + K + N, M, K, N, act_dtype="bf16")
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    _, _, packed, gamma = gpu_pack(W)
    ref_xq, ref_eta, ref_xsum = orc.quant_act(x)
    ref_yint, ref_y = orc.forward(ref_xq, ref_eta, ref_packed, ref_gamma, K, N)
    xq, eta, xsum = (torch.from_numpy(a).cuda() for a in (ref_xq, ref_eta, ref_xsum.astype(np.int32)))
    for static in (True, False):
        for out in ("bf16", "f32"):
            y, y_int = bl.forward(xq, eta, xsum, packed, gamma, N, out_dtype=DT[out], want_int=True,
                                  path="gemv", weights_static=static)
            np.testing.assert_array_equal(y_int.cpu().numpy(), ref_yint)
            np.testing.assert_array_equal(y_bits(y.cpu()), oracle_y_bits(ref_y, out))
    if M <= 4:
        register_kernels(False)
        y_ring = bl.forward(xq, eta, xsum, packed, gamma, N, out_dtype=torch.bfloat16, path="gemv")
        np.testing.assert_array_equal(y_bits(y_ring.cpu()), orc.f32_to_bf16_bits(ref_y))


@pytest.mark.parametrize("M", [3, 4, 6, 8])
@pytest.mark.parametrize("K,N", [(3200, 8640), (8640, 3200)])
def test_multi_token_linear_uses_quantiser_then_register_kernel(M, K, N):
    """bitlinear_linear for 3..8 tokens (quantiser, then the register kernel)
    on decode_3b's matrices: x~, eta, xsum, y_int and y bit-exact."""
    W, x = inputs.make_case(13500 + M + K, M, K, N, act_dtype="bf16")
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    _, _, packed, gamma = gpu_pack(W)
    ref_xq, ref_eta, ref_xsum = orc.quant_act(x)
    ref_yint, ref_y = orc.forward(ref_xq, ref_eta, ref_packed, ref_gamma, K, N)
    xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
    y, (xq, eta, xsum), y_int = bl.linear(xd, packed, gamma, N, out_dtype=torch.bfloat16, want_quant=True,
                                          want_int=True, weights_static=True)
    np.testing.assert_array_equal(xq.cpu().numpy(), ref_xq)
    np.testing.assert_array_equal(eta.cpu().numpy().view(np.uint32), ref_eta.view(np.uint32))
    np.testing.assert_array_equal(xsum.cpu().numpy(), ref_xsum)
    np.testing.assert_array_equal(y_int.cpu().numpy(), ref_yint)
    np.testing.assert_array_equal(y_bits(y.cpu()), orc.f32_to_bf16_bits(ref_y))


# ----------------------------------------------------------------- 2..32 tokens, warp-level MMA

_MMA_CASES = ([(K, 8640) for K in (1024, 2048, 3200, 4096, 6144)]
              + [(K, 3200) for K in (2048, 4096, 6144, 8640, 12288)]
              + [(K, 1000) for K in (4096, 8192, 12288, 16384, 24576)]
              + [(64, 5), (3200, 8641), (8640, 2369), (1024, 149)])


@pytest.fixture
def mma_kernel():
    yield bl.set_decode_mma
    bl.set_decode_mma(True)


@pytest.mark.parametrize("M", [9, 12, 16])
@pytest.mark.parametrize("K,N", _MMA_CASES)
def test_warp_mma_decode_kernel_every_shape(mma_kernel, M, K, N):
    """bitlinear_forward (x~ given) for 9..16 tokens on the warp-MMA kernel:
    every (token slots, row blocks, K steps) instantiation, ragged last CTAs
    and row blocks, padding words, tokens and K steps, static and non-static
    weights, fp32 and bf16 y; y_int and y bit-exact against the oracle, and
    identical with the kernel switched off."""
    if bl.decode_mma_shape(M, K, N) is None:
        # the activation slots of 16 tokens fit one CTA's shared memory up to
        # K = 12288
        assert K > 12288, "the warp-MMA kernel takes this shape"
        pytest.skip("the activation slots of this many tokens exceed one CTA's shared memory")
    W, x = inputs.make_case(14000 + 11 * M + K + N, M, K, N, act_dtype="bf16")
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    _, _, packed, gamma = gpu_pack(W)
    ref_xq, ref_eta, ref_xsum = orc.quant_act(x)
    ref_yint, ref_y = orc.forward(ref_xq, ref_eta, ref_packed, ref_gamma, K, N)
    xq, eta, xsum = (torch.from_numpy(a).cuda() for a in (ref_xq, ref_eta, ref_xsum.astype(np.int32)))
    for static in (True, False):
        for out in ("bf16", "f32"):
            y, y_int = bl.forward(xq, eta, xsum, packed, gamma, N, out_dtype=DT[out], want_int=True,
                                  path="gemv", weights_static=static)
            np.testing.assert_array_equal(y_int.cpu().numpy(), ref_yint)
            np.testing.assert_array_equal(y_bits(y.cpu()), oracle_y_bits(ref_y, out))
    mma_kernel(False)
    y_off = bl.forward(xq, eta, xsum, packed, gamma, N, out_dtype=torch.bfloat16)
    np.testing.assert_array_equal(y_bits(y_off.cpu()), orc.f32_to_bf16_bits(ref_y))


@pytest.mark.parametrize("M", [9, 16, 24])
@pytest.mark.parametrize("K,N", [(3200, 8640), (8640, 3200)])
def test_warp_mma_linear_on_decode_shapes(M, K, N):
    """bitlinear_linear for 9..24 tokens on decode_3b's matrices (quantiser,
    then the warp-MMA kernel up to 16 tokens, the tensor-core kernel above):
    x~, eta, xsum, y_int and y bit-exact."""
    W, x = inputs.make_case(14500 + M + K, M, K, N, act_dtype="bf16")
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    _, _, packed, gamma = gpu_pack(W)
    ref_xq, ref_eta, ref_xsum = orc.quant_act(x)
    ref_yint, ref_y = orc.forward(ref_xq, ref_eta, ref_packed, ref_gamma, K, N)
    xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
    want_path = "gemv" if M <= 16 else "tcgen05"  # above 16 tokens: the tensor-core kernel
    assert bl.select_path(M, K, N, xd, packed, xd) == want_path
    y, (xq, eta, xsum), y_int = bl.linear(xd, packed, gamma, N, out_dtype=torch.bfloat16, want_quant=True,
                                          want_int=True, weights_static=True)
    np.testing.assert_array_equal(xq.cpu().numpy(), ref_xq)
    np.testing.assert_array_equal(xsum.cpu().numpy(), ref_xsum)
    np.testing.assert_array_equal(y_int.cpu().numpy(), ref_yint)
    np.testing.assert_array_equal(y_bits(y.cpu()), orc.f32_to_bf16_bits(ref_y))


_REGM_FUSED_CASES = [(1024, 1000), (3200, 1000), (8640, 1000), (12288, 1000), (3200, 3200), (8640, 3200),
                     (2048, 8640), (3200, 8640), (64, 5), (3200, 8641), (8640, 2369)]


@pytest.mark.parametrize("M", [2, 3, 4, 5, 8])
@pytest.mark.parametrize("K,N", _REGM_FUSED_CASES)
def test_multi_token_fused_layer_every_shape(register_kernels, M, K, N):
    """bitlinear_linear for 2..8 bf16 tokens on the register kernel, with the
    quantiser fused at two tokens (every CTA quantises both rows) and the
    quantiser kernel before it from three tokens on: every rows-per-warp
    value, ragged last CTAs, padding words and tokens, one token whose |x|
    are all below 1e-5 (eta is the 1e-5 floor: IEEE quotients), the optional
    x~ / eta / xsum outputs present or not, static and non-static weights,
    fp32 and bf16 y; bit-exact against the oracle and against the two-kernel
    path (register kernels off)."""
    assert bl.decode_regm_shape(M, K, N) is not None, "the register kernel takes (M, K, N)"
    W, x = inputs.make_case(15000 + 13 * M + K + N, M, K, N, act_dtype="bf16")
    rng = np.random.default_rng(M + K)
    bits = rng.integers(0x3000, 0x3727, size=K).astype(np.uint32)
    x[M - 1] = ((bits << 16).view(np.float32) * np.where(rng.random(K) < 0.5, -1, 1)).astype(np.float32)
    ref_packed, ref_gamma, _ = orc.pack_weights(W)
    _, _, packed, gamma = gpu_pack(W)
    ref_xq, ref_eta, ref_xsum = orc.quant_act(x)
    ref_yint, ref_y = orc.forward(ref_xq, ref_eta, ref_packed, ref_gamma, K, N)
    xd = torch.from_numpy(x).cuda().to(torch.bfloat16)
    for static in (True, False):
        y, (xq, eta, xsum), y_int = bl.linear(xd, packed, gamma, N, out_dtype=torch.bfloat16, want_quant=True,
                                              want_int=True, weights_static=static)
        np.testing.assert_array_equal(xq.cpu().numpy(), ref_xq)
        np.testing.assert_array_equal(eta.cpu().numpy().view(np.uint32), ref_eta.view(np.uint32))
        np.testing.assert_array_equal(xsum.cpu().numpy(), ref_xsum)
        np.testing.assert_array_equal(y_int.cpu().numpy(), ref_yint)
        np.testing.assert_array_equal(y_bits(y.cpu()), orc.f32_to_bf16_bits(ref_y))
    y32 = bl.linear(xd, packed, gamma, N, out_dtype=torch.float32, weights_static=True)
    np.testing.assert_array_equal(y32.cpu().numpy().view(np.uint32), ref_y.view(np.uint32))
    register_kernels(False)
    y_off = bl.linear(xd, packed, gamma, N, out_dtype=torch.bfloat16, weights_static=True)
    np.testing.assert_array_equal(y_bits(y_off.cpu()), orc.f32_to_bf16_bits(ref_y))
