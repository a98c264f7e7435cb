"""Step-level parity of the CUDA path against the fp64 oracle (one test per
hot-path step, called through the C ABI of include/rm_ops.h)."""
import numpy as np
import pytest
import torch

import synth
import classifier_scoring_b200 as rm
from oracle import scorer as O
from tests.helpers import F32_RTOL

pytestmark = pytest.mark.gpu
BF16_REL = 2.0 ** -8      # one bf16 rounding of the output


def dev(a, dtype):
    return torch.as_tensor(np.ascontiguousarray(a)).to(dtype).cuda()


def f64(t):
    return t.detach().to(torch.float64).cpu().numpy()


@pytest.fixture(scope="module", autouse=True)
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    rm.lib()
    torch.cuda.init()


# --- GEMM (QKV / out-proj / FFN projections) -----------------------------------

# the shapes cover every tile width the launcher picks (64, 96, 128, 160, 192, 224, 256)
@pytest.mark.parametrize("M,N,K", [(1, 8, 8), (130, 936, 312), (3264, 2304, 768), (257, 768, 3072),
                                   (1000, 1200, 312), (128, 256, 64), (64, 128, 1200),
                                   (555, 3072, 768), (26112 // 16, 6144, 2048), (3328, 768, 768),
                                   (4000, 2304, 768)])
@pytest.mark.parametrize("act", [0, 1, 2])
def test_gemm_fp32_out(M, N, K, act):
    g = torch.Generator().manual_seed(M * 7 + N + K + act)
    x = (torch.randn(M, K, generator=g)).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    b = torch.randn(N, generator=g, dtype=torch.float32) * 0.1
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    xd, wd, bd = x.cuda(), w.cuda(), b.cuda()
    rm.ops.gemm(xd, wd, bd, y, rm.F32, M, N, K, act)
    torch.cuda.synchronize()
    X, W, B = f64(x), f64(w), f64(b)
    pre = O.linear(X, W, B)
    ref = pre if act == 0 else O.gelu(pre, O.GELU_ERF if act == 1 else O.GELU_TANH)
    scale = np.abs(X) @ np.abs(W).T + np.abs(B)          # sum_k |a_k b_k| + |bias|
    err = np.abs(f64(y) - ref)
    # GELU' <= 1.13; erff/tanhf add a few fp32 ulps of the output
    bound = F32_RTOL * scale * (1.0 if act == 0 else 1.2) + (0 if act == 0 else 4e-7 * np.abs(ref))
    assert np.all(err <= bound), float((err / bound).max())


# bf16 output: the epilogue stores boxes of 32 columns, so widths that are not
# a multiple of 32 (936, 1200) end in a box the store clips
@pytest.mark.parametrize("M,N,K", [(3264, 2304, 768), (77, 936, 312), (3328, 768, 768),
                                   (1000, 1200, 312), (4000, 2304, 768)])
def test_gemm_bf16_out_and_no_bias(M, N, K):
    g = torch.Generator().manual_seed(5)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    rm.ops.gemm(x.cuda(), w.cuda(), None, y, rm.BF16, M, N, K, 0)
    torch.cuda.synchronize()
    ref = O.linear(f64(x), f64(w), None)
    scale = np.abs(f64(x)) @ np.abs(f64(w)).T
    assert np.all(np.abs(f64(y) - ref) <= BF16_REL * np.abs(ref) + F32_RTOL * scale)


# Every output tile forced, on a ragged problem (partial last row and column
# tiles -- with a CTA pair the second CTA's rows or weight half can lie wholly
# outside -- and a partial last K block) and on a multi-round projection shape.
# Y is the head of a larger buffer whose rows past M must stay untouched (the
# epilogue's box stores are clipped to M rows).
GEMM_TILES = [(1, bn) for bn in (64, 96, 128, 160, 192, 224, 256)] + [(2, bn) for bn in (128, 192, 256)]


@pytest.mark.parametrize("cg,bn", GEMM_TILES, ids=[f"cg{c}-bn{b}" for c, b in GEMM_TILES])
@pytest.mark.parametrize("shape", ["ragged", "proj"])
@pytest.mark.parametrize("out", ["f32-gelu", "bf16"])
def test_gemm_every_tile(cg, bn, shape, out):
    M, N, K = (555, 2 * bn + 40, 200) if shape == "ragged" else (3328, 2304, 768)
    g = torch.Generator().manual_seed(cg * 1000 + bn + M)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    b = torch.randn(N, generator=g, dtype=torch.float32) * 0.1
    X, W, B = f64(x), f64(w), f64(b)
    scale = np.abs(X) @ np.abs(W).T + np.abs(B)
    f32 = out == "f32-gelu"
    buf = torch.full((M + 300, N), float("nan"), dtype=torch.float32 if f32 else torch.bfloat16,
                     device="cuda")
    y = buf[:M]
    if f32:
        rm.ops.gemm_tiled(x.cuda(), w.cuda(), b.cuda(), y, rm.F32, M, N, K, 1, cg, bn)
        torch.cuda.synchronize()
        ref = O.gelu(O.linear(X, W, B), O.GELU_ERF)
        bound = F32_RTOL * scale * 1.2 + 4e-7 * np.abs(ref)
    else:
        rm.ops.gemm_tiled(x.cuda(), w.cuda(), b.cuda(), y, rm.BF16, M, N, K, 0, cg, bn)
        torch.cuda.synchronize()
        ref = O.linear(X, W, B)
        bound = BF16_REL * np.abs(ref) + F32_RTOL * scale
    err = np.abs(f64(y) - ref)
    assert np.all(err <= bound), float(np.nanmax(err / bound))
    assert bool(torch.isnan(buf[M:]).all())


# Y += X.W^T + b with Y in fp32 (the decoder's residual add folded into its
# output projection and FFN2): every tile, ragged and projection shapes.  Y
# starts from seeded values; rows past M (the rest of the buffer) must keep
# theirs bit for bit.  Each element is added to once, so the result equals the
# stored product added in fp32 (the unfolded path) and repeats bit for bit.
@pytest.mark.parametrize("cg,bn", GEMM_TILES, ids=[f"cg{c}-bn{b}" for c, b in GEMM_TILES])
@pytest.mark.parametrize("shape", ["ragged", "proj"])
def test_gemm_accumulate_every_tile(cg, bn, shape):
    M, N, K = (555, 2 * bn + 40, 200) if shape == "ragged" else (3328, 768, 768)
    g = torch.Generator().manual_seed(cg * 1000 + bn + M + 1)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    b = torch.randn(N, generator=g, dtype=torch.float32) * 0.1
    y0 = torch.randn(M + 300, N, generator=g) * 2.0
    X, W, B = f64(x), f64(w), f64(b)
    ref = O.linear(X, W, B)
    scale = np.abs(X) @ np.abs(W).T + np.abs(B)
    Y0 = f64(y0[:M])
    xd, wd, bd = x.cuda(), w.cuda(), b.cuda()
    runs = []
    for _ in range(2):
        buf = y0.cuda()
        rm.ops.gemm_accumulate(xd, wd, bd, buf[:M], rm.F32, M, N, K, 0, cg, bn)
        torch.cuda.synchronize()
        runs.append(buf)
    buf = runs[0]
    # the tile's fp32 accumulation, then one fp32 rounding of the sum
    err = np.abs(f64(buf[:M]) - (Y0 + ref))
    bound = 2.0 ** -24 * np.abs(Y0 + ref) + F32_RTOL * scale * (1.0 + 2.0 ** -23)
    assert np.all(err <= bound), float(np.nanmax(err / bound))
    assert torch.equal(buf[M:].cpu(), y0[M:])
    assert torch.equal(runs[0], runs[1])
    # the same as storing the product and adding it in fp32
    prod = torch.empty(M, N, dtype=torch.float32, device="cuda")
    rm.ops.gemm_tiled(xd, wd, bd, prod, rm.F32, M, N, K, 0, cg, bn)
    torch.cuda.synchronize()
    assert torch.equal(buf[:M], y0[:M].cuda() + prod)


def test_gemm_accumulate_takes_fp32_without_activation_only():
    x = torch.zeros(16, 16, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(16, 16, dtype=torch.float32, device="cuda")
    with pytest.raises(rm.RmError):
        rm.ops.gemm_accumulate(x, x, None, y, rm.F32, 16, 16, 16, 1)
    with pytest.raises(rm.RmError):
        rm.ops.gemm_accumulate(x, x, None, x, rm.BF16, 16, 16, 16, 0)


# The tiles of the persistent grid's last, partial round run as 2 or 4 column
# slices each when the slices fit the idle SMs.  Shapes where that happens on
# a 148-SM B200 (widths 256 -> 4 slices of 64, 192 -> 2 of 96, 128 -> 2 of 64;
# and a single round of few tiles), against the oracle and bit for bit against
# 64-column tiles, which are never sliced: an element's value does not depend
# on the tile or slice it was computed in.
@pytest.mark.parametrize("bn,M,N,K", [(256, 20000, 768, 320), (192, 19000, 768, 256),
                                      (128, 9700, 768, 192), (256, 1000, 1000, 200)])
def test_gemm_tail_slices(bn, M, N, K):
    g = torch.Generator().manual_seed(bn + M)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16)
    b = torch.randn(N, generator=g, dtype=torch.float32) * 0.1
    xd, wd, bd = x.cuda(), w.cuda(), b.cuda()
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    y64 = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    rm.ops.gemm_tiled(xd, wd, bd, y, rm.F32, M, N, K, 0, 1, bn)
    rm.ops.gemm_tiled(xd, wd, bd, y64, rm.F32, M, N, K, 0, 1, 64)
    torch.cuda.synchronize()
    X, W, B = f64(x), f64(w), f64(b)
    ref = O.linear(X, W, B)
    scale = np.abs(X) @ np.abs(W).T + np.abs(B)
    err = np.abs(f64(y) - ref)
    assert np.all(err <= F32_RTOL * scale), float(np.nanmax(err / (F32_RTOL * scale)))
    assert torch.equal(y, y64)


def test_gemm_rejects_bad_shapes():
    x = torch.zeros(16, 12, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rm.RmError):
        rm.ops.gemm(x, x, None, x, rm.BF16, 16, 16, 12, 0)


# --- residual + LayerNorm ---------------------------------------------------------

@pytest.mark.parametrize("H", [128, 312, 768, 2048])
@pytest.mark.parametrize("mode", [0, 1, 2])
def test_res_ln_fp32(H, mode):
    T = 777
    rng = np.random.default_rng(H + mode)
    y = rng.normal(0, 1, (T, H)).astype(np.float32)
    x = rng.normal(0.5, 2, (T, H)).astype(np.float32)
    gm = (1 + rng.normal(0, 0.2, H)).astype(np.float32)
    bt = rng.normal(0, 0.2, H).astype(np.float32)
    yd, xd, zd = dev(y, torch.float32), dev(x, torch.float32), torch.zeros(T, H, device="cuda")
    rm.ops.res_ln(yd, xd, zd, dev(gm, torch.float32), dev(bt, torch.float32), T, H, 1e-5,
                  rm.F32, mode)
    torch.cuda.synchronize()
    u = x.astype(np.float64) + (y.astype(np.float64) if mode != 2 else 0)
    if mode == 1:
        u = u.astype(np.float32).astype(np.float64)       # the stored residual is fp32
    ref = O.layer_norm(u, gm.astype(np.float64), bt.astype(np.float64), 1e-5)
    out = f64(xd) if mode == 0 else f64(zd)
    assert np.all(np.abs(out - ref) <= F32_RTOL * (np.abs(ref) + np.abs(gm)))
    if mode == 1:
        assert np.array_equal(f64(xd), u)


@pytest.mark.parametrize("H", [312, 768, 2048])
def test_res_ln_bf16(H):
    T = 3264
    rng = np.random.default_rng(H)
    y = rng.normal(0, 1, (T, H))
    x = rng.normal(0, 1, (T, H))
    gm = (1 + rng.normal(0, 0.02, H)).astype(np.float32)
    bt = rng.normal(0, 0.02, H).astype(np.float32)
    yd, xd = dev(y, torch.bfloat16), dev(x, torch.bfloat16)
    u = f64(yd) + f64(xd)
    rm.ops.res_ln(yd, xd, None, dev(gm, torch.float32), dev(bt, torch.float32), T, H, 1e-12,
                  rm.BF16, 0)
    torch.cuda.synchronize()
    ref = O.layer_norm(u, gm.astype(np.float64), bt.astype(np.float64), 1e-12)
    assert np.all(np.abs(f64(xd) - ref) <= BF16_REL * np.abs(ref) + 1e-4 * np.abs(gm))


@pytest.mark.parametrize("H", [1024, 2048])
@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("ydt", ["bf16", "f32"])
def test_res_ln_fp32_residual_with_bf16_rows(H, mode, ydt):
    """The decoder's rows: z bf16, the residual stream x fp32, y bf16
    (RM_ROWS_RESID_F32) or fp32 (RM_ROWS_F32_IN)."""
    T = 1001
    rng = np.random.default_rng(H + 7 * mode)
    y = rng.normal(0, 1, (T, H))
    x = rng.normal(0.3, 3, (T, H)).astype(np.float32)
    gm = (1 + rng.normal(0, 0.02, H)).astype(np.float32)
    bt = rng.normal(0, 0.02, H).astype(np.float32)
    yd = dev(y, torch.bfloat16 if ydt == "bf16" else torch.float32)
    xd = dev(x, torch.float32)
    zd = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    u = x.astype(np.float64) + (f64(yd) if mode == 1 else 0)
    if mode == 1:
        u = u.astype(np.float32).astype(np.float64)       # the stored residual: one fp32 rounding
    rm.ops.res_ln(yd if mode == 1 else None, xd, zd, dev(gm, torch.float32), dev(bt, torch.float32),
                  T, H, 1e-5, rm.ROWS_RESID_F32 if ydt == "bf16" else rm.ROWS_F32_IN, mode)
    torch.cuda.synchronize()
    ref = O.layer_norm(u, gm.astype(np.float64), bt.astype(np.float64), 1e-5)
    assert np.all(np.abs(f64(zd) - ref) <= BF16_REL * np.abs(ref) + F32_RTOL * (np.abs(ref) + np.abs(gm)))
    assert np.array_equal(f64(xd), u if mode == 1 else x.astype(np.float64))


# --- softmax -------------------------------------------------------------------------

def varlen_rows(lens, nh, rng, dtype):
    off = synth.offsets_from_lengths(lens)
    rb, so = rm.ops.varlen_meta(off, nh)
    S = np.full(int(so[-1]), np.nan, dtype=np.float32)
    for i, L in enumerate(lens):
        Lp = (L + 7) // 8 * 8
        blk = S[so[i]:so[i + 1]].reshape(nh, L, Lp)
        blk[:, :, :L] = rng.normal(0, 3, (nh, L, L))
    return off, rb, so, S


@pytest.mark.parametrize("lens", [[1, 2, 3, 100, 57], [64, 128, 256], [513, 560, 7], [1024, 1000]],
                         ids=["short", "tinybert", "long", "max"])
@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("dtype", [rm.F32, rm.BF16], ids=["f32", "bf16"])
def test_softmax(lens, causal, dtype):
    nh = 3
    rng = np.random.default_rng(len(lens) + causal)
    lens = np.array(lens)
    off, rb, so, S = varlen_rows(lens, nh, rng, dtype)
    tdt = torch.float32 if dtype == rm.F32 else torch.bfloat16
    Sd = dev(S, tdt)
    S_in = f64(Sd)
    rm.ops.softmax(Sd, dtype, dev(off, torch.int32), dev(so, torch.int64), len(lens),
                   int(off[-1]), nh, int(lens.max()), causal)
    torch.cuda.synchronize()
    P = f64(Sd)
    for i, L in enumerate(lens):
        Lp = (L + 7) // 8 * 8
        got = P[so[i]:so[i + 1]].reshape(nh, L, Lp)
        s_in = S_in[so[i]:so[i + 1]].reshape(nh, L, Lp)[:, :, :L]
        allowed = np.tril(np.ones((L, L), bool)) if causal else np.ones((L, L), bool)
        ref = O.softmax_masked(s_in, np.broadcast_to(allowed, (nh, L, L)))
        g = got[:, :, :L]
        ok = np.broadcast_to(allowed, g.shape)
        tol = F32_RTOL if dtype == rm.F32 else BF16_REL
        assert np.all(np.abs(g[ok] - ref[ok]) <= tol * ref[ok] + 1e-37)
        # entries inside a written 8-wide chunk but outside the row are exactly 0
        for r in (0, L - 1):
            lim = r + 1 if causal else L
            end = min(Lp, (lim + 7) // 8 * 8)
            assert np.all(got[:, r, lim:end] == 0)


@pytest.mark.parametrize("lens", [[1, 2, 3, 100, 57], [64, 128, 256], [513, 560, 7], [1024, 1000],
                                  [5, 33, 65, 129, 257, 513, 769, 31, 8, 1]],
                         ids=["short", "tinybert", "long", "max", "mixed"])
@pytest.mark.parametrize("causal", [0, 1])
@pytest.mark.parametrize("dtype", [rm.F32, rm.BF16], ids=["f32", "bf16"])
def test_softmax_classes(lens, causal, dtype):
    """Length-class softmax against the oracle, every row of every sequence,
    the masked tail of each written chunk exactly 0, entries outside the rows
    untouched; twice in a row on the same scratch (the index is rebuilt)."""
    nh = 3
    rng = np.random.default_rng(len(lens) + causal + 101)
    lens = np.array(lens)
    off, rb, so, S = varlen_rows(lens, nh, rng, dtype)
    tdt = torch.float32 if dtype == rm.F32 else torch.bfloat16
    T = int(off[-1])
    d_off, d_so = dev(off, torch.int32), dev(so, torch.int64)
    nbytes = rm.ops.softmax_scratch_bytes(len(lens), T, nh)
    scratch = torch.full((nbytes,), 255, dtype=torch.uint8, device="cuda")
    for _ in range(2):
        Sd = dev(S, tdt)
        S_in = f64(Sd)
        rm.ops.softmax_classes(Sd, dtype, d_off, d_so, len(lens), T, nh, int(lens.max()), causal,
                               scratch)
        torch.cuda.synchronize()
        P = f64(Sd)
        for i, L in enumerate(lens):
            Lp = (L + 7) // 8 * 8
            got = P[so[i]:so[i + 1]].reshape(nh, L, Lp)
            s_in = S_in[so[i]:so[i + 1]].reshape(nh, L, Lp)[:, :, :L]
            allowed = np.tril(np.ones((L, L), bool)) if causal else np.ones((L, L), bool)
            ref = O.softmax_masked(s_in, np.broadcast_to(allowed, (nh, L, L)))
            g = got[:, :, :L]
            ok = np.broadcast_to(allowed, g.shape)
            tol = F32_RTOL if dtype == rm.F32 else BF16_REL
            assert np.all(np.abs(g[ok] - ref[ok]) <= tol * ref[ok] + 1e-37)
            before = S_in[so[i]:so[i + 1]].reshape(nh, L, Lp)
            for r in (0, L - 1):
                lim = r + 1 if causal else L
                end = min(Lp, (lim + 7) // 8 * 8)
                assert np.all(got[:, r, lim:end] == 0)
                # past the last written chunk the buffer is untouched
                assert np.array_equal(got[:, r, end:], before[:, r, end:], equal_nan=True)


def test_softmax_classes_many_sequences_against_the_oracle():
    """Thousands of sequences of every class (the planning kernels loop), sampled
    against the oracle, the longest included."""
    nh = 2
    rng = np.random.default_rng(5)
    lens = rng.integers(1, 40, 3000)
    lens[rng.integers(0, 3000, 40)] = rng.integers(40, 1025, 40)
    off, rb, so, S = varlen_rows(lens, nh, rng, rm.F32)
    T = int(off[-1])
    Sd = dev(S, torch.float32)
    S_in = f64(Sd)
    scratch = torch.empty(rm.ops.softmax_scratch_bytes(len(lens), T, nh), dtype=torch.uint8,
                          device="cuda")
    rm.ops.softmax_classes(Sd, rm.F32, dev(off, torch.int32), dev(so, torch.int64), len(lens), T, nh,
                           int(lens.max()), 0, scratch)
    torch.cuda.synchronize()
    P = f64(Sd)
    for i in list(np.linspace(0, len(lens) - 1, 40).astype(int)) + list(np.argsort(lens)[-5:]):
        L = int(lens[i])
        Lp = (L + 7) // 8 * 8
        got = P[so[i]:so[i + 1]].reshape(nh, L, Lp)[:, :, :L]
        s_in = S_in[so[i]:so[i + 1]].reshape(nh, L, Lp)[:, :, :L]
        ref = O.softmax_masked(s_in, np.ones((nh, L, L), bool))
        assert np.all(np.abs(got - ref) <= F32_RTOL * ref + 1e-37)


# --- attention scores and context -----------------------------------------------------

def qkv_for(T, H, rng):
    return rng.normal(0, 1, (T, 3 * H))


@pytest.mark.parametrize("nh,d", [(2, 64), (12, 26), (12, 64), (16, 128)])
@pytest.mark.parametrize("causal", [0, 1])
def test_attention_scores(nh, d, causal):
    H = nh * d
    lens = np.array([1, 65, 130, 64, 9])
    off = synth.offsets_from_lengths(lens)
    rb, so = rm.ops.varlen_meta(off, nh)
    rng = np.random.default_rng(nh + d + causal)
    qkv = dev(qkv_for(int(off[-1]), H, rng), torch.bfloat16)
    Q = f64(qkv)
    S = torch.full((int(so[-1]),), float("nan"), dtype=torch.bfloat16, device="cuda")
    rm.ops.attn_scores(qkv, S, dev(off, torch.int32), dev(rb, torch.int32), dev(so, torch.int64),
                       len(lens), int(rb[-1]), nh, d, causal)
    torch.cuda.synchronize()
    Sh = f64(S)
    for i, L in enumerate(lens):
        Lp = (L + 7) // 8 * 8
        blk = Sh[so[i]:so[i + 1]].reshape(nh, L, Lp)
        rows = Q[off[i]:off[i + 1]]
        for j in range(nh):
            q = rows[:, j * d:(j + 1) * d]
            k = rows[:, H + j * d:H + (j + 1) * d]
            ref = q @ k.T / np.sqrt(d)
            scale = np.abs(q) @ np.abs(k).T / np.sqrt(d)
            ok = np.tril(np.ones((L, L), bool)) if causal else np.ones((L, L), bool)
            err = np.abs(blk[j][:, :L] - ref)
            assert np.all(err[ok] <= BF16_REL * np.abs(ref[ok]) + F32_RTOL * scale[ok])


@pytest.mark.parametrize("nh,d", [(2, 64), (12, 26), (16, 128)])
@pytest.mark.parametrize("causal", [0, 1])
def test_attention_context(nh, d, causal):
    H = nh * d
    lens = np.array([1, 65, 130, 64, 9])
    off = synth.offsets_from_lengths(lens)
    rb, so = rm.ops.varlen_meta(off, nh)
    rng = np.random.default_rng(nh * d + causal)
    T = int(off[-1])
    qkv = dev(qkv_for(T, H, rng), torch.bfloat16)
    V = f64(qkv)
    # probabilities with junk (NaN) outside the allowed keys: the kernel must not read them
    P = np.full(int(so[-1]), np.nan, dtype=np.float32)
    for i, L in enumerate(lens):
        Lp = (L + 7) // 8 * 8
        blk = P[so[i]:so[i + 1]].reshape(nh, L, Lp)
        ok = np.tril(np.ones((L, L), bool)) if causal else np.ones((L, L), bool)
        s = rng.normal(0, 2, (nh, L, L))
        blk[:, :, :L] = np.where(ok, O.softmax_masked(s, np.broadcast_to(ok, s.shape)), np.nan)
    Pd = dev(P, torch.bfloat16)
    Ph = f64(Pd)
    ctx = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    rm.ops.attn_context(Pd, qkv, ctx, dev(off, torch.int32), dev(rb, torch.int32),
                        dev(so, torch.int64), len(lens), int(rb[-1]), nh, d, causal)
    torch.cuda.synchronize()
    C = f64(ctx)
    for i, L in enumerate(lens):
        Lp = (L + 7) // 8 * 8
        blk = Ph[so[i]:so[i + 1]].reshape(nh, L, Lp)[:, :, :L]
        rows = V[off[i]:off[i + 1]]
        for j in range(nh):
            p = np.nan_to_num(blk[j], nan=0.0)
            v = rows[:, 2 * H + j * d:2 * H + (j + 1) * d]
            ref = p @ v
            scale = np.abs(p) @ np.abs(v)
            got = C[off[i]:off[i + 1], j * d:(j + 1) * d]
            assert np.all(np.abs(got - ref) <= BF16_REL * np.abs(ref) + F32_RTOL * scale)


# --- embedding and head ----------------------------------------------------------------

@pytest.mark.parametrize("H,ln,xdt", [(128, True, "bf16"), (312, True, "bf16"), (768, True, "bf16"),
                                      (2048, False, "bf16"), (2048, False, "f32")])
def test_embed(H, ln, xdt):
    V, P = 1000, 600
    lens = np.array([1, 560, 33, 8])
    off = synth.offsets_from_lengths(lens)
    rng = np.random.default_rng(H)
    ids = rng.integers(0, V, int(off[-1])).astype(np.int32)
    ids[5] = V + 7            # out of range: clamped to V-1 and counted
    ids[9] = -3               # clamped to 0
    ew = dev(rng.normal(0, 0.5, (V, H)), torch.bfloat16)
    ep = dev(rng.normal(0, 0.5, (P, H)), torch.bfloat16)
    g = dev(1 + rng.normal(0, 0.1, H), torch.float32)
    b = dev(rng.normal(0, 0.1, H), torch.float32)
    f32 = xdt == "f32"
    x = torch.zeros(int(off[-1]), H, dtype=torch.float32 if f32 else torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rm.ops.embed(dev(ids, torch.int32), dev(off, torch.int32), len(lens), int(off[-1]), ew, ep,
                 g if ln else None, b if ln else None, 1e-12, V, P, H, x, err,
                 x_dtype=rm.F32 if f32 else rm.BF16)
    torch.cuda.synchronize()
    assert int(err.item()) == 2
    EW, EP = f64(ew), f64(ep)
    cid = np.clip(ids, 0, V - 1)
    for i, L in enumerate(lens):
        u = EW[cid[off[i]:off[i + 1]]] + EP[:L]
        ref = O.layer_norm(u, f64(g), f64(b), 1e-12) if ln else u
        got = f64(x)[off[i]:off[i + 1]]
        if f32:
            # the sum of two bf16 values, rounded once to fp32
            assert np.all(np.abs(got - ref) <= 2.0 ** -24 * np.abs(ref))
        else:
            assert np.all(np.abs(got - ref) <= BF16_REL * np.abs(ref) + 1e-5 * (1 + np.abs(ref)))


@pytest.mark.parametrize("last", [0, 1])
def test_head(last):
    H = 768
    lens = np.array([1, 17, 100, 2])
    off = synth.offsets_from_lengths(lens)
    rng = np.random.default_rng(last)
    x = dev(rng.normal(0, 1, (int(off[-1]), H)), torch.bfloat16)
    w = rng.normal(0, 0.05, H).astype(np.float32)
    out = torch.zeros(len(lens), dtype=torch.float32, device="cuda")
    rm.ops.head(x, dev(off, torch.int32), len(lens), dev(w, torch.float32), 0.25, H, last, out)
    torch.cuda.synchronize()
    X = f64(x)
    rows = X[off[1:] - 1] if last else X[off[:-1]]
    ref = rows @ w.astype(np.float64) + 0.25
    assert np.all(np.abs(f64(out) - ref) <= F32_RTOL * (np.abs(rows) @ np.abs(w) + 0.25))


@pytest.mark.parametrize("lens", [[1, 65, 130, 64, 9], [300, 7, 560], [100] * 8],
                         ids=["ragged", "long", "uniform"])
@pytest.mark.parametrize("nh,d", [(2, 64), (12, 26), (12, 64), (16, 128)])
@pytest.mark.parametrize("causal", [0, 1])
def test_attention_fused(lens, nh, d, causal):
    H = nh * d
    lens = np.array(lens)
    off = synth.offsets_from_lengths(lens)
    rb, so = rm.ops.varlen_meta(off, nh)
    rng = np.random.default_rng(nh * d + causal + len(lens))
    T = int(off[-1])
    qkv = dev(qkv_for(T, H, rng) * 1.5, torch.bfloat16)
    X = f64(qkv)
    ctx = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    rm.ops.attn_fused(qkv, ctx, dev(off, torch.int32), dev(rb, torch.int32), len(lens),
                      int(rb[-1]), nh, d, causal)
    torch.cuda.synchronize()
    C = f64(ctx)
    for i, L in enumerate(lens):
        rows = X[off[i]:off[i + 1]]
        for j in range(nh):
            q = rows[:, j * d:(j + 1) * d]
            k = rows[:, H + j * d:H + (j + 1) * d]
            v = rows[:, 2 * H + j * d:2 * H + (j + 1) * d]
            p = O.attention_probs(q, k, bool(causal))
            ref = p @ v
            # one bf16 rounding of the output and of every probability
            tol = BF16_REL * np.abs(ref) + 2 * BF16_REL * (p @ np.abs(v)) + F32_RTOL
            got = C[off[i]:off[i + 1], j * d:(j + 1) * d]
            assert np.all(np.abs(got - ref) <= tol), float((np.abs(got - ref) / tol).max())


def _attention_ref_check(X, C, off, nh, d, causal):
    H = nh * d
    for i in range(len(off) - 1):
        rows = X[off[i]:off[i + 1]]
        for j in range(nh):
            q = rows[:, j * d:(j + 1) * d]
            k = rows[:, H + j * d:H + (j + 1) * d]
            v = rows[:, 2 * H + j * d:2 * H + (j + 1) * d]
            p = O.attention_probs(q, k, bool(causal))
            ref = p @ v
            # one bf16 rounding of the output and of every probability
            tol = BF16_REL * np.abs(ref) + 2 * BF16_REL * (p @ np.abs(v)) + F32_RTOL
            got = C[off[i]:off[i + 1], j * d:(j + 1) * d]
            assert np.all(np.abs(got - ref) <= tol), (i, j, float((np.abs(got - ref) / tol).max()))


@pytest.mark.parametrize("lens", [
    [1, 65, 130, 64, 9],                              # ragged, tiles cut sequences
    [2, 3, 1, 5, 2, 7, 1, 1, 4, 9, 2, 3, 8, 1, 6, 2],  # many sequences per 16-row warp
    [300, 7, 560],                                    # long rows, several key chunks
    [100] * 8,                                        # uniform, sequences straddle tiles
    [64] * 3,                                         # tiles aligned with sequences
    [5],                                              # one tile, shorter than 64 rows
], ids=["ragged", "tiny", "long", "uniform", "aligned", "single"])
@pytest.mark.parametrize("nh,d", [(2, 64), (12, 64), (16, 128)])
@pytest.mark.parametrize("causal", [0, 1])
def test_attention_tiles(lens, nh, d, causal):
    """Packed-row tiles against the oracle's attention, every row and head."""
    H = nh * d
    lens = np.array(lens)
    off = synth.offsets_from_lengths(lens)
    rng = np.random.default_rng(nh * d + causal + len(lens) + 5)
    T = int(off[-1])
    qkv = dev(qkv_for(T, H, rng) * 1.5, torch.bfloat16)
    ctx = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    # the launch as rm_score sizes it (max_len = the longest row), which takes
    # more heads per CTA for short rows than the default bound (T) does
    rm.ops.attn_tiles(qkv, ctx, dev(off, torch.int32), len(lens), T, nh, d, causal,
                      max_len=int(lens.max()))
    torch.cuda.synchronize()
    _attention_ref_check(f64(qkv), f64(ctx), off, nh, d, causal)


def test_attention_tiles_bench_shape():
    """A fused call of the BERT-base stream's shape (512 sequences of 2..100
    tokens, 12 heads of 64): every output finite, sampled sequences against the
    oracle, and the per-sequence fused kernel's output finite on the same input."""
    nh, d = 12, 64
    H = nh * d
    rng = np.random.default_rng(2024)
    lens = rng.integers(2, 101, 512)
    off = synth.offsets_from_lengths(lens)
    rb, _ = rm.ops.varlen_meta(off, nh)
    T = int(off[-1])
    qkv = dev(qkv_for(T, H, rng) * 1.5, torch.bfloat16)
    a = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    b = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    d_off = dev(off, torch.int32)
    rm.ops.attn_tiles(qkv, a, d_off, len(lens), T, nh, d, 0)
    rm.ops.attn_fused(qkv, b, d_off, dev(rb, torch.int32), len(lens), int(rb[-1]), nh, d, 0)
    torch.cuda.synchronize()
    A, B = f64(a), f64(b)
    assert np.all(np.isfinite(A)) and np.all(np.isfinite(B))
    pick = np.linspace(0, len(lens) - 1, 12).astype(int)
    X = f64(qkv)
    for i in pick:
        sub = np.array([0, lens[i]], dtype=np.int64)
        _attention_ref_check(X[off[i]:off[i + 1]], A[off[i]:off[i + 1]], sub, nh, d, 0)


@pytest.mark.parametrize("kind", ["short", "mixed"])
def test_attention_tiles_repeat_bit_identical(kind):
    """Many heads per CTA and one key chunk per tile let the load ring run
    several heads ahead of the warps that read it: thirty launches (other
    launches in between change what shared memory held) must give the same
    bits, and the first must match the oracle."""
    nh, d = 12, 64
    H = nh * d
    rng = np.random.default_rng(17)
    lens = rng.integers(1, 9, 4000) if kind == "short" else rng.integers(2, 101, 500)
    off = synth.offsets_from_lengths(lens)
    T = int(off[-1])
    qkv = dev(qkv_for(T, H, rng) * 1.5, torch.bfloat16)
    other = dev(qkv_for(T, H, rng), torch.bfloat16)
    d_off = dev(off, torch.int32)
    first = None
    junk = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    for _ in range(30):
        rm.ops.attn_tiles(other, junk, d_off, len(lens), T, nh, d, 0)
        ctx = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
        rm.ops.attn_tiles(qkv, ctx, d_off, len(lens), T, nh, d, 0, max_len=int(lens.max()))
        torch.cuda.synchronize()
        if first is None:
            first = ctx
            X, C = f64(qkv), f64(ctx)
            for i in np.linspace(0, len(lens) - 1, 16).astype(int):
                sub = np.array([0, lens[i]], dtype=np.int64)
                _attention_ref_check(X[off[i]:off[i + 1]], C[off[i]:off[i + 1]], sub, nh, d, 0)
        else:
            assert torch.equal(ctx, first)


def test_attention_tiles_rejects_other_head_dims():
    x = torch.zeros(8, dtype=torch.bfloat16, device="cuda")
    off = dev(np.array([0, 4], dtype=np.int32), torch.int32)
    for d in (26, 32, 96):
        with pytest.raises(rm.RmError) as e:
            rm.ops.attn_tiles(x, x, off, 1, 4, 2, d, 0)
        assert e.value.code == rm.RM_E_INVAL


# --- tensor-core attention (head dim 64, sequences of at most 128 tokens) ------

def _attn_tc(qkv, ctx, off, nh, causal):
    tiles = rm.ops.attn_tc_tiles(off)
    rm.ops.attn_tc(qkv, ctx, dev(off, torch.int32), dev(tiles, torch.int32), len(tiles) - 1,
                   len(off) - 1, int(off[-1]), nh, causal)
    return tiles


@pytest.mark.parametrize("lens", [
    [1, 65, 128, 64, 9],                                # ragged; a full 128-row tile
    [2, 3, 1, 5, 2, 7, 1, 1, 4, 9, 2, 3, 8, 1, 6, 2],    # many sequences per tile and warp
    [100] * 8,                                          # one sequence per tile
    [127, 1, 128, 128, 2],                              # tiles of exactly 128 rows
    [5],                                                # one short tile
    [33, 31, 32, 32, 64, 17, 47],                       # sequences across 32-row warps
], ids=["ragged", "tiny", "uniform", "full", "single", "warps"])
@pytest.mark.parametrize("nh", [2, 12])
@pytest.mark.parametrize("causal", [0, 1])
def test_attention_tc(lens, nh, causal):
    """tcgen05 attention on sequence tiles against the oracle's attention,
    every row and head."""
    d = 64
    H = nh * d
    lens = np.array(lens)
    off = synth.offsets_from_lengths(lens)
    rng = np.random.default_rng(nh * 7 + causal + len(lens))
    T = int(off[-1])
    qkv = dev(qkv_for(T, H, rng) * 1.5, torch.bfloat16)
    ctx = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    _attn_tc(qkv, ctx, off, nh, causal)
    torch.cuda.synchronize()
    _attention_ref_check(f64(qkv), f64(ctx), off, nh, d, causal)


def _attn_tcl(qkv, ctx, off, nh, causal):
    items = rm.ops.attn_tcl_items(off, causal)
    rm.ops.attn_tcl(qkv, ctx, dev(off, torch.int32), dev(items, torch.int32), len(items),
                    len(off) - 1, int(off[-1]), nh, causal)
    return items


@pytest.mark.parametrize("lens", [
    [129],                                              # two key chunks, one row past a tile
    [512],                                              # four full chunks and query tiles
    [1, 512, 130, 7, 300, 256, 128],                    # ragged, chunk and tile edges
    [200] * 6,                                          # uniform
    [383, 385, 5],                                      # around the third chunk edge
], ids=["129", "512", "ragged", "uniform", "edges"])
@pytest.mark.parametrize("nh", [2, 12])
@pytest.mark.parametrize("causal", [0, 1])
def test_attention_tcl(lens, nh, causal):
    """tcgen05 attention on 128-row query tiles of sequences up to 512 tokens
    against the oracle's attention, every row and head."""
    d = 64
    H = nh * d
    lens = np.array(lens)
    off = synth.offsets_from_lengths(lens)
    rng = np.random.default_rng(nh * 11 + causal + len(lens))
    T = int(off[-1])
    qkv = dev(qkv_for(T, H, rng) * 1.5, torch.bfloat16)
    ctx = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    _attn_tcl(qkv, ctx, off, nh, causal)
    torch.cuda.synchronize()
    _attention_ref_check(f64(qkv), f64(ctx), off, nh, d, causal)


def test_attention_tcl_long_stream_against_tiles_and_oracle():
    """A fused call of the lengths-5..500 stream's shape (256 sequences, 12
    heads of 64): every output finite, within bf16 rounding of the packed-row
    tile kernel everywhere, and bit-identical on a repeat."""
    nh, d = 12, 64
    H = nh * d
    rng = np.random.default_rng(77)
    lens = rng.integers(5, 501, 256)
    off = synth.offsets_from_lengths(lens)
    T = int(off[-1])
    qkv = dev(qkv_for(T, H, rng) * 1.5, torch.bfloat16)
    a = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    a2 = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    b = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    _attn_tcl(qkv, a, off, nh, 0)
    _attn_tcl(qkv, a2, off, nh, 0)
    rm.ops.attn_tiles(qkv, b, dev(off, torch.int32), len(lens), T, nh, d, 0, max_len=500)
    torch.cuda.synchronize()
    A, B = f64(a), f64(b)
    assert np.all(np.isfinite(A))
    assert torch.equal(a, a2)
    X = f64(qkv)
    vmax = np.repeat(np.maximum.reduceat(np.abs(X[:, 2 * H:]), off[:-1], axis=0), lens, axis=0)
    assert np.all(np.abs(A - B) <= 1.5 * BF16_REL * (vmax + np.abs(B)) + 1e-6)


def test_attention_tc_bench_shape_against_tiles_and_oracle():
    """A fused call of the BERT-base stream's shape (512 sequences of 2..100
    tokens, 12 heads of 64): every output finite, within bf16 rounding of the
    packed-row tile kernel everywhere, sampled sequences against the oracle."""
    nh, d = 12, 64
    H = nh * d
    rng = np.random.default_rng(2024)
    lens = rng.integers(2, 101, 512)
    off = synth.offsets_from_lengths(lens)
    T = int(off[-1])
    qkv = dev(qkv_for(T, H, rng) * 1.5, torch.bfloat16)
    a = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    b = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    _attn_tc(qkv, a, off, nh, 0)
    rm.ops.attn_tiles(qkv, b, dev(off, torch.int32), len(lens), T, nh, d, 0, max_len=100)
    torch.cuda.synchronize()
    A, B = f64(a), f64(b)
    assert np.all(np.isfinite(A))
    X = f64(qkv)
    # Each kernel rounds every P entry to bf16 (half an ulp, 2^-9 relative:
    # at most 2^-9 * max_k |v_kc| on output column c after the division by
    # the row sum) and the output once (2^-9 |out|); the two differ by at
    # most twice that.  max_k runs over the row's own sequence.
    vmax = np.repeat(np.maximum.reduceat(np.abs(X[:, 2 * H:]), off[:-1], axis=0), lens, axis=0)
    assert np.all(np.abs(A - B) <= 1.5 * BF16_REL * (vmax + np.abs(B)) + 1e-6)
    for i in np.linspace(0, len(lens) - 1, 16).astype(int):
        sub = np.array([0, lens[i]], dtype=np.int64)
        _attention_ref_check(X[off[i]:off[i + 1]], A[off[i]:off[i + 1]], sub, nh, d, 0)


def test_attention_tc_repeat_bit_identical():
    """Twelve heads through three load slots, four TMEM regions and two softmax
    groups: thirty launches with other launches in between give the same bits."""
    nh, d = 12, 64
    H = nh * d
    rng = np.random.default_rng(23)
    lens = rng.integers(1, 129, 300)
    off = synth.offsets_from_lengths(lens)
    T = int(off[-1])
    qkv = dev(qkv_for(T, H, rng) * 1.5, torch.bfloat16)
    other = dev(qkv_for(T, H, rng), torch.bfloat16)
    junk = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    first = None
    for _ in range(30):
        _attn_tc(other, junk, off, nh, 0)
        ctx = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
        _attn_tc(qkv, ctx, off, nh, 0)
        torch.cuda.synchronize()
        if first is None:
            first = ctx
            X, C = f64(qkv), f64(ctx)
            for i in np.linspace(0, len(lens) - 1, 12).astype(int):
                sub = np.array([0, lens[i]], dtype=np.int64)
                _attention_ref_check(X[off[i]:off[i + 1]], C[off[i]:off[i + 1]], sub, nh, d, 0)
        else:
            assert torch.equal(ctx, first)


def test_gemm_gelu_epilogue_against_cuda_erf_and_oracle():
    """GELU of the epilogue (Abramowitz & Stegun 7.1.28 erf) on a dense grid of
    pre-activations: x = 0, W = 0, so y = GELU(bias)."""
    N = 8192
    u = torch.linspace(-12, 12, N, dtype=torch.float32)
    x = torch.zeros(16, 64, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(N, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(16, N, dtype=torch.float32, device="cuda")
    rm.ops.gemm(x, w, u.cuda(), y, rm.F32, 16, N, 64, 1)
    torch.cuda.synchronize()
    got = f64(y[0])
    cuda_erff = torch.nn.functional.gelu(u.cuda()).double().cpu().numpy()   # CUDA's erff
    ref = O.gelu(u.double().numpy())
    assert np.max(np.abs(got - ref)) <= 2e-6
    assert np.max(np.abs(got - cuda_erff)) <= 2e-6
    assert np.all(f64(y) == got[None, :])
