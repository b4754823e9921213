"""GPU parity of the tcgen05 block-scaled FP4 GEMM and of QSNR(AB).

C = A^Q (B^Q)^T is checked against the oracle's dequantized operands
multiplied in binary64 (the products of E2M1 values and power-of-two or
UE4M3 scales are exact; the tensor cores accumulate in binary32): normwise
relative error below 1e-3 and every element within 1e-3 * rms(C).  QSNR(AB)
(Eq. (2) of the MXFP4 paper's Sec.3) is checked against the oracle's sums,
1e-3 relative.
"""
import numpy as np
import pytest
import torch

from microscaling_block_quantization_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mx():
    from microscaling_block_quantization_b200 import build
    build.build()
    import microscaling_block_quantization_b200 as m
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return m


def chunk_layout(scales: np.ndarray, rows: int, S: int) -> np.ndarray:
    """Canonical [rows][S] scale bytes -> the 512-byte 128 x 4 chunk layout."""
    out = np.zeros(rows * S, np.uint8)
    r = np.arange(rows)[:, None]
    j = np.arange(S)[None, :]
    idx = ((r // 128) * (S // 4) + j // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + j % 4
    out[idx.ravel()] = scales.reshape(rows, S).ravel()
    return out


def configs(mx):
    return {"mxfp4": mx.Config(sf_layout=1),
            "nvfp4": mx.Config(block=16, scale_fmt=1, rule=3, tensor_scale=1, sf_layout=1)}


def ocfg(orc, name):
    if name == "mxfp4":
        return orc.Cfg()
    return orc.Cfg(block=16, scale_fmt=orc.UE4M3, rule=orc.NEAREST, tensor_scale=orc.TS_COMPUTE)


def deq(orc, name, x):
    r = orc.quantize(ocfg(orc, name), x)
    return orc.dequantize(ocfg(orc, name), r["packed"], r["scales"], r["tensor_scale"], None, None,
                          *x.shape), r


@pytest.mark.parametrize("name", ["mxfp4", "nvfp4"])
def test_scale_chunk_layout(mx, orc, name):
    x = inputs.laplace_outlier_cols(256, 512, seed=6, n_outlier_cols=2)
    cfg = configs(mx)[name]
    q = mx.quantize(x.cuda(), cfg)
    r = orc.quantize(ocfg(orc, name), x)
    S = 512 // cfg.block
    assert np.array_equal(q.codes.cpu().numpy(), r["packed"].ravel())
    assert np.array_equal(q.scales.cpu().numpy(), chunk_layout(r["scales"], 256, S))
    xh = mx.dequantize(q, torch.float32).cpu().numpy()
    oxh, _ = deq(orc, name, x)
    assert np.array_equal(xh.view(np.uint32), oxh.view(np.uint32))


def check_gemm(mx, orc, name, M, N, K, out_dtype=torch.float32, seed=0):
    a = inputs.laplace_outlier_cols(M, K, seed=6 + seed, n_outlier_cols=2)
    w = inputs.normal(N, K, sigma=0.02, seed=7 + seed)
    cfg = configs(mx)[name]
    qa = mx.quantize(a.cuda(), cfg, stats=False)
    qw = mx.quantize(w.cuda(), cfg, stats=False)
    c = mx.gemm(qa, qw, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert mx.mx_device_status() == 0
    ah, _ = deq(orc, name, a)
    wh, _ = deq(orc, name, w)
    ref = ah.astype(np.float64) @ wh.astype(np.float64).T
    got = c.float().cpu().numpy().astype(np.float64)
    tol = 1e-3 if out_dtype == torch.float32 else 8e-3      # bf16 output rounding
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel < tol, rel
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(got - ref)) <= tol * rms + tol * np.abs(ref).max() * (out_dtype != torch.float32)
    return rel


@pytest.mark.parametrize("name", ["mxfp4", "nvfp4"])
def test_gemm_single_tile(mx, orc, name):
    check_gemm(mx, orc, name, 128, 128, 256)        # 128 x 128 tile kernel
    check_gemm(mx, orc, name, 128, 256, 256)        # persistent 128 x 256 kernel


@pytest.mark.parametrize("name", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("shape", [(256, 384, 1024), (384, 256, 2048), (128, 640, 768),
                                   (384, 512, 1280), (2048, 2560, 512)])
def test_gemm_tiles_and_stage_ring(mx, orc, name, shape):
    check_gemm(mx, orc, name, *shape)


@pytest.mark.parametrize("name", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("shape", [(256, 256, 512), (384, 768, 512), (1280, 4096, 256)])
def test_gemm_bf16_output(mx, orc, name, shape):
    """bf16 C written by the epilogue's tensor stores (128 x 256 tiles; more
    tiles than CTAs in the last shape): against the oracle, and bit for bit
    the round-to-nearest-even of the binary32 C."""
    check_gemm(mx, orc, name, *shape, out_dtype=torch.bfloat16)
    M, N, K = shape
    a = inputs.laplace_outlier_cols(M, K, seed=6, n_outlier_cols=2).cuda()
    w = inputs.normal(N, K, sigma=0.02, seed=7).cuda()
    cfg = configs(mx)[name]
    qa, qw = mx.quantize(a, cfg, stats=False), mx.quantize(w, cfg, stats=False)
    c16 = mx.gemm(qa, qw, out_dtype=torch.bfloat16)
    c32 = mx.gemm(qa, qw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(c16.view(torch.int16), c32.to(torch.bfloat16).view(torch.int16))


def test_gemm_rejects_canonical_scales(mx):
    a = torch.zeros(128, 256, dtype=torch.bfloat16, device="cuda")
    q = mx.quantize(a, mx.MXFP4, stats=False)
    with pytest.raises(mx.MXError) as e:
        mx.gemm(q, q)
    assert e.value.code == -2


def _qsnr_vs_oracle(mx, orc, name, M, N, K, blas=False):
    a = inputs.laplace_outlier_cols(M, K, seed=6, n_outlier_cols=2)
    w = inputs.normal(N, K, sigma=0.02, seed=7)
    cfg = configs(mx)[name]
    qa = mx.quantize(a.cuda(), cfg, stats=False)
    qw = mx.quantize(w.cuda(), cfg, stats=False)
    st = mx.gemm_qsnr(a.cuda(), w.cuda(), qa, qw).cpu().numpy()
    assert mx.mx_device_status() == 0
    ah, _ = deq(orc, name, a)
    wh, _ = deq(orc, name, w)
    f = orc.gemm_qsnr_blas if blas else orc.gemm_qsnr
    o = f(orc.input_f32(a), orc.input_f32(w), ah, wh)
    assert abs(st[0] - o[0]) <= 1e-3 * o[0]
    assert abs(st[1] - o[1]) <= 1e-3 * o[1]
    assert abs(st[2] - o[2]) <= 1e-2
    return st


@pytest.mark.parametrize("name", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("shape", [(256, 256, 512), (384, 640, 768), (128, 128, 256)])
def test_gemm_qsnr_small(mx, orc, name, shape):
    """Both products formed tile by tile in one kernel, C never written:
    tiles of 128 x 256 (N % 256 == 0) and 128 x 128 (N = 640), against the
    oracle's binary64 sums."""
    _qsnr_vs_oracle(mx, orc, name, *shape)


@pytest.mark.parametrize("name", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("shape", [(2176, 2560, 512), (2176, 1920, 256)])
def test_gemm_qsnr_many_tiles_per_cta(mx, orc, name, shape):
    """More output tiles than CTAs (each CTA walks several tiles, the
    accumulator hand-over alternating between the two products), and a
    last group of tile rows shorter than the others."""
    _qsnr_vs_oracle(mx, orc, name, *shape, blas=True)


def test_gemm_qsnr_workspace_does_not_grow_with_c(mx):
    """The QSNR(AB) scratch is a fixed set of per-CTA records, not C."""
    lib = mx.lib()
    assert lib.mx_gemm_workspace_bytes(8192, 14336, 4096) == lib.mx_gemm_workspace_bytes(128, 128, 256)
    assert lib.mx_gemm_workspace_bytes(8192, 14336, 4096) < 1 << 20


@pytest.mark.parametrize("name", ["mxfp4", "nvfp4"])
def test_gemm_qsnr_llama_shape(mx, orc, name):
    """QSNR(AB) of the full 8192 x 4096 by 14336 x 4096 layer against the
    oracle's binary64 BLAS sums over its dequantized operands."""
    A, W = inputs.llama_linear()
    cfg = configs(mx)[name]
    qa = mx.quantize(A.cuda(), cfg, stats=False)
    qw = mx.quantize(W.cuda(), cfg, stats=False)
    st = mx.gemm_qsnr(A.cuda(), W.cuda(), qa, qw).cpu().numpy()
    assert mx.mx_device_status() == 0
    ah, _ = deq(orc, name, A)
    wh, _ = deq(orc, name, W)
    o = orc.gemm_qsnr_blas(orc.input_f32(A), orc.input_f32(W), ah, wh)
    assert abs(st[0] - o[0]) <= 1e-3 * o[0]
    assert abs(st[1] - o[1]) <= 1e-3 * o[1]
    assert abs(st[2] - o[2]) <= 1e-2


@pytest.mark.parametrize("name", ["mxfp4", "nvfp4"])
def test_gemm_llama_shape_sampled_rows(mx, orc, name):
    """The 8192 x 4096 by 14336 x 4096 layer in the benchmark's launch
    configuration: 64 sampled rows of C against the oracle's dequantized
    operands in binary64."""
    A, W = inputs.llama_linear()
    cfg = configs(mx)[name]
    qa = mx.quantize(A.cuda(), cfg, stats=False)
    qw = mx.quantize(W.cuda(), cfg, stats=False)
    c = mx.gemm(qa, qw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert mx.mx_device_status() == 0
    rows = np.sort(np.random.default_rng(1).choice(8192, 64, replace=False))
    wh, _ = deq(orc, name, W)
    r = orc.quantize(ocfg(orc, name), A)
    ah = orc.dequantize(ocfg(orc, name), r["packed"], r["scales"], r["tensor_scale"], None, None, 8192, 4096)
    ref = ah[rows].astype(np.float64) @ wh.astype(np.float64).T
    got = c[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel < 1e-3, rel
    assert np.max(np.abs(got - ref)) <= 1e-3 * np.sqrt(np.mean(ref ** 2))


def mbs_cfgs(mx, orc):
    return mx.Config(macro_block=128), orc.Cfg(macro_block=128)


def mbs_expected_sf16(orc, r, rows, cols):
    """The folded UE4M3 16-element scales and the tensor scale, from the
    oracle's E8M0 block scales and E4M3 macro scales: S_M X / 2^t, t the
    largest folded exponent minus 7."""
    sc = r["scales"].reshape(rows, cols // 32).astype(np.int64)
    mc = np.repeat(r["macro"].reshape(rows, cols // 128), 4, axis=1)
    sm = np.array([orc.scale_decode(orc.UE4M3, int(c) & 0x7F) for c in range(128)], np.float64)[mc & 0x7F]
    val = sm * np.exp2(sc - 127.0)
    live = (sc != 0) & (sc != 255) & ((mc & 0x7F) != 0x7F)
    emax = int(np.max(np.floor(np.log2(val[live]))))
    t = emax - 7
    folded = val / 2.0 ** t
    codes = np.zeros_like(sc, dtype=np.uint8)
    for idx in zip(*np.nonzero(live)):
        codes[idx] = orc.scale_encode_nearest(orc.UE4M3, float(np.float32(folded[idx])))
    codes[(sc == 255) | ((mc & 0x7F) == 0x7F)] = 0x7F
    return np.repeat(codes, 2, axis=1), 2.0 ** t


@pytest.mark.parametrize("shape", [(256, 256, 512), (384, 512, 1280)])
def test_mbs_gemm_operands(mx, orc, shape):
    """Macro Block Scaling operands through the NVFP4 GEMM kind: the folded
    scales are S_M X / s_T bit for bit, and C equals the product of the MBS
    dequantized operands (exact products, FP32 accumulation)."""
    M, N, K = shape
    a = inputs.laplace_outlier_cols(M, K, seed=6, n_outlier_cols=2)
    w = inputs.normal(N, K, sigma=0.02, seed=7)
    cfg, ocf = mbs_cfgs(mx, orc)
    qa = mx.quantize(a.cuda(), cfg, stats=False)
    qw = mx.quantize(w.cuda(), cfg, stats=False)
    fa, fw = mx.mbs_gemm_operand(qa), mx.mbs_gemm_operand(qw)
    c = mx.gemm(fa, fw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert mx.mx_device_status() == 0
    ra, rw = orc.quantize(ocf, a), orc.quantize(ocf, w)
    for f, r, rows in ((fa, ra, M), (fw, rw, N)):
        exp, ts = mbs_expected_sf16(orc, r, rows, K)
        assert np.array_equal(f.scales.cpu().numpy(), chunk_layout(exp, rows, K // 16))
        assert float(f.tensor_scale.item()) == ts
    ah = orc.dequantize(ocf, ra["packed"], ra["scales"], ra["tensor_scale"], ra["macro"], None, M, K)
    wh = orc.dequantize(ocf, rw["packed"], rw["scales"], rw["tensor_scale"], rw["macro"], None, N, K)
    ref = ah.astype(np.float64) @ wh.astype(np.float64).T
    got = c.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-3
    assert np.max(np.abs(got - ref)) <= 1e-3 * np.sqrt(np.mean(ref ** 2))


def test_mbs_gemm_scales_rejects_other_configs(mx):
    x = torch.zeros(128, 256, dtype=torch.bfloat16, device="cuda")
    q = mx.quantize(x, mx.MXFP4, stats=False)
    with pytest.raises(ValueError):
        mx.mbs_gemm_operand(q)


@pytest.mark.parametrize("ea,eb", [(2, 2), (3, 3), (2, 3)])
@pytest.mark.parametrize("shape", [(128, 256, 256), (256, 512, 768), (384, 256, 1024)])
def test_mxfp6_gemm(mx, orc, ea, eb, shape):
    """MXFP6 operands (E2M3 / E3M2 codes, one per byte, E8M0 scales per 32) on
    the tcgen05 kind::mxf8f6f4: C equals the binary64 product of the
    oracle's dequantized operands (products of FP6 values and powers of two
    are exact; FP32 accumulation)."""
    M, N, K = shape
    a = inputs.laplace_outlier_cols(M, K, seed=6, n_outlier_cols=2)
    w = inputs.normal(N, K, sigma=0.02, seed=7)
    ca, cw = mx.Config(elem=ea, sf_layout=1), mx.Config(elem=eb, sf_layout=1)
    qa = mx.quantize(a.cuda(), ca, stats=False)
    qw = mx.quantize(w.cuda(), cw, stats=False)
    for out_dtype in (torch.float32, torch.bfloat16):
        c = mx.gemm(qa, qw, out_dtype=out_dtype)
        torch.cuda.synchronize()
        assert mx.mx_device_status() == 0
        oa, ow = orc.Cfg(elem=ea), orc.Cfg(elem=eb)
        ra, rw = orc.quantize(oa, a), orc.quantize(ow, w)
        S = K // 32
        assert np.array_equal(qa.scales.cpu().numpy(), chunk_layout(ra["scales"], M, S))
        # codes in the tensor-core operand layout (16 codes in 12 bytes + 4 zero bytes)
        assert np.array_equal(qa.codes.cpu().numpy(),
                              orc.pack_tc(ea, orc.unpack(ea, ra["packed"], M, K)).ravel())
        ah = orc.dequantize(oa, ra["packed"], ra["scales"], ra["tensor_scale"], None, None, M, K)
        wh = orc.dequantize(ow, rw["packed"], rw["scales"], rw["tensor_scale"], None, None, N, K)
        # the library's dequantizer reads the tensor-core layout back
        xh = mx.dequantize(qa, torch.float32).cpu().numpy()
        assert np.array_equal(xh.view(np.uint32), ah.view(np.uint32))
        ref = ah.astype(np.float64) @ wh.astype(np.float64).T
        got = c.float().cpu().numpy().astype(np.float64)
        tol = 1e-3 if out_dtype == torch.float32 else 8e-3
        assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < tol
        rms = np.sqrt(np.mean(ref ** 2))
        assert np.max(np.abs(got - ref)) <= tol * rms + tol * np.abs(ref).max() * (out_dtype != torch.float32)


@pytest.mark.parametrize("ea,eb", [(2, 0), (0, 3), (3, 0), (0, 2)])
@pytest.mark.parametrize("shape", [(128, 256, 256), (256, 512, 768)])
def test_fp6_fp4_mixed_gemm(mx, orc, ea, eb, shape):
    """One FP6 operand (E2M3 / E3M2) and one MXFP4 operand (packed E2M1) on
    kind::mxf8f6f4, the MX6 weight / activation with MX4 gradient pairing of
    MX training: the packed E2M1 codes are expanded by the TMA to the
    kind's one-byte-per-element shared-memory form.  C equals the binary64
    product of the oracle's dequantized operands within FP32 accumulation."""
    M, N, K = shape
    a = inputs.laplace_outlier_cols(M, K, seed=6, n_outlier_cols=2)
    w = inputs.normal(N, K, sigma=0.02, seed=7)
    ca, cw = mx.Config(elem=ea, sf_layout=1), mx.Config(elem=eb, sf_layout=1)
    qa = mx.quantize(a.cuda(), ca, stats=False)
    qw = mx.quantize(w.cuda(), cw, stats=False)
    oa, ow = orc.Cfg(elem=ea), orc.Cfg(elem=eb)
    ra, rw = orc.quantize(oa, a), orc.quantize(ow, w)
    ah = orc.dequantize(oa, ra["packed"], ra["scales"], ra["tensor_scale"], None, None, M, K)
    wh = orc.dequantize(ow, rw["packed"], rw["scales"], rw["tensor_scale"], None, None, N, K)
    ref = ah.astype(np.float64) @ wh.astype(np.float64).T
    for out_dtype in (torch.float32, torch.bfloat16):
        c = mx.gemm(qa, qw, out_dtype=out_dtype)
        torch.cuda.synchronize()
        assert mx.mx_device_status() == 0
        got = c.float().cpu().numpy().astype(np.float64)
        tol = 1e-3 if out_dtype == torch.float32 else 8e-3
        assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < tol
        rms = np.sqrt(np.mean(ref ** 2))
        assert np.max(np.abs(got - ref)) <= tol * rms + tol * np.abs(ref).max() * (out_dtype != torch.float32)


@pytest.mark.parametrize("had", [16, 32])
@pytest.mark.parametrize("elem", [0, 2])
def test_rotated_operand_gemm(mx, orc, had, elem):
    """Both operands rotated by the same block Hadamard along K, quantized and
    multiplied: (A H)(W H)^T = A W^T.  The GEMM equals the binary64 product of
    the oracle's dequantized rotated operands, and its QSNR against A W^T
    beats the unrotated MXFP4 product on outlier-column activations."""
    M, N, K = 256, 256, 512
    a = inputs.laplace_outlier_cols(M, K, seed=6, n_outlier_cols=2)
    w = inputs.normal(N, K, sigma=0.02, seed=7)
    cfg = mx.Config(elem=elem, hadamard=had, sf_layout=1)
    qa = mx.quantize(a.cuda(), cfg, stats=False)
    qw = mx.quantize(w.cuda(), cfg, stats=False)
    c = mx.gemm(qa, qw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert mx.mx_device_status() == 0
    oc = orc.Cfg(elem=elem, hadamard=had)
    ra, rw = orc.quantize(oc, a), orc.quantize(oc, w)
    ah = orc.dequantize(oc, ra["packed"], ra["scales"], ra["tensor_scale"], None, None, M, K)
    wh = orc.dequantize(oc, rw["packed"], rw["scales"], rw["tensor_scale"], None, None, N, K)
    ref = ah.astype(np.float64) @ wh.astype(np.float64).T
    got = c.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-3
    exact = orc.input_f32(a).astype(np.float64) @ orc.input_f32(w).astype(np.float64).T
    if elem == 0:
        q0 = mx.quantize(a.cuda(), mx.Config(sf_layout=1), stats=False)
        w0 = mx.quantize(w.cuda(), mx.Config(sf_layout=1), stats=False)
        c0 = mx.gemm(q0, w0, out_dtype=torch.float32).cpu().numpy().astype(np.float64)
        assert np.linalg.norm(exact - got) < np.linalg.norm(exact - c0)


def test_gemm_rejects_mismatched_rotation(mx):
    x = torch.zeros(128, 256, dtype=torch.bfloat16, device="cuda")
    qa = mx.quantize(x, mx.Config(hadamard=32, sf_layout=1), stats=False)
    qb = mx.quantize(x, mx.Config(sf_layout=1), stats=False)
    with pytest.raises(mx.MXError) as e:
        mx.gemm(qa, qb)
    assert e.value.code == -2


def test_mxfp6_gemm_qsnr(mx, orc):
    M, N, K = 256, 256, 512
    a = inputs.laplace_outlier_cols(M, K, seed=6, n_outlier_cols=2)
    w = inputs.normal(N, K, sigma=0.02, seed=7)
    cfg = mx.Config(elem=2, sf_layout=1)
    qa = mx.quantize(a.cuda(), cfg, stats=False)
    qw = mx.quantize(w.cuda(), cfg, stats=False)
    st = mx.gemm_qsnr(a.cuda(), w.cuda(), qa, qw).cpu().numpy()
    oc = orc.Cfg(elem=2)
    ra, rw = orc.quantize(oc, a), orc.quantize(oc, w)
    ah = orc.dequantize(oc, ra["packed"], ra["scales"], ra["tensor_scale"], None, None, M, K)
    wh = orc.dequantize(oc, rw["packed"], rw["scales"], rw["tensor_scale"], None, None, N, K)
    o = orc.gemm_qsnr(orc.input_f32(a), orc.input_f32(w), ah, wh)
    assert abs(st[0] - o[0]) <= 1e-3 * o[0]
    assert abs(st[1] - o[1]) <= 1e-3 * o[1]


def test_mxfp6_gemm_needs_n_multiple_of_256(mx):
    a = torch.zeros(128, 256, dtype=torch.bfloat16, device="cuda")
    q = mx.quantize(a, mx.Config(elem=2, sf_layout=1), stats=False)
    with pytest.raises(mx.MXError) as e:
        mx.gemm(q, q)
    assert e.value.code == -2
