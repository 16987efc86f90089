"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Tolerance (from the arithmetic contract in include/sqz.h): for every output
    |y_gpu - y| <= 1e-3 * sum_k |w x| + 1e-6
with y the oracle's fp64 value and the bound computed by the oracle.
Dequantized weights must match the oracle bit for bit.
"""
import numpy as np
import pytest
import torch

import synth
from pins import f16_val, random_csr

pytestmark = pytest.mark.gpu

REL, ABS = 1e-3, 1e-6


@pytest.fixture(scope="module")
def B():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from lut_dequant_gemv_b200 import binding, build

    build.build()
    binding.lib()
    return binding


def upload(B, L):
    return B.create_layer_from_numpy(L.n_out, L.k_in, L.bits, L.codes, L.lut, L.rowptr, L.col, L.val)


def gpu_gemv(B, layer, x_np, ldx=None, ldy=None, n_out=None):
    batch, k_in = x_np.shape
    ldx = ldx or k_in
    n_out = layer.n_out if n_out is None else n_out
    ldy = ldy or n_out
    xd = torch.zeros((batch, ldx), dtype=torch.int16, device="cuda")
    xd[:, :k_in] = torch.from_numpy(x_np.view(np.int16)).cuda()
    yd = torch.full((batch, ldy), 0x7E00, dtype=torch.int16, device="cuda")  # NaN sentinel
    B.sqz_gemv(layer, xd, yd)
    torch.cuda.synchronize()
    return yd.cpu().numpy().view(np.uint16)


def assert_close(y16, y_ref, bound, where=""):
    yg = f16_val(y16)
    err = np.abs(yg - y_ref)
    lim = REL * bound + ABS
    bad = np.argwhere(~(err <= lim))
    assert bad.size == 0, (f"{where}: {len(bad)} outputs out of tolerance, first {bad[:5].tolist()}, "
                           f"gpu={yg[tuple(bad[0])]}, ref={y_ref[tuple(bad[0])]}, bound={bound[tuple(bad[0])]}")


def make_small(seed, n_out, k_in, bits, nnz, dup=False, unsorted=False):
    rng = np.random.default_rng(seed)
    wpr = k_in * bits // 32
    codes = rng.integers(0, 1 << 32, size=(n_out, wpr), dtype=np.uint64).astype(np.uint32)
    lut = np.sort(rng.normal(0, 0.02, size=(n_out, 1 << bits)), axis=1).astype(np.float16).view(np.uint16)
    rowptr, col, val = random_csr(rng, n_out, k_in, nnz, dup=dup, unsorted=unsorted)
    return synth.Layer(n_out, k_in, bits, codes, lut, rowptr, col, val)


SMALL = [
    # (n_out, k_in, bits, nnz, batch, dup, unsorted)
    (1, 32, 3, 0, 1, False, False),
    (1, 8, 4, 1, 1, False, False),
    (7, 96, 3, 9, 3, True, True),
    (33, 24, 4, 40, 2, False, False),
    (65, 1024, 3, 300, 1, False, True),
    (129, 1000, 4, 500, 5, True, False),
    (300, 4128, 3, 2000, 16, False, False),
    (257, 4104, 4, 1500, 7, False, False),
    (64, 2048, 3, 0, 16, False, False),
    # fewer units than warps per CTA, tiles shared by several CTAs
    (500, 2048, 3, 400, 1, False, False),
    (4096, 256, 4, 100, 1, False, True),
    (2000, 512, 3, 300, 4, True, False),
    (1000, 1024, 4, 900, 9, False, False),
]


@pytest.mark.parametrize("n_out,k_in,bits,nnz,batch,dup,unsorted", SMALL)
def test_small_shapes(B, orc, n_out, k_in, bits, nnz, batch, dup, unsorted):
    L = make_small(1000 + n_out + k_in, n_out, k_in, bits, nnz, dup, unsorted)
    x = (np.random.default_rng(7).standard_normal((batch, k_in))).astype(np.float16).view(np.uint16)
    layer = upload(B, L)
    y = gpu_gemv(B, layer, x)
    y_ref, bound = orc.gemv_layer(L, x)
    assert_close(y, y_ref, bound, f"{n_out}x{k_in} b{bits}")


def test_skewed_row(B, orc):
    """One very dense row (every column an outlier) among empty rows."""
    n_out, k_in, bits = 40, 512, 3
    L = make_small(5, n_out, k_in, bits, 0)
    counts = np.zeros(n_out, dtype=np.int64)
    counts[17] = k_in
    counts[3] = 5
    rowptr = np.zeros(n_out + 1, dtype=np.int32)
    np.cumsum(counts, out=rowptr[1:])
    col = np.concatenate([np.arange(5) * 7, np.arange(k_in)[::-1]]).astype(np.int32)
    val = np.random.default_rng(3).uniform(-0.5, 0.5, size=len(col)).astype(np.float16).view(np.uint16)
    L = synth.Layer(n_out, k_in, bits, L.codes, L.lut, rowptr, col, val)
    x = synth.make_x(2, k_in, seed=1)
    y = gpu_gemv(B, upload(B, L), x)
    y_ref, bound = orc.gemv_layer(L, x)
    assert_close(y, y_ref, bound)


def test_strided_x_and_y(B, orc):
    """ldx > K and ldy > N: padding of y is left untouched."""
    L = make_small(9, 50, 256, 4, 30)
    x = synth.make_x(3, 256, seed=2)
    layer = upload(B, L)
    y = gpu_gemv(B, layer, x, ldx=256 + 24, ldy=50 + 13)
    y_ref, bound = orc.gemv_layer(L, x)
    assert_close(y[:, :50], y_ref, bound)
    assert np.all(y[:, 50:] == 0x7E00)


def test_degenerate_sizes(B, orc):
    # N = 0: nothing written, no error
    L0 = synth.Layer(0, 64, 3, np.zeros((0, 6), np.uint32), np.zeros((0, 8), np.uint16),
                     np.zeros(1, np.int32), np.zeros(0, np.int32), np.zeros(0, np.uint16))
    layer = upload(B, L0)
    xd = torch.zeros((1, 64), dtype=torch.int16, device="cuda")
    yd = torch.zeros((1, 1), dtype=torch.int16, device="cuda")
    B.lib().sqz_gemv(layer, xd.data_ptr(), 1, 64, yd.data_ptr(), 1, None)
    # K = 0: y = 0
    Lk = synth.Layer(5, 0, 4, np.zeros((5, 0), np.uint32), np.ones((5, 16), np.uint16) * 0x3C00,
                     np.zeros(6, np.int32), np.zeros(0, np.int32), np.zeros(0, np.uint16))
    layer = upload(B, Lk)
    yd = torch.full((1, 5), 0x7E00, dtype=torch.int16, device="cuda")
    B.lib().sqz_gemv(layer, None, 1, 0, yd.data_ptr(), 5, None)
    torch.cuda.synchronize()
    assert np.all(yd.cpu().numpy() == 0)


def test_dequant_bit_exact(B, orc):
    for L in (make_small(11, 37, 4096, 3, 10), make_small(12, 19, 1032, 4, 0),
              synth.layer_for(synth.workloads()["llama7b-q-4bit"][0])):
        layer = upload(B, L)
        w = torch.empty((L.n_out, L.k_in), dtype=torch.int16, device="cuda")
        B.sqz_debug_dequant(layer, w)
        torch.cuda.synchronize()
        ref = orc.dequant(L.codes, L.lut, L.n_out, L.k_in, L.bits)
        assert np.array_equal(w.cpu().numpy().view(np.uint16), ref)


def _rows_for(shape, limit=60_000_000):
    if shape.n_out * shape.k_in * shape.batch <= limit:
        return None
    rng = np.random.default_rng(shape.n_out + shape.k_in)
    r = rng.choice(shape.n_out, size=384, replace=False)
    return np.unique(np.concatenate([r, [0, 1, shape.n_out - 2, shape.n_out - 1]])).astype(np.int32)


ALL_SHAPES = [(name, s) for name, shapes in synth.workloads().items() for s in shapes]


@pytest.mark.parametrize("name,shape", ALL_SHAPES, ids=[f"{n}:{s.key}:B{s.batch}" for n, s in ALL_SHAPES])
def test_workload_parity(B, orc, name, shape):
    """Every workload shape at full size, in the launch configuration the
    benchmark times; rows sampled where the oracle would take too long."""
    L = synth.layer_for(shape)
    x = synth.x_for(shape)
    y = gpu_gemv(B, upload(B, L), x)
    rows = _rows_for(shape)
    y_ref, bound = orc.gemv_layer(L, x, rows=rows)
    yg = y if rows is None else y[:, rows]
    assert_close(yg, y_ref, bound, shape.key)


def test_deterministic_and_batch_independent(B):
    """Two runs are bit-identical, and each column of a batch-8 call equals
    the batch-1 call on that column (same kernel, same summation order)."""
    shape = synth.workloads()["llama7b-up-3bit"][0]
    L = synth.layer_for(shape)
    layer = upload(B, L)
    x = synth.make_x(8, shape.k_in, seed=5, key="det")
    y8 = gpu_gemv(B, layer, x)
    assert np.array_equal(y8, gpu_gemv(B, layer, x))
    for b in (0, 3, 7):
        y1 = gpu_gemv(B, layer, x[b:b + 1])
        assert np.array_equal(y1[0], y8[b])
    x16 = synth.make_x(16, shape.k_in, seed=6, key="det")
    y16 = gpu_gemv(B, layer, x16)
    assert np.array_equal(y16, gpu_gemv(B, layer, x16))


def test_long_rows_deterministic_and_batch_independent(B, orc):
    """Skewed outliers: rows cut into many sparse shares have their pieces
    added by a warp in a fixed order.  Results match the oracle on sampled
    rows (the longest rows among them), repeat bit for bit, and each column
    of a batch equals the batch-1 call on it -- with the default kernel and
    with the decode-ahead kernel."""
    shape = synth.workloads()["llama7b-skew"][0]
    L = synth.layer_for(shape)
    counts = np.diff(L.rowptr)
    longest = np.argsort(counts)[-24:]
    rows = np.unique(np.concatenate([longest, np.arange(0, shape.n_out, 97)])).astype(np.int32)
    x = synth.make_x(8, shape.k_in, seed=12, key="long-rows")
    for predecode in (0, 1):
        layer = upload(B, L)
        if predecode:
            B.sqz_layer_set_predecode(layer, 1)
        y8 = gpu_gemv(B, layer, x)
        assert np.array_equal(y8, gpu_gemv(B, layer, x))
        for b in (0, 5):
            y1 = gpu_gemv(B, layer, x[b:b + 1])
            assert np.array_equal(y1[0], y8[b]), (predecode, b)
        y_ref, bound = orc.gemv_layer(L, x, rows=rows)
        assert_close(y8[:, rows], y_ref, bound, f"predecode={predecode}")
        layer.close()


def test_host_entry_point_matches_device(B):
    shape = synth.workloads()["llama7b-q-4bit"][0]
    L = synth.layer_for(shape)
    layer = upload(B, L)
    x = synth.make_x(4, shape.k_in, seed=8)
    yd = gpu_gemv(B, layer, x)
    xh = torch.from_numpy(x.view(np.int16).copy()).pin_memory()
    yh = torch.zeros((4, shape.n_out), dtype=torch.int16).pin_memory()
    B.sqz_gemv_host(layer, xh, yh)
    assert np.array_equal(yh.numpy().view(np.uint16), yd)


def test_host_entry_point_replays_read_new_inputs(B, orc):
    """Repeated host calls on the same pinned buffers (served by one captured
    graph) read each call's x and write each call's y; changing the MAC unit
    drops the captured launches; pageable buffers take the direct path."""
    L = make_small(33, 300, 1024, 3, 600)
    layer = upload(B, L)
    s = torch.cuda.Stream()
    xh = torch.empty((2, 1024), dtype=torch.int16).pin_memory()
    yh = torch.empty((2, 300), dtype=torch.int16).pin_memory()
    for trial in range(4):
        if trial == 2:
            B.sqz_layer_set_mac(layer, B.SQZ_MAC_CUDA_CORES)
        x = synth.make_x(2, 1024, seed=40 + trial)
        xh.copy_(torch.from_numpy(x.view(np.int16)))
        B.sqz_gemv_host(layer, xh, yh, stream=s, batch=2 if trial < 2 else 1)
        b = 2 if trial < 2 else 1
        y_ref, bound = orc.gemv_layer(L, x[:b])
        assert_close(yh.numpy()[:b].view(np.uint16), y_ref, bound, f"host replay {trial}")
    xp = torch.from_numpy(synth.make_x(1, 1024, seed=50).view(np.int16).copy())  # pageable
    yp = torch.zeros((1, 300), dtype=torch.int16)
    B.sqz_gemv_host(layer, xp, yp, stream=s)
    y_ref, bound = orc.gemv_layer(L, xp.numpy().view(np.uint16))
    assert_close(yp.numpy().view(np.uint16), y_ref, bound, "host pageable")


def test_host_entry_point_strided_and_unaligned_pinned_buffers(B, orc):
    """Page-locked y written by the product kernel through its device
    mapping, with row strides that are not multiples of 8 elements and
    buffers starting 2 bytes past a 16-byte boundary (x then takes a 2-D
    copy); y's padding columns stay untouched; captured and direct (legacy
    stream) calls agree."""
    L = make_small(61, 200, 512, 4, 300)
    layer = upload(B, L)
    s = torch.cuda.Stream()
    ldx, ldy = 512 + 3, 200 + 5
    xbuf = torch.zeros(3 * ldx + 1, dtype=torch.int16).pin_memory()
    ybuf = torch.full((3 * ldy + 1,), 0x7E00, dtype=torch.int16).pin_memory()
    xh = xbuf[1:1 + 3 * ldx].view(3, ldx)  # 2 bytes past the allocation's start
    yh = ybuf[1:1 + 3 * ldy].view(3, ldy)
    for trial, stream in enumerate((s, s, None)):
        x = synth.make_x(3, 512, seed=70 + trial)
        xh[:, :512].copy_(torch.from_numpy(x.view(np.int16)))
        xh[:, 512:].fill_(0x7C00)  # +inf past K must never be read
        B.sqz_gemv_host(layer, xh, yh, stream=stream)
        y_ref, bound = orc.gemv_layer(L, x)
        assert_close(yh[:, :200].numpy().view(np.uint16), y_ref, bound, f"pinned strided {trial}")
        assert np.all(yh[:, 200:].numpy() == 0x7E00)
    aligned_x = torch.from_numpy(synth.make_x(2, 512, seed=80).view(np.int16).copy()).pin_memory()
    aligned_y = torch.zeros((2, 200), dtype=torch.int16).pin_memory()
    B.sqz_gemv_host(layer, aligned_x, aligned_y, stream=s)
    y_ref, bound = orc.gemv_layer(L, aligned_x.numpy().view(np.uint16))
    assert_close(aligned_y.numpy().view(np.uint16), y_ref, bound, "pinned packed")


def test_non_default_stream(B, orc):
    L = make_small(21, 500, 2048, 3, 400)
    x = synth.make_x(2, 2048, seed=9)
    layer = upload(B, L)
    s = torch.cuda.Stream()
    xd = torch.from_numpy(x.view(np.int16)).cuda()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        yd = torch.empty((2, 500), dtype=torch.int16, device="cuda")
        B.sqz_gemv(layer, xd, yd, stream=s)
    s.synchronize()
    y_ref, bound = orc.gemv_layer(L, x)
    assert_close(yd.cpu().numpy().view(np.uint16), y_ref, bound)


@pytest.mark.parametrize("case", ["rowptr0", "decreasing", "end", "col_high", "col_neg"])
def test_malformed_csr_rejected_on_device(B, case):
    L = make_small(31, 10, 64, 3, 12)
    rowptr, col = L.rowptr.copy(), L.col.copy()
    if case == "rowptr0":
        rowptr[0] = 1
    elif case == "decreasing":
        rowptr[5] = rowptr[6] + 1
    elif case == "end":
        rowptr[-1] -= 1
    elif case == "col_high":
        col[3] = 64
    else:
        col[0] = -1
    with pytest.raises(B.SqzError) as ei:
        B.create_layer_from_numpy(10, 64, 3, L.codes, L.lut, rowptr, col, L.val)
    assert ei.value.status == B.SQZ_ERR_INVALID_ARG


def test_invalid_gemv_args(B):
    L = make_small(41, 8, 64, 4, 3)
    layer = upload(B, L)
    x = torch.zeros((17, 64), dtype=torch.int16, device="cuda")
    y = torch.zeros((17, 8), dtype=torch.int16, device="cuda")
    with pytest.raises(B.SqzError):
        B.sqz_gemv(layer, x, y)  # batch 17
    st = B.lib().sqz_gemv(layer, x.data_ptr(), 2, 63, y.data_ptr(), 8, None)  # ldx < K
    assert st == B.SQZ_ERR_INVALID_ARG
    st = B.lib().sqz_gemv(layer, x.data_ptr(), 2, 64, y.data_ptr(), 7, None)  # ldy < N
    assert st == B.SQZ_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        B.sqz_gemv(layer, x[:2, :63], y[:2])  # the binding checks tensor widths


def test_fp16_yardstick(B, orc):
    L = make_small(51, 333, 1032, 4, 0)
    w = orc.dequant(L.codes, L.lut, L.n_out, L.k_in, 4)
    x = synth.make_x(3, 1032, seed=3)
    ref = f16_val(x) @ f16_val(w).T
    bound = np.abs(f16_val(x)) @ np.abs(f16_val(w)).T
    wd = torch.from_numpy(w.view(np.int16)).cuda()
    xd = torch.from_numpy(x.view(np.int16)).cuda()
    yd = torch.empty((3, 333), dtype=torch.int16, device="cuda")
    B.sqz_fp16_gemv(wd, xd, yd)
    torch.cuda.synchronize()
    assert_close(yd.cpu().numpy().view(np.uint16), ref, bound)


@pytest.mark.parametrize("mac", ["cuda", "mixed"])
@pytest.mark.parametrize("wl", ["llama7b-q-4bit", "llama7b-up-3bit"])
def test_mac_variants_match_oracle(B, orc, wl, mac):
    """The CUDA-core and the split tensor/CUDA-core multiply-accumulate
    variants (batch 1) meet the same bound as the tensor-core one."""
    shape = synth.workloads()[wl][0]
    L = synth.layer_for(shape)
    x = synth.x_for(shape)
    layer = upload(B, L)
    y_tc = gpu_gemv(B, layer, x)
    B.sqz_layer_set_mac(layer, B.SQZ_MAC_CUDA_CORES if mac == "cuda" else B.SQZ_MAC_MIXED)
    y_v = gpu_gemv(B, layer, x)
    y_ref, bound = orc.gemv_layer(L, x)
    assert_close(y_v, y_ref, bound, mac)
    assert_close(y_tc, y_ref, bound, "tensor cores")
    assert B.sqz_layer_status(layer) == 0
    # a batch > 1 call keeps the tensor cores whatever the choice
    x3 = synth.make_x(3, shape.k_in, seed=12)
    y_ref3, bound3 = orc.gemv_layer(L, x3)
    assert_close(gpu_gemv(B, layer, x3), y_ref3, bound3, "batch 3")


@pytest.mark.parametrize("bits,k_in", [(3, 288), (3, 4128), (4, 264), (4, 1000)])
@pytest.mark.parametrize("mac", ["tensor", "mixed"])
def test_padded_columns_with_nonfinite_lut_entries(B, orc, bits, k_in, mac):
    """K not a multiple of 256: the columns past K inside the last
    super-group are padding.  Rows whose LUT holds inf/NaN entries that no
    real code selects must still give finite, exact results (the padding
    must not pick a non-finite entry), and the dequantized export must stay
    bit-exact."""
    n_out = 70
    L = make_small(61 + k_in, n_out, k_in, bits, 50)
    rng = np.random.default_rng(k_in)
    nlev = 1 << bits
    lut = L.lut.copy()
    lut[::3, 0] = 0x7C00   # +inf
    lut[1::3, 0] = 0xFC00  # -inf
    lut[1::3, 1] = 0x7E00  # NaN
    lut[2::3, :nlev - 1] = 0x7C00  # only the last entry finite
    # codes: rows 0,1 (mod 3) never use entries 0/1, rows 2 (mod 3) only the last
    codes_mat = rng.integers(2, nlev, size=(n_out, k_in))
    codes_mat[2::3] = nlev - 1
    bitsarr = ((codes_mat[:, :, None] >> np.arange(bits)) & 1).reshape(n_out, -1)
    words = np.packbits(bitsarr.astype(np.uint8), axis=1, bitorder="little").view("<u4")
    Lx = synth.Layer(n_out, k_in, bits, np.ascontiguousarray(words), lut, L.rowptr, L.col, L.val)
    layer = upload(B, Lx)
    if mac == "mixed":
        B.sqz_layer_set_mac(layer, B.SQZ_MAC_MIXED)
    for batch in (1, 3):
        x = synth.make_x(batch, k_in, seed=batch)
        y = gpu_gemv(B, layer, x)
        y_ref, bound = orc.gemv_layer(Lx, x)
        assert np.isfinite(y_ref).all()
        assert_close(y, y_ref, bound, f"batch {batch}")
    w = torch.empty((n_out, k_in), dtype=torch.int16, device="cuda")
    B.sqz_debug_dequant(layer, w)
    torch.cuda.synchronize()
    assert np.array_equal(w.cpu().numpy().view(np.uint16), orc.dequant(Lx.codes, Lx.lut, n_out, k_in, bits))


@pytest.mark.parametrize("n_out,k_in,bits,batch,ldx_pad", [
    (200, 8288, 3, 16, 0),   # x staged in K chunks; the last chunk is short
    (150, 12000, 4, 12, 0),
    (96, 9216, 3, 9, 1),     # x rows not 16-byte aligned: copied by the threads
    (300, 6144, 4, 16, 0),
    (64, 16384, 3, 8, 0),    # 8 columns that need several passes
    (40, 20000, 4, 16, 0),   # 16 columns, several passes even in launches of 8
    (300, 18432, 3, 5, 0),   # launches of 4 columns (4 carried) and 1
    (300, 18432, 3, 5, 3),
    (40, 98304, 4, 2, 0),    # one column does not fit at all: x in K chunks (7 passes, 2 carried)
    (24, 98304, 3, 3, 1),    # 9 passes, 4 carried, x rows copied by the threads
])
def test_batches_whose_x_is_staged_in_chunks(B, orc, n_out, k_in, bits, batch, ldx_pad):
    """Batches whose activations do not fit in shared memory at once: the
    batch runs as single-pass launches of fewer columns when those are fewer
    than the passes the whole batch would need, else x is staged chunk by
    chunk over several passes with per-tile sums kept between them.  Same
    tolerance, and bit-identical from run to run."""
    L = make_small(90 + k_in, n_out, k_in, bits, n_out * 12)
    x = synth.make_x(batch, k_in, seed=batch)
    layer = upload(B, L)
    y = gpu_gemv(B, layer, x, ldx=k_in + ldx_pad)
    y_ref, bound = orc.gemv_layer(L, x)
    assert_close(y, y_ref, bound, f"{n_out}x{k_in} b{bits} B{batch}")
    assert np.array_equal(y, gpu_gemv(B, layer, x, ldx=k_in + ldx_pad))
    assert B.sqz_layer_status(layer) == 0


@pytest.mark.parametrize("mode", ["balanced", "rowwise"])
@pytest.mark.parametrize("wl,idx", [("llama7b-skew", 0), ("llama7b-skew", 1), ("llama7b-up-3bit", 0)])
def test_csr_schemes_match_oracle(B, orc, wl, idx, mode):
    """Both sparse schemes -- the balanced split and the plain row-per-thread
    CSR it replaces -- on uniform and on heavily skewed outliers (Zipf rows,
    the heaviest entirely outliers), batch 1 and batch 3."""
    shape = synth.workloads()[wl][idx]
    L = synth.layer_for(shape)
    layer = upload(B, L)
    if mode == "rowwise":
        B.sqz_layer_set_csr_mode(layer, B.SQZ_CSR_ROWWISE)
    for batch in (1, 3):
        x = synth.make_x(batch, shape.k_in, seed=batch, key="csr-modes")
        y = gpu_gemv(B, layer, x)
        rows = _rows_for(synth.Shape(shape.name, shape.n_out, shape.k_in, shape.bits, shape.density, batch))
        y_ref, bound = orc.gemv_layer(L, x, rows=rows)
        assert_close(y if rows is None else y[:, rows], y_ref, bound, f"{shape.key} {mode} B{batch}")
    assert B.sqz_layer_status(layer) == 0
    with pytest.raises(B.SqzError):
        B.sqz_layer_set_csr_mode(layer, 5)


def test_chained_calls_read_the_previous_output(B, orc):
    """Back-to-back calls on one stream where each call's x is the previous
    call's y: a launch may start before the previous kernel ends, and must
    still read x only after that kernel has written it."""
    dims = [4096, 1024, 2048, 4096, 512]
    layers, hosts = [], []
    for i in range(len(dims) - 1):
        L = make_small(70 + i, dims[i + 1], dims[i], 3 if i % 2 == 0 else 4, dims[i + 1] * 3)
        hosts.append(L)
        layers.append(upload(B, L))
    x0 = synth.make_x(1, dims[0], seed=4)
    bufs = [torch.from_numpy(x0.view(np.int16)).cuda()]
    for d in dims[1:]:
        bufs.append(torch.full((1, d), 0x7E00, dtype=torch.int16, device="cuda"))
    torch.cuda.synchronize()
    for rep in range(3):
        for i, layer in enumerate(layers):
            B.sqz_gemv(layer, bufs[i], bufs[i + 1])
        torch.cuda.synchronize()
        x = x0
        for i, L in enumerate(hosts):
            y = bufs[i + 1].cpu().numpy().view(np.uint16)
            y_ref, bound = orc.gemv_layer(L, x)
            assert_close(y, y_ref, bound, f"rep {rep} layer {i}")
            x = y  # the next layer's input is what the GPU produced
        for b in bufs[1:]:
            b.fill_(0x7E00)


def test_status_word_clear_after_runs(B):
    shape = synth.workloads()["llama65b-3bit-t3"][2]
    L = synth.layer_for(shape)
    layer = upload(B, L)
    x = synth.x_for(shape)
    for _ in range(3):
        gpu_gemv(B, layer, x)
    assert B.sqz_layer_status(layer) == 0
    with pytest.raises(B.SqzError):
        B.sqz_layer_set_mac(layer, 7)


@pytest.mark.parametrize("wl", ["llama7b-up-3bit", "llama7b-q-4bit"])
def test_layer_holds_the_compressed_weights_once(B, wl):
    """A handle's device memory is the compressed layer (codes, LUTs, CSR)
    once, in the kernel's layout, plus the fixed staging buffers of the host
    entry point (16 columns of x and of y): no second copy of the weights
    (summary page §5 "Inference Latency and Memory Benchmarking", Table 3:
    the memory footprint is the point of the method)."""
    from lut_dequant_gemv_b200 import accounting as acc

    shape = synth.workloads()[wl][0]
    L = synth.layer_for(shape)
    layer = upload(B, L)
    info = B.sqz_layer_info(layer)
    weights = (acc.code_bytes(L.n_out, L.k_in, L.bits) + acc.lut_bytes(L.n_out, L.bits)
               + acc.csr_bytes(L.n_out, L.nnz))
    staging = 2 * 16 * (L.k_in + L.n_out)
    assert info["device_bytes"] <= 1.05 * (weights + staging), (info["device_bytes"], weights, staging)
    # and it still computes the product
    x = synth.x_for(shape)
    y16 = gpu_gemv(B, layer, x)
    import oracle

    rows = np.arange(0, L.n_out, 97, dtype=np.int32)
    y_ref, bound = oracle.default().gemv_layer(L, x, rows=rows)
    assert_close(y16[:, rows], y_ref, bound, wl)
    layer.close()


@pytest.mark.parametrize("n_out,k_in,bits,nnz,batch", [
    (300, 4096, 3, 5000, 1), (257, 1032, 4, 1000, 3), (2000, 3072, 3, 30000, 8), (5000, 512, 4, 0, 2),
    (33, 96, 3, 10, 1), (4100, 2048, 4, 9000, 5), (150, 20000, 3, 400, 1)])
def test_decode_ahead_and_plain_kernels_match_oracle(B, orc, n_out, k_in, bits, nnz, batch):
    """The kernel that decodes ahead of x into tensor memory (an option of
    the handle, batches of 1..8) and the default kernel agree with the oracle
    on the same inputs; the two CTA shapes of the decode-ahead kernel give the
    same bits, and its results do not depend on how many quads a warp parked
    before x arrived (the same MMAs run in the same order either way)."""
    L = make_small(90 + n_out % 17, n_out, k_in, bits, nnz)
    x = synth.make_x(batch, k_in, seed=3, key="pd")
    layer = upload(B, L)
    y_ref, bound = orc.gemv_layer(L, x)
    y_plain = gpu_gemv(B, layer, x)
    assert_close(y_plain, y_ref, bound, "default kernel")
    assert B.sqz_plan_query(n_out, k_in, bits, batch, predecode=1)["predecode"] == 1
    B.sqz_layer_set_predecode(layer, 1)
    y_pd = gpu_gemv(B, layer, x)
    assert_close(y_pd, y_ref, bound, "decode-ahead")
    for _ in range(3):
        assert np.array_equal(gpu_gemv(B, layer, x), y_pd)
    for shape_nw in (8, 16):
        plan = B.sqz_plan_query(n_out, k_in, bits, batch, predecode=shape_nw)
        if not plan["predecode"]:
            continue  # that CTA shape does not fit this call
        assert plan["threads"] == (shape_nw + 1) * 32
        B.sqz_layer_set_predecode(layer, shape_nw)
        assert np.array_equal(gpu_gemv(B, layer, x), y_pd), f"decode-ahead with {shape_nw} dense warps"
    B.sqz_layer_set_predecode(layer, 0)
    assert np.array_equal(gpu_gemv(B, layer, x), y_plain)
    assert B.sqz_layer_status(layer) == 0
    layer.close()


def test_decode_ahead_chained_calls_read_the_previous_output(B, orc):
    """The decode-ahead kernel starts decoding before the previous kernel of
    the stream has finished; x must still be read only after it has."""
    dims = [4096, 1024, 2048, 4096, 512]
    layers, hosts = [], []
    for i in range(len(dims) - 1):
        L = make_small(170 + i, dims[i + 1], dims[i], 3 if i % 2 == 0 else 4, dims[i + 1] * 3)
        hosts.append(L)
        layers.append(upload(B, L))
        B.sqz_layer_set_predecode(layers[-1], 1)
    x0 = synth.make_x(1, dims[0], seed=14)
    bufs = [torch.from_numpy(x0.view(np.int16)).cuda()]
    for d in dims[1:]:
        bufs.append(torch.full((1, d), 0x7E00, dtype=torch.int16, device="cuda"))
    torch.cuda.synchronize()
    for rep in range(3):
        for i, layer in enumerate(layers):
            B.sqz_gemv(layer, bufs[i], bufs[i + 1])
        torch.cuda.synchronize()
        x = x0
        for i, L in enumerate(hosts):
            y = bufs[i + 1].cpu().numpy().view(np.uint16)
            y_ref, bound = orc.gemv_layer(L, x)
            assert_close(y, y_ref, bound, f"rep {rep} layer {i}")
            x = y
        for b in bufs[1:]:
            b.fill_(0x7E00)
