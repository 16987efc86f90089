"""sqz_check_csr_static: the CSR check for callers that cannot allocate
device memory (serving loops that must avoid cudaMalloc's implicit
synchronisation, runtimes with all device memory reserved up front).

Its verdict must equal the one sqz_create_layer reaches with its own,
allocating, check on the same arrays -- on consecutive calls, since every
call reuses the same fixed device array and must clear what the previous
call left there.  The flag word is an integer, so the comparison is exact.

This file is named to be collected last, so that a run stopping at the
first failure has already run every other test; it also passes on its own.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

FLAG_WORDS = {1: "rowptr[0]!=0", 2: "rowptr[N]!=nnz", 4: "rowptr decreasing", 8: "column outside [0,K)"}


@pytest.fixture(scope="module")
def B():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from lut_dequant_gemv_b200 import binding, build

    build.build()
    binding.lib()
    return binding


def csr_cases():
    """(name, layer, expected flags) with the same codes/LUT and a CSR that is
    well formed or broken in one way."""
    base = synth.make_layer(64, 256, 3, 0.02, seed=3, key="noalloc")
    out = [("valid", base, 0)]
    empty_rows = synth.make_layer(64, 256, 3, 0.001, seed=4, key="noalloc-sparse")
    out.append(("valid_empty_rows", empty_rows, 0))

    def broken(name, flag, edit):
        rp, col = base.rowptr.copy(), base.col.copy()
        edit(rp, col)
        out.append((name, synth.Layer(base.n_out, base.k_in, base.bits, base.codes, base.lut, rp, col, base.val),
                    flag))

    broken("rowptr0", 1, lambda rp, col: rp.__setitem__(0, 1))
    broken("end", 2, lambda rp, col: rp.__setitem__(-1, rp[-1] - 1))
    broken("decreasing", 4, lambda rp, col: rp.__setitem__(10, rp[11] + 1))
    broken("col_high", 8, lambda rp, col: col.__setitem__(5, 256))
    broken("col_neg", 8, lambda rp, col: col.__setitem__(0, -3))
    out.append(("bench_layer", synth.layer_for(synth.workloads()["llama7b-up-3bit"][0]), 0))
    return out


def create_verdict(B, L):
    """Flags implied by sqz_create_layer: 0 on success, else the reasons its
    message lists."""
    try:
        layer = B.create_layer_from_numpy(L.n_out, L.k_in, L.bits, L.codes, L.lut, L.rowptr, L.col, L.val)
    except B.SqzError as e:
        assert e.status == B.SQZ_ERR_INVALID_ARG
        return sum(bit for bit, word in FLAG_WORDS.items() if word in str(e))
    layer.close()
    return 0


def test_static_check_matches_create_on_consecutive_calls(B):
    cases = csr_cases()
    dev = [(name, torch.from_numpy(L.rowptr).cuda(), torch.from_numpy(L.col).cuda(), L, flag)
           for name, L, flag in cases]
    torch.cuda.synchronize()
    # interleave broken and valid matrices so a stale flag would show
    order = [0, 2, 1, 3, 0, 4, 5, 1, 6, 7, 0]
    for idx in order:
        name, rp, col, L, flag = dev[idx]
        first = B.sqz_check_csr_static(rp, col, L.n_out, L.k_in)
        second = B.sqz_check_csr_static(rp, col, L.n_out, L.k_in)
        assert first == second == flag, (name, first, second, flag)
        assert create_verdict(B, L) == first, name


def test_static_check_rejects_out_of_range_sizes(B):
    rp = torch.zeros(2, dtype=torch.int32, device="cuda")
    col = torch.zeros(1, dtype=torch.int32, device="cuda")
    import ctypes

    flags = ctypes.c_int32(0)
    lib = B.lib()
    assert lib.sqz_check_csr_static(rp.data_ptr(), col.data_ptr(), 1, 4, (1 << 31), None,
                                    ctypes.byref(flags)) == B.SQZ_ERR_INVALID_ARG
    assert "nnz" in B.sqz_last_error()
    assert lib.sqz_check_csr_static(rp.data_ptr(), col.data_ptr(), -1, 4, 1, None,
                                    ctypes.byref(flags)) == B.SQZ_ERR_INVALID_ARG
    assert lib.sqz_check_csr_static(rp.data_ptr(), col.data_ptr(), 1, 4, 1, None, None) == B.SQZ_ERR_INVALID_ARG
    # nnz == 0: accepted without touching the arrays, like sqz_create_layer
    assert lib.sqz_check_csr_static(None, None, 1, 4, 0, None, ctypes.byref(flags)) == B.SQZ_OK
    assert flags.value == 0


def test_static_check_on_a_side_stream(B):
    L = synth.make_layer(300, 512, 4, 0.01, seed=8, key="noalloc-stream")
    rp, col = torch.from_numpy(L.rowptr).cuda(), torch.from_numpy(L.col).cuda()
    bad = col.clone()
    bad[7] = 512
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        assert B.sqz_check_csr_static(rp, bad, L.n_out, L.k_in, stream=s) == 8
        assert B.sqz_check_csr_static(rp, col, L.n_out, L.k_in, stream=s) == 0


def test_static_check_refuses_a_capturing_stream(B):
    """The check reads its verdict back and synchronises, which a graph
    capture cannot contain: on a capturing stream it must return
    SQZ_ERR_UNSUPPORTED without enqueuing anything, and the capture must
    still end cleanly and replay."""
    L = synth.make_layer(64, 256, 3, 0.02, seed=9, key="noalloc-capture")
    rp, col = torch.from_numpy(L.rowptr).cuda(), torch.from_numpy(L.col).cuda()
    out = torch.zeros(4, device="cuda")
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            out.add_(1.0)
            with pytest.raises(B.SqzError) as ei:
                B.sqz_check_csr_static(rp, col, L.n_out, L.k_in, stream=s)
            assert ei.value.status == B.SQZ_ERR_UNSUPPORTED
            assert "captured" in str(ei.value)
            out.add_(1.0)
    g.replay()
    torch.cuda.synchronize()
    assert torch.all(out == 2.0)
    # outside the capture the same call works and clears what it finds
    assert B.sqz_check_csr_static(rp, col, L.n_out, L.k_in) == 0
